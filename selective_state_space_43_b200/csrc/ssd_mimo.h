// ssd_mimo.h -- arguments and launcher of the MIMO decode step (ssd_mimo.cu).
// Free of CUDA headers, like ssd_backward.h, so that ssd_mimo.cu also compiles for the tests'
// host emulation of the CUDA execution model.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace ssd {
namespace mimo {

struct MimoArgs {
    int64_t batch;
    int H, P, N, G, R;
    bool act_bf16;  // x, dt, B, C, z are bf16 (else fp32)
    bool y_bf16;    // y is bf16 (else fp32)
    const float *A, *D, *dt_bias;  // [H]
    const void *x, *z;             // [batch][H][R][P]
    const void* dt;                // [batch][H]
    const void *B, *C;             // [batch][G][R][N]
    float* ssm_state;              // [batch][H][P][N], updated in place
    void* y;                       // [batch][H][R][P]
    void* ev_before = nullptr;     // optional cudaEvent_t pair around the step kernel
    void* ev_after = nullptr;
};

// Dynamic shared memory of the step kernel: the head's P x N fp32 state, x, B, C and y of one
// (sequence, head), and the state load's mbarrier.
inline size_t smem_bytes(int R, int P, int N) {
    return (size_t)(P * N + 2 * R * P + 2 * R * N) * sizeof(float) + 16;
}

}  // namespace mimo
}  // namespace ssd
