// ssd_backward.h -- arguments and launcher of the prefill backward (ssd_backward.cu).
//
// Kept free of CUDA headers so that ssd_backward.cu also compiles as plain C++
// for the tests' host emulation of the CUDA execution model (SSD_EMU), which
// supplies cudaError_t and cudaStream_t itself.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace ssd {
namespace bwd {

struct BwdArgs {
    int64_t batch, L;
    int H, P, N, G;
    bool act_bf16;  // x, dt, B, C, z, init_conv_state are bf16 (else fp32)
    bool dy_bf16;   // dy is bf16 (else fp32)
    const float *A, *D, *dt_bias, *conv_w, *conv_b;
    const void *x, *dt, *B, *C, *z, *dy;
    const float* init_state;      // [batch][H][P][N] or nullptr (zeros)
    const void* init_conv_state;  // [batch][conv_dim][3] or nullptr (zeros)
    const float* d_final;         // [batch][H][P][N] or nullptr (zeros)
    // gradients (fp32, written, never accumulated into)
    float *dx, *ddt, *dB, *dC, *dz;              // [batch][L][...] like the inputs
    float *dA, *dD, *ddt_bias;                   // [H]
    float *dconv_w, *dconv_b;                    // [conv_dim][4], [conv_dim]
    float *d_init_state, *d_init_conv_state;     // nullable
    void* workspace;
    // optional cudaEvent_t pair recorded around chunk_bwd_kernel (the dominant kernel), or nullptr
    void* ev_before = nullptr;
    void* ev_after = nullptr;
};

// Inputs and outputs of the tensor-core version of the per-chunk state sums (ssd_backward_tc.cu): the
// workspace's post-conv channels U [batch][L][conv_dim], dt and in-chunk cumsum DT, CS [batch][H][L], and
// the chunk-local sums SP, LM [batch][nchunks][H][P][N] it writes.
struct ChunkStateTcArgs {
    int64_t batch, L;
    int H, G, N;
    bool act_bf16, dy_bf16;
    const float *U, *DT, *CS;
    const void *dy, *z;
    float *SP, *LM;
};

// Inputs and outputs of the tensor-core per-chunk backward (ssd_backward_tc.cu), which writes exactly what
// the CUDA-core chunk kernel writes: dz, ddt, the post-conv gradients of x (DU) and of B, C (DU for the
// first half of each group's heads, DU2 for the second), and the per-chunk partials PH.
// The entering states and leaving adjoints come as the state pass's fp16 tiles SPH, LMH
// [batch][nchunks][H][N/64][64][64] (128-byte swizzled rows, row p scaled by s_p) with the inverse row
// scales SPS, LMS [batch][nchunks][H][64].
struct ChunkBwdTcArgs {
    int64_t batch, L;
    int H, G, N, split, nsplit_pf;  // heads-per-group halves (1 or 2); partial sums per chunk in PF
    bool act_bf16, dy_bf16;
    const float *A, *D, *dt_bias;
    const void *dt, *z, *dy;
    const float *U, *DT, *CS;
    const void *SPH, *LMH;
    const float *SPS, *LMS, *PF;
    float *dz, *ddt, *DU, *DU2, *PH;
};

// Bytes of workspace launch_prefill_backward needs (every region 256-byte aligned).
size_t workspace_bytes(int64_t batch, int64_t L, int H, int P, int N, int G);

// Dynamic shared memory of the per-chunk backward kernel for d_state N.
size_t chunk_bwd_smem_bytes(int N);

}  // namespace bwd
}  // namespace ssd
