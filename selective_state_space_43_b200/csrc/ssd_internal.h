// ssd_internal.h -- launch arguments and launcher entry points shared by the
// C-ABI layer (ssd_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// Activation / output types: fp32 in and out; bf16 in and out; bf16 in, fp32 y.
enum class ActKind { F32, BF16, BF16_YF32 };

// Records the caller's events around the dominant kernel (benchmark hook).
struct TimingHook {
    cudaEvent_t ev_before = nullptr, ev_after = nullptr;
    void before(cudaStream_t s) const {
        if (ev_before) cudaEventRecord(ev_before, s);
    }
    void after(cudaStream_t s) const {
        if (ev_after) cudaEventRecord(ev_after, s);
    }
};

struct DecodeArgs {
    int H, P, N, G, HP, GN, conv_dim, hpg;
    const float *A, *D, *dt_bias, *conv_w, *conv_b;
    const void *x, *dt, *B, *C, *z;
    void* conv_state;
    float* ssm_state;
    void* y;
};

struct PrefillArgs {
    int64_t batch, L, nchunks;
    int H, P, N, G, Q, HP, GN, conv_dim, hpg;
    const float *A, *D, *dt_bias, *conv_w, *conv_b;
    const void *x, *dt, *B, *C, *z;
    const float* init_state;
    const void* init_conv_state;
    void* y;
    float* final_state;
    void* conv_state;
    void* workspace;  // tensor-core path: post-conv B and C, [batch*L][2][G][N] bf16
    // Packed variable-length batch: device array of batch+1 row offsets (cu[0] = 0, cu[batch] = L);
    // sequence b is rows cu[b] .. cu[b+1]-1 of [L][...] activations.  nullptr: batch x L layout.
    const int64_t* cu = nullptr;
    int* err = nullptr;  // device error word (bit 1: a sequence's offsets were invalid)
    // Elements between consecutive rows (tokens) of each input; a batch is L rows.  The contiguous
    // widths HP, HP, H, GN, GN unless the inputs are views into a wider array (e.g. the in_proj output).
    int64_t rs_x = 0, rs_z = 0, rs_dt = 0, rs_B = 0, rs_C = 0;
    // Tests of the timeout path only (0 otherwise): the tensor-core scan's MMA warp first waits this
    // many ns on a barrier that nothing arrives on, then gives up and aborts its CTA.
    uint64_t stall_ns = 0;
};

// Device error word bits, read back by ssd_device_status.
constexpr int kErrTimeout = 1, kErrBadSeqlens = 2;

// Rows of sequence b: the first row in the [rows][...] activation arrays, the length, and whether its
// offsets were valid (0 <= cu[b] <= cu[b+1] <= L); an invalid sequence is treated as empty.
struct SeqSpan {
    int64_t row0, len;
    bool ok;
};
__device__ inline SeqSpan seq_span(const PrefillArgs& a, int64_t b) {
    if (!a.cu) return SeqSpan{b * a.L, a.L, true};
    const int64_t r0 = a.cu[b], r1 = a.cu[b + 1];
    if (r0 < 0 || r1 < r0 || r1 > a.L) return SeqSpan{0, 0, false};
    return SeqSpan{r0, r1 - r0, true};
}

// The device error word of the current device (nullptr if it cannot be found).
int* device_error_flag();

cudaError_t launch_decode(const DecodeArgs& a, int64_t batch, ActKind kind, cudaStream_t st, const TimingHook& hook);

// CUDA-core chunked SSD (any supported shape, fp32 or bf16 activations).
cudaError_t launch_prefill_simt(const PrefillArgs& a, ActKind kind, cudaStream_t st, const TimingHook& hook);

// tcgen05 tensor-core chunked SSD (bf16 activations, P = 64, Q = 128, N in {64, 128}).
bool prefill_tc_supported(int P, int N, int Q, int H, bool bf16);
size_t prefill_tc_workspace_bytes(int64_t batch, int64_t L, int G, int N);
cudaError_t launch_prefill_tc(const PrefillArgs& a, ActKind kind, cudaStream_t st, const TimingHook& hook);
// Synchronises `st`, then reads and clears the tensor-core kernel's timeout flag.
cudaError_t read_and_clear_tc_error(int* flag, cudaStream_t st);

// Reads and clears the decode step's error word (nonzero: a state load never landed).  Does not
// synchronise: call after the stream is idle.
cudaError_t read_and_clear_decode_error(int* flag);

namespace mimo {
struct MimoArgs;
// The MIMO decode step (ssd_mimo.cu); sizes and pointers validated by the caller.
cudaError_t launch_mimo_decode(const MimoArgs& a, cudaStream_t st);
// Reads and clears the MIMO kernel's error word (nonzero: a state load never landed).  Does not
// synchronise: call after the stream is idle.
cudaError_t read_and_clear_mimo_error(int* flag);
}  // namespace mimo

namespace bwd {
struct BwdArgs;
// The prefill backward (ssd_backward.cu); sizes and pointers validated by the caller.
cudaError_t launch_prefill_backward(const BwdArgs& a, cudaStream_t st);
// Reads and clears the error word of the backward's tensor-core kernel (ssd_backward_tc.cu; nonzero: a
// bounded wait gave up).  Does not synchronise: call after the stream is idle.
cudaError_t read_and_clear_bwd_tc_error(int* flag);
// The same for the tensor-core per-chunk backward (ssd_chunk_bwd_tc.cu).
cudaError_t read_and_clear_chunk_bwd_tc_error(int* flag);
}  // namespace bwd

}  // namespace ssd
