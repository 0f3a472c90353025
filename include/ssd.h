/*
 * ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 selective-SSM layer core.
 *
 * Two operations, both from the Mamba-2 layer used by the hybrid models on
 * the pages ("Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성
 * 분석", §1.4 Mamba-2 구성 and §3.2 접근법 A):
 *
 *   ssd_prefill      the chunked state-space-duality (SSD) scan over a whole
 *                    sequence ("EP6. 트랜스포머 대체 신경망 연구" §7, §8:
 *                    Mamba-2's SSD is exactly a masked, attention-like form);
 *   ssd_decode_step  one token of the recurrence for a batch of sequences,
 *                    streaming the fixed-size state once ("Mamba-3: 추론을
 *                    우선한 상태 공간 모델", opening section: with a scalar
 *                    transition the decode step is memory-bandwidth bound).
 *
 * Per token t, head h (group g = h / (H/G)), with u = SiLU(causal conv4(.)+b)
 * applied to the channels [x | B | C]:
 *     dt  = softplus(dt_raw[t,h] + dt_bias[h])
 *     S_h = exp(dt * A[h]) * S_h + dt * u_x[t,h,:] (outer) u_B[t,g,:]   (P x N)
 *     y   = (S_h . u_C[t,g,:] + D[h] * u_x[t,h,:]) * SiLU(z[t,h,:])
 *
 * Conventions shared by every entry point
 *  - Pointers: all tensor pointers are DEVICE pointers, row-major and
 *    contiguous, owned by the caller.  The library allocates no memory and
 *    keeps no pointer after it returns.
 *  - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *    default stream).  Calls are asynchronous: a returned SSD_OK means the
 *    work was enqueued; faults during execution surface on the stream.
 *  - Validation happens before any launch; a failing check returns its status
 *    and writes nothing.
 *  - Activation dtype (`dtype`): applies to x, dt, B, C, z, y, conv_state and
 *    init_conv_state (y is fp32 under SSD_BF16_YF32).  Parameters and SSM
 *    states are always fp32.
 *  - Shapes: headdim P = 64; d_state N in {16, 32, 64, 128}; nheads % ngroups
 *    == 0; d_conv = 4; chunk Q in {64, 128}.  conv_dim = H*P + 2*G*N.
 *  - Alignment: every tensor pointer 16-byte aligned.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_NULL = 1,        /* a required pointer is NULL                              */
    SSD_ERR_SHAPE = 2,       /* a size is out of range or inconsistent                  */
    SSD_ERR_DTYPE = 3,       /* unknown activation dtype                                */
    SSD_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned                        */
    SSD_ERR_UNSUPPORTED = 5, /* valid but not implemented (e.g. aliasing outputs)      */
    SSD_ERR_CUDA = 6,        /* a CUDA runtime call failed (launch or query)            */
    SSD_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than ssd_prefill_workspace_bytes */
    SSD_ERR_TIMEOUT = 8,     /* a bounded device-side wait gave up                      */
    SSD_ERR_RANGE = 9        /* a backward operand beyond the tensor-core path's fp16 range */
} ssd_status;

/* Activation dtype.  SSD_BF16_YF32 reads bf16 activations (and keeps the conv
 * state in bf16) but writes y in fp32: the same arithmetic as SSD_BF16, whose y
 * is exactly the round-to-nearest-even bf16 of this fp32 y. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1, SSD_BF16_YF32 = 2 } ssd_dtype;

typedef struct {
    int64_t batch;   /* sequences                                       */
    int64_t seqlen;  /* tokens per sequence (ignored by decode)          */
    int32_t nheads;  /* H                                                */
    int32_t headdim; /* P (must be 64)                                   */
    int32_t d_state; /* N                                                */
    int32_t ngroups; /* G; heads h*G/H .. share one B/C group            */
    int32_t chunk;   /* Q, the SSD chunk length (64 or 128)              */
    int32_t d_conv;  /* conv taps (must be 4)                            */
} ssd_dims;

/* Layer parameters, fp32 device pointers. */
typedef struct {
    const float* A;       /* [H]  per-head transition rate, A < 0                   */
    const float* D;       /* [H]  skip weight                                       */
    const float* dt_bias; /* [H]  added to dt_raw before softplus                   */
    const float* conv_w;  /* [conv_dim][4] depthwise taps, tap 3 = current token   */
    const float* conv_b;  /* [conv_dim]                                            */
} ssd_params;

/* Human-readable name of a status code (static storage). */
SSD_API const char* ssd_status_string(ssd_status s);

/* Library build identification (static storage). */
SSD_API const char* ssd_version(void);

/*
 * Bytes of device workspace ssd_prefill needs for these sizes (0 if none).
 * The workspace holds the post-conv, post-SiLU B and C channels of every
 * token ([batch][seqlen][2][G][N] in the activation dtype) on the tensor-core
 * path.  Returns 0 for invalid sizes.
 */
SSD_API size_t ssd_prefill_workspace_bytes(const ssd_dims* dims, ssd_dtype dtype);

/*
 * Which kernel path ssd_prefill takes for these sizes:
 *   1 = tcgen05 tensor-core chunk scan (bf16 activations, P=64, N in {64, 128},
 *       Q in {64, 128}, nheads a multiple of 8).  It always works in chunks of
 *       128 tokens (Q = 64 gives the same result up to rounding: the chunk
 *       length is a tiling choice), and runs N = 64 in the N = 128 tiles with
 *       the upper 64 state channels zero;
 *   2 = CUDA-core chunk scan (every other supported shape, and fp32);
 *  <0 = -(ssd_status) for invalid sizes.
 */
SSD_API int ssd_prefill_path(const ssd_dims* dims, ssd_dtype dtype);

/*
 * Chunked SSD prefill over batch x seqlen tokens.
 *   x, z        [batch][seqlen][H*P]     dtype
 *   dt          [batch][seqlen][H]       dtype (dt_raw, before bias and softplus)
 *   B, C        [batch][seqlen][G][N]    dtype (pre-conv)
 *   init_state  [batch][H][P][N] fp32, or NULL for zeros; may equal final_state
 *   init_conv_state [batch][conv_dim][3] dtype, tokens -3..-1 of the conv
 *               history, or NULL for zeros; must not alias conv_state
 *   y           [batch][seqlen][H*P]     dtype, fp32 for SSD_BF16_YF32 (out);
 *               must not alias x or z
 *   final_state [batch][H][P][N] fp32 (out): the state after the last token
 *   conv_state  [batch][conv_dim][3] dtype (out): pre-conv inputs of tokens
 *               seqlen-3 .. seqlen-1 (history-filled when seqlen < 3)
 *   workspace   device scratch of at least ssd_prefill_workspace_bytes()
 *               bytes (may be NULL when that is 0)
 * seqlen == 0 is valid: final_state = init_state (or zeros), conv_state =
 * the history, y untouched; x, dt, B, C, z and y may then be NULL.
 */
SSD_API ssd_status ssd_prefill(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                       const void* x, const void* dt, const void* B, const void* C, const void* z,
                       const float* init_state, const void* init_conv_state,
                       void* y, float* final_state, void* conv_state,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Elements between consecutive tokens (rows) of each prefill input.  Lets
 * x, z, dt, B and C be views into one wider per-token array -- the in_proj
 * output [batch][seqlen][z | x | B | C | dt] of a Mamba-2 block -- read in
 * place instead of being copied out first.  Batch b starts at row b*seqlen.
 * Each stride must be at least its row width (H*P, H*P, H, G*N, G*N) and a
 * multiple of 16 bytes (SSD_ERR_SHAPE / SSD_ERR_ALIGN otherwise).
 */
typedef struct {
    int64_t x, z, dt, B, C;
} ssd_row_strides;

/*
 * ssd_prefill on strided inputs (row_strides NULL = contiguous rows, the same
 * as ssd_prefill).  y, the states and the workspace are laid out as for
 * ssd_prefill; y must not overlap any input.
 */
SSD_API ssd_status ssd_prefill_strided(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                                       const ssd_row_strides* row_strides, const void* x, const void* dt,
                                       const void* B, const void* C, const void* z, const float* init_state,
                                       const void* init_conv_state, void* y, float* final_state, void* conv_state,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode token for each of `batch` sequences (dims->seqlen is ignored).
 *   x, z        [batch][H*P]   dtype
 *   dt          [batch][H]     dtype
 *   B, C        [batch][G][N]  dtype (pre-conv)
 *   conv_state  [batch][conv_dim][3] dtype, in/out: rolled by one token
 *   ssm_state   [batch][H][P][N] fp32, in/out, updated in place
 *   y           [batch][H*P]   dtype, fp32 for SSD_BF16_YF32 (out)
 * Two launches: the state stream (all heads) and the roll of the shared B/C
 * conv channels, which must follow every head's read of them.  Both are
 * programmatic dependent launches (CUDA's programmatic stream serialization):
 * the state kernel issues its ssm_state load before it waits for the kernel
 * ahead of it in the stream, and reads everything else after.  So a kernel
 * that precedes this call on the stream and lets its dependents start early
 * (griddepcontrol.launch_dependents) must not write ssm_state after doing so;
 * kernels that do not, copies and events order the call as usual.  In this
 * library only the two decode kernels and the prefill's first kernel (always
 * followed by the prefill's own scan) let dependents start early.  Back-to-back
 * decode steps overlap the next step's state load with the previous roll.
 */
SSD_API ssd_status ssd_decode_step(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                           const void* x, const void* dt, const void* B, const void* C, const void* z,
                           void* conv_state, float* ssm_state, void* y, void* stream);

/*
 * Size of the built-in scratch array used by ssd_prefill_noalloc: 16 MiB,
 * enough for batch * seqlen * 2 * ngroups * d_state * 2 bytes, e.g. 4096
 * tokens of a layer with 8 groups of d_state 128.
 */
#define SSD_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * ssd_prefill without a workspace argument, for callers that cannot allocate
 * device memory themselves (no access to an allocator, or an allocation would
 * synchronise or break a pre-reserved memory budget).  No counterpart in the
 * pages: this is a packaging of ssd_prefill, not another step of the method.
 * Arguments, layouts and results are exactly those of ssd_prefill; the
 * scratch lives in a fixed SSD_NOALLOC_SCRATCH_BYTES array inside the
 * library, held on every GPU that loads it until the process exits.
 *  - Returns SSD_ERR_WORKSPACE, launching nothing, when the sizes need more
 *    scratch than that (ssd_prefill_workspace_bytes() > SSD_NOALLOC_SCRATCH_BYTES).
 *  - Allocates nothing: no cudaMalloc / cudaFree or allocating library call.
 *  - The first call on a device (with that device current) looks up the
 *    array's address there; make it before any stream capture.  The address
 *    stays cached for the process: do not use this entry point across a
 *    cudaDeviceReset (the cached address would be stale).
 *  - All calls share the array: calls whose kernels overlap on the GPU race.
 *    Each call rewrites every scratch element it reads, so no clearing is
 *    needed between calls.
 */
SSD_API ssd_status ssd_prefill_noalloc(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                               const void* x, const void* dt, const void* B, const void* C, const void* z,
                               const float* init_state, const void* init_conv_state,
                               void* y, float* final_state, void* conv_state, void* stream);

/*
 * Packed variable-length prefill (continuous batching).  dims->batch = nseq
 * sequences of different lengths are laid back to back along the token axis;
 * dims->seqlen = T, their total.  Sequence s is rows cu_seqlens[s] ..
 * cu_seqlens[s+1]-1; each is scanned on its own, from its own initial states,
 * exactly as ssd_prefill scans one sequence of a batch (chunked prefill with
 * per-sequence states, the serving-stack gap the "EP6" survey's vLLM section
 * names).
 *   cu_seqlens  DEVICE array of nseq+1 int64 (8-byte aligned): 0 = cu[0] <= cu[1]
 *               <= ... <= cu[nseq] = T; empty sequences are allowed.  The kernels
 *               read it; a sequence whose offsets are out of order or outside
 *               [0, T] is treated as empty and ssd_device_status() then reports
 *               SSD_ERR_SHAPE.
 *   x, z        [T][H*P]     dtype;  dt [T][H];  B, C [T][G][N];  y [T][H*P] (out)
 *   init_state  [nseq][H][P][N] fp32 or NULL;  init_conv_state [nseq][conv_dim][3] or NULL
 *   final_state [nseq][H][P][N] fp32 (out);   conv_state [nseq][conv_dim][3] (out)
 *   workspace   at least ssd_prefill_varlen_workspace_bytes() bytes (the
 *               post-conv B/C of all T rows on the tensor-core path, else 0)
 * Same kernel paths, argument rules and error codes as ssd_prefill.
 */
SSD_API size_t ssd_prefill_varlen_workspace_bytes(const ssd_dims* dims, ssd_dtype dtype);
SSD_API ssd_status ssd_prefill_varlen(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                                      const int64_t* cu_seqlens, const void* x, const void* dt, const void* B,
                                      const void* C, const void* z, const float* init_state,
                                      const void* init_conv_state, void* y, float* final_state,
                                      void* conv_state, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Context parallelism: one sequence split into W consecutive segments, one per
 * rank.  The state after a segment is affine in the state before it,
 * S_out = exp(A * sum_t dt_t) * S_in + S_loc, with S_loc the state the segment
 * reaches from zero, so one exchange suffices: each rank scans its segment
 * from zero (ssd_prefill, final_state = S_loc) with the 3 pre-conv tokens
 * before the segment as its init_conv_state (ssd_conv_window of the previous
 * rank's segment), sums its dt (ssd_dt_sum), all ranks gather (S_loc, sums),
 * each folds the segments before its own into its initial state
 * (ssd_cp_combine) and scans its segment again from that state.  Segments
 * must be at least 3 tokens long.  The library provides the three steps; the
 * gather is the caller's (see selective_state_space_43_b200/cp.py).
 *
 * ssd_conv_window: conv_state [batch][conv_dim][3] (out) = pre-conv x|B|C of
 *   tokens seqlen-3 .. seqlen-1 (from init_conv_state, or zero, before token 0);
 *   the conv_state output of ssd_prefill, without the scan.
 * ssd_dt_sum: dt_sum [batch][H] fp32 (out) = sum over the seqlen tokens of
 *   softplus(dt_raw + dt_bias[h]); deterministic.
 * ssd_cp_combine: state_in [batch][H][P][N] fp32 (out) = init_state (or zero)
 *   folded with segments 0 .. upto-1: S <- exp(A_h dt_sums[q]) S + seg_states[q],
 *   with dt_sums [nseg][batch][H] and seg_states [nseg][batch][H][P][N].
 *   dims supplies batch, nheads, headdim and d_state; seqlen is ignored.
 */
SSD_API ssd_status ssd_conv_window(const ssd_dims* dims, ssd_dtype dtype, const void* x, const void* B,
                                   const void* C, const void* init_conv_state, void* conv_state, void* stream);
SSD_API ssd_status ssd_dt_sum(const ssd_dims* dims, ssd_dtype dtype, const float* dt_bias, const void* dt,
                              float* dt_sum, void* stream);
SSD_API ssd_status ssd_cp_combine(const ssd_dims* dims, int nseg, int upto, const float* A, const float* dt_sums,
                                  const float* seg_states, const float* init_state, float* state_in, void* stream);

/*
 * RMSNorm of the gated output before a block's output projection (the
 * "Mamba-3" page, 정규화 section: Mamba-2's norm, kept in hybrids).  Applied
 * after the gate, over norm_groups contiguous channel groups of each row
 * (norm_groups = ngroups for Mamba-2's grouped norm, 1 for one norm over all
 * channels):  out[r][c] = y[r][c] * rsqrt(mean over c's group of y^2 + eps) * weight[c].
 *   y, out      [rows][channels] in dtype (SSD_BF16 or SSD_F32); out may equal y
 *   weight      [channels] fp32
 * channels / norm_groups must be a multiple of 8; pointers 16-byte aligned.
 */
SSD_API ssd_status ssd_gated_rmsnorm(int64_t rows, int32_t channels, int32_t norm_groups, float eps,
                                     ssd_dtype dtype, const void* y, const float* weight, void* out, void* stream);

/*
 * One decode token of the multi-input multi-output (MIMO) SSM for a batch of
 * sequences ("Mamba-3: 추론을 우선한 상태 공간 모델", opening section: several SSMs
 * modelled in parallel per head at almost no cost to decode latency; 아키텍처:
 * the MIMO projection widens B and C).  Rank R = `rank` (1, 2, 4 or 8), on the
 * Mamba-2 scalar decay and without the short conv (the page drops it):
 *   dt = softplus(dt_raw + dt_bias[h]),  a = exp(dt * A[h])
 *   S[h] <- a * S[h] + dt * sum_{k<R} x_k[h] (outer) B_k[g]
 *   y_k[h] = (S[h] . C_k[g] + D[h] * x_k[h]) * silu(z_k[h])
 * R = 1 is the Mamba-2 decode step without its conv.
 *   x, z        [batch][H][R][P]     dtype (post-projection, no conv)
 *   dt          [batch][H]           dtype (dt_raw)
 *   B, C        [batch][G][R][N]     dtype
 *   ssm_state   [batch][H][P][N] fp32, updated in place
 *   y           [batch][H][R][P]     dtype, fp32 for SSD_BF16_YF32 (out)
 * params: A, D, dt_bias are used; conv_w and conv_b are ignored (may be NULL).
 * y must not overlap any input or the state (SSD_ERR_UNSUPPORTED).
 * dims->seqlen and dims->chunk are ignored; the other fields are validated as
 * for the decode step (d_conv included, although the MIMO step has no conv).
 * SSD_ERR_SHAPE for any other rank.
 */
SSD_API ssd_status ssd_mimo_decode_step(const ssd_dims* dims, int32_t rank, ssd_dtype dtype,
                                        const ssd_params* params, const void* x, const void* dt, const void* B,
                                        const void* C, const void* z, float* ssm_state, void* y, void* stream);

/*
 * Gradients of ssd_prefill, for training ("Nemotron-H 스타일 Hybrid Mamba-Transformer
 * 3B 모델 구현 타당성 분석" §3.1/§3.2: the hybrid is trained from scratch and the
 * new Mamba-2 layer's forward and backward are checked).  The gradients are
 * those of the loss  sum(dy * y) + sum(d_final_state * final_state)  with y and
 * final_state the outputs of ssd_prefill on the same inputs; the conv_state
 * output carries none.  Every gradient is fp32 and is written, never added to.
 *
 *   inputs        exactly as for ssd_prefill (contiguous rows; dims->chunk is
 *                 validated but the backward uses its own 64-token chunks)
 *   dy            [batch][seqlen][H*P]: bf16 for SSD_BF16, fp32 for SSD_F32 and
 *                 SSD_BF16_YF32 (the dtype of the forward's y)
 *   d_final_state [batch][H][P][N] fp32, or NULL for zero
 *   grads         dx, dz [batch][seqlen][H*P]; ddt [batch][seqlen][H] (of dt_raw);
 *                 dB, dC [batch][seqlen][G][N] (pre-conv inputs);
 *                 dA, dD, ddt_bias [H]; dconv_w [conv_dim][4]; dconv_b [conv_dim]
 *                 (summed over the batch); d_init_state [batch][H][P][N] and
 *                 d_init_conv_state [batch][conv_dim][3], each NULL when not
 *                 wanted (they are the gradients for the given initial states,
 *                 or for zero ones when those are NULL)
 *   workspace     device scratch of ssd_prefill_backward_workspace_bytes()
 *                 (the post-conv channels and their gradients, fp32, a second
 *                 copy of the B/C gradients, and two fp32
 *                 [batch][ceil(seqlen/64)][H][P][N] state arrays)
 * All pointers device memory, 16-byte aligned; gradients must not overlap the
 * inputs, the workspace or one another (SSD_ERR_UNSUPPORTED otherwise).  The result is deterministic (every sum is taken in a
 * fixed order).  seqlen == 0 is valid: d_init_state = d_final_state (or zero),
 * the parameter gradients and d_init_conv_state are zero.  Errors as for
 * ssd_prefill; SSD_ERR_SHAPE also when ceil(seqlen/64) or batch exceeds 65535.
 */
typedef struct {
    float *dx, *ddt, *dB, *dC, *dz;
    float *dA, *dD, *ddt_bias, *dconv_w, *dconv_b;
    float *d_init_state, *d_init_conv_state;
} ssd_grads;

SSD_API size_t ssd_prefill_backward_workspace_bytes(const ssd_dims* dims);
SSD_API ssd_status ssd_prefill_backward(const ssd_dims* dims, ssd_dtype dtype, const ssd_params* params,
                                        const void* x, const void* dt, const void* B, const void* C, const void* z,
                                        const float* init_state, const void* init_conv_state, const void* dy,
                                        const float* d_final_state, const ssd_grads* grads, void* workspace,
                                        size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream` and reports whether a kernel launched by this library
 * gave up on a bounded device-side wait since the last call (SSD_ERR_TIMEOUT;
 * its outputs are then incomplete), whether a tensor-core backward kernel met
 * an operand that fp16 cannot hold even after its power-of-two state scaling
 * (SSD_ERR_RANGE; |value| >= 65504, the gradients of that call are invalid),
 * or whether the stream holds a CUDA error (SSD_ERR_CUDA).  Clears the flags.  Every wait inside the kernels is bounded
 * (about 2 s), so a kernel can never hang the device.
 */
SSD_API ssd_status ssd_device_status(void* stream);

/*
 * Testing aid for the timeout path (no counterpart in the pages; off unless
 * a test calls it).  While wait_ns is nonzero, every tensor-core prefill
 * (ssd_prefill, ssd_prefill_strided, ssd_prefill_varlen, ssd_prefill_noalloc)
 * launched from this host thread makes each CTA wait wait_ns nanoseconds on a
 * barrier that nothing arrives on before its first tensor-core step; the wait
 * gives up, the CTA lets its copies in flight land, frees its tensor memory
 * and exits, and ssd_device_status() then reports SSD_ERR_TIMEOUT (the
 * outputs of that call are incomplete).  Pass 0 to switch it off.  Nothing
 * faults or hangs: it exercises the same bounded-wait exit a real stall would
 * take.  Thread-local; always returns SSD_OK.
 */
SSD_API ssd_status ssd_test_stall_prefill(uint64_t wait_ns);

/*
 * Optional timing hook for benchmarks.  When both are non-NULL, the next
 * ssd_prefill / ssd_decode_step calls on this host thread record
 * `before_main` (a cudaEvent_t) on their stream immediately before the
 * dominant kernel launch and `after_main` immediately after it.  Pass NULLs
 * to switch it off.  Thread-local; never synchronises.
 */
SSD_API ssd_status ssd_set_timing_events(void* before_main, void* after_main);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
