// ssd_backward.cu -- gradients of the chunked SSD prefill (the training backward).
//
// The layer is trained from scratch in "Nemotron-H 스타일 Hybrid Mamba-Transformer
// 3B 모델 구현 타당성 분석" (§3.1: the new Mamba-2 layer needs its forward and
// backward checked; §3.2 phase 2).  The backward differentiates the loss
//   sum dy . y + sum d_final . final_state
// through the whole layer core: conv1d (k=4) + SiLU on [x | B | C], dt =
// softplus(dt_raw + dt_bias), the scalar-decay state recurrence, the D skip
// and the SiLU(z) gate.
//
// It works on its own 64-token chunks (the chunk length is an implementation
// choice; the gradients do not depend on it beyond rounding).  With, inside a
// chunk, cs_i the inclusive cumulative sum of dt*A, L_ij = exp(cs_i - cs_j)
// (i >= j), g_i = dy_i * silu(z_i), Sp the state entering the chunk and Lm the
// adjoint of the state leaving it:
//
//   y_i   = sum_{j<=i} (C_i.B_j) L_ij dt_j x_j + exp(cs_i) Sp C_i + D x_i
//   dx_j  = dt_j [sum_{i>=j} (C_i.B_j) L_ij g_i + exp(cs_last - cs_j) Lm B_j] + D g_j
//   dB_j  = dt_j [sum_{i>=j} (g_i.x_j) L_ij C_i + exp(cs_last - cs_j) x_j Lm]     (summed over the group's heads)
//   dC_i  = sum_{j<=i} (g_i.x_j) L_ij dt_j B_j + exp(cs_i) g_i Sp                  (summed over the group's heads)
//   d(dA_k) = sum_{i>=k} sum_{j<k} M_ij + sum_{i>=k} E_i + F + sum_{j<k} W_j,
//     M_ij = (g_i.x_j)(C_i.B_j) L_ij dt_j,  E_i = exp(cs_i) g_i.(Sp C_i),
//     F = exp(cs_last) <Lm, Sp>,  W_j = exp(cs_last - cs_j) dt_j x_j.(Lm B_j)
//   ddt_j = sum_i M_ij / dt_j + W_j / dt_j + A d(dA_j)   (the first two formed without dividing)
//   Lm of chunk c-1 = exp(cs_last,c) Lm_c + sum_{i in c} exp(cs_i) g_i (outer) C_i
//
// Kernels, in launch order (all fp32 arithmetic):
//   post_conv_kernel    u = silu(conv(xBC)) of every channel and token           -> U
//   dt_kernel           dt and the in-chunk cumsum of dt*A                       -> DT, CS
//   chunk_state_kernel  per (chunk, head): sum exp(cs_last-cs_j) dt_j x_j B_j^T and
//                       sum exp(cs_i) g_i C_i^T                                   -> SP, LM
//   state_pass_kernel   per head (4 CTAs, one slice of the state each): forward scan of
//                       SP into the entering states, reverse scan of LM into the leaving
//                       adjoints, F per chunk (4 partial sums), d_init_state
//   chunk_bwd_kernel    per (chunk, group, half of the group's heads), heads in turn: dz,
//                       ddt, the post-conv gradients of x (per head) and of B, C (summed
//                       over the half; the conv backward adds the two halves)
//   conv_bwd_kernel     per (channel, 32-token tile): through SiLU' and the taps to
//                       the pre-conv gradients, per-tile conv_w/conv_b partial sums,
//                       d_init_conv_state
//   reduce_kernel       sums of the per-tile / per-chunk partials in a fixed order
//                       -> dconv_w, dconv_b, dA, dD, ddt_bias (deterministic)
//
// SSD_EMU: compiled as plain C++ by the tests' host emulation (one thread per
// CUDA thread, a real barrier for __syncthreads), which runs this same source
// on the CPU under AddressSanitizer; the library is always built with nvcc.
#ifdef SSD_EMU
#include "emu_cuda.h"
#define SSD_LAUNCH(kern, grid, block, smem, st, ...) \
    ((void)(st), ::emu::launch((grid), (block), (smem), [&]() { kern(__VA_ARGS__); }))
#define SSD_SET_SMEM(kern, bytes) cudaSuccess
#define SSD_DYN_SMEM() (::emu::smem())
#else
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#define SSD_LAUNCH(kern, grid, block, smem, st, ...) kern<<<(grid), (block), (smem), (st)>>>(__VA_ARGS__)
#define SSD_SET_SMEM(kern, bytes) \
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes))
extern __shared__ __align__(16) unsigned char ssd_bwd_smem[];
#define SSD_DYN_SMEM() (ssd_bwd_smem)
#endif

#include <type_traits>

#include "ssd_backward.h"

namespace ssd {
namespace bwd {

#ifndef SSD_EMU
// The tensor-core per-chunk state sums (ssd_backward_tc.cu), used in place of chunk_state_kernel for bf16
// activations with P = 64 and N in {64, 128}.
bool chunk_state_tc_supported(int P, int N, bool act_bf16);
cudaError_t launch_chunk_state_tc(const ChunkStateTcArgs& a, int64_t nchunks, cudaStream_t st);
// The tensor-core per-chunk backward (ssd_chunk_bwd_tc.cu), used in place of chunk_bwd_kernel under the
// same conditions (and 16-byte aligned dy, z, dz).
bool chunk_bwd_tc_supported(int P, int N, bool act_bf16, const void* dy, const void* z, const void* dz);
cudaError_t launch_chunk_bwd_tc(const ChunkBwdTcArgs& a, int64_t nchunks, cudaStream_t st);
#endif

constexpr int kQ = 64;    // backward chunk (tokens)
constexpr int kT = 256;   // threads per block
constexpr int kP = 64;    // head dimension
constexpr int kS = kQ + 4;  // row stride of the 64-wide shared tiles: a multiple of 4 floats (16-byte rows)
constexpr int kTS = kQ + 1; // row stride of the prefix-sum tile (written row by row, one row per thread)
constexpr int kSplit = 4;   // CTAs per head in the chunk-to-chunk state scans

struct Ws {
    float* U;   // [batch][L][conv_dim]  post-conv, post-SiLU channels
    float* DU;  // [batch][L][conv_dim]  their gradients
    float* DT;  // [batch][H][L]         dt
    float* CS;  // [batch][H][L]         in-chunk inclusive cumsum of dt*A
    float* SP;  // [batch][nc][H][P][N]  chunk-local states, then the states entering each chunk
    float* LM;  // [batch][nc][H][P][N]  chunk-local adjoints, then the adjoints leaving each chunk
    float* PF;  // [batch][nc][H][kSplit]  F = exp(cs_last) <Lm, Sp>, in kSplit partial sums
    float* PH;  // [batch][nc][H][3]     per-chunk partial dA, dD, ddt_bias
    float* PW;  // [batch][ntile][conv_dim][5]  per-tile partial dconv_w (4), dconv_b
    float* DU2; // [batch][L][2 G N]     dB | dC of the second half of each group's heads (when split)
    // for the tensor-core chunk backward (else unused): the entering states and leaving adjoints as fp16
    // tiles, [batch][nc][H][N/64 boxes][64 rows p][64 n] with 128-byte rows and the 128-byte swizzle (the
    // shared-memory image its MMAs read), each row p scaled by a power of two s_p <= 1 that keeps it below
    // 2^14, and the inverses 1/s_p [batch][nc][H][64]
    float* SPH;
    float* LMH;
    float* SPS;
    float* LMS;
};

namespace {

__host__ __device__ inline int64_t nchunks(int64_t L) { return (L + kQ - 1) / kQ; }
constexpr int kCT = 32;   // tokens per tile of the two conv kernels (twice the threads of a 64-token tile)
__host__ __device__ inline int64_t ntiles(int64_t L) { return L > 0 ? (L + kCT - 1) / kCT : 1; }
// CTAs per (chunk, group) in the chunk backward: the group's heads in two halves when there are two or more
__host__ __device__ inline int head_split(int H, int G) { return H / G >= 2 ? 2 : 1; }
inline size_t round256(size_t v) { return (v + 255) & ~size_t(255); }

// Carves the workspace; returns the bytes used (base may be null to only count).
size_t carve(int64_t batch, int64_t L, int H, int P, int N, int G, char* base, Ws* ws) {
    const int64_t conv_dim = (int64_t)H * P + 2LL * G * N, nc = nchunks(L), nt = ntiles(L);
    const size_t sizes[14] = {
        (size_t)(batch * L * conv_dim), (size_t)(batch * L * conv_dim), (size_t)(batch * H * L),
        (size_t)(batch * H * L),        (size_t)(batch * nc * H * P * N), (size_t)(batch * nc * H * P * N),
        (size_t)(batch * nc * H * kSplit), (size_t)(batch * nc * H * 3),  (size_t)(batch * nt * conv_dim * 5),
        (size_t)(batch * L * 2 * G * N), (size_t)(batch * nc * H * P * N / 2), (size_t)(batch * nc * H * P * N / 2),
        (size_t)(batch * nc * H * P),   (size_t)(batch * nc * H * P)};
    float** slots[14] = {&ws->U,  &ws->DU, &ws->DT,  &ws->CS,  &ws->SP,  &ws->LM,  &ws->PF,
                         &ws->PH, &ws->PW, &ws->DU2, &ws->SPH, &ws->LMH, &ws->SPS, &ws->LMS};
    size_t off = 0;
    for (int k = 0; k < 14; ++k) {
        if (base) *slots[k] = reinterpret_cast<float*>(base + off);
        off += round256(sizes[k] * sizeof(float));
    }
    return off;
}

__device__ __forceinline__ float ld_act(const void* p, int64_t i, bool bf16) {
    if (bf16) return __uint_as_float(static_cast<unsigned>(static_cast<const unsigned short*>(p)[i]) << 16);
    return static_cast<const float*>(p)[i];
}
__device__ __forceinline__ float act_to_f(unsigned short v) { return __uint_as_float(static_cast<unsigned>(v) << 16); }
__device__ __forceinline__ float act_to_f(float v) { return v; }

// A 16-byte global -> shared copy that takes no registers while in flight (cp.async, cached in L2 only); the
// bytes past src_bytes (0 or 16) are zero-filled, and none is read when src_bytes is 0.
#ifdef SSD_EMU
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    memset(dst, 0, 16);
    if (src_bytes) memcpy(dst, src, src_bytes);
}
__device__ __forceinline__ void cp_async_wait_all() {}
#else
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(sa), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}
#endif
__device__ __forceinline__ float sigmoid_f(float v) { return 1.f / (1.f + expf(-v)); }
__device__ __forceinline__ float silu_f(float v) { return v * sigmoid_f(v); }
__device__ __forceinline__ float dsilu_f(float v) {
    const float s = sigmoid_f(v);
    return s * (1.f + v * (1.f - s));
}
__device__ __forceinline__ float softplus_f(float v) { return v > 20.f ? v : log1pf(expf(v)); }
// The same with the fast exponential and division (a few ulp; 0 and 1 at the far ends): the two conv kernels
// evaluate one per channel and token, and there the instruction count is what competes with HBM.
__device__ __forceinline__ float sigmoid_fast(float v) { return __fdividef(1.f, 1.f + __expf(-v)); }
__device__ __forceinline__ float silu_fast(float v) { return v * sigmoid_fast(v); }
__device__ __forceinline__ float dsilu_fast(float v) {
    const float s = sigmoid_fast(v);
    return s * (1.f + v * (1.f - s));
}

// Pre-conv value of channel c at token s of sequence b (s in [-3, L)); history or zero before 0.
__device__ __forceinline__ float raw_at(const BwdArgs& a, int64_t b, int64_t s, int64_t c) {
    const int64_t HP = (int64_t)a.H * a.P, GN = (int64_t)a.G * a.N, conv_dim = HP + 2 * GN;
    if (s < 0)
        return a.init_conv_state ? ld_act(a.init_conv_state, (b * conv_dim + c) * 3 + (s + 3), a.act_bf16) : 0.f;
    const int64_t row = b * a.L + s;
    if (c < HP) return ld_act(a.x, row * HP + c, a.act_bf16);
    if (c < HP + GN) return ld_act(a.B, row * GN + (c - HP), a.act_bf16);
    return ld_act(a.C, row * GN + (c - HP - GN), a.act_bf16);
}

// The two conv kernels spread a kCT-token tile over several threads per channel: each thread takes a short
// window, loads all of it, then computes, so that many loads are in flight without long per-thread chains
// (measured: both the 2-token streaming loop and one thread per whole tile leave HBM well under half busy).
constexpr int kPC = 64;                // post_conv: channel pairs per CTA
constexpr int kPST = kCT * kPC / kT;   // post_conv: tokens per thread (kT / kPC sub-tiles of the tile)
static_assert(kPST * (kT / kPC) == kCT, "the sub-tiles cover the tile");
// conv_bwd stages its tile in shared memory instead: kCB channels x (kCT + 6) pre-conv rows and (kCT + 3) du
// rows arrive by cp.async, so the loads in flight hold no registers, and each row is read as one kCB-channel
// run (DRAM serves long runs of a row better than many short ones); then each thread takes a channel pair
// (packed fp32 arithmetic) and kBST tokens of the tile, in two passes through shared memory.
constexpr int kCB = 128;                     // channels per CTA
constexpr int kBPairs = kCB / 2;             // channel pairs per CTA
constexpr int kBSUB = kT / kBPairs;          // sub-tiles per tile
constexpr int kBST = kCT / kBSUB;            // tokens per thread
constexpr int kRawRows = kCT + 6, kDuRows = kCT + 3;
static_assert(kBST * kBSUB == kCT && kCB % 8 == 0 && kBPairs % 32 == 0,
              "the sub-tiles cover the tile; whole 16-byte chunks per row; a warp within one sub-tile");
// shared memory of conv_bwd_kernel: the staged pre-conv rows (element size esz), du and du2 rows, partials
inline size_t conv_bwd_smem(size_t esz) {
    return (size_t)kRawRows * kCB * esz + 2 * (size_t)kDuRows * kCB * 4 + (size_t)kBSUB * 5 * kCB * 4;
}

// Channels c, c + 1 of one token from its row: bf16 pairs as one 32-bit load, fp32 pairs as one 64-bit load.
__device__ __forceinline__ float2 act_pair(const unsigned short* p) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ float2 act_pair(const float* p) { return *reinterpret_cast<const float2*>(p); }

// grid (ceil(conv_dim / (2 kPC)), ntiles, batch), kT threads: thread (pair lc, sub-tile) takes channels
// c, c + 1 and tokens t0 .. t0 + kPST - 1; it loads their pre-conv values and those of the 3 tokens before
// (the conv history before token 0), then writes u = silu(conv) for its tokens.  Token indices are 32-bit
// and every load is a 32-bit offset from one row pointer: the index arithmetic is most of the kernel's
// instructions otherwise.  kBf16: the inputs are bf16 (a.act_bf16); kHist: a conv history is given
// (a.init_conv_state; without one the tokens before 0 are zero and take no registers).
template <bool kBf16, bool kHist>
__global__ void __launch_bounds__(kT) post_conv_kernel(BwdArgs a, Ws ws) {
    using T = typename std::conditional<kBf16, unsigned short, float>::type;
    const int HP = a.H * a.P, GN = a.G * a.N, conv_dim = HP + 2 * GN, L = static_cast<int>(a.L);
    const int lc = threadIdx.x % kPC, sub = threadIdx.x / kPC;
    const int c = (blockIdx.x * kPC + lc) * 2;
    const int b = blockIdx.z, t0 = blockIdx.y * kCT + sub * kPST;
    if (c >= conv_dim || t0 >= L) return;
    float w[2][4], bias[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float4 wv = *reinterpret_cast<const float4*>(a.conv_w + (c + k) * 4);
        w[k][0] = wv.x, w[k][1] = wv.y, w[k][2] = wv.z, w[k][3] = wv.w;
        bias[k] = a.conv_b[c + k];
    }
    // the pre-conv array of channels c, c + 1 (x, B or C), its row stride, and the pointer at token t0
    const T* src;
    int rs;
    if (c < HP) {
        src = static_cast<const T*>(a.x) + c, rs = HP;
    } else if (c < HP + GN) {
        src = static_cast<const T*>(a.B) + (c - HP), rs = GN;
    } else {
        src = static_cast<const T*>(a.C) + (c - HP - GN), rs = GN;
    }
    src += ((int64_t)b * L + t0) * rs;
    float2 r[kPST + 3];  // tokens t0 - 3 .. t0 + kPST - 1
#pragma unroll
    for (int i = 0; i < kPST + 3; ++i) {
        const int s = t0 - 3 + i;
        if (s >= L || (!kHist && i < 3 && s < 0))
            r[i] = make_float2(0.f, 0.f);
        else if (i < 3 && s < 0)
            r[i] = make_float2(raw_at(a, b, s, c), raw_at(a, b, s, c + 1));
        else
            r[i] = act_pair(src + (i - 3) * rs);
    }
    float* u = ws.U + ((int64_t)b * L + t0) * conv_dim + c;
#pragma unroll
    for (int i = 0; i < kPST; ++i) {
        if (t0 + i < L) {
            float2 v;
            v.x = silu_fast(bias[0] + w[0][0] * r[i].x + w[0][1] * r[i + 1].x + w[0][2] * r[i + 2].x + w[0][3] * r[i + 3].x);
            v.y = silu_fast(bias[1] + w[1][0] * r[i].y + w[1][1] * r[i + 1].y + w[1][2] * r[i + 2].y + w[1][3] * r[i + 3].y);
            *reinterpret_cast<float2*>(u + i * conv_dim) = v;
        }
    }
}

// grid (nchunks, ceil(H / (kT / 32)), batch), kT threads: one warp per (chunk, head), lane l holding tokens
// t0 + l and t0 + l + 32: dt = softplus(dt_raw + dt_bias) and the in-chunk inclusive cumulative sum of dt * A
// (a warp scan), stored with consecutive lanes on consecutive tokens.
__global__ void __launch_bounds__(kT) dt_kernel(BwdArgs a, Ws ws) {
    const int lane = threadIdx.x & 31;
    const int64_t h = (int64_t)blockIdx.y * (kT / 32) + (threadIdx.x >> 5);
    if (h >= a.H) return;
    const int64_t b = blockIdx.z, t0 = (int64_t)blockIdx.x * kQ;
    const int64_t t1 = t0 + kQ < a.L ? t0 + kQ : a.L;
    const float Ah = a.A[h], bias = a.dt_bias[h];
    float dt[2], v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int64_t t = t0 + lane + 32 * u;
        dt[u] = t < t1 ? softplus_f(ld_act(a.dt, (b * a.L + t) * a.H + h, a.act_bf16) + bias) : 0.f;
        v[u] = dt[u] * Ah;
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float p0 = __shfl_up_sync(0xffffffffu, v[0], o), p1 = __shfl_up_sync(0xffffffffu, v[1], o);
        if (lane >= o) {
            v[0] += p0;
            v[1] += p1;
        }
    }
    v[1] += __shfl_sync(0xffffffffu, v[0], 31);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int64_t t = t0 + lane + 32 * u;
        if (t < t1) {
            ws.DT[(b * a.H + h) * a.L + t] = dt[u];
            ws.CS[(b * a.H + h) * a.L + t] = v[u];
        }
    }
}

// Register-tiled product of two shared-memory operands, the building block of the chunk kernels:
//   acc[r][c] += sum_{k < K} A(ty + 16 r, k) * B(tx + 16 c, k),
//   A(m, k) = A[m * sam + k * sak],  B(n, k) = B[n * sbn + k * sbk],
// with the kT threads as a 16 x 16 grid (ty = tid / 16, tx = tid % 16).  Each k costs TM + TN
// shared loads for TM * TN FMAs.  Rows and columns are interleaved by 16, so a warp (two ty, all 16
// tx) reads two A addresses and 16 B addresses per k: bank-conflict free when sam is not a multiple
// of 32 and sbn is odd.
template <int TM, int TN>
__device__ __forceinline__ void tile_mma(float (&acc)[TM][TN], const float* A, int sam, int sak, const float* B,
                                         int sbn, int sbk, int K, int ty, int tx) {
    for (int k = 0; k < K; ++k) {
        float av[TM], bv[TN];
#pragma unroll
        for (int r = 0; r < TM; ++r) av[r] = A[(ty + 16 * r) * sam + k * sak];
#pragma unroll
        for (int c = 0; c < TN; ++c) bv[c] = B[(tx + 16 * c) * sbn + k * sbk];
#pragma unroll
        for (int r = 0; r < TM; ++r)
#pragma unroll
            for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
    }
}

// 16-byte shared load (the address must be 16-byte aligned; the host emulation checks it).
__device__ __forceinline__ float4 lds4(const float* p) {
#ifdef SSD_EMU
    emu_check_aligned(p, 16);
#endif
    return *reinterpret_cast<const float4*>(p);
}

__device__ __forceinline__ float f4c(const float4& v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// tile_mma for A and B both contiguous along k (sak = sbk = 1), four k per 16-byte load of each:
// per four k, TM + TN loads (a warp's A loads: two rows, one wavefront; its B loads: 16 rows, two
// wavefronts) for 4 TM TN FMAs.  K a multiple of 4; rows and the bases 16-byte aligned.
template <int TM, int TN>
__device__ __forceinline__ void tile_mma_kk(float (&acc)[TM][TN], const float* A, int sam, const float* B, int sbn,
                                            int K, int ty, int tx) {
    for (int k = 0; k < K; k += 4) {
        float4 av[TM], bv[TN];
#pragma unroll
        for (int r = 0; r < TM; ++r) av[r] = lds4(A + (ty + 16 * r) * sam + k);
#pragma unroll
        for (int c = 0; c < TN; ++c) bv[c] = lds4(B + (tx + 16 * c) * sbn + k);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int r = 0; r < TM; ++r)
#pragma unroll
                for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(f4c(av[r], i), f4c(bv[c], i), acc[r][c]);
    }
}

// tile_mma for A contiguous along k (sak = 1), B any: A four k per 16-byte load, B scalar.
template <int TM, int TN>
__device__ __forceinline__ void tile_mma_ak(float (&acc)[TM][TN], const float* A, int sam, const float* B, int sbn,
                                            int sbk, int K, int ty, int tx) {
    for (int k = 0; k < K; k += 4) {
        float4 av[TM];
#pragma unroll
        for (int r = 0; r < TM; ++r) av[r] = lds4(A + (ty + 16 * r) * sam + k);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float bv[TN];
#pragma unroll
            for (int c = 0; c < TN; ++c) bv[c] = B[(tx + 16 * c) * sbn + (k + i) * sbk];
#pragma unroll
            for (int r = 0; r < TM; ++r)
#pragma unroll
                for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(f4c(av[r], i), bv[c], acc[r][c]);
        }
    }
}

// Column n of a thread's c-th output column in the products whose B runs along n (N-wide results, TN =
// N/16 columns per thread): contiguous groups of four, 4 tx .. 4 tx + 3 within each 64-column block, so
// that the 16 column threads of a warp read 256 contiguous bytes per load (two wavefronts).  TN = 2:
// pairs 2 tx, 2 tx + 1; TN = 1: column tx.
template <int TN>
__device__ __forceinline__ int ncol(int tx, int c) {
    if constexpr (TN >= 4) return 64 * (c / 4) + 4 * tx + (c % 4);
    else if constexpr (TN == 2) return 2 * tx + c;
    else return tx;
}

// The TN values of row k of B (B(n, k) = B[n + k * sbk], n = ncol(tx, c)) in as few loads as the
// layout allows: 16-byte loads for TN >= 4, 8-byte for TN = 2 (sbk a multiple of 4, base 16-byte aligned).
template <int TN>
__device__ __forceinline__ void load_ncols(float (&bv)[TN], const float* Bk, int tx) {
    if constexpr (TN >= 4) {
#pragma unroll
        for (int h = 0; h < TN / 4; ++h) {
            const float4 v = lds4(Bk + 64 * h + 4 * tx);
            bv[4 * h] = v.x;
            bv[4 * h + 1] = v.y;
            bv[4 * h + 2] = v.z;
            bv[4 * h + 3] = v.w;
        }
    } else if constexpr (TN == 2) {
        const float* p = Bk + 2 * tx;
#ifdef SSD_EMU
        emu_check_aligned(p, 8);
#endif
        const float2 v = *reinterpret_cast<const float2*>(p);
        bv[0] = v.x;
        bv[1] = v.y;
    } else {
        bv[0] = Bk[tx];
    }
}

// tile_mma with A contiguous along k (four k per 16-byte load) and B running along n (ncol columns);
// rows 4 ty + r (four contiguous rows per thread: with sam = 68 a warp's two ty read rows 4 apart, 16
// banks apart, one wavefront).
template <int TM, int TN>
__device__ __forceinline__ void tile_mma_ak_nc(float (&acc)[TM][TN], const float* A, int sam, const float* B,
                                               int sbk, int K, int ty, int tx) {
    for (int k = 0; k < K; k += 4) {
        float4 av[TM];
#pragma unroll
        for (int r = 0; r < TM; ++r) av[r] = lds4(A + (TM * ty + r) * sam + k);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float bv[TN];
            load_ncols(bv, B + (k + i) * sbk, tx);
#pragma unroll
            for (int r = 0; r < TM; ++r)
#pragma unroll
                for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(f4c(av[r], i), bv[c], acc[r][c]);
        }
    }
}

// tile_mma for the chunk-state sums: rows m = 4 ty + r (four contiguous rows per thread, A(m, k) =
// A[m + k * sak], one 16-byte load per k; a warp's two ty read 32 contiguous bytes) and B along n
// (ncol columns).  sak a multiple of 4, A 16-byte aligned.
template <int TN>
__device__ __forceinline__ void tile_mma_mc_nc(float (&acc)[4][TN], const float* A, int sak, const float* B,
                                               int sbk, int K, int ty, int tx) {
    for (int k = 0; k < K; ++k) {
        const float4 a4 = lds4(A + 4 * ty + k * sak);
        float bv[TN];
        load_ncols(bv, B + k * sbk, tx);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < TN; ++c) acc[r][c] = fmaf(f4c(a4, r), bv[c], acc[r][c]);
    }
}

template <int TM, int TN>
__device__ __forceinline__ void tile_zero(float (&acc)[TM][TN]) {
#pragma unroll
    for (int r = 0; r < TM; ++r)
#pragma unroll
        for (int c = 0; c < TN; ++c) acc[r][c] = 0.f;
}

// grid (nchunks, H, batch), kT threads.  Chunk-local state and adjoint sums of one head:
//   SP[p][n] = sum_j exp(cs_last - cs_j) dt_j x_j[p] B_j[n],  LM[p][n] = sum_i exp(cs_i) g_i[p] C_i[n].
// Each thread owns rows p = 4 ty + r (r < 4) and columns n = ncol(tx, c) (c < N/16) of both.
template <int N>
__global__ void __launch_bounds__(kT) chunk_state_kernel(BwdArgs a, Ws ws) {
    constexpr int TN = N / 16;
    const int64_t nc = nchunks(a.L), HP = (int64_t)a.H * kP, GN = (int64_t)a.G * N, conv_dim = HP + 2 * GN;
    const int64_t c = blockIdx.x, b = blockIdx.z;
    const int h = blockIdx.y, g = h / (a.H / a.G), tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int64_t t0 = c * kQ;
    const int Qv = static_cast<int>(a.L - t0 < kQ ? a.L - t0 : kQ);

    float* sm = reinterpret_cast<float*>(SSD_DYN_SMEM());
    float* wx = sm;               // [kQ][kP]
    float* wg = wx + kQ * kP;     // [kQ][kP]
    float* Bs = wg + kQ * kP;     // [kQ][N]
    float* Cs = Bs + kQ * N;      // [kQ][N]
    float* fx = Cs + kQ * N;      // [kQ]
    float* fg = fx + kQ;          // [kQ]

    const float* dtp = ws.DT + (b * a.H + h) * a.L + t0;
    const float* csp = ws.CS + (b * a.H + h) * a.L + t0;
    if (tid < kQ) {
        if (tid < Qv) {
            fx[tid] = dtp[tid] * expf(csp[Qv - 1] - csp[tid]);
            fg[tid] = expf(csp[tid]);
        } else {
            fx[tid] = 0.f;
            fg[tid] = 0.f;
        }
    }
    __syncthreads();
    for (int e = tid; e < kQ * kP; e += kT) {
        const int j = e / kP, p = e % kP;
        if (j < Qv) {
            const int64_t row = b * a.L + t0 + j;
            wx[e] = ws.U[row * conv_dim + (int64_t)h * kP + p] * fx[j];
            const int64_t yi = row * HP + (int64_t)h * kP + p;
            wg[e] = ld_act(a.dy, yi, a.dy_bf16) * silu_f(ld_act(a.z, yi, a.act_bf16)) * fg[j];
        } else {
            wx[e] = 0.f;
            wg[e] = 0.f;
        }
    }
    for (int e = tid; e < kQ * N; e += kT) {
        const int j = e / N, n = e % N;
        if (j < Qv) {
            const int64_t row = (b * a.L + t0 + j) * conv_dim;
            Bs[e] = ws.U[row + HP + (int64_t)g * N + n];
            Cs[e] = ws.U[row + HP + GN + (int64_t)g * N + n];
        } else {
            Bs[e] = 0.f;
            Cs[e] = 0.f;
        }
    }
    __syncthreads();
    const int64_t base = ((b * nc + c) * a.H + h) * (int64_t)kP * N;
    float acc[4][TN];
    tile_zero(acc);
    tile_mma_mc_nc(acc, wx, kP, Bs, N, Qv, ty, tx);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < TN; ++q) ws.SP[base + (int64_t)(4 * ty + r) * N + ncol<TN>(tx, q)] = acc[r][q];
    tile_zero(acc);
    tile_mma_mc_nc(acc, wg, kP, Cs, N, Qv, ty, tx);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int q = 0; q < TN; ++q) ws.LM[base + (int64_t)(4 * ty + r) * N + ncol<TN>(tx, q)] = acc[r][q];
}

// Sum of v over the block (kT threads); every thread gets the total.  red: kT floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
    const int tid = threadIdx.x;
    red[tid] = v;
    __syncthreads();
    for (int s = kT / 2; s > 0; s >>= 1) {
        if (tid < s) red[tid] += red[tid + s];
        __syncthreads();
    }
    const float total = red[0];
    __syncthreads();
    return total;
}

// M consecutive floats (16-byte aligned when M is a multiple of 4).
template <int M>
__device__ __forceinline__ void ld_vec(const float* p, float (&v)[M]) {
    if constexpr (M % 4 == 0) {
#pragma unroll
        for (int m = 0; m < M; m += 4) {
            const float4 t = *reinterpret_cast<const float4*>(p + m);
            v[m] = t.x, v[m + 1] = t.y, v[m + 2] = t.z, v[m + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int m = 0; m < M; ++m) v[m] = p[m];
    }
}
template <int M>
__device__ __forceinline__ void st_vec(float* p, const float (&v)[M]) {
    if constexpr (M % 4 == 0) {
#pragma unroll
        for (int m = 0; m < M; m += 4) *reinterpret_cast<float4*>(p + m) = make_float4(v[m], v[m + 1], v[m + 2], v[m + 3]);
    } else {
#pragma unroll
        for (int m = 0; m < M; ++m) p[m] = v[m];
    }
}

#ifndef SSD_EMU
// Writes this thread's M (8 or 4) consecutive elements n0.. of state row p as fp16 into the swizzled tile of one
// (chunk, head) (see Ws::SPH), scaled by the row's power of two s_p <= 1 (the 16 lanes that hold row p agree on
// it), and 1/s_p into the row's scale slot.
template <int M>
__device__ __forceinline__ void store_half_row(const float (&v)[M], int p, int n0, char* tile, float* inv_scale) {
    float mx = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) mx = fmaxf(mx, fabsf(v[m]));
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sc = 1.f;
    if (!(mx < 16384.f)) {
        const int e = min(((__float_as_int(mx) >> 23) & 0xff) - 127, 128);  // mx in [2^e, 2^(e+1))
        sc = __int_as_float((127 + 13 - e) << 23);                           // mx * sc in [2^13, 2^14)
    }
    uint32_t w[M / 2];
#pragma unroll
    for (int m = 0; m < M; m += 2) {
        __half2 hv = __floats2half2_rn(v[m] * sc, v[m + 1] * sc);
        w[m / 2] = *reinterpret_cast<uint32_t*>(&hv);
    }
    const int k8 = n0 >> 3;
    char* dst = tile + (k8 >> 3) * 8192 + p * 128 + (((k8 & 7) ^ (p & 7)) << 4) + ((n0 & 7) ? 8 : 0);
    if constexpr (M == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    if ((threadIdx.x & 15) == 0) inv_scale[p] = 1.f / sc;
}
#endif

#ifndef SSD_EMU
// The M (8 or 4) elements n0.. of row p of one (chunk, head) fp16 tile (see Ws::SPH), unscaled.
template <int M>
__device__ __forceinline__ void load_half_row(const char* tile, const float* inv_scale, int p, int n0, float (&v)[M]) {
    const int k8 = n0 >> 3;
    const char* src = tile + (k8 >> 3) * 8192 + p * 128 + (((k8 & 7) ^ (p & 7)) << 4) + ((n0 & 7) ? 8 : 0);
    uint32_t w[M / 2];
    if constexpr (M == 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(src);
        w[0] = q.x, w[1] = q.y, w[2] = q.z, w[3] = q.w;
    } else {
        const uint2 q = *reinterpret_cast<const uint2*>(src);
        w[0] = q.x, w[1] = q.y;
    }
    const float is = inv_scale[p];
#pragma unroll
    for (int m = 0; m < M; m += 2) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[m / 2]));
        v[m] = f.x * is;
        v[m + 1] = f.y * is;
    }
}
#endif

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr int kWin = 32;  // chunks per window of the state pass (one decay per lane, one F flush)

// Shared memory of the state pass: the per-warp partial F sums of a window, by window parity.
constexpr size_t state_pass_smem() { return 2 * (size_t)kWin * (kT / 32) * sizeof(float); }

// grid (H * kSplit, batch), kT threads: the P*N state elements of a head in kSplit slices of P / kSplit whole
// rows p; a thread holds M = P*N / (kSplit * kT) consecutive elements of one row (16 threads per row).  The
// forward scan turns SP into the states entering each chunk, the reverse scan turns LM into the adjoints
// leaving each chunk and leaves each slice's part of F.  The next chunk's values are loaded before the
// current chunk's are stored, so the loads of consecutive chunks overlap; the chunks' decays are loaded 32 at
// a time (one per lane) and F is reduced per warp, with one block barrier per 32 chunks.  For the
// tensor-core chunk backward (ws.SPH set) the entering states are written only as scaled fp16 tiles, the
// reverse scan takes them from there for F, and the leaving adjoints are written only as such tiles (the fp32
// arrays have no other reader).
template <int N>
__global__ void __launch_bounds__(kT) state_pass_kernel(BwdArgs a, Ws ws) {
    constexpr int M = kP * N / (kSplit * kT);
    constexpr int SLICE = kP * N / kSplit;
    constexpr int NW = kT / 32;
    const int64_t nc = nchunks(a.L), b = blockIdx.y;
    const int h = blockIdx.x / kSplit, sp = blockIdx.x % kSplit, tid = threadIdx.x;
    const int lane = tid & 31, wid = tid >> 5;
    float* fw = reinterpret_cast<float*>(SSD_DYN_SMEM());  // [2][kWin][NW]
    const int64_t off = (int64_t)sp * SLICE + (int64_t)tid * M;  // this thread's first element in a P x N block
    const int64_t head = (b * a.H + h) * (int64_t)kP * N + off;
    const int prow = static_cast<int>(off / N), n0 = static_cast<int>(off % N);
    const float* csh = ws.CS + (b * a.H + h) * a.L;
#ifndef SSD_EMU
    const bool half_tiles = (M == 4 || M == 8) && ws.SPH != nullptr;
#else
    const bool half_tiles = false;
#endif
    auto blk = [&](int64_t c) { return ((b * nc + c) * a.H + h) * (int64_t)kP * N; };
    // exp(cs at the last token) of chunk w * kWin + lane, for the window w
    auto window_decays = [&](int64_t w) {
        const int64_t c = w * kWin + lane;
        float d = 0.f;
        if (c < nc) {
            const int64_t last = (c * kQ + kQ - 1 < a.L ? c * kQ + kQ - 1 : a.L - 1);
            d = expf(csh[last]);
        }
        return d;
    };

    float s[M], cur[M], nxt[M];
#pragma unroll
    for (int m = 0; m < M; ++m) s[m] = cur[m] = nxt[m] = 0.f;
    if (a.init_state) ld_vec<M>(a.init_state + head, s);
    if (nc > 0) ld_vec<M>(ws.SP + blk(0) + off, cur);
    float dwin = 0.f;
    for (int64_t c = 0; c < nc; ++c) {
        if ((c % kWin) == 0) dwin = window_decays(c / kWin);
        const float decay = __shfl_sync(0xffffffffu, dwin, static_cast<int>(c % kWin));
        if (c + 1 < nc) ld_vec<M>(ws.SP + blk(c + 1) + off, nxt);
        if (!half_tiles) st_vec<M>(ws.SP + blk(c) + off, s);
#ifndef SSD_EMU
        if constexpr (M == 4 || M == 8) {
            if (half_tiles)
                store_half_row<M>(s, prow, n0, reinterpret_cast<char*>(ws.SPH) + blk(c) * 2,
                                  ws.SPS + ((b * nc + c) * a.H + h) * kP);
        }
#endif
#pragma unroll
        for (int m = 0; m < M; ++m) {
            s[m] = decay * s[m] + cur[m];
            cur[m] = nxt[m];
        }
    }

    // reverse: the adjoints leaving each chunk, and F = decay <Lm, Sp> per chunk (this slice's part)
    float l[M], lcur[M], lnxt[M], scur[M], snxt[M];
#pragma unroll
    for (int m = 0; m < M; ++m) l[m] = lcur[m] = lnxt[m] = scur[m] = snxt[m] = 0.f;
    if (a.d_final) ld_vec<M>(a.d_final + head, l);
    // the state entering chunk c: the fp32 array, or the fp16 tile and its row scale
    auto load_sp = [&](int64_t c, float (&v)[M]) {
#ifndef SSD_EMU
        if constexpr (M == 4 || M == 8) {
            if (half_tiles) {
                load_half_row<M>(reinterpret_cast<const char*>(ws.SPH) + blk(c) * 2,
                                 ws.SPS + ((b * nc + c) * a.H + h) * kP, prow, n0, v);
                return;
            }
        }
#endif
        ld_vec<M>(ws.SP + blk(c) + off, v);
    };
    if (nc > 0) {
        ld_vec<M>(ws.LM + blk(nc - 1) + off, lcur);
        load_sp(nc - 1, scur);
    }
    for (int64_t c = nc - 1; c >= 0; --c) {
        const int64_t w = c / kWin;
        const int ci = static_cast<int>(c % kWin);
        if (c == nc - 1 || ci == kWin - 1) dwin = window_decays(w);
        const float decay = __shfl_sync(0xffffffffu, dwin, ci);
        if (c > 0) {
            ld_vec<M>(ws.LM + blk(c - 1) + off, lnxt);
            load_sp(c - 1, snxt);
        }
#ifndef SSD_EMU
        if constexpr (M == 4 || M == 8) {
            if (half_tiles)
                store_half_row<M>(l, prow, n0, reinterpret_cast<char*>(ws.LMH) + blk(c) * 2,
                                  ws.LMS + ((b * nc + c) * a.H + h) * kP);
            else
                st_vec<M>(ws.LM + blk(c) + off, l);
        } else {
            st_vec<M>(ws.LM + blk(c) + off, l);
        }
#else
        st_vec<M>(ws.LM + blk(c) + off, l);
#endif
        float f = 0.f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            f += l[m] * scur[m];
            l[m] = decay * l[m] + lcur[m];
            lcur[m] = lnxt[m];
            scur[m] = snxt[m];
        }
        f = warp_sum_f(f);
        if (lane == 0) fw[((w & 1) * kWin + ci) * NW + wid] = f;
        if (ci == 0) {
            // the window is done: its chunks' F, the warps' sums in a fixed order, times the chunk's decay
            // (lane t of every warp holds chunk w * kWin + t's)
            __syncthreads();
            if (tid < kWin && w * kWin + tid < nc) {
                float t = 0.f;
#pragma unroll
                for (int q = 0; q < NW; ++q) t += fw[((w & 1) * kWin + tid) * NW + q];
                ws.PF[((b * nc + w * kWin + tid) * a.H + h) * kSplit + sp] = dwin * t;
            }
        }
    }
    if (a.d_init_state) st_vec<M>(a.d_init_state + head, l);
}

template <int N>
constexpr size_t chunk_bwd_floats() {
    // Bs, Cs [kQ][N+4]; CB, LCB, LGX, xs, gs [kQ][kS]; Tm [kQ][kTS] (+3 to keep 16-byte alignment);
    // X [kP][N+4]; red [kQ][17] (+4); 7 vectors of kQ; 3 x kT block sums
    return 2 * (size_t)kQ * (N + 4) + 5 * (size_t)kQ * kS + ((size_t)kQ * kTS + 3) / 4 * 4 + (size_t)kP * (N + 4) +
           ((size_t)kQ * 17 + 3) / 4 * 4 + 7 * (size_t)kQ + 3 * (size_t)kT;
}

// grid (nchunks, G, batch), kT threads.  One chunk of one group; the group's heads in turn.  The
// contractions are register-tiled shared-memory products (tile_mma): a thread owns rows ty + 16 r and
// columns tx + 16 c of every 64-row result, and of the group's dB / dC, which stay in registers across
// the heads.  The causal (triangular) sums run over the whole chunk: the operands are zero above the
// diagonal.
template <int N>
__global__ void __launch_bounds__(kT, 1) chunk_bwd_kernel(BwdArgs a, Ws ws) {
    constexpr int NS = N + 4;      // row stride of the N-wide tiles (16-byte rows)
    constexpr int TN = N / 16;     // columns per thread of the N-wide results
    constexpr int RS = 17;         // row stride of the per-row partial sums
    const int64_t nc = nchunks(a.L), HP = (int64_t)a.H * kP, GN = (int64_t)a.G * N, conv_dim = HP + 2 * GN;
    const int64_t c = blockIdx.x, b = blockIdx.z, t0 = c * kQ;
    const int hpg = a.H / a.G, split = head_split(a.H, a.G), tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int g = blockIdx.y / split, half = blockIdx.y % split;
    const int hl0 = half * hpg / split, hl1 = (half + 1) * hpg / split;  // this CTA's heads of the group
    const int Qv = static_cast<int>(a.L - t0 < kQ ? a.L - t0 : kQ);
    // causal sums over the chunk's rows, rounded up to whole 16-byte loads: the operands are zero past Qv
    const int Q4 = (Qv + 3) & ~3;

    float* sm = reinterpret_cast<float*>(SSD_DYN_SMEM());
    float* Bs = sm;                  // [kQ][NS]  post-conv B of the group
    float* Cs = Bs + kQ * NS;        // [kQ][NS]
    float* CB = Cs + kQ * NS;        // [kQ][kS]  C_i . B_j
    float* LCB = CB + kQ * kS;       // [kQ][kS]  L_ij dt_j C_i . B_j         (i >= j, else 0)
    float* LGX = LCB + kQ * kS;      // [kQ][kS]  L_ij g_i . x_j, then times dt_j (i >= j, else 0)
    float* xs = LGX + kQ * kS;       // [kQ][kS]  post-conv x of the head
    float* gs = xs + kQ * kS;        // [kQ][kS]  g = dy * silu(z)
    float* X = gs + kQ * kS;         // [kP][NS]  Sp, then Lm
    float* Tm = X + kP * NS;         // [kQ][kTS] row prefix sums of M
    float* red = Tm + (kQ * kTS + 3) / 4 * 4;    // [kQ][RS]  per-row partial sums over the 16 column threads
    float* dts = red + (kQ * RS + 3) / 4 * 4;    // [kQ]
    float* css = dts + kQ;
    float* ex = css + kQ;            // exp(cs_i)
    float* el = ex + kQ;             // exp(cs_last - cs_j)
    float* Ev = el + kQ;             // exp(cs_i) g_i . (Sp C_i)
    float* Wv = Ev + kQ;             // exp(cs_last - cs_j) x_j . (Lm B_j)
    float* Dr = Wv + kQ;             // ddt without the decay term
    float* bsum = Dr + kQ;           // [3][kT]

    // the group's post-conv B and C, and C_i . B_j
    for (int e = tid; e < kQ * N; e += kT) {
        const int j = e / N, n = e % N;
        float bv = 0.f, cv = 0.f;
        if (j < Qv) {
            const int64_t row = (b * a.L + t0 + j) * conv_dim;
            bv = ws.U[row + HP + (int64_t)g * N + n];
            cv = ws.U[row + HP + GN + (int64_t)g * N + n];
        }
        Bs[j * NS + n] = bv;
        Cs[j * NS + n] = cv;
    }
    __syncthreads();
    {
        float acc[4][4];
        tile_zero(acc);
        tile_mma_kk(acc, Cs, NS, Bs, NS, N, ty, tx);
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int q = 0; q < 4; ++q) CB[(ty + 16 * r) * kS + tx + 16 * q] = acc[r][q];
    }

    float dBa[4][TN], dCa[4][TN];  // rows j (or i) = 4 ty + r, columns n = ncol(tx, c)
    tile_zero(dBa);
    tile_zero(dCa);

    for (int hl = hl0; hl < hl1; ++hl) {
        const int h = g * hpg + hl;
        const float Dh = a.D[h], Ah = a.A[h], bias = a.dt_bias[h];
        const int64_t hrow = (b * a.H + h) * a.L + t0;
        const int64_t sbase = ((b * nc + c) * a.H + h) * (int64_t)kP * N;

        // 1: dt, cs, x and g of the head
        if (tid < kQ) {
            dts[tid] = tid < Qv ? ws.DT[hrow + tid] : 0.f;
            css[tid] = tid < Qv ? ws.CS[hrow + tid] : 0.f;
        }
        for (int e = tid; e < kQ * kP; e += kT) {
            const int j = e / kP, p = e % kP;
            float xv = 0.f, gv = 0.f;
            if (j < Qv) {
                const int64_t row = b * a.L + t0 + j;
                xv = ws.U[row * conv_dim + (int64_t)h * kP + p];
                const int64_t yi = row * HP + (int64_t)h * kP + p;
                gv = ld_act(a.dy, yi, a.dy_bf16) * silu_f(ld_act(a.z, yi, a.act_bf16));
            }
            xs[j * kS + p] = xv;
            gs[j * kS + p] = gv;
        }
        __syncthreads();

        // 2: decay factors; L-weighted g.x (LGX, without dt for now) and dt-weighted C.B (LCB); Sp
        const float cl = css[Qv - 1];
        if (tid < kQ) {
            ex[tid] = tid < Qv ? expf(css[tid]) : 0.f;
            el[tid] = tid < Qv ? expf(cl - css[tid]) : 0.f;
        }
        {
            float acc[4][4];
            tile_zero(acc);
            tile_mma_kk(acc, gs, kS, xs, kS, kP, ty, tx);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = ty + 16 * r, j = tx + 16 * q;
                    float lgx = 0.f, lcb = 0.f;
                    if (j <= i && i < Qv) {
                        const float Lij = expf(css[i] - css[j]);
                        lgx = acc[r][q] * Lij;
                        lcb = CB[i * kS + j] * Lij * dts[j];
                    }
                    LGX[i * kS + j] = lgx;
                    LCB[i * kS + j] = lcb;
                }
        }
        for (int e = tid; e < kP * N; e += kT) X[(e / N) * NS + e % N] = ws.SP[sbase + e];
        __syncthreads();

        // 3: y recomputed for dz (Sp C_i and the intra-chunk sum), E_i, dC_i += exp(cs_i) g_i Sp;
        //    the direct part of ddt from the pairs (before LGX takes dt)
        if (tid < kQ) {
            float dr = 0.f;
            for (int i = tid; i < Qv; ++i) dr += LGX[i * kS + tid] * CB[i * kS + tid];
            Dr[tid] = dr;
        }
        float pD = 0.f;
        {
            float spc[4][4], yin[4][4];
            tile_zero(spc);
            tile_zero(yin);
            tile_mma_kk(spc, Cs, NS, X, NS, N, ty, tx);            // [i][p] = sum_n C_i[n] Sp[p][n]
            tile_mma_ak(yin, LCB, kS, xs, 1, kS, Q4, ty, tx);      // [i][p] = sum_j LCB[i][j] x_j[p]
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = ty + 16 * r;
                float epart = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int p = tx + 16 * q;
                    const float gv = gs[i * kS + p], xv = xs[i * kS + p];
                    epart += gv * spc[r][q];
                    pD += gv * xv;
                    if (i < Qv) {
                        const float yv = yin[r][q] + ex[i] * spc[r][q] + Dh * xv;
                        const int64_t yi = (b * a.L + t0 + i) * HP + (int64_t)h * kP + p;
                        a.dz[yi] = ld_act(a.dy, yi, a.dy_bf16) * yv * dsilu_f(ld_act(a.z, yi, a.act_bf16));
                    }
                }
                red[i * RS + tx] = epart;
            }
        }
        {
            float acc[4][TN];
            tile_zero(acc);
            tile_mma_ak_nc(acc, gs, kS, X, NS, kP, ty, tx);        // [i][n] = sum_p g_i[p] Sp[p][n]
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < TN; ++q) dCa[r][q] += ex[4 * ty + r] * acc[r][q];
        }
        __syncthreads();

        // 4: E_i; LGX takes dt_j; the leaving adjoint Lm
        if (tid < kQ) {
            float e = 0.f;
            for (int k = 0; k < 16; ++k) e += red[tid * RS + k];
            Ev[tid] = ex[tid] * e;
        }
        for (int e = tid; e < kQ * kQ; e += kT) LGX[(e / kQ) * kS + e % kQ] *= dts[e % kQ];
        for (int e = tid; e < kP * N; e += kT) X[(e / N) * NS + e % N] = ws.LM[sbase + e];
        __syncthreads();

        // 5: dx (Lm B_j and the intra-chunk sum), W_j; dB_j += dt_j exp(cs_last - cs_j) x_j Lm and the
        //    intra-chunk parts of dB and dC
        {
            float lmb[4][4], dxi[4][4];
            tile_zero(lmb);
            tile_zero(dxi);
            tile_mma_kk(lmb, Bs, NS, X, NS, N, ty, tx);            // [j][p] = sum_n B_j[n] Lm[p][n]
            tile_mma(dxi, LCB, 1, kS, gs, 1, kS, Qv, ty, tx);    // [j][p] = sum_i LCB[i][j] g_i[p]
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = ty + 16 * r;
                float wpart = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int p = tx + 16 * q;
                    wpart += xs[j * kS + p] * lmb[r][q];
                    if (j < Qv) {
                        const float d = dxi[r][q] + dts[j] * el[j] * lmb[r][q] + Dh * gs[j * kS + p];
                        ws.DU[(b * a.L + t0 + j) * conv_dim + (int64_t)h * kP + p] = d;
                    }
                }
                red[j * RS + tx] = wpart;
            }
        }
        {
            float acc[4][TN];
            tile_zero(acc);
            tile_mma_ak_nc(acc, xs, kS, X, NS, kP, ty, tx);        // [j][n] = sum_p x_j[p] Lm[p][n]
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = 4 * ty + r;
#pragma unroll
                for (int q = 0; q < TN; ++q) dBa[r][q] += dts[j] * el[j] * acc[r][q];
            }
            tile_zero(acc);
            tile_mma_mc_nc(acc, LGX, kS, Cs, NS, Qv, ty, tx);      // [j][n] = sum_i LGX[i][j] dt_j C_i[n]
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < TN; ++q) dBa[r][q] += acc[r][q];
            tile_zero(acc);
            tile_mma_ak_nc(acc, LGX, kS, Bs, NS, Q4, ty, tx);      // [i][n] = sum_j LGX[i][j] dt_j B_j[n]
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int q = 0; q < TN; ++q) dCa[r][q] += acc[r][q];
        }
        __syncthreads();

        // 6: W_j and the rest of the direct part of ddt; row prefix sums of M_ij = LGX[i][j] C_i . B_j
        if (tid < kQ) {
            float w = 0.f;
            for (int k = 0; k < 16; ++k) w += red[tid * RS + k];
            w *= el[tid];
            Wv[tid] = w;
            Dr[tid] += w;
            float run = 0.f;
            for (int k = 0; k <= tid; ++k) {
                Tm[tid * kTS + k] = run;
                run += LGX[tid * kS + k] * CB[tid * kS + k];
            }
        }
        __syncthreads();

        // 7: d(dA_k) = sum_{i>=k} sum_{j<k} M_ij + sum_{i>=k} E_i + F + sum_{j<k} dt_j W_j; ddt; partials
        float F = 0.f;
#pragma unroll
        for (int k = 0; k < kSplit; ++k) F += ws.PF[((b * nc + c) * a.H + h) * kSplit + k];
        float pdA = 0.f, pbias = 0.f;
        if (tid < Qv) {
            const int k = tid;
            float R = 0.f, Es = 0.f, Wsum = 0.f;
            for (int i = k; i < Qv; ++i) {
                R += Tm[i * kTS + k];
                Es += Ev[i];
            }
            for (int j = 0; j < k; ++j) Wsum += dts[j] * Wv[j];
            const float dda = R + Es + F + Wsum;
            const float ddt = Dr[k] + Ah * dda;
            const int64_t di = (b * a.L + t0 + k) * a.H + h;
            const float dr = ddt * sigmoid_f(ld_act(a.dt, di, a.act_bf16) + bias);
            a.ddt[di] = dr;
            pdA = dts[k] * dda;
            pbias = dr;
        }
        const float sA = block_sum(pdA, bsum), sD = block_sum(pD, bsum + kT), sB = block_sum(pbias, bsum + 2 * kT);
        if (tid == 0) {
            float* ph = ws.PH + ((b * nc + c) * a.H + h) * 3;
            ph[0] = sA;
            ph[1] = sD;
            ph[2] = sB;
        }
        __syncthreads();
    }

    // this half's dB | dC: the first half into the B/C part of DU, the second into DU2; the conv
    // backward adds the two in that order
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int j = 4 * ty + r;
        if (j < Qv) {
            float* dst = half == 0 ? ws.DU + (b * a.L + t0 + j) * conv_dim + HP
                                   : ws.DU2 + (b * a.L + t0 + j) * 2 * GN;
#pragma unroll
            for (int q = 0; q < TN; ++q) {
                dst[(int64_t)g * N + ncol<TN>(tx, q)] = dBa[r][q];
                dst[GN + (int64_t)g * N + ncol<TN>(tx, q)] = dCa[r][q];
            }
        }
    }
}

// The pre-conv array holding channel c (x, B or C), offset to c's column, and its row stride.
template <typename T>
__device__ __forceinline__ const T* raw_col(const BwdArgs& a, int c, int HP, int GN, int& rs) {
    rs = c < HP ? HP : GN;
    if (c < HP) return static_cast<const T*>(a.x) + c;
    if (c < HP + GN) return static_cast<const T*>(a.B) + (c - HP);
    return static_cast<const T*>(a.C) + (c - HP - GN);
}

// Channels c, c + 1 of a staged row (c even): one 32-bit (bf16) or 64-bit (fp32) shared load.
__device__ __forceinline__ float2 pair_at(const unsigned short* row, int c) { return act_pair(row + c); }
__device__ __forceinline__ float2 pair_at(const float* row, int c) { return *reinterpret_cast<const float2*>(row + c); }
__device__ __forceinline__ float2 dsilu_fast2(float2 v) { return make_float2(dsilu_fast(v.x), dsilu_fast(v.y)); }

// grid (ceil(conv_dim / kCB), ntiles, batch), kT threads, conv_bwd_smem(sizeof(T)) bytes of dynamic shared memory.
// With v_t the pre-SiLU conv output, dv_t = du_t silu'(v_t), and the pre-conv gradient of token s is
// w0 dv_{s+3} + w1 dv_{s+2} + w2 dv_{s+1} + w3 dv_s.  The CTA first stages the pre-conv values of tokens
// tb - 3 .. tb + kCT + 2 (tb the tile's first token; the conv history, or zero, before token 0) and du (plus
// the second half's dB | dC) of tokens tb .. tb + kCT + 2, zero past the sequence.  Then thread (pair pr,
// sub-tile) computes dv of its kBST tokens once (the last sub-tile also the 3 tokens after the tile), in place
// of du, with its share of the tile's conv_w / conv_b partials; and, after a barrier, the kBST gradients from
// dv of its tokens and the 3 after.  The partials are summed over the sub-tiles in their order.
// HP = 64 H and GN = G N (N a multiple of 16) are multiples of 8, so a 16-byte chunk of a row never straddles
// x / B / C or conv_dim, every chunk is 16-byte aligned (the entry point rejects unaligned arrays), and a
// channel pair never straddles an array.  kBf16 = a.act_bf16, kHist = (a.init_conv_state != null).
template <bool kBf16, bool kHist>
__global__ void __launch_bounds__(kT) conv_bwd_kernel(BwdArgs a, Ws ws) {
    using T = typename std::conditional<kBf16, unsigned short, float>::type;
    constexpr int kE = 16 / sizeof(T);  // elements per 16-byte chunk
    unsigned char* smem = SSD_DYN_SMEM();
    T* raw_s = reinterpret_cast<T*>(smem);                                               // [kRawRows][kCB]
    float* du_s = reinterpret_cast<float*>(smem + (size_t)kRawRows * kCB * sizeof(T));  // [kDuRows][kCB]: du, then dv
    float* du2_s = du_s + kDuRows * kCB;                                        // [kDuRows][kCB]
    float* part = du2_s + kDuRows * kCB;                                        // [kBSUB][5][kCB]
    const int HP = a.H * a.P, GN = a.G * a.N, conv_dim = HP + 2 * GN, L = static_cast<int>(a.L);
    const int tid = threadIdx.x, c0 = blockIdx.x * kCB, b = blockIdx.z, tile = blockIdx.y, tb = tile * kCT;
    const int64_t row0 = (int64_t)b * L;
    const bool add2 = head_split(a.H, a.G) == 2 && c0 + kCB > HP;  // the second half's dB | dC apply here
    for (int e = tid; e < kRawRows * (kCB / kE); e += kT) {
        const int i = e / (kCB / kE), c = c0 + (e - i * (kCB / kE)) * kE, s = tb - 3 + i;
        if (s < 0) continue;  // history rows: below
        const bool ok = s < L && c < conv_dim;
        int rs = 0;
        const T* g = ok ? raw_col<T>(a, c, HP, GN, rs) : static_cast<const T*>(a.x);
        cp_async16(raw_s + i * kCB + (c - c0), ok ? g + (row0 + s) * rs : g, ok ? 16 : 0);
    }
    for (int e = tid; e < kDuRows * (kCB / 4); e += kT) {
        const int i = e / (kCB / 4), c = c0 + (e - i * (kCB / 4)) * 4, t = tb + i;
        const bool ok = t < L && c < conv_dim;
        cp_async16(du_s + i * kCB + (c - c0), ok ? ws.DU + (row0 + t) * conv_dim + c : ws.DU, ok ? 16 : 0);
        if (add2) {
            const bool ok2 = ok && c >= HP;
            cp_async16(du2_s + i * kCB + (c - c0), ok2 ? ws.DU2 + (row0 + t) * 2 * GN + (c - HP) : ws.DU, ok2 ? 16 : 0);
        }
    }
    if (tb == 0) {
        // tokens -3 .. -1: the conv history (layout [batch][conv_dim][3]) or zero
        for (int e = tid; e < 3 * kCB; e += kT) {
            const int i = e / kCB, c = c0 + (e - i * kCB);
            T v = 0;
            if (kHist && c < conv_dim) v = static_cast<const T*>(a.init_conv_state)[((int64_t)b * conv_dim + c) * 3 + i];
            raw_s[i * kCB + (c - c0)] = v;
        }
    }
    cp_async_wait_all();
    __syncthreads();

    const int pr = tid % kBPairs, sub = tid / kBPairs;  // sub is the warp: every branch on it is uniform
    const int lcp = 2 * pr, c = c0 + lcp, i0 = sub * kBST;  // channels c, c + 1; rows i0 .. of the tile
    const bool live = c < conv_dim;  // conv_dim is even: both channels of the pair or neither
    const int cc = live ? c : 0;
    float2 w[4], bias;
    {
        const float4 wa = *reinterpret_cast<const float4*>(a.conv_w + (size_t)cc * 4);
        const float4 wb = *reinterpret_cast<const float4*>(a.conv_w + (size_t)cc * 4 + 4);
        w[0] = make_float2(wa.x, wb.x), w[1] = make_float2(wa.y, wb.y);
        w[2] = make_float2(wa.z, wb.z), w[3] = make_float2(wa.w, wb.w);
        bias = make_float2(a.conv_b[cc], a.conv_b[cc + 1]);
    }
    // pass 1: dv of tokens tb + i0 .. (kBST of them; kBST + 3 for the last sub-tile), from the pre-conv rows
    // i0 .. i0 + n1 + 2 (staged row k holds token tb - 3 + k)
    constexpr int kN1 = kBST + 3;
    const int n1 = sub == kBSUB - 1 ? kN1 : kBST;
    const bool second = add2 && c >= HP;
    // a sliding window over the staged rows: r0..r2 the three before token tb + i0 + k, r3 its own
    float2 r0 = pair_at(raw_s + i0 * kCB, lcp), r1 = pair_at(raw_s + (i0 + 1) * kCB, lcp),
           r2 = pair_at(raw_s + (i0 + 2) * kCB, lcp);
    float2 g[5];
#pragma unroll
    for (int k = 0; k < 5; ++k) g[k] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kN1; ++k) {
        if (k < n1) {
            const int i = i0 + k, t = tb + i;
            const float2 r3 = pair_at(raw_s + (i + 3) * kCB, lcp);
            float2 v = __ffma2_rn(w[0], r0, bias);
            v = __ffma2_rn(w[1], r1, v);
            v = __ffma2_rn(w[2], r2, v);
            v = __ffma2_rn(w[3], r3, v);
            float2* dup = reinterpret_cast<float2*>(du_s + i * kCB + lcp);
            float2 du = *dup;
            if (second) du = __fadd2_rn(du, *reinterpret_cast<const float2*>(du2_s + i * kCB + lcp));
            const float2 dv = t < L ? __fmul2_rn(du, dsilu_fast2(v)) : make_float2(0.f, 0.f);
            *dup = dv;
            if (i < kCT) {  // the tile's own tokens (dv is zero past the sequence)
                g[0] = __ffma2_rn(dv, r0, g[0]);
                g[1] = __ffma2_rn(dv, r1, g[1]);
                g[2] = __ffma2_rn(dv, r2, g[2]);
                g[3] = __ffma2_rn(dv, r3, g[3]);
                g[4] = __fadd2_rn(dv, g[4]);
            }
            r0 = r1;
            r1 = r2;
            r2 = r3;
        }
    }
#pragma unroll
    for (int k = 0; k < 5; ++k) *reinterpret_cast<float2*>(part + (sub * 5 + k) * kCB + lcp) = g[k];
    __syncthreads();
    // pass 2: the gradients of tokens tb + i0 .. tb + i0 + kBST - 1 from dv of rows i0 .. i0 + kBST + 2
    if (live) {
        const auto dv_at = [&](int k) { return *reinterpret_cast<const float2*>(du_s + (i0 + k) * kCB + lcp); };
        const int rs = cc < HP ? HP : GN;
        float* out = cc < HP ? a.dx + cc : (cc < HP + GN ? a.dB + (cc - HP) : a.dC + (cc - HP - GN));
        out += (row0 + tb + i0) * rs;
        const int n = L - tb - i0;  // tokens of the sub-tile that exist (may be <= 0)
        // a sliding window: d0..d3 = dv of tokens j .. j + 3 of the sub-tile
        float2 d0 = dv_at(0), d1 = dv_at(1), d2 = dv_at(2);
        const float2 e0 = d0, e1 = d1, e2 = d2;  // for the conv history below
#pragma unroll
        for (int j = 0; j < kBST; ++j) {
            const float2 d3 = dv_at(j + 3);
            float2 o = __fmul2_rn(w[0], d3);
            o = __ffma2_rn(w[1], d2, o);
            o = __ffma2_rn(w[2], d1, o);
            o = __ffma2_rn(w[3], d0, o);
            if (j < n) *reinterpret_cast<float2*>(out + j * rs) = o;
            d0 = d1;
            d1 = d2;
            d2 = d3;
        }
        if (tb + i0 == 0 && a.d_init_conv_state) {
            // the history tokens s = -3, -2, -1 of channels c, c + 1 (dv is zero before token 0)
            float* dh = a.d_init_conv_state + ((int64_t)b * conv_dim + cc) * 3;
            const float2 h0 = __fmul2_rn(w[0], e0);
            const float2 h1 = __ffma2_rn(w[1], e0, __fmul2_rn(w[0], e1));
            const float2 h2 = __ffma2_rn(w[2], e0, __ffma2_rn(w[1], e1, __fmul2_rn(w[0], e2)));
            dh[0] = h0.x, dh[1] = h1.x, dh[2] = h2.x;
            dh[3] = h0.y, dh[4] = h1.y, dh[5] = h2.y;
        }
    }
    if (tid < kCB && c0 + tid < conv_dim) {
        float* pw = ws.PW + (((int64_t)b * ntiles(a.L) + tile) * conv_dim + c0 + tid) * 5;
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            float v = part[k * kCB + tid];
#pragma unroll
            for (int q = 1; q < kBSUB; ++q) v += part[(5 * q + k) * kCB + tid];
            pw[k] = v;
        }
    }
}

// grid (ceil(conv_dim / 32) + ceil(H / 32)), kT threads: 32 channels (or heads) per CTA, each summed by
// 8 threads over the tiles (chunks) t = j, j + 8, ... of every sequence, then the 8 partials in a fixed order
// -> dconv_w, dconv_b per channel; dA, dD, ddt_bias per head (deterministic).
__global__ void __launch_bounds__(kT) reduce_kernel(BwdArgs a, Ws ws) {
    constexpr int NJ = kT / 32;
    float(*part)[NJ][32] = reinterpret_cast<float(*)[NJ][32]>(SSD_DYN_SMEM());  // [5][NJ][32]
    const int64_t conv_dim = (int64_t)a.H * a.P + 2LL * a.G * a.N, nc = nchunks(a.L), nt = ntiles(a.L);
    const int64_t cblocks = (conv_dim + 31) / 32;
    const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
    const bool heads = blockIdx.x >= cblocks;
    const int64_t idx = (heads ? blockIdx.x - cblocks : blockIdx.x) * 32 + lane;
    const int K = heads ? 3 : 5;
    const int64_t limit = heads ? a.H : conv_dim;
    float s[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    if (idx < limit) {
        for (int64_t b = 0; b < a.batch; ++b) {
            if (heads) {
                for (int64_t c = j; c < nc; c += NJ) {
                    const float* ph = ws.PH + ((b * nc + c) * a.H + idx) * 3;
                    for (int k = 0; k < 3; ++k) s[k] += ph[k];
                }
            } else {
                for (int64_t t = j; t < nt; t += NJ) {
                    const float* pw = ws.PW + ((b * nt + t) * conv_dim + idx) * 5;
                    for (int k = 0; k < 5; ++k) s[k] += pw[k];
                }
            }
        }
    }
    for (int k = 0; k < 5; ++k) part[k][j][lane] = s[k];
    __syncthreads();
    if (j == 0 && idx < limit) {
        float t[5];
        for (int k = 0; k < K; ++k) {
            t[k] = 0.f;
            for (int q = 0; q < NJ; ++q) t[k] += part[k][q][lane];
        }
        if (heads) {
            a.dA[idx] = t[0];
            a.dD[idx] = t[1];
            a.ddt_bias[idx] = t[2];
        } else {
            for (int k = 0; k < 4; ++k) a.dconv_w[idx * 4 + k] = t[k];
            a.dconv_b[idx] = t[4];
        }
    }
}

// grid ceil(batch * H * P * N / kT): d_init_state = d_final when there are no tokens.
__global__ void __launch_bounds__(kT) copy_adjoint_kernel(BwdArgs a) {
    const int64_t n = a.batch * a.H * (int64_t)a.P * a.N;
    const int64_t i = (int64_t)blockIdx.x * kT + threadIdx.x;
    if (i < n) a.d_init_state[i] = a.d_final ? a.d_final[i] : 0.f;
}

template <int N>
cudaError_t launch_n(const BwdArgs& a, const Ws& ws, cudaStream_t st) {
    const int64_t conv_dim = (int64_t)a.H * a.P + 2LL * a.G * a.N, nc = nchunks(a.L), nt = ntiles(a.L);
    const unsigned cgrid = static_cast<unsigned>((conv_dim + 2 * kPC - 1) / (2 * kPC));  // post-conv channel pairs
    cudaError_t err;
    if (a.batch > 0 && nc > 0) {
        const size_t state_smem = (2 * (size_t)kQ * kP + 2 * (size_t)kQ * N + 2 * kQ) * sizeof(float);
        const size_t chunk_smem = chunk_bwd_floats<N>() * sizeof(float);
        if ((err = SSD_SET_SMEM(chunk_state_kernel<N>, state_smem)) != cudaSuccess) return err;
        if ((err = SSD_SET_SMEM(chunk_bwd_kernel<N>, chunk_smem)) != cudaSuccess) return err;
        const dim3 tiles(cgrid, static_cast<unsigned>(ntiles(a.L)), static_cast<unsigned>(a.batch));
        const bool hist = a.init_conv_state != nullptr;
        void (*post_conv)(BwdArgs, Ws) = a.act_bf16 ? (hist ? post_conv_kernel<true, true> : post_conv_kernel<true, false>)
                                                    : (hist ? post_conv_kernel<false, true> : post_conv_kernel<false, false>);
        SSD_LAUNCH(post_conv, tiles, dim3(kT), 0, st, a, ws);
        SSD_LAUNCH(dt_kernel,
                   dim3(static_cast<unsigned>(nc), static_cast<unsigned>((a.H + kT / 32 - 1) / (kT / 32)),
                        static_cast<unsigned>(a.batch)),
                   dim3(kT), 0, st, a, ws);
        const dim3 chunk_heads(static_cast<unsigned>(nc), static_cast<unsigned>(a.H), static_cast<unsigned>(a.batch));
        Ws wsp = ws;  // the state pass writes the fp16 state tiles only for the tensor-core chunk backward
#ifndef SSD_EMU
        const bool tc_chunk = chunk_bwd_tc_supported(a.P, N, a.act_bf16, a.dy, a.z, a.dz);
#else
        const bool tc_chunk = false;
#endif
        if (!tc_chunk) wsp.SPH = wsp.LMH = wsp.SPS = wsp.LMS = nullptr;
#ifndef SSD_EMU
        if (chunk_state_tc_supported(a.P, N, a.act_bf16)) {
            ChunkStateTcArgs t{a.batch, a.L, a.H, a.G, N, a.act_bf16, a.dy_bf16, ws.U, ws.DT, ws.CS, a.dy, a.z,
                               ws.SP, ws.LM};
            if ((err = launch_chunk_state_tc(t, nc, st)) != cudaSuccess) return err;
        } else {
            SSD_LAUNCH(chunk_state_kernel<N>, chunk_heads, dim3(kT), state_smem, st, a, ws);
        }
#else
        SSD_LAUNCH(chunk_state_kernel<N>, chunk_heads, dim3(kT), state_smem, st, a, ws);
#endif
        SSD_LAUNCH(state_pass_kernel<N>, dim3(static_cast<unsigned>(a.H * kSplit), static_cast<unsigned>(a.batch)),
                   dim3(kT), state_pass_smem(), st, a, wsp);
        const dim3 chunk_groups(static_cast<unsigned>(nc), static_cast<unsigned>(a.G * head_split(a.H, a.G)),
                                static_cast<unsigned>(a.batch));
#ifndef SSD_EMU
        if (a.ev_before) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_before), st);
#endif
#ifndef SSD_EMU
        if (tc_chunk) {
            ChunkBwdTcArgs t{a.batch,  a.L,   a.H,    a.G,    N,      head_split(a.H, a.G), kSplit, a.act_bf16,
                             a.dy_bf16, a.A,  a.D,    a.dt_bias, a.dt, a.z, a.dy, ws.U, ws.DT, ws.CS, ws.SPH, ws.LMH,
                             ws.SPS,   ws.LMS, ws.PF, a.dz,   a.ddt,  ws.DU,  ws.DU2, ws.PH};
            if ((err = launch_chunk_bwd_tc(t, nc, st)) != cudaSuccess) return err;
        } else {
            SSD_LAUNCH(chunk_bwd_kernel<N>, chunk_groups, dim3(kT), chunk_smem, st, a, ws);
        }
#else
        SSD_LAUNCH(chunk_bwd_kernel<N>, chunk_groups, dim3(kT), chunk_smem, st, a, ws);
#endif
#ifndef SSD_EMU
        if (a.ev_after) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_after), st);
#endif
    } else if (a.batch > 0 && a.d_init_state) {
        const int64_t n = a.batch * a.H * (int64_t)a.P * a.N;
        SSD_LAUNCH(copy_adjoint_kernel, dim3(static_cast<unsigned>((n + kT - 1) / kT)), dim3(kT), 0, st, a);
    }
    if (a.batch > 0) {
        const dim3 grid(static_cast<unsigned>((conv_dim + kCB - 1) / kCB), static_cast<unsigned>(nt),
                        static_cast<unsigned>(a.batch));
        const size_t smem = conv_bwd_smem(a.act_bf16 ? 2 : 4);
        const bool hist = a.init_conv_state != nullptr;
        void (*conv_bwd)(BwdArgs, Ws) = a.act_bf16 ? (hist ? conv_bwd_kernel<true, true> : conv_bwd_kernel<true, false>)
                                                   : (hist ? conv_bwd_kernel<false, true> : conv_bwd_kernel<false, false>);
        if ((err = SSD_SET_SMEM(conv_bwd, smem)) != cudaSuccess) return err;
        SSD_LAUNCH(conv_bwd, grid, dim3(kT), smem, st, a, ws);
    }
    SSD_LAUNCH(reduce_kernel, dim3(static_cast<unsigned>((conv_dim + 31) / 32 + (a.H + 31) / 32)), dim3(kT),
               5 * (size_t)kT * sizeof(float), st, a, ws);
    return cudaGetLastError();
}

}  // namespace

size_t workspace_bytes(int64_t batch, int64_t L, int H, int P, int N, int G) {
    Ws ws;
    return carve(batch, L, H, P, N, G, nullptr, &ws);
}

size_t chunk_bwd_smem_bytes(int N) {
    switch (N) {
        case 16: return chunk_bwd_floats<16>() * sizeof(float);
        case 32: return chunk_bwd_floats<32>() * sizeof(float);
        case 64: return chunk_bwd_floats<64>() * sizeof(float);
        default: return chunk_bwd_floats<128>() * sizeof(float);
    }
}

// Runs the backward on `st`.  Sizes, pointers and the workspace are validated by the caller
// (P = 64, N in {16, 32, 64, 128}, H % G == 0, workspace >= workspace_bytes()).
cudaError_t launch_prefill_backward(const BwdArgs& a, cudaStream_t st) {
    Ws ws;
    carve(a.batch, a.L, a.H, a.P, a.N, a.G, static_cast<char*>(a.workspace), &ws);
    switch (a.N) {
        case 16: return launch_n<16>(a, ws, st);
        case 32: return launch_n<32>(a, ws, st);
        case 64: return launch_n<64>(a, ws, st);
        default: return launch_n<128>(a, ws, st);
    }
}

}  // namespace bwd
}  // namespace ssd
