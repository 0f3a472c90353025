// ssd_backward_tc.cu -- the per-chunk state sums of the prefill backward on the sm_100a tensor cores.
//
// For every 64-token chunk c and head h the backward needs two P x N sums over the chunk's tokens j
// ("Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석" §3.1/§3.2 train the layer, so its
// backward is needed; the sums are the chunked form of the adjoint recurrence, as in ssd_backward.cu):
//   SP_c = sum_j exp(cs_last - cs_j) dt_j x_j (outer) B_j      (the state a chunk adds, from zero)
//   LM_c = sum_i exp(cs_i) g_i (outer) C_i,  g = dy * silu(z)   (the adjoint a chunk adds)
// with x, B, C the post-conv channels.  Both are dense contractions over the chunk (K = 64 tokens), so
// they run as tcgen05 MMAs, transposed so that the 128 state rows n are the MMA's M:
//   SP_c^T = B^T X',  X'_j = exp(cs_last - cs_j) dt_j x_j        [N x P], K = the chunk's tokens
//   LM_c^T = C^T G'', G''_i = exp(cs_i) g_i
// (the same operand shapes as the forward's chunk-state MMA: A = B^T read MN-major from a [token][n]
// tile, B = X' MN-major from a [token][p] tile; fp16 operands, whose 11-bit significand keeps the
// gradients that flow through these sums (the initial-state gradient, dA, ddt_bias) well inside the
// layer's tolerance where bf16's 8 bits do not; fp32 accumulators in TMEM).  The operands are activations
// (post-conv B, C, x and g scaled by decays <= 1 and dt): a magnitude fp16 cannot hold (>= 65504) sets
// bit 1 of the error word, which ssd_device_status reports as SSD_ERR_RANGE.  One
// 128-thread CTA per (chunk, head, sequence): the threads convert their slices of the fp32 post-conv
// channels, dy and z into the fp16 tiles (128-byte swizzle), one thread issues the two MMAs, and each
// thread reads its TMEM lane n (state row n) back and writes SP[p][n] / LM[p][n] for p = 0..63.  For
// d_state 64 the upper 64 rows of the B / C tiles are zero.  The wait for the MMAs is bounded; a wait that
// gives up sets this file's error word (reported by ssd_device_status) and writes nothing.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ssd_backward.h"
#include "ssd_sm100.cuh"

namespace ssd {
namespace bwd {

__device__ int g_bwd_tc_error = 0;

namespace {

using namespace sm100;

constexpr int kQc = 64;       // the backward's chunk (tokens) = the MMAs' K
constexpr int kPc = 64;       // head dimension
constexpr int kNc = 128;      // state rows in the tiles (d_state 64 uses the first 64)
constexpr int kThreadsC = 128;

// shared memory (bytes from a 1024-byte aligned base); every tile is [64 tokens][64 columns] fp16 with
// 128-byte rows and the 128-byte swizzle, 8 KB
constexpr uint32_t OFF_BT = 0;        // B: two tiles, n 0..63 and 64..127
constexpr uint32_t OFF_CT = 16384;    // C: two tiles
constexpr uint32_t OFF_XW = 32768;    // X' [j][p]
constexpr uint32_t OFF_GW = 40960;    // G'' [i][p]
constexpr uint32_t OFF_BAR = 49152;   // mbarrier
constexpr uint32_t OFF_TMH = OFF_BAR + 8;
constexpr uint32_t SMEM_C = OFF_TMH + 8 + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS_C = 128;            // SP^T in columns 0..63, LM^T in 64..127

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi, float& range) {
    range = fmaxf(range, fmaxf(fabsf(lo), fabsf(hi)));
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// Eight values (two float4) times s as fp16, tracking `range`.
__device__ __forceinline__ uint4 pack8f(float4 a, float4 b, float s, float& range) {
    return make_uint4(pack_h2(a.x * s, a.y * s, range), pack_h2(a.z * s, a.w * s, range), pack_h2(b.x * s, b.y * s, range),
                      pack_h2(b.z * s, b.w * s, range));
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// grid (nchunks, H, batch), kThreadsC threads, SMEM_C bytes of dynamic shared memory
__global__ void __launch_bounds__(kThreadsC) chunk_state_tc_kernel(const ChunkStateTcArgs a) {
    extern __shared__ uint8_t smem_c[];
    uint8_t* sm = smem_c + ((1024u - (smem_u32(smem_c) & 1023u)) & 1023u);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMH);
    const int64_t c = blockIdx.x, b = blockIdx.z;
    const int h = blockIdx.y, g = h / (a.H / a.G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t t0 = c * kQc, nc = (a.L + kQc - 1) / kQc;
    const int Qv = static_cast<int>(a.L - t0 < kQc ? a.L - t0 : kQc);
    const int64_t HP = (int64_t)a.H * kPc, GN = (int64_t)a.G * a.N, conv_dim = HP + 2 * GN;

    if (warp == 0) {
        tmem_alloc(tm_holder, TMEM_COLS_C);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }

    float range = 0.f;  // largest magnitude this thread writes to an fp16 tile
    // B and C of the chunk (rows j >= Qv and channels n >= N zero): 64 rows x 16 chunks of 8 channels, eight
    // per thread in two passes of four, each pass's loads issued before its stores (the stores could alias
    // the loads as far as the compiler knows, so it would not move later loads above them)
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        float4 v[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + kThreadsC * (4 * pass + i), r = e >> 4, n0 = 8 * (e & 15);
            if (r < Qv && n0 < a.N) {
                const float* row = a.U + (b * a.L + t0 + r) * conv_dim + HP + (int64_t)g * a.N + n0;
                v[i][0] = *reinterpret_cast<const float4*>(row);
                v[i][1] = *reinterpret_cast<const float4*>(row + 4);
                v[i][2] = *reinterpret_cast<const float4*>(row + GN);
                v[i][3] = *reinterpret_cast<const float4*>(row + GN + 4);
            } else {
                v[i][0] = v[i][1] = v[i][2] = v[i][3] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + kThreadsC * (4 * pass + i), r = e >> 4, k8 = e & 15;
            const uint32_t off = (uint32_t)(k8 >> 3) * 8192u + sw128_off(r, k8 & 7);
            *reinterpret_cast<uint4*>(sm + OFF_BT + off) = pack8f(v[i][0], v[i][1], 1.f, range);
            *reinterpret_cast<uint4*>(sm + OFF_CT + off) = pack8f(v[i][2], v[i][3], 1.f, range);
        }
    }
    // X' and G'' (64 rows x 8 chunks of 8 head channels; rows tid / 8 + 16 i), all loads first
    const float* dtp = a.DT + (b * a.H + h) * a.L + t0;
    const float* csp = a.CS + (b * a.H + h) * a.L + t0;
    const float cs_last = csp[Qv - 1];
    const int k8 = tid & 7, p0 = 8 * k8;
    float4 xv[4][2], dyv[4][2];
    uint4 zw[4];
    float dtr[4], csr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = (tid >> 3) + 16 * i;
        xv[i][0] = xv[i][1] = dyv[i][0] = dyv[i][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        zw[i] = make_uint4(0u, 0u, 0u, 0u);
        dtr[i] = csr[i] = 0.f;
        if (r < Qv) {
            dtr[i] = dtp[r];
            csr[i] = csp[r];
            const int64_t row = b * a.L + t0 + r;
            const float* xr = a.U + row * conv_dim + (int64_t)h * kPc + p0;
            xv[i][0] = *reinterpret_cast<const float4*>(xr);
            xv[i][1] = *reinterpret_cast<const float4*>(xr + 4);
            const int64_t yi = row * HP + (int64_t)h * kPc + p0;
            if (a.dy_bf16) {
                const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(a.dy) + yi);
                dyv[i][0] = make_float4(bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y));
                dyv[i][1] = make_float4(bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w));
            } else {
                dyv[i][0] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.dy) + yi);
                dyv[i][1] = *reinterpret_cast<const float4*>(static_cast<const float*>(a.dy) + yi + 4);
            }
            zw[i] = *reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(a.z) + yi);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = (tid >> 3) + 16 * i;
        const bool on = r < Qv;
        const float fx = on ? dtr[i] * __expf(cs_last - csr[i]) : 0.f, fg = on ? __expf(csr[i]) : 0.f;
        const float zf[8] = {bf_lo(zw[i].x), bf_hi(zw[i].x), bf_lo(zw[i].y), bf_hi(zw[i].y),
                             bf_lo(zw[i].z), bf_hi(zw[i].z), bf_lo(zw[i].w), bf_hi(zw[i].w)};
        const float dyf[8] = {dyv[i][0].x, dyv[i][0].y, dyv[i][0].z, dyv[i][0].w,
                              dyv[i][1].x, dyv[i][1].y, dyv[i][1].z, dyv[i][1].w};
        float4 g0, g1;
        float* gp[8] = {&g0.x, &g0.y, &g0.z, &g0.w, &g1.x, &g1.y, &g1.z, &g1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) *gp[q] = dyf[q] * zf[q] * __fdividef(1.f, 1.f + __expf(-zf[q]));
        *reinterpret_cast<uint4*>(sm + OFF_XW + sw128_off(r, k8)) = pack8f(xv[i][0], xv[i][1], fx, range);
        *reinterpret_cast<uint4*>(sm + OFF_GW + sw128_off(r, k8)) = pack8f(g0, g1, fg, range);
    }
    if (!(range < 65504.f)) atomicOr(&g_bwd_tc_error, 2);
    fence_async_smem();  // the tiles are read by the tensor cores (async proxy)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tm_holder;

    if (tid == 0) {
        // fp16 A and B (format 0), fp32 D; A MN-major (B^T / C^T), B MN-major (X' / G'')
        constexpr uint32_t ID = (1u << 4) | (1u << 15) | (1u << 16) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
        const uint64_t dB = sw128_desc(smem_u32(sm + OFF_BT), 8192, 1024);
        const uint64_t dC = sw128_desc(smem_u32(sm + OFF_CT), 8192, 1024);
        const uint64_t dX = sw128_desc(smem_u32(sm + OFF_XW), 8192, 1024);
        const uint64_t dG = sw128_desc(smem_u32(sm + OFF_GW), 8192, 1024);
        // K = 64 tokens in four steps of 16 rows; an MN-major operand advances 16 rows x 128 bytes per step
#pragma unroll
        for (uint32_t kk = 0; kk < 4; ++kk) mma_bf16(tmem, dB + kk * (2048 >> 4), dX + kk * (2048 >> 4), ID, kk > 0);
#pragma unroll
        for (uint32_t kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + 64, dC + kk * (2048 >> 4), dG + kk * (2048 >> 4), ID, kk > 0);
        mma_commit(bar);
    }
    const bool done = __all_sync(0xffffffffu, mbar_wait(bar, 0, nullptr));
    tc_fence_after();
    const int n = warp * 32 + lane;  // this thread's TMEM lane = state row n
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    if (done) {
        const int64_t base = ((b * nc + c) * a.H + h) * (int64_t)kPc * a.N;
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            float* out = which ? a.LM : a.SP;
#pragma unroll 1
            for (int p0 = 0; p0 < kPc; p0 += 16) {
                float v[16];
                tmem_ld16(tmem + lane_base + which * 64 + p0, v);
                tmem_wait_ld();
                if (n < a.N) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) out[base + (int64_t)(p0 + k) * a.N + n] = v[k];
                }
            }
        }
    } else if (tid == 0) {
        atomicOr(&g_bwd_tc_error, 1);  // bit 0: the wait gave up
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS_C);
    }
}

}  // namespace

bool chunk_state_tc_supported(int P, int N, bool act_bf16) { return act_bf16 && P == kPc && (N == 64 || N == kNc); }

cudaError_t launch_chunk_state_tc(const ChunkStateTcArgs& a, int64_t nchunks, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(chunk_state_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_C);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(nchunks), static_cast<unsigned>(a.H), static_cast<unsigned>(a.batch));
    chunk_state_tc_kernel<<<grid, kThreadsC, SMEM_C, st>>>(a);
    return cudaGetLastError();
}

cudaError_t read_and_clear_bwd_tc_error(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_bwd_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_tc_error, &zero, sizeof(int));
}

}  // namespace bwd
}  // namespace ssd
