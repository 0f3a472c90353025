// ssd_chunk_bwd_tc.cu -- the per-chunk backward of the prefill on the sm_100a tensor cores.
//
// The layer is trained ("Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석" §3.1/§3.2), so the
// SSD prefill needs its backward.  Inside one 64-token chunk, with cs the in-chunk cumulative sum of dt*A,
// L_ij = exp(cs_i - cs_j) (i >= j), g = dy * silu(z), Sp the state entering the chunk and Lm the adjoint
// of the state leaving it, every gradient of the chunk is built from ten dense products over the chunk
// (K = 64 tokens or 64 head channels) or over the state (K = N):
//   CB  = C B^T                  GX  = g x^T                 (token x token)
//   SPC = C Sp^T   LMB = B Lm^T  YIN = LCB x   DXI = LCB^T g  (token x head channel)
//   dB^T += Lm^T X'^T + C^T LGX'   dC^T += Sp^T G''^T + B^T LGX'^T   (state x token, summed over heads)
// with LCB_ij = CB_ij L_ij dt_j and LGX'_ij = GX_ij L_ij dt_j (zero above the diagonal), X'_j =
// exp(cs_last - cs_j) dt_j x_j and G''_i = exp(cs_i) g_i.  From them, elementwise:
//   y_i  = YIN_i + exp(cs_i) SPC_i + D x_i,  dz_i = dy_i silu'(z_i) y_i
//   dx_j = DXI_j + dt_j exp(cs_last - cs_j) LMB_j + D g_j
//   E_i  = exp(cs_i) g_i . SPC_i,  W_j = exp(cs_last - cs_j) x_j . LMB_j
//   M_ij = LGX'_ij CB_ij,  Dr_j = sum_i GX_ij L_ij CB_ij (the column sums of M / dt_j)
//   d(dA_k) = R_k + sum_{i>=k} E_i + F + sum_{j<k} dt_j W_j,
//     R_k = sum_{i>=k} sum_{j<k} M_ij = sum_{m<k} (colsum_m(M) - rowsum_m(M))  (M is lower triangular)
//   ddt_k = Dr_k + W_k + A d(dA_k), then through softplus
// (the same quantities, in the same fp32 epilogue arithmetic, as the CUDA-core chunk kernel of
// ssd_backward.cu; there R comes from explicit prefix sums of M).
//
// Operands are fp16 (11-bit significand; bf16's 8 bits lose too much in the sums behind ddt).  The
// entering states and leaving adjoints arrive as the state pass's fp16 tiles, row p scaled by a power of
// two s_p <= 1 that keeps it below 2^14; SPC and LMB column p are multiplied back by 1/s_p, and the
// partners of the head-summed products (X', G'') take 1/s_p on their column p.  Any other value fp16
// cannot hold (>= 65504) sets bit 1 of this file's error word (SSD_ERR_RANGE).  The elementwise terms
// read x, g and dy silu'(z) back from the same fp16 tiles the MMAs use.
//
// One CTA per (chunk, group, half of the group's heads), heads in turn; 512 threads in four roles:
//   row warps 0, 1, 4, 5, 8, 9, 12, 13 (TMEM lanes 0..63 = the chunk's tokens; warp w takes tokens
//                         32 (w & 3) .. +31 and columns 16 (w >> 2) .. +15): the elementwise work above,
//                         the LCB / LGX' tiles, dz, dx and per-row partial sums (16 columns a thread keeps
//                         each thread's dependent chains short; 16 warps cap registers at 128);
//   loader warps 2, 3, 6, 7, 10, 11: the head's tiles, two heads deep: Sp and Lm by bulk copy, x, X', g, G''
//                         and dy silu'(z) converted from global memory;
//   warp 14             : TMEM allocation and, on one thread, the MMAs;
//   warp 15             : each head's per-token scalars from the partial sums (the prefix / suffix sums
//                         behind d(dA), ddt) and the per-chunk partials of dA, dD, ddt_bias.
// Every MMA is M = 128, N = 64 with fp32 accumulators in TMEM (512 columns: CB, GX, SPC, LMB, YIN, DXI,
// dB^T, dC^T).  The token-major products use only rows 0..63 of their 128-row result: the A tile's rows
// 64..127 are whatever follows it in shared memory (always in bounds), and the result lanes 64..127 are
// never read.  dB^T and dC^T have the state index n as M (rows past N unused).
// All waits are bounded mbarrier waits that also watch a shared abort word; a wait that gives up sets
// bit 0 of the error word (SSD_ERR_TIMEOUT from ssd_device_status), and the CTA leaves without writing
// its dB / dC.  No atomics on results: every sum runs in a fixed order (deterministic).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "ssd_backward.h"
#include "ssd_sm100.cuh"

namespace ssd {
namespace bwd {

__device__ int g_chunk_bwd_tc_error = 0;

namespace {

using namespace sm100;

constexpr int kQb = 64;   // chunk (tokens)
constexpr int kPb = 64;   // head dimension
constexpr int kThreadsB = 512;
constexpr int kRows = 256;     // row threads (warps 0, 1, 4, 5, 8, 9, 12, 13)
constexpr int kWarpMma = 14, kWarpScalar = 15;
constexpr int kLoaders = 192;  // loader threads (warps 2, 3, 6, 7, 10, 11)
constexpr int kSplitPf = 4;    // partial sums of F per (chunk, head) from the state pass

// shared memory (bytes from a 1024-byte aligned base).  A "box" is [64 rows][64 fp16] with 128-byte rows
// and the 128-byte swizzle (8 KB); an N-wide tile is one box per 64 state columns.
constexpr uint32_t OFF_TC = 0;          // C [i][n], two boxes
constexpr uint32_t OFF_TB = 16384;      // B [j][n], two boxes
constexpr uint32_t OFF_LCB = 32768;     // LCB [i][j]
constexpr uint32_t OFF_LGX = 40960;     // LGX' [i][j]
constexpr uint32_t OFF_BUF = 49152;     // two per-head buffers of BUF_BYTES:
constexpr uint32_t B_SP = 0;            //   s Sp [p][n], two boxes
constexpr uint32_t B_LM = 16384;        //   s Lm [p][n], two boxes
constexpr uint32_t B_X = 32768;         //   x [j][p]
constexpr uint32_t B_XP = 40960;        //   X' [j][p]
constexpr uint32_t B_G = 49152;         //   g [i][p]
constexpr uint32_t B_GP = 57344;        //   G'' [i][p]
constexpr uint32_t B_DS = 65536;        //   dy silu'(z) [i][p]
constexpr uint32_t BUF_BYTES = 73728;
constexpr uint32_t OFF_VEC = OFF_BUF + 2 * BUF_BYTES;  // fp32 vectors:
constexpr uint32_t V_DT = 0;            //   dt [2 buffers][64]
constexpr uint32_t V_CS = 512;          //   cs [2][64]
constexpr uint32_t V_COL = 1024;        //   column sums of GX L CB [2 head parities][2 token halves][64]
constexpr uint32_t V_ROWM = 2048;       //   row sums of M [2][4 column quarters][64]
constexpr uint32_t V_E = 4096;          //   g_i . SPC_i partials [2][4][64]
constexpr uint32_t V_W = 6144;          //   W_j partials [2][4][64]
constexpr uint32_t V_PD = 8192;         //   sum g . x per row warp [2][8]
constexpr uint32_t V_ISC = 8256;        //   inverse row scales of each buffer's Sp, Lm tiles [2][2][64]
constexpr uint32_t VEC_BYTES = 9280;
constexpr uint32_t OFF_BAR = OFF_VEC + VEC_BYTES;
enum : int { TILE_FULL0, TILE_FULL1, TILE_FREE0, TILE_FREE1, SPLM_FULL0, SPLM_FULL1, GX_DONE, B1_DONE, LT_FULL,
             B2_DONE, ACC_FREE, WSYNC, SCALAR_FREE, FINAL, NBAR };
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // abort word, TMEM base
constexpr uint32_t SMEM_B = OFF_MISC + 16 + 1024;  // + alignment slack

// TMEM columns (lane = token or state row)
constexpr uint32_t COL_CB = 0, COL_GX = 64, COL_SPC = 128, COL_LMB = 192, COL_YIN = 256, COL_DXI = 320,
                   COL_DB = 384, COL_DC = 448, TMEM_COLS_B = 512;

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}
// Instruction descriptor for kind::f16 with fp16 A/B (format 0) and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float sigm(float v) { return 1.f / (1.f + expf(-v)); }

// Eight consecutive activations from element i (a multiple of 8) of a bf16 or fp32 array (16-byte aligned).
__device__ __forceinline__ void load8(const void* p, int64_t i, bool bf16, float (&v)[8]) {
    if (bf16) {
        const uint4 w = *reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(p) + i);
        v[0] = bf_lo(w.x), v[1] = bf_hi(w.x), v[2] = bf_lo(w.y), v[3] = bf_hi(w.y);
        v[4] = bf_lo(w.z), v[5] = bf_hi(w.z), v[6] = bf_lo(w.w), v[7] = bf_hi(w.w);
    } else {
        const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
        const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(p) + i + 4);
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    }
}
// Eight values times s as fp16; `range` keeps the largest magnitude packed (>= 65504 does not fit).
__device__ __forceinline__ uint4 pack8(const float (&v)[8], float s, float& range) {
    float w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        w[q] = v[q] * s;
        range = fmaxf(range, fabsf(w[q]));
    }
    return make_uint4(pack_h2(w[0], w[1]), pack_h2(w[2], w[3]), pack_h2(w[4], w[5]), pack_h2(w[6], w[7]));
}
// Eight values v[q] f[q] s as fp16 (f: the per-column inverse state scales, in shared memory), tracking
// `range` likewise.
__device__ __forceinline__ uint4 pack8s(const float (&v)[8], const float* f, float s, float& range) {
    float w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = v[q] * f[q];
    return pack8(w, s, range);
}
// The eight fp16 values of 16-byte chunk `chunk` of row r of a swizzled tile, as fp32.
__device__ __forceinline__ void unpack8(const uint8_t* tile, int r, int chunk, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(tile + sw128_off(r, chunk));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// D (+)= A B over K = 16 * steps; a K-major operand steps 32 bytes inside a box and 8 KB from box to box,
// an MN-major one 16 rows (2 KB) per step.  The first step overwrites D unless acc.
__device__ __forceinline__ void mma_steps(uint32_t d, uint64_t a0, bool a_mn, uint64_t b0, bool b_mn, uint32_t idesc,
                                          int steps, bool acc) {
    for (int kk = 0; kk < steps; ++kk) {
        const uint32_t kmaj = ((uint32_t)(kk >> 2) * 8192u + (uint32_t)(kk & 3) * 32u) >> 4;
        const uint32_t mnmaj = ((uint32_t)kk * 2048u) >> 4;
        mma_bf16(d, a0 + (a_mn ? mnmaj : kmaj), b0 + (b_mn ? mnmaj : kmaj), idesc, (acc || kk > 0) ? 1u : 0u);
    }
}

constexpr uint32_t ID_KK = idesc_f16_f32(128, 64, false, false);
constexpr uint32_t ID_KM = idesc_f16_f32(128, 64, false, true);
constexpr uint32_t ID_MK = idesc_f16_f32(128, 64, true, false);
constexpr uint32_t ID_MM = idesc_f16_f32(128, 64, true, true);
__device__ __forceinline__ uint64_t kdesc(const uint8_t* p) { return sw128_desc(smem_u32(p), 16, 1024); }
__device__ __forceinline__ uint64_t mdesc(const uint8_t* p) { return sw128_desc(smem_u32(p), 8192, 1024); }

// The first MMAs of head k (operands: the head's buffer and C, B): GX first (the row warps start on it), then
// SPC, LMB and the Sp / Lm parts of dB^T, dC^T (which the first head starts).
__device__ __forceinline__ void issue_batch1(const uint8_t* sm, uint32_t tmem, int k, int nbox, uint64_t* gx_done,
                                             uint64_t* done) {
    const uint8_t* bo = sm + OFF_BUF + (k & 1) * BUF_BYTES;
    mma_steps(tmem + COL_GX, kdesc(bo + B_G), false, kdesc(bo + B_X), false, ID_KK, 4, false);
    mma_commit(gx_done);
    mma_steps(tmem + COL_SPC, kdesc(sm + OFF_TC), false, kdesc(bo + B_SP), false, ID_KK, 4 * nbox, false);
    mma_steps(tmem + COL_LMB, kdesc(sm + OFF_TB), false, kdesc(bo + B_LM), false, ID_KK, 4 * nbox, false);
    mma_steps(tmem + COL_DB, mdesc(bo + B_LM), true, kdesc(bo + B_XP), false, ID_MK, 4, k > 0);
    mma_steps(tmem + COL_DC, mdesc(bo + B_SP), true, kdesc(bo + B_GP), false, ID_MK, 4, k > 0);
    mma_commit(done);
}
// The MMAs that need the row warps' LCB / LGX' tiles: YIN, DXI (then `done`), and the intra-chunk parts of
// dB^T, dC^T (then `free_buf`: the head's buffer and the LCB / LGX' tiles are free).
__device__ __forceinline__ void issue_batch2(const uint8_t* sm, uint32_t tmem, int k, uint64_t* done,
                                             uint64_t* free_buf) {
    const uint8_t* bo = sm + OFF_BUF + (k & 1) * BUF_BYTES;
    mma_steps(tmem + COL_YIN, kdesc(sm + OFF_LCB), false, mdesc(bo + B_X), true, ID_KM, 4, false);
    mma_steps(tmem + COL_DXI, mdesc(sm + OFF_LCB), true, mdesc(bo + B_G), true, ID_MM, 4, false);
    mma_commit(done);
    mma_steps(tmem + COL_DB, mdesc(sm + OFF_TC), true, mdesc(sm + OFF_LGX), true, ID_MM, 4, true);
    mma_steps(tmem + COL_DC, mdesc(sm + OFF_TB), true, kdesc(sm + OFF_LGX), false, ID_MK, 4, true);
    mma_commit(free_buf);
}

// A warp-uniform bounded wait: true when the phase of `parity` completed for every lane.
__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity, volatile int* abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}
__device__ __forceinline__ void give_up(volatile int* abort) {
    *abort = 1;
    atomicOr(&g_chunk_bwd_tc_error, 1);
}

// Sum over the warp's 32 lanes of each of v[0..15]: lane l ends with the sum of v[l & 15] (both halves
// of the warp add up, then a butterfly: at each step a lane keeps the half of its values whose index bit
// matches its lane bit and adds the partner's).
__device__ __forceinline__ float column_sums16(float (&v)[16], int lane) {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], 16);
#pragma unroll
    for (int s = 8; s >= 1; s >>= 1) {
        const bool up = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = up ? v[i] : v[i + s];
            const float keep = up ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return v[0];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
    return v;
}

// Exclusive prefix sums over the 64 tokens held two per lane (token lane and lane + 32).
__device__ __forceinline__ void scan_excl(const float (&v)[2], float (&out)[2], int lane) {
    float s0 = v[0], s1 = v[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t0 = __shfl_up_sync(0xffffffffu, s0, o), t1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
            s0 += t0;
            s1 += t1;
        }
    }
    const float tot0 = __shfl_sync(0xffffffffu, s0, 31);
    out[0] = s0 - v[0];
    out[1] = tot0 + s1 - v[1];
}

// grid (nchunks, G * split, batch), kThreadsB threads, SMEM_B bytes of dynamic shared memory
__global__ void __launch_bounds__(kThreadsB, 1) chunk_bwd_tc_kernel(const ChunkBwdTcArgs a) {
    extern __shared__ uint8_t smem_b[];
    uint8_t* sm = smem_b + ((1024u - (smem_u32(smem_b) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + OFF_MISC);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(sm + OFF_MISC + 8);
    float* vec = reinterpret_cast<float*>(sm + OFF_VEC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t c = blockIdx.x, b = blockIdx.z, t0 = c * kQb, nc = (a.L + kQb - 1) / kQb;
    const int hpg = a.H / a.G, g = blockIdx.y / a.split, half = blockIdx.y % a.split;
    const int hl0 = half * hpg / a.split, nh = (half + 1) * hpg / a.split - hl0;
    const int Qv = static_cast<int>(a.L - t0 < kQb ? a.L - t0 : kQb);
    const int N = a.N, nbox = N / 64;
    const int64_t HP = (int64_t)a.H * kPb, GN = (int64_t)a.G * N, conv_dim = HP + 2 * GN;
    const int64_t row0 = b * a.L + t0;  // first token row of the chunk

    if (warp == kWarpMma) {
        tmem_alloc(tm_holder, TMEM_COLS_B);
        tmem_relinquish();
    }
    if (tid == 0) {
        *abort = 0;
        mbar_init(&bars[TILE_FULL0], kLoaders);
        mbar_init(&bars[TILE_FULL1], kLoaders);
        mbar_init(&bars[TILE_FREE0], 1 + kRows + 32);  // the MMAs' commit, the row threads, the scalar warp
        mbar_init(&bars[TILE_FREE1], 1 + kRows + 32);
        mbar_init(&bars[SPLM_FULL0], 1);    // the bulk copies' transaction bytes
        mbar_init(&bars[SPLM_FULL1], 1);
        mbar_init(&bars[GX_DONE], 1);
        mbar_init(&bars[B1_DONE], 1);
        mbar_init(&bars[LT_FULL], kRows);
        mbar_init(&bars[B2_DONE], 1);
        mbar_init(&bars[ACC_FREE], kRows);
        mbar_init(&bars[WSYNC], kRows);
        mbar_init(&bars[SCALAR_FREE], 32);
        mbar_init(&bars[FINAL], 1);
        fence_mbar_init();
    }
    // the group's post-conv B and C (rows past Qv zero): 64 rows x N/8 chunks of 8 channels
    for (int e = tid; e < kQb * (N / 8); e += kThreadsB) {
        const int r = e / (N / 8), k8 = e % (N / 8);
        uint4 pb = make_uint4(0u, 0u, 0u, 0u), pc = pb;
        if (r < Qv) {
            const float* src = a.U + (row0 + r) * conv_dim + HP + (int64_t)g * N + 8 * k8;
            float v[8], range = 0.f;
            load8(src, 0, false, v);
            pb = pack8(v, 1.f, range);
            load8(src + GN, 0, false, v);
            pc = pack8(v, 1.f, range);
            if (!(range < 65504.f)) atomicOr(&g_chunk_bwd_tc_error, 2);
        }
        const uint32_t off = (uint32_t)(k8 >> 3) * 8192u + sw128_off(r, k8 & 7);
        *reinterpret_cast<uint4*>(sm + OFF_TB + off) = pb;
        *reinterpret_cast<uint4*>(sm + OFF_TC + off) = pc;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tm_holder;

    if (warp == kWarpMma) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            mma_steps(tmem + COL_CB, kdesc(sm + OFF_TC), false, kdesc(sm + OFF_TB), false, ID_KK, 4 * nbox, false);
            bool ok = true;
            for (int k = 0; k < nh && ok; ++k) {
                const int buf = k & 1;
                ok = mbar_wait(&bars[TILE_FULL0 + buf], (k >> 1) & 1, abort) &&
                     mbar_wait(&bars[SPLM_FULL0 + buf], (k >> 1) & 1, abort) &&
                     (k == 0 || mbar_wait(&bars[ACC_FREE], (k - 1) & 1, abort));
                if (!ok) break;
                tc_fence_after();
                issue_batch1(sm, tmem, k, nbox, &bars[GX_DONE], &bars[B1_DONE]);
                ok = mbar_wait(&bars[LT_FULL], k & 1, abort);
                if (!ok) break;
                tc_fence_after();
                issue_batch2(sm, tmem, k, &bars[B2_DONE], &bars[TILE_FREE0 + buf]);
            }
            if (!ok) give_up(abort);
            mma_commit(&bars[FINAL]);  // every MMA issued so far
        }
        __syncwarp();
    } else if (warp == kWarpScalar) {
        // ---------------- scalar warp: each head's ddt and per-chunk partial sums (tokens lane, lane + 32) -------
        bool ok = true;
        for (int k = 0; k < nh && ok; ++k) {
            const int buf = k & 1, par = k & 1;
            const int h = g * hpg + hl0 + k;
            // the global inputs first: F, the raw dt of the two tokens, A, dt_bias
            const float* pf = a.PF + ((b * nc + c) * a.H + h) * kSplitPf;
            const float F = (pf[0] + pf[1]) + (pf[2] + pf[3]);
            float raw[2] = {0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int kk = lane + 32 * u;
                if (kk < Qv) raw[u] = bf_lo(static_cast<const unsigned short*>(a.dt)[(row0 + kk) * a.H + h]);
            }
            const float Ah = a.A[h], bias = a.dt_bias[h];
            // dt and exp(cs) of the two tokens from the head's buffer (TILE_FULL), then the row warps' sums (WSYNC)
            if (!wait_all(&bars[TILE_FULL0 + buf], (k >> 1) & 1, abort)) {
                ok = false;
                break;
            }
            const float* dts = vec + (V_DT >> 2) + buf * 64;
            const float* css = vec + (V_CS >> 2) + buf * 64;
            float dtk[2], exk[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int kk = lane + 32 * u;
                dtk[u] = dts[kk];
                exk[u] = kk < Qv ? expf(css[kk]) : 0.f;
            }
            if (!wait_all(&bars[WSYNC], par, abort)) {
                ok = false;
                break;
            }
            const float* col = vec + (V_COL >> 2) + par * 128;
            const float* rwm = vec + (V_ROWM >> 2) + par * 256;
            const float* ev = vec + (V_E >> 2) + par * 256;
            const float* wv = vec + (V_W >> 2) + par * 256;
            const float* pdw = vec + (V_PD >> 2) + par * 8;
            // the four column quarters' partial sums of token kk, in a fixed order
            auto q4 = [](const float* v, int kk) { return (v[kk] + v[64 + kk]) + (v[128 + kk] + v[192 + kk]); };
            float dr0[2], d[2], e[2], w[2], dw[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int kk = lane + 32 * u;
                dr0[u] = col[kk] + col[64 + kk];
                d[u] = dtk[u] * dr0[u] - q4(rwm, kk);
                e[u] = exk[u] * q4(ev, kk);
                w[u] = q4(wv, kk);
                dw[u] = dtk[u] * w[u];
            }
            const float pD = ((pdw[0] + pdw[1]) + (pdw[2] + pdw[3])) + ((pdw[4] + pdw[5]) + (pdw[6] + pdw[7]));
            __syncwarp();
            mbar_arrive(&bars[SCALAR_FREE]);  // the partial sums are read: the row warps may write the next ones
            // exclusive prefix sums of d and dt W, inclusive suffix sums of E, over the 64 tokens
            float R[2], Wp[2], Ex[2], Es[2];
            scan_excl(d, R, lane);
            scan_excl(dw, Wp, lane);
            scan_excl(e, Ex, lane);
            const float etot = __shfl_sync(0xffffffffu, Ex[1] + e[1], 31);
            Es[0] = etot - Ex[0];
            Es[1] = etot - Ex[1];
            float pdA = 0.f, pbias = 0.f;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int kk = lane + 32 * u;
                if (kk < Qv) {
                    const float dda = R[u] + Es[u] + F + Wp[u];
                    const float ddt = dr0[u] + w[u] + Ah * dda;
                    const float dr = ddt * sigm(raw[u] + bias);
                    a.ddt[(row0 + kk) * a.H + h] = dr;
                    pdA += dtk[u] * dda;
                    pbias += dr;
                }
            }
            pdA = warp_sum(pdA);
            pbias = warp_sum(pbias);
            if (lane == 0) {
                float* ph = a.PH + ((b * nc + c) * a.H + h) * 3;
                ph[0] = pdA;
                ph[1] = pD;
                ph[2] = pbias;
            }
            mbar_arrive(&bars[TILE_FREE0 + buf]);
        }
        if (!ok) give_up(abort);
    } else if ((warp & 3) >= 2) {
        // ---------------- loaders: warps 2, 3, 6, 7, 10, 11 (14 and 15 took the branches above) ----------------
        const int lt = ((warp >> 2) * 2 + (warp & 3) - 2) * 32 + lane;  // 0..kLoaders-1
        const int k8 = lt & 7;  // this thread's 16-byte chunk (8 head channels) of rows lt / 8 + 24 m
        for (int k = 0; k < nh; ++k) {
            const int buf = k & 1;
            if (k >= 2 && !wait_all(&bars[TILE_FREE0 + buf], ((k >> 1) - 1) & 1, abort)) {
                give_up(abort);
                break;
            }
            uint8_t* bo = sm + OFF_BUF + buf * BUF_BYTES;
            const int h = g * hpg + hl0 + k;
            const int64_t hrow = (b * a.H + h) * a.L + t0;
            // Sp and Lm: the state pass's fp16 tiles and their inverse row scales, four bulk copies onto this
            // buffer's barrier
            const int64_t ti = (b * nc + c) * a.H + h;
            const uint32_t tile_bytes = 8192u * (uint32_t)nbox;
            float* isc = vec + (V_ISC >> 2) + buf * 128;  // 1/s_p of Sp [64], then of Lm [64]
            if (lt == 0) {
                uint64_t* bar = &bars[SPLM_FULL0 + buf];
                mbar_arrive_expect_tx(bar, 2 * tile_bytes + 2 * 256);
                bulk_load(bo + B_SP, static_cast<const char*>(a.SPH) + ti * tile_bytes, tile_bytes, bar);
                bulk_load(bo + B_LM, static_cast<const char*>(a.LMH) + ti * tile_bytes, tile_bytes, bar);
                bulk_load(isc, a.SPS + ti * 64, 256, bar);
                bulk_load(isc + 64, a.LMS + ti * 64, 256, bar);
            }
            // x, X', g, G'', dy silu'(z): 64 rows x 8 chunks of 8 channels, up to three chunks per thread (rows
            // lt / 8 + 24 m below 64), all loads first
            const float cs_last = a.CS[hrow + Qv - 1];
            float xv[3][8], gv[3][8], zv[3][8], dtr[3], csr[3];
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                const int r = (lt >> 3) + 24 * m;
                if (r < Qv) {
                    dtr[m] = a.DT[hrow + r];
                    csr[m] = a.CS[hrow + r];
                    load8(a.U, (row0 + r) * conv_dim + (int64_t)h * kPb + 8 * k8, false, xv[m]);
                    const int64_t yi = (row0 + r) * HP + (int64_t)h * kPb + 8 * k8;
                    load8(a.dy, yi, a.dy_bf16, gv[m]);
                    load8(a.z, yi, a.act_bf16, zv[m]);
                } else {
                    dtr[m] = csr[m] = 0.f;
#pragma unroll
                    for (int q = 0; q < 8; ++q) xv[m][q] = gv[m][q] = zv[m][q] = 0.f;
                }
            }
            float range = 0.f;  // largest magnitude written to an fp16 tile
            if (!wait_all(&bars[SPLM_FULL0 + buf], (k >> 1) & 1, abort)) {
                give_up(abort);
                break;
            }
            // X' takes Lm's inverse row scales and G'' Sp's (column p of X', G'' meets row p of Lm, Sp)
            const float* is = isc + 8 * k8;
            const float* il = isc + 64 + 8 * k8;
#pragma unroll
            for (int m = 0; m < 3; ++m) {
                const int r = (lt >> 3) + 24 * m;
                if (r >= kQb) break;
                float ds[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float zq = zv[m][q], s = __fdividef(1.f, 1.f + __expf(-zq)), dy = gv[m][q];
                    gv[m][q] = dy * zq * s;                       // g = dy silu(z)
                    ds[q] = dy * s * (1.f + zq * (1.f - s));      // dy silu'(z)
                }
                const bool on = r < Qv;
                const uint32_t off = sw128_off(r, k8);
                *reinterpret_cast<uint4*>(bo + B_X + off) = pack8(xv[m], 1.f, range);
                *reinterpret_cast<uint4*>(bo + B_XP + off) =
                    pack8s(xv[m], il, on ? dtr[m] * __expf(cs_last - csr[m]) : 0.f, range);
                *reinterpret_cast<uint4*>(bo + B_G + off) = pack8(gv[m], 1.f, range);
                *reinterpret_cast<uint4*>(bo + B_GP + off) = pack8s(gv[m], is, on ? __expf(csr[m]) : 0.f, range);
                *reinterpret_cast<uint4*>(bo + B_DS + off) = pack8(ds, 1.f, range);
                if (k8 == 0) {
                    vec[(V_DT >> 2) + buf * 64 + r] = dtr[m];
                    vec[(V_CS >> 2) + buf * 64 + r] = csr[m];
                }
            }
            if (!(range < 65504.f)) atomicOr(&g_chunk_bwd_tc_error, 2);
            fence_async_smem();
            mbar_arrive(&bars[TILE_FULL0 + buf]);
        }
    } else {
        // ---------------- row warps 0, 1, 4, 5, 8, 9, 12, 13 ----------------
        const int rq = warp & 3;           // token half: rows 32 rq .. 32 rq + 31
        const int cq = warp >> 2;          // column quarter: 16 cq .. 16 cq + 15
        const int r = 32 * rq + lane, c0 = 16 * cq;
        const int wi = rq + 2 * cq;        // 0..7
        const uint32_t lb = (uint32_t)(32 * rq) << 16;
        bool ok = true;
        for (int k = 0; k < nh && ok; ++k) {
            const int buf = k & 1, par = k & 1;
            const int h = g * hpg + hl0 + k;
            const float Dh = a.D[h];
            // the head's tiles (TILE_FULL), then GX (GX_DONE)
            if (!wait_all(&bars[TILE_FULL0 + buf], (k >> 1) & 1, abort) || !wait_all(&bars[GX_DONE], par, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint8_t* bo = sm + OFF_BUF + buf * BUF_BYTES;
            const float* dts = vec + (V_DT >> 2) + buf * 64;
            const float* css = vec + (V_CS >> 2) + buf * 64;
            const float cs_r = css[r], dt_r = dts[r], cs_last = css[Qv - 1];
            // the inverse row scales of this head's Sp, Lm tiles: SPC and LMB column p come out of TMEM times s_p
            const float* isp = vec + (V_ISC >> 2) + buf * 128 + c0;
            const float* ilm = isp + 64;
            // phase B: LCB and LGX' rows, the row sums of M and the column sums of GX L CB
            float rowm = 0.f, range = 0.f;
            {
                float gx[16], cb[16];
                tmem_ld16(tmem + lb + COL_GX + c0, gx);
                tmem_ld16(tmem + lb + COL_CB + c0, cb);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    uint32_t plcb[4], plgx[4];
#pragma unroll
                    for (int w2 = 0; w2 < 4; ++w2) {
                        float lc[2], lg[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int q = 8 * q8 + 2 * w2 + u, j = c0 + q;
                            const bool on = j <= r && r < Qv;
                            const float L = on ? __expf(cs_r - css[j]) : 0.f;
                            const float lgx = gx[q] * L, dtj = dts[j];
                            lc[u] = cb[q] * L * dtj;
                            lg[u] = lgx * dtj;
                            rowm += lg[u] * cb[q];
                            gx[q] = lgx * cb[q];  // becomes this row's share of column j's sum
                        }
                        plcb[w2] = pack_h2(lc[0], lc[1]);
                        plgx[w2] = pack_h2(lg[0], lg[1]);
                        range = fmaxf(range, fmaxf(fmaxf(fabsf(lc[0]), fabsf(lc[1])), fmaxf(fabsf(lg[0]), fabsf(lg[1]))));
                    }
                    const uint32_t off = sw128_off(r, 2 * cq + q8);
                    *reinterpret_cast<uint4*>(sm + OFF_LCB + off) = make_uint4(plcb[0], plcb[1], plcb[2], plcb[3]);
                    *reinterpret_cast<uint4*>(sm + OFF_LGX + off) = make_uint4(plgx[0], plgx[1], plgx[2], plgx[3]);
                }
                fence_async_smem();
                mbar_arrive(&bars[LT_FULL]);
                if (!(range < 65504.f)) atomicOr(&g_chunk_bwd_tc_error, 2);
                // the scalar warp is done with the previous head's partial sums before these are written
                if (k > 0 && !wait_all(&bars[SCALAR_FREE], (k - 1) & 1, abort)) {
                    ok = false;
                    break;
                }
                const float col = column_sums16(gx, lane);
                if (lane < 16) vec[(V_COL >> 2) + (par * 2 + rq) * 64 + c0 + lane] = col;
            }
            vec[(V_ROWM >> 2) + (par * 4 + cq) * 64 + r] = rowm;
            // E partial (g . SPC) and sum g . x over this thread's columns, once SPC is there (B1_DONE)
            if (!wait_all(&bars[B1_DONE], par, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float pd = 0.f;
            {
                float spc[16];
                tmem_ld16(tmem + lb + COL_SPC + c0, spc);
                tmem_wait_ld();
                float e = 0.f;
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    float gq[8], xq[8];
                    unpack8(bo + B_G, r, 2 * cq + q8, gq);
                    unpack8(bo + B_X, r, 2 * cq + q8, xq);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        e += gq[q] * spc[8 * q8 + q] * isp[8 * q8 + q];
                        pd += gq[q] * xq[q];
                    }
                }
                vec[(V_E >> 2) + (par * 4 + cq) * 64 + r] = e;
            }
            if (!wait_all(&bars[B2_DONE], par, abort)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // phase C: dz from the recomputed y; dx; W
            const float ex_r = r < Qv ? expf(cs_r) : 0.f, el_r = r < Qv ? expf(cs_last - cs_r) : 0.f;
            {
                float yin[16], spc[16];
                tmem_ld16(tmem + lb + COL_YIN + c0, yin);
                tmem_ld16(tmem + lb + COL_SPC + c0, spc);
                tmem_wait_ld();
                float* dz = a.dz + (row0 + r) * HP + (int64_t)h * kPb + c0;
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    float xq[8], dq[8], o[8];
                    unpack8(bo + B_X, r, 2 * cq + q8, xq);
                    unpack8(bo + B_DS, r, 2 * cq + q8, dq);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int qq = 8 * q8 + q;
                        o[q] = dq[q] * (yin[qq] + ex_r * isp[qq] * spc[qq] + Dh * xq[q]);
                    }
                    if (r < Qv) {
                        *reinterpret_cast<float4*>(dz + 8 * q8) = make_float4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<float4*>(dz + 8 * q8 + 4) = make_float4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
            float wpart = 0.f;
            {
                float lmb[16], dxi[16];
                tmem_ld16(tmem + lb + COL_LMB + c0, lmb);
                tmem_ld16(tmem + lb + COL_DXI + c0, dxi);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&bars[ACC_FREE]);  // the head's last TMEM read: the next head's MMAs may start
                const float f = dt_r * el_r;
                float* du = a.DU + (row0 + r) * conv_dim + (int64_t)h * kPb + c0;
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    float xq[8], gq[8], o[8];
                    unpack8(bo + B_X, r, 2 * cq + q8, xq);
                    unpack8(bo + B_G, r, 2 * cq + q8, gq);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int qq = 8 * q8 + q;
                        const float lm = lmb[qq] * ilm[qq];
                        o[q] = dxi[qq] + f * lm + Dh * gq[q];
                        wpart += xq[q] * lm;
                    }
                    if (r < Qv) {
                        *reinterpret_cast<float4*>(du + 8 * q8) = make_float4(o[0], o[1], o[2], o[3]);
                        *reinterpret_cast<float4*>(du + 8 * q8 + 4) = make_float4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
            vec[(V_W >> 2) + (par * 4 + cq) * 64 + r] = el_r * wpart;
            pd = warp_sum(pd);
            if (lane == 0) vec[(V_PD >> 2) + par * 8 + wi] = pd;
            mbar_arrive(&bars[WSYNC]);
            mbar_arrive(&bars[TILE_FREE0 + buf]);
        }
        if (!ok) give_up(abort);
    }

    // every role is done issuing; dB^T and dC^T are final once the last MMAs complete
    const bool done = __all_sync(0xffffffffu, mbar_wait(&bars[FINAL], 0, nullptr));
    tc_fence_after();
    __syncthreads();
    if (warp < 8 && done && *abort == 0) {
        const int n = 32 * (warp & 3) + lane, j0 = 32 * (warp >> 2);
        const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
        float db[32], dc[32];
        tmem_ld32(tmem + lb + COL_DB + j0, db);
        tmem_ld32(tmem + lb + COL_DC + j0, dc);
        tmem_wait_ld();
        if (n < N) {
            for (int q = 0; q < 32; ++q) {
                const int j = j0 + q;
                if (j < Qv) {
                    float* dst = half == 0 ? a.DU + (row0 + j) * conv_dim + HP : a.DU2 + (row0 + j) * 2 * GN;
                    dst[(int64_t)g * N + n] = db[q];
                    dst[GN + (int64_t)g * N + n] = dc[q];
                }
            }
        }
    } else if (tid == 0 && !done) {
        atomicOr(&g_chunk_bwd_tc_error, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS_B);
    }
}

}  // namespace

bool chunk_bwd_tc_supported(int P, int N, bool act_bf16, const void* dy, const void* z, const void* dz) {
    const uintptr_t bits = reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(z) |
                           reinterpret_cast<uintptr_t>(dz);
    return act_bf16 && P == kPb && (N == 64 || N == 128) && (bits & 15u) == 0;
}

cudaError_t read_and_clear_chunk_bwd_tc_error(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_chunk_bwd_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_chunk_bwd_tc_error, &zero, sizeof(int));
}

cudaError_t launch_chunk_bwd_tc(const ChunkBwdTcArgs& a, int64_t nchunks, cudaStream_t st) {
    if (a.nsplit_pf != kSplitPf || !a.act_bf16) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_B);
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(nchunks), static_cast<unsigned>(a.G * a.split),
                    static_cast<unsigned>(a.batch));
    chunk_bwd_tc_kernel<<<grid, kThreadsB, SMEM_B, st>>>(a);
    return cudaGetLastError();
}

}  // namespace bwd
}  // namespace ssd
