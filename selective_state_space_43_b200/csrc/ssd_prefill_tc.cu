// ssd_prefill_tc.cu -- chunked SSD prefill on the sm_100a tensor cores.
//
// Mamba-2's state-space duality splits the scan into chunks of Q tokens:
// inside a chunk the layer is a causal, decay-masked attention-like product,
// across chunks one P x N state per head is passed on ("EP6. 트랜스포머 대체
// 신경망 연구" §7-§8; chunk_size 128 and the layer sizes from "Nemotron-H 스타일
// Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석" table 1.4).  Per chunk c,
// head h (group g), with u = SiLU(conv4 + b) of the x / B / C channels,
// cs = inclusive cumsum of dt*A inside the chunk:
//   G      = C_c B_c^T                                   [Q x Q]  (tcgen05, K = N)
//   M[i,j] = G[i,j] exp(cs_i - cs_j) dt_j   (j <= i)     [Q x Q]  (CUDA cores)
//   Y      = M X_c                                       [Q x P]  (tcgen05, K = Q)
//   Y2     = C_c S_prev^T                                [Q x P]  (tcgen05, K = N)
//   S_c^T  = B_c^T X'_c,  X'_j = exp(cs_last - cs_j) dt_j x_j     [N x P]  (tcgen05, K = Q)
//   y      = (Y + exp(cs_i) Y2 + D x) SiLU(z)
//   S_prev <- exp(cs_last) S_prev + S_c
//
// Two kernels:
//   bc_prologue  SiLU(conv4) of the B and C channels of every token, written
//                once per group to the workspace in bf16 (the 16 heads of a
//                group then read it from L2 instead of recomputing it), and
//                the conv_state tail of all channels.
//   chunk_scan   one CTA per (sequence b, head h) walks the chunks in order;
//                all accumulators live in TMEM; 7 warps:
//                  warp 0  TMA producer: raw x and z tiles (2-stage ring)
//                  warp 1  TMEM allocator + single-thread tcgen05.mma issuer
//                  warp 2  TMA producer: post-conv B and C tiles
//                  warps 3-6  128 compute threads, thread i <-> token row i
//                           <-> TMEM lane i: x conv, decay mask, state pass,
//                           epilogue (D skip, z gate, y store).
// Every mbarrier wait is bounded; a wait that gives up raises a device error
// flag (read back by ssd_device_status) and the CTA drains and exits.
#include <cuda.h>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_sm100.cuh"

namespace ssd {

__device__ int g_tc_error = 0;  // set by a chunk_scan CTA whose bounded wait gave up

namespace {

using namespace sm100;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr int kThreads = 224;
constexpr int kWarpRaw = 0, kWarpMma = 1, kWarpBc = 2, kFirstCompute = 3;
constexpr int kComputeThreads = 128;

// shared memory map (bytes from a 1024-byte aligned base)
constexpr uint32_t OFF_C = 0;          // u_C tile: two boxes [128 tok][64 n] bf16, 128B swizzle
constexpr uint32_t OFF_B = 32768;      // u_B tile
constexpr uint32_t OFF_X = 65536;      // X  [j][p] bf16 (MN-major B operand)
constexpr uint32_t OFF_XP = 81920;     // X' [j][p] bf16
constexpr uint32_t OFF_M = 98304;      // M  [i][j] bf16, two K blocks of 64 (K-major A operand)
constexpr uint32_t OFF_S = 131072;     // S_prev [n][p] bf16 (MN-major B operand)
constexpr uint32_t OFF_RAWX = 147456;  // 2 x raw x tile [tok][p] bf16 (TMA, 128B swizzle)
constexpr uint32_t OFF_RAWZ = 180224;  // 2 x raw z tile
constexpr uint32_t OFF_SMALL = 212992;
// small region
constexpr uint32_t OFF_W = OFF_SMALL;              // conv taps of the head's x channels  [64] float4
constexpr uint32_t OFF_CB = OFF_W + 64 * 16;       // conv bias [64] float
constexpr uint32_t OFF_HALO = OFF_CB + 64 * 4;     // [2][3][64] bf16 raw x history
constexpr uint32_t OFF_CS = OFF_HALO + 2 * 3 * 64 * 2;  // cs [128] float
constexpr uint32_t OFF_DT = OFF_CS + 128 * 4;      // dt [128] float
constexpr uint32_t OFF_WTOT = OFF_DT + 128 * 4;    // warp totals of the dA scan [4] float
constexpr uint32_t OFF_BAR = OFF_WTOT + 16;        // mbarriers (8 B each)
constexpr int NBAR = 13;
constexpr uint32_t OFF_TMEM = OFF_BAR + NBAR * 8;  // TMEM base address
constexpr uint32_t OFF_ABORT = OFF_TMEM + 4;
constexpr uint32_t SMEM_USED = OFF_ABORT + 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

enum Bar { FULL_RAW0 = 0, FULL_RAW1, EMPTY_RAW0, EMPTY_RAW1, FULL_BC, EMPTY_BC, XREADY, MREADY, G_FULL, SC_FULL,
           Y_FULL, MMA_DONE, COMPUTE_SYNC };

// TMEM columns (fp32 accumulators, 128 lanes)
constexpr uint32_t COL_G = 0, COL_Y = 128, COL_Y2 = 192, COL_SC = 256, COL_SRUN = 320, TMEM_COLS = 512;

struct TcParams {
    PrefillArgs a;
    CUtensorMap tm_x, tm_z, tm_bc;
};

// Barrier among the 128 compute threads, on an mbarrier so that it is bounded
// like every other wait (a named barrier could not give up).
__device__ __forceinline__ bool compute_sync(uint64_t* bar, uint32_t& phase, volatile int* abort_flag) {
    mbar_arrive(bar);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, phase, abort_flag));
    phase ^= 1u;
    return ok;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// A compute warp proceeds only if every lane saw the phase complete, so that the
// warp-collective tcgen05.ld / st that follow are never reached by part of a warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_tc_error, 1);
}

template <typename TY>
__global__ void __launch_bounds__(kThreads, 1) chunk_scan_kernel(const __grid_constant__ TcParams prm) {
    const PrefillArgs& a = prm.a;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_ABORT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int g = h / a.hpg;
    const int nc = (int)a.nchunks;

    if (threadIdx.x == 0) {
        mbar_init(&bars[FULL_RAW0], 1);
        mbar_init(&bars[FULL_RAW1], 1);
        mbar_init(&bars[EMPTY_RAW0], kComputeThreads);
        mbar_init(&bars[EMPTY_RAW1], kComputeThreads);
        mbar_init(&bars[FULL_BC], 1);
        mbar_init(&bars[EMPTY_BC], 1);
        mbar_init(&bars[XREADY], kComputeThreads);
        mbar_init(&bars[MREADY], kComputeThreads);
        mbar_init(&bars[G_FULL], 1);
        mbar_init(&bars[SC_FULL], 1);
        mbar_init(&bars[Y_FULL], 1);
        mbar_init(&bars[MMA_DONE], 1);
        mbar_init(&bars[COMPUTE_SYNC], kComputeThreads);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp >= kFirstCompute) {
        const int i = threadIdx.x - kFirstCompute * 32;
        if (i < kP) {
            const int ch = h * kP + i;
            reinterpret_cast<float4*>(sm + OFF_W)[i] = *reinterpret_cast<const float4*>(a.conv_w + (size_t)ch * 4);
            reinterpret_cast<float*>(sm + OFF_CB)[i] = a.conv_b[ch];
            // conv history of token 0: the initial conv state (tokens -3..-1) or zeros
            __nv_bfloat16* halo = reinterpret_cast<__nv_bfloat16*>(sm + OFF_HALO);
            for (int k = 0; k < 3; ++k) {
                __nv_bfloat16 v = __float2bfloat16_rn(0.f);
                if (a.init_conv_state)
                    v = static_cast<const __nv_bfloat16*>(a.init_conv_state)[((size_t)b * a.conv_dim + ch) * 3 + k];
                halo[k * 64 + i] = v;
            }
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == kWarpRaw) {
        // ---------------- raw x / z producer ----------------
        if (lane == 0) {
            prefetch_tmap(&prm.tm_x);
            prefetch_tmap(&prm.tm_z);
            int issued[2] = {-1, -1};
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !mbar_wait(&bars[EMPTY_RAW0 + s], ((c >> 1) + 1) & 1, abort_flag)) {
                    raise_abort(abort_flag);
                    break;
                }
                mbar_arrive_expect_tx(&bars[FULL_RAW0 + s], 2 * 16384);
                tma_load_3d(sm + OFF_RAWX + s * 16384, &prm.tm_x, &bars[FULL_RAW0 + s], h * kP, c * kQ, b);
                tma_load_3d(sm + OFF_RAWZ + s * 16384, &prm.tm_z, &bars[FULL_RAW0 + s], h * kP, c * kQ, b);
                issued[s] = c;
            }
            if (*abort_flag) {  // let copies still in flight land before the CTA exits
                for (int s = 0; s < 2; ++s)
                    if (issued[s] >= 0) mbar_wait(&bars[FULL_RAW0 + s], (issued[s] >> 1) & 1, nullptr, 100000000ull);
            }
        }
    } else if (warp == kWarpBc) {
        // ---------------- post-conv B / C producer ----------------
        if (lane == 0) {
            prefetch_tmap(&prm.tm_bc);
            int last = -1;
            for (int c = 0; c < nc; ++c) {
                if (c >= 1 && !mbar_wait(&bars[EMPTY_BC], (c - 1) & 1, abort_flag)) {
                    raise_abort(abort_flag);
                    break;
                }
                mbar_arrive_expect_tx(&bars[FULL_BC], 4 * 16384);
                const int xc = a.GN + g * kN, xb = g * kN;
                tma_load_3d(sm + OFF_C, &prm.tm_bc, &bars[FULL_BC], xc, c * kQ, b);
                tma_load_3d(sm + OFF_C + 16384, &prm.tm_bc, &bars[FULL_BC], xc + 64, c * kQ, b);
                tma_load_3d(sm + OFF_B, &prm.tm_bc, &bars[FULL_BC], xb, c * kQ, b);
                tma_load_3d(sm + OFF_B + 16384, &prm.tm_bc, &bars[FULL_BC], xb + 64, c * kQ, b);
                last = c;
            }
            if (*abort_flag && last >= 0) mbar_wait(&bars[FULL_BC], last & 1, nullptr, 100000000ull);
        }
    } else if (warp == kWarpMma) {
        // ---------------- tcgen05.mma issuer ----------------
        if (lane == 0) {
            constexpr uint32_t ID_G = idesc_bf16_f32(128, 128, false, false);   // C (K-major) x B (K-major)
            constexpr uint32_t ID_Y = idesc_bf16_f32(128, 64, false, true);     // M (K-major) x X (MN-major)
            constexpr uint32_t ID_Y2 = idesc_bf16_f32(128, 64, false, true);    // C (K-major) x S (MN-major)
            constexpr uint32_t ID_SC = idesc_bf16_f32(128, 64, true, true);     // B^T (MN-major) x X' (MN-major)
            const uint32_t sC = smem_u32(sm + OFF_C), sB = smem_u32(sm + OFF_B);
            const uint32_t sX = smem_u32(sm + OFF_X), sXp = smem_u32(sm + OFF_XP);
            const uint32_t sM = smem_u32(sm + OFF_M), sS = smem_u32(sm + OFF_S);
            for (int c = 0; c < nc; ++c) {
                if (!mbar_wait(&bars[FULL_BC], c & 1, abort_flag)) { raise_abort(abort_flag); break; }
                if (c >= 1 && !mbar_wait(&bars[MREADY], (c - 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tmem + COL_G, sw128_desc(sC + koff, 16, 1024), sw128_desc(sB + koff, 16, 1024), ID_G,
                             kk > 0);
                }
                mma_commit(&bars[G_FULL]);
                if (!mbar_wait(&bars[XREADY], c & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tmem + COL_Y2, sw128_desc(sC + koff, 16, 1024), sw128_desc(sS + kk * 2048, 16384, 1024),
                             ID_Y2, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_bf16(tmem + COL_SC, sw128_desc(sB + kk * 2048, 16384, 1024),
                             sw128_desc(sXp + kk * 2048, 16384, 1024), ID_SC, kk > 0);
                }
                mma_commit(&bars[SC_FULL]);
                mma_commit(&bars[EMPTY_BC]);
                if (!mbar_wait(&bars[MREADY], c & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (kk >> 2) * 16384 + (kk & 3) * 32;
                    mma_bf16(tmem + COL_Y, sw128_desc(sM + koff, 16, 1024), sw128_desc(sX + kk * 2048, 16384, 1024),
                             ID_Y, kk > 0);
                }
                mma_commit(&bars[Y_FULL]);
            }
            // nothing may still be running on the tensor cores when TMEM is released
            mma_commit(&bars[MMA_DONE]);
            mbar_wait(&bars[MMA_DONE], 0, nullptr, 100000000ull);
        }
    } else {
        // ---------------- compute warps ----------------
        const int q = warp & 3;                       // TMEM lane quadrant of this warp
        const int i = q * 32 + lane;                  // token row / TMEM lane / state row n
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float A = a.A[h], Dh = a.D[h], dtb = a.dt_bias[h];
        const __nv_bfloat16* dtp = static_cast<const __nv_bfloat16*>(a.dt);
        float* s_cs = reinterpret_cast<float*>(sm + OFF_CS);
        float* s_dt = reinterpret_cast<float*>(sm + OFF_DT);
        float* s_wtot = reinterpret_cast<float*>(sm + OFF_WTOT);
        const float4* s_w = reinterpret_cast<const float4*>(sm + OFF_W);
        const float* s_cb = reinterpret_cast<const float*>(sm + OFF_CB);
        uint8_t* sX = sm + OFF_X;
        uint8_t* sXp = sm + OFF_XP;
        uint8_t* sMm = sm + OFF_M;
        uint8_t* sS = sm + OFF_S;

        // initial state: S_run (TMEM, fp32) and its bf16 copy (smem) for the first chunk's C S^T
        {
            const float* init = a.init_state ? a.init_state + ((size_t)b * a.H + h) * kP * kN : nullptr;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float v[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) v[k] = init ? init[(size_t)(half * 32 + k) * kN + i] : 0.f;
                tmem_st32(tmem + lane_base + COL_SRUN + half * 32, v);
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint4 w;
                    w.x = pack_bf2(v[k4 * 8 + 0], v[k4 * 8 + 1]);
                    w.y = pack_bf2(v[k4 * 8 + 2], v[k4 * 8 + 3]);
                    w.z = pack_bf2(v[k4 * 8 + 4], v[k4 * 8 + 5]);
                    w.w = pack_bf2(v[k4 * 8 + 6], v[k4 * 8 + 7]);
                    *reinterpret_cast<uint4*>(sS + sw128_off(i, half * 4 + k4)) = w;
                }
            }
            tmem_wait_st();
        }

        float u[kP];  // post-conv x of row i, kept for the D skip
        bool ok = true;
        uint32_t sync_phase = 0;
        for (int c = 0; c < nc && ok; ++c) {
            const int s = c & 1;
            const int64_t t0 = (int64_t)c * kQ;
            const int Qc = (int)(a.L - t0 < kQ ? a.L - t0 : kQ);
            const bool valid = i < Qc;

            // (b) dt, in-chunk inclusive cumsum of dt*A
            float dtv = 0.f, dA = 0.f;
            if (valid) {
                dtv = softplus_f(__bfloat162float(dtp[((size_t)b * a.L + t0 + i) * a.H + h]) + dtb);
                dA = dtv * A;
            }
            float inc = dA;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += up;
            }
            if (lane == 31) s_wtot[q] = inc;
            if (!compute_sync(&bars[COMPUTE_SYNC], sync_phase, abort_flag)) { raise_abort(abort_flag); ok = false; break; }
            float off = 0.f;
            for (int k = 0; k < q; ++k) off += s_wtot[k];
            const float cs_i = inc + off;
            const float cs_last = s_wtot[0] + s_wtot[1] + s_wtot[2] + s_wtot[3];
            s_cs[i] = cs_i;
            s_dt[i] = dtv;
            const float wx = valid ? __expf(cs_last - cs_i) * dtv : 0.f;  // weight of x_i in the chunk state
            const float ecs = __expf(cs_i);                               // decay of S_prev up to row i

            // (c) raw x tile -> conv + SiLU -> X, X'
            if (!warp_wait(&bars[FULL_RAW0 + s], (c >> 1) & 1, abort_flag)) { raise_abort(abort_flag); ok = false; break; }
            const uint8_t* rx = sm + OFF_RAWX + s * 16384;
            const __nv_bfloat16* halo_in = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_HALO) + (c & 1) * 192;
#pragma unroll
            for (int k8 = 0; k8 < 8; ++k8) {  // 8 channels (16 bytes) at a time
                float acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = s_cb[k8 * 8 + e];
#pragma unroll
                for (int tap = 0; tap < 4; ++tap) {
                    const int r = i - 3 + tap;
                    uint4 w;
                    if (r >= 0) {
                        w = *reinterpret_cast<const uint4*>(rx + sw128_off(r, k8));
                    } else {
                        w = *reinterpret_cast<const uint4*>(halo_in + (r + 3) * 64 + k8 * 8);
                    }
                    const float xv[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                                         bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 wt = s_w[k8 * 8 + e];
                        const float tw = tap == 0 ? wt.x : (tap == 1 ? wt.y : (tap == 2 ? wt.z : wt.w));
                        acc[e] = fmaf(tw, xv[e], acc[e]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) u[k8 * 8 + e] = valid ? silu_f(acc[e]) : 0.f;
                uint4 o1, o2;
                o1.x = pack_bf2(u[k8 * 8 + 0], u[k8 * 8 + 1]);
                o1.y = pack_bf2(u[k8 * 8 + 2], u[k8 * 8 + 3]);
                o1.z = pack_bf2(u[k8 * 8 + 4], u[k8 * 8 + 5]);
                o1.w = pack_bf2(u[k8 * 8 + 6], u[k8 * 8 + 7]);
                o2.x = pack_bf2(u[k8 * 8 + 0] * wx, u[k8 * 8 + 1] * wx);
                o2.y = pack_bf2(u[k8 * 8 + 2] * wx, u[k8 * 8 + 3] * wx);
                o2.z = pack_bf2(u[k8 * 8 + 4] * wx, u[k8 * 8 + 5] * wx);
                o2.w = pack_bf2(u[k8 * 8 + 6] * wx, u[k8 * 8 + 7] * wx);
                *reinterpret_cast<uint4*>(sX + sw128_off(i, k8)) = o1;
                *reinterpret_cast<uint4*>(sXp + sw128_off(i, k8)) = o2;
            }
            if (i >= kQ - 3) {  // raw history of the next chunk
                __nv_bfloat16* halo_out = reinterpret_cast<__nv_bfloat16*>(sm + OFF_HALO) + ((c + 1) & 1) * 192;
#pragma unroll
                for (int k8 = 0; k8 < 8; ++k8)
                    *reinterpret_cast<uint4*>(halo_out + (i - (kQ - 3)) * 64 + k8 * 8) =
                        *reinterpret_cast<const uint4*>(rx + sw128_off(i, k8));
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[XREADY]);
            // s_cs / s_dt of this chunk visible to every compute thread
            if (!compute_sync(&bars[COMPUTE_SYNC], sync_phase, abort_flag)) { raise_abort(abort_flag); ok = false; break; }

            // (e) decay mask: M[i, j] = G[i, j] exp(cs_i - cs_j) dt_j for j <= i
            if (!warp_wait(&bars[G_FULL], c & 1, abort_flag)) { raise_abort(abort_flag); ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {  // 32 columns j at a time
                uint32_t packed[16];
                if (kb <= q) {  // warp-uniform: blocks right of the diagonal are all zero
                    float gv[32];
                    tmem_ld32(tmem + lane_base + COL_G + kb * 32, gv);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int j = kb * 32 + e;
                        const float m0 = j <= i ? gv[e] * __expf(cs_i - s_cs[j]) * s_dt[j] : 0.f;
                        const float m1 = j + 1 <= i ? gv[e + 1] * __expf(cs_i - s_cs[j + 1]) * s_dt[j + 1] : 0.f;
                        packed[e >> 1] = pack_bf2(m0, m1);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 16; ++e) packed[e] = 0u;
                }
                uint8_t* mrow = sMm + (kb >> 1) * 16384;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int chunk = (kb & 1) * 4 + k4;
                    *reinterpret_cast<uint4*>(mrow + sw128_off(i, chunk)) =
                        make_uint4(packed[k4 * 4 + 0], packed[k4 * 4 + 1], packed[k4 * 4 + 2], packed[k4 * 4 + 3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[MREADY]);

            // (f) state passing: S_run <- exp(cs_last) S_run + S_c  (lane i = state row n)
            if (!warp_wait(&bars[SC_FULL], c & 1, abort_flag)) { raise_abort(abort_flag); ok = false; break; }
            tc_fence_after();
            {
                const float dl = __expf(cs_last);
                const bool last = c == nc - 1;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float sc[32], sr[32];
                    tmem_ld32(tmem + lane_base + COL_SC + half * 32, sc);
                    tmem_ld32(tmem + lane_base + COL_SRUN + half * 32, sr);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) sr[k] = fmaf(dl, sr[k], sc[k]);
                    tmem_st32(tmem + lane_base + COL_SRUN + half * 32, sr);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        uint4 w;
                        w.x = pack_bf2(sr[k4 * 8 + 0], sr[k4 * 8 + 1]);
                        w.y = pack_bf2(sr[k4 * 8 + 2], sr[k4 * 8 + 3]);
                        w.z = pack_bf2(sr[k4 * 8 + 4], sr[k4 * 8 + 5]);
                        w.w = pack_bf2(sr[k4 * 8 + 6], sr[k4 * 8 + 7]);
                        *reinterpret_cast<uint4*>(sS + sw128_off(i, half * 4 + k4)) = w;
                    }
                    if (last) {
                        float* fs = a.final_state + ((size_t)b * a.H + h) * kP * kN;
#pragma unroll
                        for (int k = 0; k < 32; ++k) fs[(size_t)(half * 32 + k) * kN + i] = sr[k];
                    }
                }
                tmem_wait_st();
            }

            // (g) epilogue: y = (Y + exp(cs_i) Y2 + D x) SiLU(z)
            if (!warp_wait(&bars[Y_FULL], c & 1, abort_flag)) { raise_abort(abort_flag); ok = false; break; }
            tc_fence_after();
            {
                const uint8_t* rz = sm + OFF_RAWZ + s * 16384;
                TY* yrow = static_cast<TY*>(a.y) + ((size_t)b * a.L + t0 + i) * a.HP + (size_t)h * kP;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float y1[32], y2[32];
                    tmem_ld32(tmem + lane_base + COL_Y + half * 32, y1);
                    tmem_ld32(tmem + lane_base + COL_Y2 + half * 32, y2);
                    tmem_wait_ld();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const uint4 zw = *reinterpret_cast<const uint4*>(rz + sw128_off(i, half * 4 + k4));
                        const float zv[8] = {bf_lo(zw.x), bf_hi(zw.x), bf_lo(zw.y), bf_hi(zw.y),
                                             bf_lo(zw.z), bf_hi(zw.z), bf_lo(zw.w), bf_hi(zw.w)};
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int k = k4 * 8 + e;
                            const float yv = fmaf(ecs, y2[k], y1[k]) + Dh * u[half * 32 + k];
                            o[e] = yv * silu_f(zv[e]);
                        }
                        if (valid) {
                            if constexpr (sizeof(TY) == 2) {
                                uint4 w;
                                w.x = pack_bf2(o[0], o[1]);
                                w.y = pack_bf2(o[2], o[3]);
                                w.z = pack_bf2(o[4], o[5]);
                                w.w = pack_bf2(o[6], o[7]);
                                *reinterpret_cast<uint4*>(yrow + half * 32 + k4 * 8) = w;
                            } else {
                                float4* dst = reinterpret_cast<float4*>(yrow + half * 32 + k4 * 8);
                                dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                                dst[1] = make_float4(o[4], o[5], o[6], o[7]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars[EMPTY_RAW0 + s]);
        }
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// SiLU(conv4) of the B and C channels into the workspace [b][t][2][G*N] (bf16),
// plus the conv_state tail of every channel.  Block: 256 threads = 256 channel
// pairs of one token block; each thread slides a 4-tap window along 64 tokens.
constexpr int kProTok = 64;

__global__ void __launch_bounds__(256) bc_prologue_kernel(PrefillArgs a) {
    const int64_t b = blockIdx.y;
    const int64_t t0 = (int64_t)blockIdx.x * kProTok;
    const int pairs = a.GN;  // (2 arrays x GN channels) / 2 per pair
    const int pair = blockIdx.z * 256 + threadIdx.x;
    const __nv_bfloat16* hist = static_cast<const __nv_bfloat16*>(a.init_conv_state);
    if (pair < pairs) {
        const int sel = pair >= a.GN / 2;                      // 0 = B, 1 = C
        const int ch0 = (pair - sel * (a.GN / 2)) * 2;         // channel within the array
        const int cglob = a.HP + sel * a.GN + ch0;             // conv channel index
        const uint32_t* src = static_cast<const uint32_t*>(sel ? a.C : a.B);
        uint32_t* dst = static_cast<uint32_t*>(a.workspace);
        const float4 w0 = *reinterpret_cast<const float4*>(a.conv_w + (size_t)cglob * 4);
        const float4 w1 = *reinterpret_cast<const float4*>(a.conv_w + (size_t)(cglob + 1) * 4);
        const float b0 = a.conv_b[cglob], b1 = a.conv_b[cglob + 1];
        float h0[3], h1[3];  // window: tokens t-3, t-2, t-1
#pragma unroll
        for (int k = 0; k < 3; ++k) {
            const int64_t t = t0 - 3 + k;
            if (t >= 0) {
                const uint32_t v = src[((size_t)b * a.L + t) * (a.GN / 2) + ch0 / 2];
                h0[k] = bf_lo(v);
                h1[k] = bf_hi(v);
            } else if (hist) {
                h0[k] = __bfloat162float(hist[((size_t)b * a.conv_dim + cglob) * 3 + (t + 3)]);
                h1[k] = __bfloat162float(hist[((size_t)b * a.conv_dim + cglob + 1) * 3 + (t + 3)]);
            } else {
                h0[k] = h1[k] = 0.f;
            }
        }
        const int64_t tend = t0 + kProTok < a.L ? t0 + kProTok : a.L;
        for (int64_t t = t0; t < tend; ++t) {
            const uint32_t v = src[((size_t)b * a.L + t) * (a.GN / 2) + ch0 / 2];
            const float x0 = bf_lo(v), x1 = bf_hi(v);
            const float p0 = b0 + w0.x * h0[0] + w0.y * h0[1] + w0.z * h0[2] + w0.w * x0;
            const float p1 = b1 + w1.x * h1[0] + w1.y * h1[1] + w1.z * h1[2] + w1.w * x1;
            dst[(((size_t)b * a.L + t) * 2 + sel) * (a.GN / 2) + ch0 / 2] = pack_bf2(silu_f(p0), silu_f(p1));
            h0[0] = h0[1]; h0[1] = h0[2]; h0[2] = x0;
            h1[0] = h1[1]; h1[1] = h1[2]; h1[2] = x1;
        }
    }
    // conv_state tail (pre-conv inputs of tokens L-3..L-1) for every channel, by the last token block
    if (blockIdx.x == gridDim.x - 1 && blockIdx.z == 0) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.conv_state);
        for (int c = threadIdx.x; c < a.conv_dim; c += 256) {
            for (int k = 0; k < 3; ++k) {
                const int64_t t = a.L - 3 + k;
                __nv_bfloat16 v;
                if (t >= 0) {
                    if (c < a.HP) v = static_cast<const __nv_bfloat16*>(a.x)[((size_t)b * a.L + t) * a.HP + c];
                    else if (c < a.HP + a.GN)
                        v = static_cast<const __nv_bfloat16*>(a.B)[((size_t)b * a.L + t) * a.GN + (c - a.HP)];
                    else
                        v = static_cast<const __nv_bfloat16*>(a.C)[((size_t)b * a.L + t) * a.GN + (c - a.HP - a.GN)];
                } else {
                    v = hist ? hist[((size_t)b * a.conv_dim + c) * 3 + (t + 3)] : __float2bfloat16_rn(0.f);
                }
                out[((size_t)b * a.conv_dim + c) * 3 + k] = v;
            }
        }
    }
}

// ---- host side ------------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 map over [batch][L][width] with a [1][128][64] box and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t width, int64_t L, int64_t batch) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)width * 2, (cuuint64_t)(width * L * 2)};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int P, int N, int Q, bool bf16) { return bf16 && P == kP && N == kN && Q == kQ; }

size_t prefill_tc_workspace_bytes(int64_t batch, int64_t L, int G, int N) {
    return (size_t)batch * (size_t)L * 2 * (size_t)G * (size_t)N * 2;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, ActKind kind, cudaStream_t st, const TimingHook& hook) {
    if (a.L == 0) return launch_prefill_simt(a, kind, st, hook);  // nothing to scan: states pass through
    TcParams prm;
    prm.a = a;
    if (!make_map(&prm.tm_x, a.x, a.HP, a.L, a.batch) || !make_map(&prm.tm_z, a.z, a.HP, a.L, a.batch) ||
        !make_map(&prm.tm_bc, a.workspace, 2 * a.GN, a.L, a.batch))
        return cudaErrorInvalidValue;
    const dim3 pgrid((unsigned)((a.L + kProTok - 1) / kProTok), (unsigned)a.batch, (unsigned)((a.GN + 255) / 256));
    bc_prologue_kernel<<<pgrid, 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto kern = kind == ActKind::BF16_YF32 ? chunk_scan_kernel<float> : chunk_scan_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    hook.before(st);
    kern<<<(unsigned)(a.batch * a.H), kThreads, SMEM_BYTES, st>>>(prm);
    hook.after(st);
    return cudaGetLastError();
}

cudaError_t read_and_clear_tc_error(int* flag, cudaStream_t st) {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(flag, g_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

}  // namespace ssd
