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
// Two kernels (the second launched with programmatic dependent launch):
//   bc_prologue  SiLU(conv4) of the B and C channels of every token, written
//                once per group to the workspace in bf16 (the 16 heads of a
//                group then read it from L2 instead of recomputing it);
//                The same launch writes the conv_state output (last 3 pre-conv
//                tokens of every channel).
//   chunk_scan   one CTA per (sequence b, head h) walks the chunks in order;
//                all accumulators live in TMEM; 20 warps:
//                  warp 0  TMA producer: raw x tiles two chunks ahead (2-stage
//                           ring), z of the current chunk (one buffer, which
//                           the epilogue overwrites with y for the TMA store)
//                  warp 1  TMEM allocator + single-thread tcgen05.mma issuer
//                  warp 2  each chunk's dt and cumsum of dt*A one chunk ahead
//                           (double-buffered), from a raw dt tile that warp 0
//                           loads with the chunk's raw x; then the chunk's
//                           decay tables, once the previous chunk's mask is done
//                  warp 3  TMA producer: post-conv B and C tiles
//                  warps 4-11  group A, two threads per token row i (= TMEM
//                           lane i), each owning two 8-column groups of each of
//                           the 4 decay-mask column blocks and 32 output
//                           columns: the decay mask of chunk c, then its
//                           epilogue (D skip, z gate, y store)
//                  warps 12-19 group B, two threads per row: the x conv of
//                           chunk c+1 (32 channels each; fp32 output kept in
//                           TMEM for the D skip), then the state pass of chunk
//                           c+1 (32 state columns of row n = i)
//                The two groups run a chunk apart, so the mask / epilogue of one
//                chunk overlaps the conv / state pass of the next instead of all
//                16 warps walking the four phases in lock step.  Elementwise
//                math uses the packed fp32x2 FMA / MUL of sm_100.
// The decay exp(cs_i - cs_j) dt_j of M is assembled from tables that the
// cumsum warp writes for each chunk, so the mask itself needs no MUFU work.
// With g(i) the 8-row group of i and cs_end(g) the cumsum at the group's last
// row: inside a group an exact table exp(cs_i - cs_j) dt_j; below it the
// product exp(cs_i - cs_end(g(i)-1)) exp(cs_end(g(i)-1) - cs_end(g(j)))
// exp(cs_end(g(j)) - cs_j) dt_j.  With A < 0 the cumsum does not increase, so
// every factor is <= 1: none overflows, and one underflows only where the true
// product is below ~1e-38.
// Every mbarrier wait is bounded; a wait that gives up raises a device error
// flag (read back by ssd_device_status) and the CTA drains and exits.
#include <cuda.h>

#include <mutex>

#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_sm100.cuh"

namespace ssd {

__device__ int g_tc_error = 0;  // device error word: kErrTimeout | kErrBadSeqlens

namespace {

using namespace sm100;

constexpr int kQ = 128, kP = 64, kN = 128;
constexpr int kThreads = 640;
// Warp w issues from scheduler w % 4, which it shares with the compute warps of TMEM lane quadrant w % 4.
// The causal mask gives quadrant q (rows 32q .. 32q + 31) about q + 1 times quadrant 0's work, so the
// busiest single-warp role (the cumsum / tables warp, ~800 instructions per chunk) sits on scheduler 0 and
// the light TMA producer on scheduler 2.
constexpr int kWarpRaw = 2, kWarpMma = 1, kWarpCs = 0, kWarpBc = 3, kFirstCompute = 4;
// The 16 compute warps form two groups of 8 (two warps per TMEM lane quadrant in each), specialised by
// phase so that the phases of neighbouring chunks overlap: group A (warps 4-11) builds each chunk's decay
// mask and runs its epilogue, group B (warps 12-19) runs the x conv and the state pass.
constexpr int kFirstGroupB = 12;
constexpr int kGroupThreads = 256;

// shared memory map (bytes from a 1024-byte aligned base)
constexpr uint32_t OFF_C = 0;          // u_C tile: two boxes [128 tok][64 n] bf16, 128B swizzle
constexpr uint32_t OFF_B = 32768;      // u_B tile
constexpr uint32_t OFF_X = 65536;      // 2 x X [j][p] bf16 (MN-major B operand), by chunk parity
constexpr uint32_t OFF_XP = 98304;     // X' [j][p] bf16
constexpr uint32_t OFF_M = 114688;     // M  [i][j] bf16, two K blocks of 64 (K-major A operand)
constexpr uint32_t OFF_S = 147456;     // S_prev [n][p] bf16 (MN-major B operand)
constexpr uint32_t OFF_RAWX = 163840;  // 2 stages [tok][p] bf16 (TMA, 128B swizzle): raw x of chunks c, c+1
constexpr uint32_t OFF_Z = 196608;     // [tok][p] bf16 (TMA, 128B swizzle): a chunk's z, then its y
constexpr uint32_t OFF_SMALL = 212992;
// small region
constexpr uint32_t OFF_DTRAW = OFF_SMALL;              // 2 stages [128 tok][8 heads] bf16 raw dt (TMA, with x)
constexpr uint32_t OFF_WT = OFF_DTRAW + 2 * 2048;      // conv taps of the head's x channels [4][64] float
constexpr uint32_t OFF_CB = OFF_WT + 4 * 64 * 4;       // conv bias [64] float
constexpr uint32_t OFF_HALO = OFF_CB + 64 * 4;         // [2][3][64] bf16 raw x history
// the cumsum warp's per-chunk vectors, three chunks deep (slot c % 3), so that it can run ahead of both
// compute groups: a slot is rewritten once both groups are done with the chunk three back
constexpr int kCsSlots = 3;
constexpr uint32_t OFF_CS = OFF_HALO + 2 * 3 * 64 * 2;      // cs [3][128] float
constexpr uint32_t OFF_COLF = OFF_CS + kCsSlots * 128 * 4;  // exp(cs_end(g(j)) - cs_j) dt_j [3][128]
constexpr uint32_t OFF_WX = OFF_COLF + kCsSlots * 128 * 4;  // weight of x_j in the chunk state [3][128]
// decay tables of one chunk (single buffer: rewritten once every thread's mask of the previous chunk is done);
// g = 8-row group, cs_end(g) = cs at the group's last row
constexpr uint32_t OFF_RFAC = OFF_WX + kCsSlots * 128 * 4;  // exp(cs_i - cs_end(g(i)-1)) [128]
constexpr uint32_t OFF_PG = OFF_RFAC + 128 * 4;        // exp(cs_end(gi-1) - cs_end(g)), g < gi: [16 gi][4 q][4 kb]
constexpr uint32_t OFF_DG = OFF_PG + 256 * 4;          // exp(cs_i - cs_j) dt_j inside a group, j <= i: [16][8][8]
constexpr uint32_t OFF_BAR = OFF_DG + 1024 * 4;        // mbarriers (8 B each)
constexpr int NBAR = 23;
constexpr uint32_t OFF_TMEM = OFF_BAR + NBAR * 8;  // TMEM base address
constexpr uint32_t OFF_ABORT = OFF_TMEM + 4;
constexpr uint32_t SMEM_USED = OFF_ABORT + 4;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// FULL_RAW / XREADY / EPI_DONE come in pairs by chunk parity, CS_* in threes by chunk mod 3 (a waiter of one group may be a whole
// chunk behind the other group, and a barrier must never run two phases past a waiter); EPI_DONE = a
// chunk's epilogue is complete (its Y / Y2 / z / conv output read, its y written); EMPTY_BC = the chunk's
// last B / C reader (Y2) is complete; SREADY = the state entering the next chunk is in shared memory.
enum Bar { FULL_RAW0 = 0, FULL_RAW1, XREADY0, XREADY1, FULL_Z, EPI_DONE0, EPI_DONE1, FULL_BC, EMPTY_BC, MREADY,
           G_FULL, SC_FULL, Y_FULL, MMA_DONE, CS_READY0, CS_READY1, CS_READY2, CS_FREE0, CS_FREE1, CS_FREE2,
           TAB_READY, SREADY, NEVER };  // NEVER: nothing arrives on it (the test stall of the timeout path waits on it)
static_assert(NEVER + 1 == NBAR, "barrier count");

// TMEM columns (fp32, 128 lanes): G = C B^T, Y = M X, Y2 = C S^T, S_c, the running state, and the
// post-conv x of two chunks (for the D skip)
constexpr uint32_t COL_G = 0, COL_Y = 128, COL_Y2 = 192, COL_SC = 256, COL_SRUN = 320, COL_U = 384, TMEM_COLS = 512;

struct TcParams {
    PrefillArgs a;
    CUtensorMap tm_x, tm_z, tm_y, tm_bc, tm_dt;
};

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
// Two (three) phases at once: the try_waits are issued back to back, so when the phases have completed
// (the usual case in the pipeline's steady state) their latencies overlap; otherwise one by one.
__device__ __forceinline__ bool warp_wait2(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1,
                                           volatile int* abort_flag) {
    const bool r0 = mbar_try_wait(b0, p0), r1 = mbar_try_wait(b1, p1);
    if (__all_sync(0xffffffffu, r0 & r1)) return true;
    return warp_wait(b0, p0, abort_flag) && warp_wait(b1, p1, abort_flag);
}
__device__ __forceinline__ bool warp_wait3(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint64_t* b2,
                                           uint32_t p2, volatile int* abort_flag) {
    const bool r0 = mbar_try_wait(b0, p0), r1 = mbar_try_wait(b1, p1), r2 = mbar_try_wait(b2, p2);
    if (__all_sync(0xffffffffu, r0 & r1 & r2)) return true;
    return warp_wait(b0, p0, abort_flag) && warp_wait(b1, p1, abort_flag) && warp_wait(b2, p2, abort_flag);
}

// SiLU(v) = v sigmoid(v) with sigmoid(v) = (1 + tanh(v/2)) / 2: one MUFU
// operation (the hardware tanh approximation, relative error ~2^-11) instead
// of an exponential and a reciprocal.
__device__ __forceinline__ float tanh_approx(float v) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}

// softplus(v) = log(1 + e^v) with the fast exp / log (absolute error ~1e-7
// for the small dt this layer uses); above 20 the correction is below 2.1e-9.
__device__ __forceinline__ float softplus_fast(float v) { return v > 20.f ? v : __logf(1.f + __expf(v)); }

__device__ __forceinline__ float2 silu2(float2 v) {
    const float2 hv = __fmul2_rn(v, make_float2(0.5f, 0.5f));
    return __ffma2_rn(hv, make_float2(tanh_approx(hv.x), tanh_approx(hv.y)), hv);
}

__device__ __forceinline__ float s_wx_at(const uint8_t* sm, int buf, int row) {
    return reinterpret_cast<const float*>(sm + OFF_WX)[buf * 128 + row];
}

// D (+)= A B over K = 128 in eight K = 16 steps, from base descriptors (see sw128_desc); a descriptor's
// start address field holds the byte address / 16, so a step adds its byte offset / 16.
template <bool a_mn, bool b_mn>
__device__ __forceinline__ void mma_k128(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc) {
#pragma unroll
    for (uint32_t kk = 0; kk < 8; ++kk) {
        const uint32_t kmaj = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4, mnmaj = (kk * 2048) >> 4;
        mma_bf16(d_tmem, a0 + (a_mn ? mnmaj : kmaj), b0 + (b_mn ? mnmaj : kmaj), idesc, kk > 0);
    }
}

// Whether bf16 y of chunk c leaves through the TMA store of its smem tile.  The store clips rows beyond
// the tensor map (the end of a [batch][L] row), but in a packed batch the rows past a sequence's end
// belong to the next sequence, so a partial last chunk there is stored from registers instead.
template <bool kVarlen>
__device__ __forceinline__ bool tma_y_chunk(int64_t Ls, int c) {
    return !kVarlen || Ls - (int64_t)c * kQ >= kQ;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(&g_tc_error, kErrTimeout);
}

// Row-major x conv of chunk cc for the calling thread of group B: token row i, channels 32*half .. +31
// (two 16-channel quarters).  Writes X and X' (bf16, smem operands) and the fp32 conv output into TMEM
// (for the D skip), and the raw history of the next chunk.  Returns false if a wait gave up.
__device__ __forceinline__ bool conv_chunk(const PrefillArgs& a, uint8_t* sm, uint64_t* bars, volatile int* abort_flag,
                                           uint32_t tmem, uint32_t lane_base, int cc, int nc, int64_t Ls, int i,
                                           int half) {
    const int buf = cc & 1;
    // this chunk's cumsum (its raw x tile arrived before it) and raw x
    if (!warp_wait2(&bars[CS_READY0 + cc % kCsSlots], (cc / kCsSlots) & 1, &bars[FULL_RAW0 + buf], (cc >> 1) & 1,
                    abort_flag))
        return false;
    // the raw history rows were written by other threads in the previous chunk's conv; the X tile and the
    // conv output of this parity were last read by chunk cc-2's Y MMA and epilogue
    if (cc >= 2) {
        if (!warp_wait2(&bars[XREADY0 + ((cc - 1) & 1)], ((cc - 1) >> 1) & 1, &bars[EPI_DONE0 + buf],
                        ((cc - 2) >> 1) & 1, abort_flag))
            return false;
    } else if (cc == 1 && !warp_wait(&bars[XREADY0], 0, abort_flag)) {
        return false;
    }
    const int64_t t0 = (int64_t)cc * kQ;
    const int Qc = (int)(Ls - t0 < kQ ? Ls - t0 : kQ);
    const bool valid = i < Qc;
    const uint8_t* rx = sm + OFF_RAWX + buf * 16384;
    const uint4* halo_in = reinterpret_cast<const uint4*>(sm + OFF_HALO + (cc & 1) * 384);
    const float4* wt = reinterpret_cast<const float4*>(sm + OFF_WT);   // [tap][64 channels]
    const float4* cb = reinterpret_cast<const float4*>(sm + OFF_CB);
    const float wxr = s_wx_at(sm, cc % kCsSlots, i);
    uint8_t* sX = sm + OFF_X + buf * 16384;
    uint8_t* sXp = sm + OFF_XP;
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
        const int quarter = 2 * half + sub;
        float2 acc[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 bv = cb[quarter * 4 + m];
            acc[2 * m] = make_float2(bv.x, bv.y);
            acc[2 * m + 1] = make_float2(bv.z, bv.w);
        }
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) {
            const int r = i - 3 + tap;
            uint4 w[2];
#pragma unroll
            for (int k = 0; k < 2; ++k)
                w[k] = r >= 0 ? *reinterpret_cast<const uint4*>(rx + sw128_off(r, quarter * 2 + k))
                              : halo_in[(r + 3) * 8 + quarter * 2 + k];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 tv = wt[tap * 16 + quarter * 4 + m];
                const uint32_t lo = (m & 1) ? w[m >> 1].z : w[m >> 1].x;
                const uint32_t hi = (m & 1) ? w[m >> 1].w : w[m >> 1].y;
                acc[2 * m] = __ffma2_rn(make_float2(tv.x, tv.y), make_float2(bf_lo(lo), bf_hi(lo)), acc[2 * m]);
                acc[2 * m + 1] = __ffma2_rn(make_float2(tv.z, tv.w), make_float2(bf_lo(hi), bf_hi(hi)), acc[2 * m + 1]);
            }
        }
        float u[16];
        uint32_t xo[8], xpo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 uv = valid ? silu2(acc[k]) : make_float2(0.f, 0.f);
            u[2 * k] = uv.x;
            u[2 * k + 1] = uv.y;
            xo[k] = pack_bf2(uv.x, uv.y);
            const float2 up = __fmul2_rn(uv, make_float2(wxr, wxr));
            xpo[k] = pack_bf2(up.x, up.y);
        }
        tmem_st16(tmem + lane_base + COL_U + buf * 64 + quarter * 16, u);
        // X' is single-buffered: the previous chunk's S_c must have read it
        if (sub == 0 && cc >= 1 && !warp_wait(&bars[SC_FULL], (cc - 1) & 1, abort_flag)) return false;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            *reinterpret_cast<uint4*>(sX + sw128_off(i, quarter * 2 + k)) =
                make_uint4(xo[4 * k], xo[4 * k + 1], xo[4 * k + 2], xo[4 * k + 3]);
            *reinterpret_cast<uint4*>(sXp + sw128_off(i, quarter * 2 + k)) =
                make_uint4(xpo[4 * k], xpo[4 * k + 1], xpo[4 * k + 2], xpo[4 * k + 3]);
        }
        if (i >= kQ - 3 && cc + 1 < nc) {  // raw history (rows 125..127) of the next chunk
            uint4* halo_out = reinterpret_cast<uint4*>(sm + OFF_HALO + ((cc + 1) & 1) * 384);
#pragma unroll
            for (int k = 0; k < 2; ++k)
                halo_out[(i - (kQ - 3)) * 8 + quarter * 2 + k] =
                    *reinterpret_cast<const uint4*>(rx + sw128_off(i, quarter * 2 + k));
        }
    }
    tmem_wait_st();  // the conv output is read by a group-A thread, the running state again by this one
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(&bars[XREADY0 + buf]);
    return true;
}

// The running state is split between the two compute groups by columns: the thread (quadrant q, half) of
// group A owns state columns 32*half .. +15 of row n = i (= TMEM lane i), the matching thread of group B
// columns 32*half + 16 .. +31.  Each writes its part of the bf16 copy that is the Y2 operand and arrives on
// SREADY (256 + 256 arrivals per phase; phase 0 = the initial state, phase c+1 = the state entering chunk c+1).

// Initial state (or zeros) of the calling thread's 16 columns col .. col+15: S_run in TMEM, bf16 in smem.
__device__ __forceinline__ void state_init(const PrefillArgs& a, uint8_t* sm, uint64_t* bars, uint32_t tmem,
                                           uint32_t lane_base, int b, int h, int i, int col) {
    // state row n = i exists for i < N; with N = 64 the rows 64..127 stay zero throughout
    const float* init = a.init_state && i < a.N ? a.init_state + ((size_t)b * a.H + h) * kP * a.N : nullptr;
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = init ? init[(size_t)(col + k) * a.N + i] : 0.f;
    tmem_st16(tmem + lane_base + COL_SRUN + col, v);
    uint8_t* sS = sm + OFF_S;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
        uint4 w;
        w.x = pack_bf2(v[k2 * 8 + 0], v[k2 * 8 + 1]);
        w.y = pack_bf2(v[k2 * 8 + 2], v[k2 * 8 + 3]);
        w.z = pack_bf2(v[k2 * 8 + 4], v[k2 * 8 + 5]);
        w.w = pack_bf2(v[k2 * 8 + 6], v[k2 * 8 + 7]);
        *reinterpret_cast<uint4*>(sS + sw128_off(i, col / 8 + k2)) = w;
    }
    tmem_wait_st();
    fence_async_smem();
    mbar_arrive(&bars[SREADY]);
}

// State pass of chunk c for the calling thread's 16 columns: S_run <- exp(cs_last) S_run + S_c (TMEM), then,
// once Y2 and S_c of chunk c are complete, the bf16 state entering chunk c+1 into smem.  Returns false if a
// wait gave up.
__device__ __forceinline__ bool state_half(uint8_t* sm, uint64_t* bars, volatile int* abort_flag, uint32_t tmem,
                                           uint32_t lane_base, int c, float cs_last, int i, int col) {
    if (!warp_wait(&bars[SC_FULL], c & 1, abort_flag)) return false;
    tc_fence_after();
    const float dl = __expf(cs_last);
    const float2 dl2 = make_float2(dl, dl);
    float sc[16], sr[16];
    tmem_ld16(tmem + lane_base + COL_SC + col, sc);
    tmem_ld16(tmem + lane_base + COL_SRUN + col, sr);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
        const float2 v = __ffma2_rn(dl2, make_float2(sr[k], sr[k + 1]), make_float2(sc[k], sc[k + 1]));
        sr[k] = v.x;
        sr[k + 1] = v.y;
    }
    tmem_st16(tmem + lane_base + COL_SRUN + col, sr);
    // S_prev is overwritten once Y2 = C S_prev^T of this chunk has read it
    if (!warp_wait(&bars[EMPTY_BC], c & 1, abort_flag)) return false;
    uint8_t* sS = sm + OFF_S;
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
        uint4 w;
        w.x = pack_bf2(sr[k2 * 8 + 0], sr[k2 * 8 + 1]);
        w.y = pack_bf2(sr[k2 * 8 + 2], sr[k2 * 8 + 3]);
        w.z = pack_bf2(sr[k2 * 8 + 4], sr[k2 * 8 + 5]);
        w.w = pack_bf2(sr[k2 * 8 + 6], sr[k2 * 8 + 7]);
        *reinterpret_cast<uint4*>(sS + sw128_off(i, col / 8 + k2)) = w;  // the state entering chunk c+1
    }
    tmem_wait_st();
    tc_fence_before();  // this chunk's S_c reads are done before the next S_c MMA may overwrite it
    fence_async_smem();
    mbar_arrive(&bars[SREADY]);
    return true;
}

// Final state of the calling thread's 16 columns (rows n < N).
__device__ __forceinline__ void state_final(const PrefillArgs& a, uint32_t tmem, uint32_t lane_base, int b, int h,
                                            int i, int col) {
    if (i >= a.N) return;
    tmem_wait_st();
    float sr[16];
    tmem_ld16(tmem + lane_base + COL_SRUN + col, sr);
    tmem_wait_ld();
    float* fs = a.final_state + ((size_t)b * a.H + h) * kP * a.N;
#pragma unroll
    for (int k = 0; k < 16; ++k) fs[(size_t)(col + k) * a.N + i] = sr[k];
}

// kVarlen: a packed variable-length batch (a.cu set); the batch x L layout otherwise.
template <typename TY, bool kVarlen>
__global__ void __launch_bounds__(kThreads, 1) chunk_scan_kernel(const __grid_constant__ TcParams prm) {
    const PrefillArgs& a = prm.a;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, formed as an offset from the shared array so that every access through it
    // stays a shared-window access (32-bit addresses) rather than a generic one
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + OFF_TMEM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_ABORT);
    float* s_cs = reinterpret_cast<float*>(sm + OFF_CS);      // [3][128] by chunk mod 3
    float* s_colf = reinterpret_cast<float*>(sm + OFF_COLF);
    float* s_wx = reinterpret_cast<float*>(sm + OFF_WX);
    constexpr bool kTmaStoreY = sizeof(TY) == 2;  // bf16 y goes out through TMA from the stage it was written in

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int g = h / a.hpg;
    // sequence b: its rows in the activation arrays, its length and chunk count; the tensor maps are
    // [batch][L][width] (coordinates: token c*Q, batch b) or, for a packed batch, [1][rows][width]
    // (coordinates: token row0 + c*Q, batch 0)
    const SeqSpan span = kVarlen ? seq_span(a, b) : SeqSpan{(int64_t)b * a.L, a.L, true};
    if (!span.ok && threadIdx.x == 0) atomicOr(&g_tc_error, kErrBadSeqlens);
    const int64_t Ls = span.len;
    const int nc = (int)((Ls + kQ - 1) / kQ);
    const int tok0 = kVarlen ? (int)span.row0 : 0;
    const int mb = kVarlen ? 0 : b;

    if (threadIdx.x == 0) {
        for (int k = 0; k < NBAR; ++k) {
            uint32_t cnt = 1;
            if (k == XREADY0 || k == XREADY1) cnt = kGroupThreads;                      // group B
            if (k == EPI_DONE0 || k == EPI_DONE1 || k == MREADY) cnt = kGroupThreads;   // group A
            if (k == CS_FREE0 || k == CS_FREE1 || k == CS_FREE2 || k == SREADY) cnt = 2 * kGroupThreads;  // both
            if (k == CS_READY0 || k == CS_READY1 || k == CS_READY2 || k == TAB_READY) cnt = 32;
            mbar_init(&bars[k], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp >= kFirstCompute) {
        const int i = threadIdx.x - kFirstCompute * 32;
        if (a.N < kN) {  // d_state 64: the upper 64 channels of the B / C tiles are zero for the whole launch
            for (int e = i; e < 16384 / 16; e += 2 * kGroupThreads) {
                reinterpret_cast<uint4*>(sm + OFF_C + 16384)[e] = make_uint4(0u, 0u, 0u, 0u);
                reinterpret_cast<uint4*>(sm + OFF_B + 16384)[e] = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_async_smem();
        }
        if (i < kP) {
            const int ch = h * kP + i;
            // conv taps [tap][channel], bias, and the history of token 0 (initial conv state or zeros)
            const float4 w4 = *reinterpret_cast<const float4*>(a.conv_w + (size_t)ch * 4);
            float* wt = reinterpret_cast<float*>(sm + OFF_WT);
            wt[0 * 64 + i] = w4.x;
            wt[1 * 64 + i] = w4.y;
            wt[2 * 64 + i] = w4.z;
            wt[3 * 64 + i] = w4.w;
            reinterpret_cast<float*>(sm + OFF_CB)[i] = a.conv_b[ch];
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
        // ---------------- raw x / z producer, y store ----------------
        // Raw x runs two chunks ahead: stage c&1 is refilled with x(c+2) as soon as chunk c's conv
        // has read it.  The z buffer holds z(c) until chunk c's epilogue has read it and written
        // y(c) over it; y(c) is then stored and z(c+1) loaded.  The waits follow the order in which
        // the compute threads complete the two events (conv(c+1) before epilogue(c)).
        if (lane == 0) {
            prefetch_tmap(&prm.tm_x);
            prefetch_tmap(&prm.tm_z);
            prefetch_tmap(&prm.tm_dt);
            int issued_x0 = -1, issued_x1 = -1, issued_z = -1;  // last chunk loaded into each buffer
            auto load_x = [&](int c) {  // raw x of chunk c and its dt (the 8-head column block holding h)
                const int s = c & 1;
                mbar_arrive_expect_tx(&bars[FULL_RAW0 + s], 16384 + 2048);
                tma_load_3d(sm + OFF_RAWX + s * 16384, &prm.tm_x, &bars[FULL_RAW0 + s], h * kP, tok0 + c * kQ, mb);
                tma_load_3d(sm + OFF_DTRAW + s * 2048, &prm.tm_dt, &bars[FULL_RAW0 + s], h & ~7, tok0 + c * kQ, mb);
                if (s) issued_x1 = c;
                else issued_x0 = c;
            };
            auto load_z = [&](int c) {
                mbar_arrive_expect_tx(&bars[FULL_Z], 16384);
                tma_load_3d(sm + OFF_Z, &prm.tm_z, &bars[FULL_Z], h * kP, tok0 + c * kQ, mb);
                issued_z = c;
            };
            for (int c = 0; c < nc && c < 2; ++c) load_x(c);
            if (nc > 0) load_z(0);
            for (int c = 0; c < nc; ++c) {
                if (c + 2 < nc) {  // x(c+2), once chunk c's conv has consumed x(c)
                    if (!mbar_wait(&bars[XREADY0 + (c & 1)], (c >> 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                    load_x(c + 2);
                }
                // y(c) out of the z buffer once chunk c's epilogue is complete, then z(c+1) in
                if (!mbar_wait(&bars[EPI_DONE0 + (c & 1)], (c >> 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                if (kTmaStoreY && tma_y_chunk<kVarlen>(Ls, c)) {
                    tma_store_3d(&prm.tm_y, sm + OFF_Z, h * kP, tok0 + c * kQ, mb);
                    bulk_commit();
                    bulk_wait_read_all();  // the buffer may be refilled once the store has read it
                }
                if (c + 1 < nc) load_z(c + 1);
            }
            if constexpr (kTmaStoreY) bulk_wait_all();
            // Every load this thread issued lands before the CTA exits.  Normally each was consumed
            // already and the waits return at once; after an abort (which another warp may raise after
            // this loop has ended) a load can still be in flight.
            if (issued_x0 >= 0) mbar_wait(&bars[FULL_RAW0], (issued_x0 >> 1) & 1, nullptr, 100000000ull);
            if (issued_x1 >= 0) mbar_wait(&bars[FULL_RAW1], (issued_x1 >> 1) & 1, nullptr, 100000000ull);
            if (issued_z >= 0) mbar_wait(&bars[FULL_Z], issued_z & 1, nullptr, 100000000ull);
        }
    } else if (warp == kWarpBc) {
        // ---------------- post-conv B / C producer ----------------
        if (lane == 0) {
            prefetch_tmap(&prm.tm_bc);
            // the post-conv B/C come from the prologue kernel launched just before this one
            asm volatile("griddepcontrol.wait;" ::: "memory");
            int last = -1;
            for (int c = 0; c < nc; ++c) {
                // B / C of chunk c, once chunk c-1's last reader of the tiles (Y2) is complete
                if (c >= 1 && !mbar_wait(&bars[EMPTY_BC], (c - 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                // one 64-wide box per 64 state channels; with N = 64 the upper boxes stay zero
                mbar_arrive_expect_tx(&bars[FULL_BC], (a.N == kN ? 4 : 2) * 16384);
                const int xc = a.GN + g * a.N, xb = g * a.N;
                tma_load_3d(sm + OFF_C, &prm.tm_bc, &bars[FULL_BC], xc, tok0 + c * kQ, mb);
                tma_load_3d(sm + OFF_B, &prm.tm_bc, &bars[FULL_BC], xb, tok0 + c * kQ, mb);
                if (a.N == kN) {
                    tma_load_3d(sm + OFF_C + 16384, &prm.tm_bc, &bars[FULL_BC], xc + 64, tok0 + c * kQ, mb);
                    tma_load_3d(sm + OFF_B + 16384, &prm.tm_bc, &bars[FULL_BC], xb + 64, tok0 + c * kQ, mb);
                }
                last = c;
            }
            // the last B / C load lands before the CTA exits (at once unless a consumer aborted)
            if (last >= 0) mbar_wait(&bars[FULL_BC], last & 1, nullptr, 100000000ull);
        }
    } else if (warp == kWarpCs) {
        // ---------------- chunk dt / cumsum (whole warp; lane l owns rows 4l .. 4l+3) ----------------
        const float A = a.A[h], dtb = a.dt_bias[h];
        for (int c = 0; c < nc; ++c) {
            // dt = softplus(dt_raw + bias) and the inclusive cumsum of dt*A over the chunk's 128 rows,
            // into slot c % 3 once every compute thread is done with chunk c - 3; the raw dt tile arrives
            // with the chunk's raw x (stage c & 1)
            const int buf = c & 1, cb = c % kCsSlots;
            if (c >= kCsSlots && !warp_wait(&bars[CS_FREE0 + cb], ((c / kCsSlots) + 1) & 1, abort_flag)) {
                raise_abort(abort_flag);
                break;
            }
            if (!warp_wait(&bars[FULL_RAW0 + buf], (c >> 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
            const int Qc = (int)(Ls - (int64_t)c * kQ < kQ ? Ls - (int64_t)c * kQ : kQ);
            const __nv_bfloat16* dtr = reinterpret_cast<const __nv_bfloat16*>(sm + OFF_DTRAW + buf * 2048) + (h & 7);
            float dtv[4], cs[4];
            float run = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = 4 * lane + k;
                dtv[k] = r < Qc ? softplus_fast(__bfloat162float(dtr[r * 8]) + dtb) : 0.f;
                run += dtv[k] * A;
                cs[k] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += up;
            }
            const float excl = incl - run;
            // The decay factors of the chunk are products of the per-row decays a_r = exp(dt_r A):
            // exp(cs_i - cs_j) = a_{j+1} ... a_i.  Lane l holds rows 4l .. 4l+3 of the 8-row group gi = l/2;
            // the pair (2gi, 2gi+1) shares the group's 8 decays, and T_g = a_{8g} ... a_{8g+7}.
            const int gi = lane >> 1;
            float ga[8], gdt[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float ak = __expf(dtv[k] * A);
                const float oak = __shfl_xor_sync(0xffffffffu, ak, 1), odt = __shfl_xor_sync(0xffffffffu, dtv[k], 1);
                ga[k] = (lane & 1) ? oak : ak;
                ga[4 + k] = (lane & 1) ? ak : oak;
                gdt[k] = (lane & 1) ? odt : dtv[k];
                gdt[4 + k] = (lane & 1) ? dtv[k] : odt;
            }
            float pre[8], suf[8];  // a_{8gi} .. a_m  and  a_{m+1} .. a_{8gi+7}
            {
                float p = 1.f, q = 1.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    p *= ga[m];
                    pre[m] = p;
                    suf[7 - m] = q;
                    q *= ga[7 - m];
                }
            }
            const float tg = pre[7];
            float tall[16];  // T_g of every group of the chunk
#pragma unroll
            for (int g = 0; g < 16; ++g) tall[g] = __shfl_sync(0xffffffffu, tg, 2 * g);
            float later = 1.f;  // T_{gi+1} ... T_15
#pragma unroll
            for (int g = 15; g > 0; --g)
                if (g > gi) later *= tall[g];
            const bool odd = lane & 1;  // this lane holds rows 4..7 of its group (else 0..3)
            float csr[4], cf[4], wx[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float sm_k = odd ? suf[4 + k] : suf[k];  // (register selects, no indexed local array)
                csr[k] = cs[k] + excl;
                cf[k] = sm_k * dtv[k];             // exp(cs_end(gi) - cs_j) dt_j
                wx[k] = sm_k * later * dtv[k];     // exp(cs_last - cs_j) dt_j
            }
            reinterpret_cast<float4*>(s_cs + cb * 128)[lane] = make_float4(csr[0], csr[1], csr[2], csr[3]);
            reinterpret_cast<float4*>(s_colf + cb * 128)[lane] = make_float4(cf[0], cf[1], cf[2], cf[3]);
            reinterpret_cast<float4*>(s_wx + cb * 128)[lane] = make_float4(wx[0], wx[1], wx[2], wx[3]);
            mbar_arrive(&bars[CS_READY0 + cb]);

            // decay tables of this chunk, once every thread's mask of the previous chunk has read them
            if (c >= 1 && !warp_wait(&bars[MREADY], (c - 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
            float rfac[4];  // exp(cs_i - cs_end(gi-1)) = a_{8gi} ... a_i
#pragma unroll
            for (int k = 0; k < 4; ++k) rfac[k] = gi > 0 ? (odd ? pre[4 + k] : pre[k]) : 0.f;
            reinterpret_cast<float4*>(sm + OFF_RFAC)[lane] = make_float4(rfac[0], rfac[1], rfac[2], rfac[3]);
            // group-to-group factors of row group gi, exp(cs_end(gi-1) - cs_end(g)) = T_{g+1} ... T_{gi-1}
            // for g < gi: entries e = 8 (l&1) .. +7 of [4 q][4 kb], g = 4 kb + q
            float between[16];
            {
                float p = 1.f;
#pragma unroll
                for (int g = 15; g >= 0; --g) {
                    between[g] = g < gi ? p : 0.f;
                    if (g < gi) p *= tall[g];
                }
            }
            float pg[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {  // e = 8 (l&1) + k: g = 4 (k & 3) + (k >> 2) + 2 (l&1)
                const int g0 = 4 * (k & 3) + (k >> 2);
                pg[k] = odd ? between[g0 + 2] : between[g0];
            }
            float4* pg4 = reinterpret_cast<float4*>(sm + OFF_PG) + gi * 4 + (lane & 1) * 2;
            pg4[0] = make_float4(pg[0], pg[1], pg[2], pg[3]);
            pg4[1] = make_float4(pg[4], pg[5], pg[6], pg[7]);
            // in-group decay of this lane's rows r = 4 (l&1) + k against the group's 8 columns:
            // exp(cs_r - cs_j) dt_j = a_{j+1} ... a_r dt_j for j <= r, zero above
            float4* dg4 = reinterpret_cast<float4*>(sm + OFF_DG) + (gi * 8 + 4 * (lane & 1)) * 2;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int r = 4 * (lane & 1) + k;
                float dv[8];
                float prod = 1.f;  // a_{j+1} ... a_r, built from j = r downwards
#pragma unroll
                for (int cix = 7; cix >= 0; --cix) {
                    dv[cix] = cix <= r ? prod * gdt[cix] : 0.f;
                    if (cix <= r) prod *= ga[cix];
                }
                dg4[2 * k] = make_float4(dv[0], dv[1], dv[2], dv[3]);
                dg4[2 * k + 1] = make_float4(dv[4], dv[5], dv[6], dv[7]);
            }
            mbar_arrive(&bars[TAB_READY]);
        }
    } else if (warp == kWarpMma) {
        // ---------------- tcgen05.mma issuer ----------------
        if (lane == 0) {
            constexpr uint32_t ID_G = idesc_bf16_f32(128, 128, false, false);   // C (K-major) x B (K-major)
            constexpr uint32_t ID_Y = idesc_bf16_f32(128, 64, false, true);     // M (K-major) x X (MN-major)
            constexpr uint32_t ID_Y2 = idesc_bf16_f32(128, 64, false, true);    // C (K-major) x S (MN-major)
            constexpr uint32_t ID_SC = idesc_bf16_f32(128, 64, true, true);     // B^T (MN-major) x X' (MN-major)
            // base descriptors; a K step of 16 advances a K-major operand by 32 bytes inside its 64-wide
            // swizzle atom (and to the second atom after four steps), an MN-major one by 16 rows (2048 bytes)
            const uint64_t dC = sw128_desc(smem_u32(sm + OFF_C), 16, 1024);
            const uint64_t dB = sw128_desc(smem_u32(sm + OFF_B), 16, 1024);
            const uint64_t dBt = sw128_desc(smem_u32(sm + OFF_B), 16384, 1024);
            const uint64_t dXp = sw128_desc(smem_u32(sm + OFF_XP), 16384, 1024);
            const uint64_t dM = sw128_desc(smem_u32(sm + OFF_M), 16, 1024);
            const uint64_t dS = sw128_desc(smem_u32(sm + OFF_S), 16384, 1024);
            const uint64_t dX0 = sw128_desc(smem_u32(sm + OFF_X), 16384, 1024);
            // test stall of the timeout path: a wait on a barrier nothing arrives on, bounded by
            // a.stall_ns, gives up and aborts the CTA before its first MMA (off unless a test sets it)
            if (a.stall_ns && !mbar_wait(&bars[NEVER], 0, abort_flag, a.stall_ns)) raise_abort(abort_flag);
            for (int c = 0; c < nc; ++c) {
                const uint64_t dX = dX0 + (uint64_t)((c & 1) * (16384 >> 4));
                if (!mbar_wait(&bars[FULL_BC], c & 1, abort_flag)) { raise_abort(abort_flag); break; }
                if (c >= 1 && !mbar_wait(&bars[MREADY], (c - 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
                mma_k128<false, false>(tmem + COL_G, dC, dB, ID_G);
                mma_commit(&bars[G_FULL]);
                // Y2 = C S_prev^T, once the state passes of the previous chunk (or the initial state, phase 0)
                // have written S_prev and the previous chunk's epilogue has read the previous Y2
                if (!mbar_wait(&bars[SREADY], c & 1, abort_flag) ||
                    (c >= 1 && !mbar_wait(&bars[EPI_DONE0 + ((c - 1) & 1)], ((c - 1) >> 1) & 1, abort_flag))) {
                    raise_abort(abort_flag);
                    break;
                }
                tc_fence_after();
                mma_k128<false, true>(tmem + COL_Y2, dC, dS, ID_Y2);
                // chunk state S_c = B^T X' (needs this chunk's conv; the S_c columns are free since both state
                // passes of the previous chunk, in the SREADY phase waited above, have read them)
                if (!mbar_wait(&bars[XREADY0 + (c & 1)], (c >> 1) & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
                mma_k128<true, true>(tmem + COL_SC, dBt, dXp, ID_SC);
                mma_commit(&bars[SC_FULL]);
                mma_commit(&bars[EMPTY_BC]);  // B / C tiles and S_prev free (Y2 and S_c complete)
                // Y = M X, once every row's decay mask is written
                if (!mbar_wait(&bars[MREADY], c & 1, abort_flag)) { raise_abort(abort_flag); break; }
                tc_fence_after();
                mma_k128<false, true>(tmem + COL_Y, dM, dX, ID_Y);
                mma_commit(&bars[Y_FULL]);
            }
            // nothing may still be running on the tensor cores when TMEM is released
            mma_commit(&bars[MMA_DONE]);
            mbar_wait(&bars[MMA_DONE], 0, nullptr, 100000000ull);
        }
    } else if (warp < kFirstGroupB) {
        // ---------------- group A: decay mask, half of the state pass, epilogue ----------------
        // Thread (quadrant q, half) owns token row i = TMEM lane i, the 8-column groups 2*half and 2*half+1
        // of each 32-column mask block, state columns 32*half .. +15 and output columns 32*half .. +31.
        const int q = warp & 3;                            // TMEM lane quadrant of this warp
        const int half = (warp - kFirstCompute) >> 2;      // 0 or 1
        const int i = q * 32 + lane;                       // token row / TMEM lane
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const float Dh = a.D[h];
        uint8_t* sMm = sm + OFF_M;
        state_init(a, sm, bars, tmem, lane_base, b, h, i, 32 * half);
        for (int c = 0; c < nc; ++c) {
            const int buf = c & 1;
            const int64_t t0 = (int64_t)c * kQ;
            const int Qc = (int)(Ls - t0 < kQ ? Ls - t0 : kQ);
            const bool tma_y = kTmaStoreY && tma_y_chunk<kVarlen>(Ls, c);  // else y is stored from registers

            // (e) decay mask of row i, once G and this chunk's decay tables (written after its cumsum, so the
            // cumsum buffer is ready too) are
            if (!warp_wait2(&bars[G_FULL], c & 1, &bars[TAB_READY], c & 1, abort_flag)) {
                raise_abort(abort_flag);
                break;
            }
            tc_fence_after();
            {
                // decay of row i (group gi) against column group g = 4 kb + quarter (columns 8g .. 8g+7):
                //   g < gi: exp(cs_i - cs_end(gi-1)) exp(cs_end(gi-1) - cs_end(g)) exp(cs_end(g) - cs_j) dt_j
                //   g = gi: the in-group table;  g > gi: zero
                const int gi = i >> 3;
                const float rfac = reinterpret_cast<const float*>(sm + OFF_RFAC)[i];
                const float4 p4a = reinterpret_cast<const float4*>(sm + OFF_PG)[gi * 4 + 2 * half];
                const float4 p4b = reinterpret_cast<const float4*>(sm + OFF_PG)[gi * 4 + 2 * half + 1];
                const float pk[2][4] = {{p4a.x, p4a.y, p4a.z, p4a.w}, {p4b.x, p4b.y, p4b.z, p4b.w}};
                const float4* drow = reinterpret_cast<const float4*>(sm + OFF_DG) + (gi * 8 + (i & 7)) * 2;
                const float* colf_b = s_colf + (c % kCsSlots) * 128;
#pragma unroll
                for (int kb2 = 0; kb2 < 4; kb2 += 2) {
                    float gv[2][16];  // two 32-column blocks per TMEM round trip (warp-uniform: blocks right of
                                      // the diagonal block are zero and not loaded)
                    if (kb2 <= q) tmem_ld16(tmem + lane_base + COL_G + kb2 * 32 + half * 16, gv[0]);
                    if (kb2 + 1 <= q) tmem_ld16(tmem + lane_base + COL_G + (kb2 + 1) * 32 + half * 16, gv[1]);
                    if (kb2 <= q) tmem_wait_ld();
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        const int kb = kb2 + kk;
#pragma unroll
                        for (int sub = 0; sub < 2; ++sub) {
                            const int quarter = 2 * half + sub;
                            const int g = 4 * kb + quarter;
                            uint4 packed = make_uint4(0u, 0u, 0u, 0u);
                            if (kb <= q && g <= gi) {
                                float4 fa, fb;
                                if (g < gi) {
                                    const float4* colf = reinterpret_cast<const float4*>(colf_b + 8 * g);
                                    const float rf = rfac * pk[sub][kb];
                                    fa = colf[0];
                                    fb = colf[1];
                                    fa = make_float4(fa.x * rf, fa.y * rf, fa.z * rf, fa.w * rf);
                                    fb = make_float4(fb.x * rf, fb.y * rf, fb.z * rf, fb.w * rf);
                                } else {
                                    fa = drow[0];
                                    fb = drow[1];
                                }
                                const float* gg = gv[kk] + 8 * sub;
                                const float2 m0 = __fmul2_rn(make_float2(gg[0], gg[1]), make_float2(fa.x, fa.y));
                                const float2 m1 = __fmul2_rn(make_float2(gg[2], gg[3]), make_float2(fa.z, fa.w));
                                const float2 m2 = __fmul2_rn(make_float2(gg[4], gg[5]), make_float2(fb.x, fb.y));
                                const float2 m3 = __fmul2_rn(make_float2(gg[6], gg[7]), make_float2(fb.z, fb.w));
                                packed = make_uint4(pack_bf2(m0.x, m0.y), pack_bf2(m1.x, m1.y), pack_bf2(m2.x, m2.y),
                                                    pack_bf2(m3.x, m3.y));
                            }
                            *reinterpret_cast<uint4*>(sMm + (kb >> 1) * 16384 +
                                                      sw128_off(i, (kb & 1) * 4 + quarter)) = packed;
                        }
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[MREADY]);

            // (f) this thread's half of the state pass of chunk c
            if (!state_half(sm, bars, abort_flag, tmem, lane_base, c, s_cs[(c % kCsSlots) * 128 + kQ - 1], i, 32 * half)) {
                raise_abort(abort_flag);
                break;
            }

            // (g) epilogue: y = (Y + exp(cs_i) Y2 + D x) SiLU(z), columns 32*half .. +31, once z, Y (Y2 before
            // it) and this chunk's conv output (written by group B; complete before the Y MMA was issued,
            // waited on here as well so that its TMEM stores are ordered before these loads directly) are in
            if (!warp_wait3(&bars[FULL_Z], c & 1, &bars[Y_FULL], c & 1, &bars[XREADY0 + buf], (c >> 1) & 1,
                            abort_flag)) {
                raise_abort(abort_flag);
                break;
            }
            tc_fence_after();
            {
                uint8_t* rz = sm + OFF_Z;  // z in, y out (same positions, this thread's only)
                const float ecs = __expf(s_cs[(c % kCsSlots) * 128 + i]);  // decay of S_prev up to row i
                const float2 e2 = make_float2(ecs, ecs), d2 = make_float2(Dh, Dh);
#pragma unroll 1
                for (int sub = 0; sub < 2; ++sub) {
                    const int quarter = 2 * half + sub;
                    float y1[16], y2[16], uu[16];
                    tmem_ld16(tmem + lane_base + COL_Y + quarter * 16, y1);
                    tmem_ld16(tmem + lane_base + COL_Y2 + quarter * 16, y2);
                    tmem_ld16(tmem + lane_base + COL_U + buf * 64 + quarter * 16, uu);
                    // the gate SiLU(z) of these 16 columns while the TMEM loads are in flight
                    float2 gz[8];
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        const uint4 zw = *reinterpret_cast<const uint4*>(rz + sw128_off(i, quarter * 2 + k2));
                        const uint32_t zr[4] = {zw.x, zw.y, zw.z, zw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) gz[k2 * 4 + e] = silu2(make_float2(bf_lo(zr[e]), bf_hi(zr[e])));
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int k2 = 0; k2 < 2; ++k2) {
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; e += 2) {
                            const int f = k2 * 8 + e;
                            float2 yv = __ffma2_rn(e2, make_float2(y2[f], y2[f + 1]), make_float2(y1[f], y1[f + 1]));
                            yv = __ffma2_rn(d2, make_float2(uu[f], uu[f + 1]), yv);
                            const float2 ov = __fmul2_rn(yv, gz[k2 * 4 + (e >> 1)]);
                            o[e] = ov.x;
                            o[e + 1] = ov.y;
                        }
                        if (tma_y) {
                            *reinterpret_cast<uint4*>(rz + sw128_off(i, quarter * 2 + k2)) =
                                make_uint4(pack_bf2(o[0], o[1]), pack_bf2(o[2], o[3]), pack_bf2(o[4], o[5]),
                                           pack_bf2(o[6], o[7]));
                        } else if (i < Qc) {
                            TY* yrow = static_cast<TY*>(a.y) + ((size_t)span.row0 + t0 + i) * a.HP + (size_t)h * kP +
                                       quarter * 16;
                            if constexpr (sizeof(TY) == 2) {
                                *reinterpret_cast<uint4*>(yrow + k2 * 8) =
                                    make_uint4(pack_bf2(o[0], o[1]), pack_bf2(o[2], o[3]), pack_bf2(o[4], o[5]),
                                               pack_bf2(o[6], o[7]));
                            } else {
                                float4* dst = reinterpret_cast<float4*>(yrow + k2 * 8);
                                dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                                dst[1] = make_float4(o[4], o[5], o[6], o[7]);
                            }
                        }
                    }
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[EPI_DONE0 + buf]);
            mbar_arrive(&bars[CS_FREE0 + c % kCsSlots]);  // group A's reads of this chunk's cumsum slot are done
        }
        // final state of this thread's columns (an empty sequence passes its initial state through)
        if (!*abort_flag) state_final(a, tmem, lane_base, b, h, i, 32 * half);
    } else {
        // ---------------- group B: x conv (one chunk ahead), the other half of the state pass ----------------
        // Thread (quadrant q, half) owns token row i = TMEM lane i of the conv (channels 32*half .. +31) and
        // state columns 32*half + 16 .. +31 of row n = i.
        const int q = warp & 3;
        const int half = (warp - kFirstGroupB) >> 2;
        const int i = q * 32 + lane;
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        state_init(a, sm, bars, tmem, lane_base, b, h, i, 32 * half + 16);
        bool ok = nc == 0 || conv_chunk(a, sm, bars, abort_flag, tmem, lane_base, 0, nc, Ls, i, half);
        if (!ok) raise_abort(abort_flag);
        for (int c = 0; c < nc && ok; ++c) {
            // (c) the next chunk's x conv first: this chunk's S_c (needed below) completes meanwhile
            if (c + 1 < nc && !conv_chunk(a, sm, bars, abort_flag, tmem, lane_base, c + 1, nc, Ls, i, half)) {
                raise_abort(abort_flag);
                break;
            }
            // (f) this thread's half of the state pass of chunk c
            if (!state_half(sm, bars, abort_flag, tmem, lane_base, c, s_cs[(c % kCsSlots) * 128 + kQ - 1], i,
                            32 * half + 16)) {
                raise_abort(abort_flag);
                break;
            }
            mbar_arrive(&bars[CS_FREE0 + c % kCsSlots]);  // group B's reads of this chunk's cumsum slot are done
        }
        if (!*abort_flag) state_final(a, tmem, lane_base, b, h, i, 32 * half + 16);
    }

    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// SiLU(conv4) of the B and C channels into the workspace [row][2][G*N] (bf16),
// and the conv_state output (pre-conv inputs of the last 3 tokens of every channel).
// Blocks with blockIdx.x < ntok: 256 channel pairs (bf16x2) over kProTok rows each; the
// block stages its kProTok + 3 input rows in shared memory before the first FMA.  Blocks with
// blockIdx.x >= ntok (and blockIdx.z == 0): the conv_state tail, one element per thread.
// In a packed batch (a.cu) the window runs over all rows; taps that reach before the
// start of a row's sequence take that sequence's initial conv state (or zero) instead.
constexpr int kProTok = 32;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// Pre-conv value of channel c at position t (< 3 tokens before the start) of sequence b's history.
__device__ __forceinline__ __nv_bfloat16 conv_history(const PrefillArgs& a, int64_t b, int c, int64_t t) {
    const __nv_bfloat16* hist = static_cast<const __nv_bfloat16*>(a.init_conv_state);
    return hist ? hist[((size_t)b * a.conv_dim + c) * 3 + (t + 3)] : __float2bfloat16_rn(0.f);
}

template <bool kVarlen>
__global__ void __launch_bounds__(256, 5) bc_prologue_kernel(PrefillArgs a, int ntok) {
    // the chunk scan may start its launch now; it waits for this grid before reading the workspace
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if ((int)blockIdx.x >= ntok) {
        if (blockIdx.z != 0) return;
        const int64_t e = ((int64_t)(blockIdx.x - ntok) * gridDim.y + blockIdx.y) * 256 + threadIdx.x;
        if (e >= a.batch * a.conv_dim * 3) return;
        const int k = (int)(e % 3);
        const int c = (int)((e / 3) % a.conv_dim);
        const int64_t b = e / (3 * (int64_t)a.conv_dim);
        const SeqSpan sp = kVarlen ? seq_span(a, b) : SeqSpan{b * a.L, a.L, true};
        const int64_t t = sp.len - 3 + k;  // position in the sequence
        __nv_bfloat16 v;
        if (t >= 0) {
            const size_t row = (size_t)(sp.row0 + t);
            if (c < a.HP) v = static_cast<const __nv_bfloat16*>(a.x)[row * a.rs_x + c];
            else if (c < a.HP + a.GN) v = static_cast<const __nv_bfloat16*>(a.B)[row * a.rs_B + (c - a.HP)];
            else v = static_cast<const __nv_bfloat16*>(a.C)[row * a.rs_C + (c - a.HP - a.GN)];
        } else {
            v = conv_history(a, b, c, t);
        }
        static_cast<__nv_bfloat16*>(a.conv_state)[e] = v;
        return;
    }
    const int64_t b = blockIdx.y;  // 0 for a packed batch
    const int64_t t0 = (int64_t)blockIdx.x * kProTok;  // first row of the window within [0, L)
    // packed batch: the sequence of row t0 (the largest s with cu[s] <= t0; empty sequences are skipped),
    // searched once per block
    __shared__ int64_t s_seq[3];  // the sequence, its first row and the first row after it
    if constexpr (kVarlen) {
        if (threadIdx.x == 0) {
            int64_t lo = 0, hi = a.batch;
            while (hi - lo > 1) {
                const int64_t mid = (lo + hi) >> 1;
                if (a.cu[mid] <= t0) lo = mid;
                else hi = mid;
            }
            s_seq[0] = lo;
            s_seq[1] = a.cu[lo];
            s_seq[2] = a.cu[lo + 1];
        }
        __syncthreads();
    }
    const int half_gn = a.GN / 2;                    // channel pairs per array
    const int pair = blockIdx.z * 256 + threadIdx.x;  // 0 .. GN-1 over both arrays
    const int sel = pair >= half_gn;                // 0 = B, 1 = C
    const int cp = pair - sel * half_gn;            // pair index within the array
    const int cglob = a.HP + sel * a.GN + 2 * cp;   // conv channel of the pair's first element
    uint32_t* dst = static_cast<uint32_t*>(a.workspace) + ((size_t)b * a.L * 2 + sel) * half_gn + cp;
    // The block's window (rows t0-3 .. t0+kProTok-1 of its 256 pairs, the rows inside [0, L)) lands in
    // shared memory by 16-byte cp.async pieces (4 pairs each), so the loads in flight hold no registers.
    // The entry points guarantee the alignment: B and C 16-byte aligned, rows a multiple of 16 bytes apart,
    // and every array a multiple of 4 channel pairs wide (so a piece never spans B and C).
    __shared__ __align__(16) uint32_t s_win[kProTok + 3][256];
    {
        const int64_t row0 = b * a.L + t0 - 3;
        for (int q = threadIdx.x; q < (kProTok + 3) * 64; q += 256) {
            const int k = q >> 6, c4 = (q & 63) * 4;
            const int gp = blockIdx.z * 256 + c4;  // first pair of the piece
            const int64_t t = t0 - 3 + k;
            if (gp < a.GN && t >= 0 && t < a.L) {
                const int gsel = gp >= half_gn;
                const int64_t grs = (gsel ? a.rs_C : a.rs_B) / 2;
                const uint32_t* g =
                    static_cast<const uint32_t*>(gsel ? a.C : a.B) + (size_t)(row0 + k) * grs + (gp - gsel * half_gn);
                cp_async16(&s_win[k][c4], g);
            }
        }
    }
    cp_async_wait_all();
    __syncthreads();
    if (pair >= a.GN) return;
    const float4 w0 = *reinterpret_cast<const float4*>(a.conv_w + (size_t)cglob * 4);
    const float4 w1 = *reinterpret_cast<const float4*>(a.conv_w + (size_t)(cglob + 1) * 4);
    const float2 bias = make_float2(a.conv_b[cglob], a.conv_b[cglob + 1]);
    // Interior windows (all rows inside [0, L) and, in a packed batch, inside one sequence): no per-row
    // checks and no history taps; the last three rows slide along in registers.
    bool interior = t0 >= 3 && t0 + kProTok <= a.L;
    if constexpr (kVarlen) interior = interior && s_seq[1] <= t0 - 3 && t0 + kProTok <= s_seq[2];
    if (interior) {
        uint32_t* q = dst + (size_t)t0 * 2 * half_gn;
        const int qs = 2 * half_gn;  // workspace row stride in channel pairs
        uint32_t r = s_win[0][threadIdx.x];
        float2 x0 = make_float2(bf_lo(r), bf_hi(r));
        r = s_win[1][threadIdx.x];
        float2 x1 = make_float2(bf_lo(r), bf_hi(r));
        r = s_win[2][threadIdx.x];
        float2 x2 = make_float2(bf_lo(r), bf_hi(r));
#pragma unroll
        for (int k = 0; k < kProTok; ++k) {
            r = s_win[k + 3][threadIdx.x];
            const float2 x3 = make_float2(bf_lo(r), bf_hi(r));
            float2 acc = bias;
            acc = __ffma2_rn(make_float2(w0.x, w1.x), x0, acc);
            acc = __ffma2_rn(make_float2(w0.y, w1.y), x1, acc);
            acc = __ffma2_rn(make_float2(w0.z, w1.z), x2, acc);
            acc = __ffma2_rn(make_float2(w0.w, w1.w), x3, acc);
            const float2 u = silu2(acc);
            q[k * qs] = pack_bf2(u.x, u.y);
            x0 = x1;
            x1 = x2;
            x2 = x3;
        }
        return;
    }
    // Edge windows (the first rows of a batch row or of a sequence, or a window past L): one row at a
    // time; a tap before the start of the row's sequence reads that sequence's conv history.
    int64_t seq = b, start = 0, next = a.L;
    if constexpr (kVarlen) {
        seq = s_seq[0];
        start = s_seq[1];
        next = s_seq[2];
    }
    const float wt0[4] = {w0.x, w0.y, w0.z, w0.w}, wt1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll 1
    for (int k = 0; k < kProTok; ++k) {
        const int64_t t = t0 + k;
        if (t >= a.L) break;
        if constexpr (kVarlen) {
            while (t >= next && seq + 1 < a.batch) {  // row t opens a later sequence
                ++seq;
                start = next;
                next = a.cu[seq + 1];
            }
        }
        float2 acc = bias;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t tt = t - 3 + j;  // window row k + j
            float2 x;
            if (tt >= start) {
                const uint32_t r = s_win[k + j][threadIdx.x];
                x = make_float2(bf_lo(r), bf_hi(r));
            } else {
                x = make_float2(__bfloat162float(conv_history(a, seq, cglob, tt - start)),
                                __bfloat162float(conv_history(a, seq, cglob + 1, tt - start)));
            }
            acc = __ffma2_rn(make_float2(wt0[j], wt1[j]), x, acc);
        }
        const float2 u = silu2(acc);
        dst[(size_t)t * 2 * half_gn] = pack_bf2(u.x, u.y);
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

// 3-D bf16 map over [batch][L][width] (rows row_stride elements apart) with a [1][128][64] box and
// 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t width, int64_t row_stride, int64_t L, int64_t batch) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)(row_stride * L * 2)};
    const cuuint32_t box[3] = {64, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over dt [batch][L][H] with a [1][128][8] box (8 heads x 128 tokens, no swizzle); needs H % 8 == 0.
bool make_dt_map(CUtensorMap* m, const void* base, int64_t H, int64_t row_stride, int64_t L, int64_t batch) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || H % 8 != 0) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)(row_stride * L * 2)};
    const cuuint32_t box[3] = {8, 128, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// d_state 64 runs the d_state 128 tiles with the upper 64 channels zero; a requested chunk of 64 runs in
// chunks of 128 (the chunk length is a tiling choice: the results agree up to rounding).  The dt tiles are
// loaded 8 heads wide, and dt rows must be a multiple of 16 bytes for the tensor map.
bool prefill_tc_supported(int P, int N, int Q, int H, bool bf16) {
    return bf16 && P == kP && (N == kN || N == 64) && (Q == kQ || Q == 64) && H % 8 == 0;
}

size_t prefill_tc_workspace_bytes(int64_t batch, int64_t L, int G, int N) {
    return (size_t)batch * (size_t)L * 2 * (size_t)G * (size_t)N * 2;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a, ActKind kind, cudaStream_t st, const TimingHook& hook) {
    if (a.L == 0) return launch_prefill_simt(a, kind, st, hook);  // nothing to scan: states pass through
    TcParams prm;
    prm.a = a;
    const int64_t mbatch = a.cu ? 1 : a.batch;  // a packed batch is one [L] row of the maps
    if (!make_map(&prm.tm_x, a.x, a.HP, a.rs_x, a.L, mbatch) || !make_map(&prm.tm_z, a.z, a.HP, a.rs_z, a.L, mbatch) ||
        (kind == ActKind::BF16 && !make_map(&prm.tm_y, a.y, a.HP, a.HP, a.L, mbatch)) ||
        !make_map(&prm.tm_bc, a.workspace, 2 * a.GN, 2 * a.GN, a.L, mbatch) ||
        !make_dt_map(&prm.tm_dt, a.dt, a.H, a.rs_dt, a.L, mbatch))
        return cudaErrorInvalidValue;
    const int ntok = (int)((a.L + kProTok - 1) / kProTok);
    const int64_t tail = a.batch * (int64_t)a.conv_dim * 3;
    const int tail_blocks = (int)((tail + 256 * mbatch - 1) / (256 * mbatch));
    const dim3 pgrid((unsigned)(ntok + tail_blocks), (unsigned)mbatch, (unsigned)((a.GN + 255) / 256));
    // the prologue's 16-byte window pieces (the entry points check the pointers and strides already)
    if (reinterpret_cast<uintptr_t>(a.B) % 16 != 0 || reinterpret_cast<uintptr_t>(a.C) % 16 != 0 || a.rs_B % 8 != 0 ||
        a.rs_C % 8 != 0 || (a.GN / 2) % 4 != 0)
        return cudaErrorInvalidValue;
    if (a.cu) bc_prologue_kernel<true><<<pgrid, 256, 0, st>>>(a, ntok);
    else bc_prologue_kernel<false><<<pgrid, 256, 0, st>>>(a, ntok);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    auto kern = kind == ActKind::BF16_YF32 ? (a.cu ? chunk_scan_kernel<float, true> : chunk_scan_kernel<float, false>)
                                           : (a.cu ? chunk_scan_kernel<__nv_bfloat16, true>
                                                   : chunk_scan_kernel<__nv_bfloat16, false>);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the scan's set-up (TMEM, barriers, state, first x conv)
    // overlaps the prologue; only its B/C loads wait for the prologue grid to complete
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.batch * a.H));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    hook.before(st);
    e = cudaLaunchKernelEx(&cfg, kern, prm);
    if (e != cudaSuccess) return e;
    hook.after(st);
    return cudaGetLastError();
}

// The flag's address is looked up once per device and cached for the process (like every device
// symbol here, it does not survive a cudaDeviceReset).
int* device_error_flag() {
    static int* ptrs[64] = {};
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> guard(lock);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_tc_error) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int*>(p);
    }
    return ptrs[dev];
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
