// ssd_mimo.cu -- one decode token of the multi-input multi-output (MIMO) SSM for a batch.
//
// "Mamba-3: 추론을 우선한 상태 공간 모델" (opening section, third change; 아키텍처: the MIMO
// projection widens B and C) models several SSMs in parallel per head instead of one, at almost
// no cost to decode latency.  Read here on the Mamba-2 scalar decay, with no short conv (the
// same page drops it):
//   dt = softplus(dt_raw + dt_bias[h]),  a = exp(dt A[h])
//   S  <- a S + dt sum_{k<R} x_k (outer) B_k           (a rank-R update of the P x N state)
//   y_k = (S C_k + D x_k) silu(z_k),   k < R
// The state is still read once and written once, now with 2R FMAs per element instead of 2, so
// the step stays bound by HBM bandwidth for R <= 8 (at most 4 flops per state byte against a
// B200 fp32/HBM ridge of about 11): this is why MIMO leaves decode latency nearly unchanged.
//
// Design: one 256-thread CTA per (sequence, head).  The P x N fp32 state of the head moves as one
// bulk copy (cp.async.bulk) into shared memory and one back out, so the bytes in flight per SM
// are set by the CTAs resident (4 per SM, 38 KB of shared memory each at R = 4, N = 128), not by
// registers; while the load lands the CTA stages x, B and C of the head.  A state row of N floats
// is covered by N/4 lanes (a float4 each); at R <= 4 each lane holds its four columns of every
// B_k and C_k in registers for all of its rows.  The R read-outs of a row are a segmented
// butterfly reduce-scatter over the row's lanes.  The wait for the state load is bounded: if it
// gives up, the CTA sets the MIMO error word (reported by ssd_device_status) and writes nothing.
//
// SSD_EMU: compiled as plain C++ by the tests' host emulation (one thread per CUDA thread, real
// barriers for __syncthreads and the warp shuffles, the bulk copies as plain copies) under
// AddressSanitizer; the library is always built with nvcc.
#ifdef SSD_EMU
#include "emu_cuda.h"
#define SSD_LAUNCH(kern, grid, block, smem, st, ...) \
    ((void)(st), ::emu::launch((grid), (block), (smem), [&]() { kern(__VA_ARGS__); }))
#define SSD_DYN_SMEM() (::emu::smem())
#else
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_sm100.cuh"
#define SSD_LAUNCH(kern, grid, block, smem, st, ...) kern<<<(grid), (block), (smem), (st)>>>(__VA_ARGS__)
extern __shared__ __align__(16) unsigned char ssd_mimo_smem[];
#define SSD_DYN_SMEM() (ssd_mimo_smem)
#endif

#include "ssd_mimo.h"

namespace ssd {
namespace mimo {
namespace {

constexpr int kT = 256;
constexpr int kP = 64;
#define COMMA ,

#ifndef SSD_EMU
__device__ int g_mimo_error = 0;  // set when a CTA's state load never landed (bounded wait gave up)
__device__ __forceinline__ void flag_error() { atomicOr(&g_mimo_error, 1); }
#else
inline void flag_error() { ::emu::g_error = 1; }
#endif

__device__ __forceinline__ float ld_act(const void* p, int64_t i, bool bf16) {
    if (bf16) return __uint_as_float(static_cast<unsigned>(static_cast<const unsigned short*>(p)[i]) << 16);
    return static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_out(void* p, int64_t i, float v, bool bf16) {
    if (bf16)
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    else
        static_cast<float*>(p)[i] = v;
}
// 16-byte shared load (the address must be 16-byte aligned; the host emulation checks it).
__device__ __forceinline__ float4 lds4(const float* p) {
#ifdef SSD_EMU
    emu_check_aligned(p, 16);
#endif
    return *reinterpret_cast<const float4*>(p);
}
// 16-byte shared store (same alignment rule)
__device__ __forceinline__ void sts4(float* p, float4 v) {
#ifdef SSD_EMU
    emu_check_aligned(p, 16);
#endif
    *reinterpret_cast<float4*>(p) = v;
}
__device__ __forceinline__ float silu_f(float v) { return v / (1.f + __expf(-v)); }
__device__ __forceinline__ float softplus_f(float v) { return v > 20.f ? v : log1pf(__expf(v)); }

// Segmented reduce-scatter of CNT partial sums over the lanes of a state row (offsets O, O/2, .., 1
// inside segments of 2*O lanes).  While more than one sum is left, each level swaps half of them with
// the partner lane (lane ^ o): the lane keeps the upper half if its bit o is set, else the lower half,
// and adds what it receives; then the remaining single sum is reduced plainly.  Costs CNT/2 + CNT/4 +
// .. shuffles for the scatter levels instead of CNT per level.  On return vals[0 .. left) hold the
// full sums of outputs first .. first+left-1 (first built from the lane's scatter bits), the same in
// every lane that shares those bits.
template <int CNT, int O>
struct RowReduce {
    static __device__ __forceinline__ void run(float* vals, int lane, int& first, int& left) {
        if constexpr (O == 0) {
            left = CNT;
        } else if constexpr (CNT > 1) {
            constexpr int HALF = CNT / 2;
            const bool upper = (lane & O) != 0;
            float keep[HALF];
#pragma unroll
            for (int i = 0; i < HALF; ++i) {
                const float send = upper ? vals[i] : vals[HALF + i];
                const float mine = upper ? vals[HALF + i] : vals[i];
                keep[i] = mine + __shfl_xor_sync(0xffffffffu, send, O);
            }
#pragma unroll
            for (int i = 0; i < HALF; ++i) vals[i] = keep[i];
            if (upper) first += HALF;
            RowReduce<HALF, O / 2>::run(vals, lane, first, left);
        } else {
            vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], O);
            RowReduce<1, O / 2>::run(vals, lane, first, left);
        }
    }
};

#ifndef SSD_EMU
using sm100::bulk_commit;
using sm100::bulk_load;
using sm100::bulk_store;
using sm100::bulk_wait_read_all;
using sm100::fence_async_smem;
using sm100::fence_mbar_init;
using sm100::mbar_arrive_expect_tx;
using sm100::mbar_init;
using sm100::mbar_wait;
#endif

// grid batch * H, kT threads, smem_bytes(R, P, N) of dynamic shared memory.
template <int R, int N>
__global__ void __launch_bounds__(kT, (R <= 4 ? 5 : 3)) mimo_decode_kernel(MimoArgs a) {
    constexpr int LPR = N / 4;            // lanes per state row (a float4 each)
    constexpr int RPW = 32 / LPR;         // rows per warp per pass
    constexpr int ITER = kP / (8 * RPW);  // passes over the P rows with 8 warps
    constexpr bool kRegBC = R <= 4;       // B_k / C_k columns of the lane held in registers
    constexpr uint32_t kStateBytes = kP * N * 4;
    float* s_st = reinterpret_cast<float*>(SSD_DYN_SMEM());  // [P][N] the head's state
    float* s_x = s_st + kP * N;                              // [R][P]
    float* s_B = s_x + R * kP;                               // [R][N]
    float* s_C = s_B + R * N;                                // [R][N]
    float* s_y = s_C + R * N;                                // [R][P]
    uint64_t* bar = reinterpret_cast<uint64_t*>(s_y + R * kP);

    const int64_t bh = blockIdx.x;
    const int64_t b = bh / a.H;
    const int h = static_cast<int>(bh - b * a.H);
    const int g = h / (a.H / a.G);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rsub = lane / LPR, n0 = (lane % LPR) * 4;
    float* gstate = a.ssm_state + bh * kP * N;

    // the state load first: it is the step's traffic
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, kStateBytes);
        bulk_load(s_st, gstate, kStateBytes, bar);
    }
    const int64_t xo = bh * R * kP, bo = (b * a.G + g) * R * N;
    for (int i = tid; i < R * kP; i += kT) s_x[i] = ld_act(a.x, xo + i, a.act_bf16);
    for (int i = tid; i < R * N; i += kT) {
        s_B[i] = ld_act(a.B, bo + i, a.act_bf16);
        s_C[i] = ld_act(a.C, bo + i, a.act_bf16);
    }
    const float dtv = softplus_f(ld_act(a.dt, bh, a.act_bf16) + a.dt_bias[h]);
    const float decay = __expf(dtv * a.A[h]);
    __syncthreads();  // x, B, C staged; the barrier's initialisation visible to every thread

    float4 bq[kRegBC ? R : 1], cq[kRegBC ? R : 1];
    if constexpr (kRegBC) {
#pragma unroll
        for (int k = 0; k < R; ++k) {
            bq[k] = lds4(s_B + k * N + n0);
            cq[k] = lds4(s_C + k * N + n0);
        }
    }
    // bounded wait for the state (about 2 s); a CTA whose load never lands flags it and writes nothing
    const bool landed = mbar_wait(bar, 0, nullptr);
    if (__syncthreads_or(landed ? 0 : 1)) {
        if (tid == 0) flag_error();
        return;
    }

#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int p = (it * 8 + warp) * RPW + rsub;
        float* srow = s_st + p * N + n0;
        float4 s = lds4(srow);
        float ix = 0.f, iy = 0.f, iz = 0.f, iw = 0.f;
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const float xk = s_x[k * kP + p];
            const float4 bk = kRegBC ? bq[kRegBC ? k : 0] : lds4(s_B + k * N + n0);
            ix += xk * bk.x;
            iy += xk * bk.y;
            iz += xk * bk.z;
            iw += xk * bk.w;
        }
        s.x = fmaf(decay, s.x, dtv * ix);
        s.y = fmaf(decay, s.y, dtv * iy);
        s.z = fmaf(decay, s.z, dtv * iz);
        s.w = fmaf(decay, s.w, dtv * iw);
        sts4(srow, s);
        float part[R];
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const float4 ck = kRegBC ? cq[kRegBC ? k : 0] : lds4(s_C + k * N + n0);
            part[k] = s.x * ck.x + s.y * ck.y + s.z * ck.z + s.w * ck.w;
        }
        int first = 0, left = R;
        RowReduce<R, LPR / 2>::run(part, lane, first, left);
        // the scatter levels used the lane's highest segment bits; the lanes whose remaining bits are
        // zero write the sums they hold
        constexpr int SCAT = (R < LPR ? R : LPR);  // lanes that end up with distinct sums
        if ((lane % (LPR / SCAT)) == 0) {
#pragma unroll
            for (int k = 0; k < R; ++k)
                if (k < left) s_y[(first + k) * kP + p] = part[k];
        }
    }
    // the updated state goes back in one bulk store, once every thread's writes are visible to it
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        bulk_store(gstate, s_st, kStateBytes);
        bulk_commit();
    }
    const float Dh = a.D[h];
    for (int i = tid; i < R * kP; i += kT) {
        const float yv = s_y[i] + Dh * s_x[i];
        st_out(a.y, xo + i, yv * silu_f(ld_act(a.z, xo + i, a.act_bf16)), a.y_bf16);
    }
    if (tid == 0) bulk_wait_read_all();  // shared memory must outlive the store's reads
}

template <int R, int N>
void launch_rn(const MimoArgs& a, cudaStream_t st) {
    const dim3 grid(static_cast<unsigned>(a.batch * a.H));
    SSD_LAUNCH(mimo_decode_kernel<R COMMA N>, grid, dim3(kT), smem_bytes(R, kP, N), st, a);
}

template <int R>
cudaError_t launch_r(const MimoArgs& a, cudaStream_t st) {
    switch (a.N) {
        case 16: launch_rn<R, 16>(a, st); break;
        case 32: launch_rn<R, 32>(a, st); break;
        case 64: launch_rn<R, 64>(a, st); break;
        default: launch_rn<R, 128>(a, st); break;
    }
    return cudaGetLastError();
}

}  // namespace

#ifndef SSD_EMU
cudaError_t read_and_clear_mimo_error(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_mimo_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_mimo_error, &zero, sizeof(int));
}
#endif

// Runs the step on `st`.  Validated by the caller: P = 64, N in {16, 32, 64, 128}, R in {1, 2, 4, 8},
// H % G == 0, batch * H >= 1 and below 2^31.
cudaError_t launch_mimo_decode(const MimoArgs& a, cudaStream_t st) {
#ifndef SSD_EMU
    if (a.ev_before) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_before), st);
#endif
    cudaError_t e;
    switch (a.R) {
        case 1: e = launch_r<1>(a, st); break;
        case 2: e = launch_r<2>(a, st); break;
        case 4: e = launch_r<4>(a, st); break;
        default: e = launch_r<8>(a, st); break;
    }
#ifndef SSD_EMU
    if (a.ev_after) cudaEventRecord(static_cast<cudaEvent_t>(a.ev_after), st);
#endif
    return e;
}

}  // namespace mimo
}  // namespace ssd
