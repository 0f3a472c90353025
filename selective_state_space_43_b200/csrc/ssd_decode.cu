// ssd_decode.cu -- one decode token of the Mamba-2 selective SSM for a batch.
//
// The step is a fixed-size state update per token: with the scalar-times-
// identity transition each fp32 state element is read once, updated with one
// FMA pair and written once, so the step is bound by HBM bandwidth
// ("Mamba-3: 추론을 우선한 상태 공간 모델", opening section; "Bamba-9B" page,
// 부록: 연산 강도).  Design:
//   * one 256-thread CTA per (sequence b, head h); the CTA first computes the
//     post-conv channels it needs (64 x channels of its head, 2N B/C channels
//     of its group) from the 3-column conv window plus the new token, and
//     rolls the window of its own x channels;
//   * the P x N fp32 state moves as one bulk copy (cp.async.bulk) into shared
//     memory and one back out, so the bytes in flight per SM are set by the
//     CTAs resident (6 per SM, ~34 KB of shared memory each at N = 128), not by
//     registers; the CTA computes the conv channels while the load lands; a
//     row of N floats is updated by N/4 lanes, a float4 each.  The wait for the
//     load is bounded: a CTA whose load never lands sets the decode error word
//     (reported by ssd_device_status as SSD_ERR_TIMEOUT) and writes no state;
//   * y = S.C is a segmented warp reduction over the N/4 lanes of a row;
//   * the shared B/C conv channels are rolled by a second, tiny kernel that
//     runs after every head has read the old window;
//   * both kernels are programmatic dependents of the kernel before them: the
//     roll waits for the state kernel's grid before it touches the windows, and
//     lets the next step's state kernel start, whose state load (written by the
//     previous state kernel, complete once the roll has passed its wait) then
//     overlaps the roll; that kernel waits for the roll before reading the B/C
//     windows.
#include "ssd_common.cuh"
#include "ssd_internal.h"
#include "ssd_sm100.cuh"

extern __shared__ __align__(16) unsigned char ssd_decode_smem[];

namespace ssd {

__device__ int g_decode_error = 0;  // set when a CTA's state load never landed (bounded wait gave up)

namespace {
constexpr int kDecodeCtas = 6;  // resident CTAs per SM the register budget is sized for
// shared memory of decode_state_kernel: the [P][N] state, the P + 2N post-conv channels, P read-outs, a barrier
constexpr size_t decode_smem_bytes(int P, int N) { return ((size_t)P * N + P + 2 * N + P) * 4 + 8; }
}  // namespace

template <typename T, typename TY, int N>
__global__ void __launch_bounds__(256, kDecodeCtas) decode_state_kernel(DecodeArgs a) {
    constexpr int P = 64;
    constexpr int LPR = N / 4;           // lanes per state row (float4 each)
    constexpr int RPW = 32 / LPR;        // rows per warp per pass
    constexpr int ITER = P / (8 * RPW);  // passes over the P rows with 8 warps
    constexpr uint32_t kStateBytes = P * N * 4;
    float* s_st = reinterpret_cast<float*>(ssd_decode_smem);  // [P][N] the head's state
    float* s_u = s_st + P * N;                                // post-conv x (P), B (N), C (N)
    float* s_y = s_u + P + 2 * N;                             // [P]
    uint64_t* bar = reinterpret_cast<uint64_t*>(s_y + P);

    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh - b * a.H;
    const int g = h / a.hpg;
    const int tid = threadIdx.x;
    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.B);
    const T* Cm = static_cast<const T*>(a.C);
    T* conv_state = static_cast<T*>(a.conv_state);
    float* gstate = a.ssm_state + (size_t)bh * P * N;

    // the state load first: it is the step's traffic
    if (tid == 0) {
        sm100::mbar_init(bar, 1);
        sm100::fence_mbar_init();
        sm100::mbar_arrive_expect_tx(bar, kStateBytes);
        sm100::bulk_load(s_st, gstate, kStateBytes, bar);
    }
    // the roll of the previous step may launch now (it waits for this grid), and this grid reads the conv
    // windows only once the kernel before it (that roll, when it is) has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int i = tid; i < P + 2 * N; i += 256) {
        int c;
        float xin;
        if (i < P) {
            c = h * P + i;
            xin = to_f32(x[(size_t)b * a.HP + c]);
        } else if (i < P + N) {
            const int n = i - P;
            c = a.HP + g * N + n;
            xin = to_f32(Bm[((size_t)b * a.G + g) * N + n]);
        } else {
            const int n = i - P - N;
            c = a.HP + a.GN + g * N + n;
            xin = to_f32(Cm[((size_t)b * a.G + g) * N + n]);
        }
        T* cs = conv_state + ((size_t)b * a.conv_dim + c) * 3;
        const float h0 = to_f32(cs[0]), h1 = to_f32(cs[1]), h2 = to_f32(cs[2]);
        const float* w = a.conv_w + (size_t)c * 4;
        const float pre = a.conv_b[c] + w[0] * h0 + w[1] * h1 + w[2] * h2 + w[3] * xin;
        s_u[i] = silu_f(pre);
        if (i < P) {  // this head owns its x channels: roll them now
            cs[0] = cs[1];
            cs[1] = cs[2];
            cs[2] = x[(size_t)b * a.HP + c];
        }
    }
    const float dtv = softplus_f(to_f32(static_cast<const T*>(a.dt)[(size_t)b * a.H + h]) + a.dt_bias[h]);
    const float decay = __expf(dtv * a.A[h]);
    __syncthreads();  // the post-conv channels staged; the barrier's initialisation visible to every thread

    const int warp = tid >> 5, lane = tid & 31;
    const int rsub = lane / LPR, n0 = (lane % LPR) * 4;
    const float4 bq = make_float4(s_u[P + n0], s_u[P + n0 + 1], s_u[P + n0 + 2], s_u[P + n0 + 3]);
    const float4 cq = make_float4(s_u[P + N + n0], s_u[P + N + n0 + 1], s_u[P + N + n0 + 2], s_u[P + N + n0 + 3]);
    // bounded wait for the state (about 2 s); a CTA whose load never lands flags it and writes no state
    const bool landed = sm100::mbar_wait(bar, 0, nullptr);
    if (__syncthreads_or(landed ? 0 : 1)) {
        if (tid == 0) atomicOr(&g_decode_error, 1);
        return;
    }
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int p = (it * 8 + warp) * RPW + rsub;
        float4* srow = reinterpret_cast<float4*>(s_st + p * N + n0);
        const float xd = dtv * s_u[p];
        float4 s = *srow;
        s.x = fmaf(decay, s.x, xd * bq.x);
        s.y = fmaf(decay, s.y, xd * bq.y);
        s.z = fmaf(decay, s.z, xd * bq.z);
        s.w = fmaf(decay, s.w, xd * bq.w);
        *srow = s;
        float part = s.x * cq.x + s.y * cq.y + s.z * cq.z + s.w * cq.w;
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((lane % LPR) == 0) s_y[p] = part;
    }
    // the updated state goes back in one bulk store, once every thread's writes are visible to it
    sm100::fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        sm100::bulk_store(gstate, s_st, kStateBytes);
        sm100::bulk_commit();
    }
    if (tid < P) {
        const size_t off = (size_t)b * a.HP + (size_t)h * P + tid;
        const float yv = s_y[tid] + a.D[h] * s_u[tid];
        const float zv = to_f32(static_cast<const T*>(a.z)[off]);
        static_cast<TY*>(a.y)[off] = from_f32<TY>(yv * silu_f(zv));
    }
    if (tid == 0) sm100::bulk_wait_read_all();  // shared memory must outlive the store's reads
}

// Roll the 2*G*N shared B/C conv channels by one token (after every head read them).
template <typename T>
__global__ void __launch_bounds__(256) decode_roll_bc_kernel(DecodeArgs a, int64_t total) {
    // every head has read the old window once the state kernel's grid is complete; the next step's state
    // kernel may then start (its state load no longer races the state kernel that wrote it)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int two_gn = 2 * a.GN;
    const int64_t b = idx / two_gn;
    const int j = (int)(idx - b * two_gn);
    const T xin = j < a.GN ? static_cast<const T*>(a.B)[b * a.GN + j]
                           : static_cast<const T*>(a.C)[b * a.GN + (j - a.GN)];
    T* cs = static_cast<T*>(a.conv_state) + ((size_t)b * a.conv_dim + a.HP + j) * 3;
    cs[0] = cs[1];
    cs[1] = cs[2];
    cs[2] = xin;
}

// A launch that may start before the kernel ahead of it in the stream completes (that kernel allows it
// with griddepcontrol.launch_dependents; this one waits for it with griddepcontrol.wait).
template <typename... Params, typename... Args>
static cudaError_t launch_dependent(void (*kern)(Params...), unsigned grid, size_t smem, cudaStream_t st,
                                    Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <typename T, typename TY, int N>
static cudaError_t launch_decode_t(const DecodeArgs& a, int64_t batch, cudaStream_t st, const TimingHook& hook) {
    hook.before(st);
    cudaError_t e = launch_dependent(decode_state_kernel<T, TY, N>, (unsigned)(batch * a.H), decode_smem_bytes(64, N),
                                     st, a);
    if (e != cudaSuccess) return e;
    hook.after(st);
    const int64_t total = batch * 2 * a.GN;
    if (total > 0) {
        e = launch_dependent(decode_roll_bc_kernel<T>, (unsigned)((total + 255) / 256), 0, st, a, total);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, int64_t batch, ActKind kind, cudaStream_t st,
                          const TimingHook& hook) {
    using bf16 = __nv_bfloat16;
    switch (a.N) {
#define SSD_DEC_CASE(NN)                                                                    \
    case NN:                                                                                \
        switch (kind) {                                                                     \
            case ActKind::BF16: return launch_decode_t<bf16, bf16, NN>(a, batch, st, hook);  \
            case ActKind::BF16_YF32: return launch_decode_t<bf16, float, NN>(a, batch, st, hook); \
            default: return launch_decode_t<float, float, NN>(a, batch, st, hook);           \
        }
        SSD_DEC_CASE(16)
        SSD_DEC_CASE(32)
        SSD_DEC_CASE(64)
        SSD_DEC_CASE(128)
#undef SSD_DEC_CASE
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t read_and_clear_decode_error(int* flag) {
    cudaError_t e = cudaMemcpyFromSymbol(flag, g_decode_error, sizeof(int));
    if (e != cudaSuccess) return e;
    const int zero = 0;
    return cudaMemcpyToSymbol(g_decode_error, &zero, sizeof(int));
}

}  // namespace ssd
