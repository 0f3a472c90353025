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
//   * the P x N fp32 state is streamed with 16-byte vectors: a row of N floats
//     is covered by N/4 lanes, every load of the CTA is issued before the first
//     FMA (P*N*4/256 bytes in flight per thread), loads and stores use the
//     streaming cache hint since nothing is re-read within the step;
//   * y = S.C is a segmented warp reduction over the N/4 lanes of a row;
//   * the shared B/C conv channels are rolled by a second, tiny kernel that
//     runs after every head has read the old window.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

template <typename T, typename TY, int N>
__global__ void __launch_bounds__(256) decode_state_kernel(DecodeArgs a) {
    constexpr int P = 64;
    constexpr int LPR = N / 4;           // lanes per state row (float4 each)
    constexpr int RPW = 32 / LPR;        // rows per warp per pass
    constexpr int ITER = P / (8 * RPW);  // passes over the P rows with 8 warps
    __shared__ float s_u[P + 2 * N];     // post-conv x (P), B (N), C (N)
    __shared__ float s_y[P];

    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh - b * a.H;
    const int g = h / a.hpg;
    const int tid = threadIdx.x;
    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.B);
    const T* Cm = static_cast<const T*>(a.C);
    T* conv_state = static_cast<T*>(a.conv_state);

    // Issue the state loads first: they are the step's traffic.
    const int warp = tid >> 5, lane = tid & 31;
    const int rsub = lane / LPR, n0 = (lane % LPR) * 4;
    float4* S = reinterpret_cast<float4*>(a.ssm_state + (size_t)bh * P * N);
    float4 v[ITER];
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int p = (it * 8 + warp) * RPW + rsub;
        v[it] = __ldcs(S + ((p * N + n0) >> 2));
    }

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
    __syncthreads();

    const float4 bq = make_float4(s_u[P + n0], s_u[P + n0 + 1], s_u[P + n0 + 2], s_u[P + n0 + 3]);
    const float4 cq = make_float4(s_u[P + N + n0], s_u[P + N + n0 + 1], s_u[P + N + n0 + 2], s_u[P + N + n0 + 3]);
#pragma unroll
    for (int it = 0; it < ITER; ++it) {
        const int p = (it * 8 + warp) * RPW + rsub;
        const float xd = dtv * s_u[p];
        float4 s = v[it];
        s.x = fmaf(decay, s.x, xd * bq.x);
        s.y = fmaf(decay, s.y, xd * bq.y);
        s.z = fmaf(decay, s.z, xd * bq.z);
        s.w = fmaf(decay, s.w, xd * bq.w);
        __stcs(S + ((p * N + n0) >> 2), s);
        float part = s.x * cq.x + s.y * cq.y + s.z * cq.z + s.w * cq.w;
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if ((lane % LPR) == 0) s_y[p] = part;
    }
    __syncthreads();
    if (tid < P) {
        const size_t off = (size_t)b * a.HP + (size_t)h * P + tid;
        const float yv = s_y[tid] + a.D[h] * s_u[tid];
        const float zv = to_f32(static_cast<const T*>(a.z)[off]);
        static_cast<TY*>(a.y)[off] = from_f32<TY>(yv * silu_f(zv));
    }
}

// Roll the 2*G*N shared B/C conv channels by one token (after every head read them).
template <typename T>
__global__ void __launch_bounds__(256) decode_roll_bc_kernel(DecodeArgs a, int64_t total) {
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

template <typename T, typename TY, int N>
static cudaError_t launch_decode_t(const DecodeArgs& a, int64_t batch, cudaStream_t st, const TimingHook& hook) {
    hook.before(st);
    decode_state_kernel<T, TY, N><<<(unsigned)(batch * a.H), 256, 0, st>>>(a);
    hook.after(st);
    const int64_t total = batch * 2 * a.GN;
    if (total > 0) decode_roll_bc_kernel<T><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a, total);
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

}  // namespace ssd
