// ssd_prefill_simt.cu -- chunked SSD prefill on the CUDA cores (fp32 math).
//
// The general path: every supported shape and both activation dtypes.  It
// computes the same chunked decomposition as the tensor-core path, with fp32
// FMAs instead of tcgen05 tiles (Mamba-2 state-space duality: inside a chunk
// the layer is a masked attention-like product, across chunks a state is
// passed on; "EP6. 트랜스포머 대체 신경망 연구" §7-§8).
//
// One 256-thread CTA per (sequence b, head h) walks the chunks in order and
// keeps the running P x N state in shared memory.  Per chunk of Qc <= Q tokens:
//   1. u = SiLU(conv4(raw) + bias) for the head's x channels and its group's
//      B and C channels (history from the previous chunk, the initial conv
//      state or zeros);  dt = softplus(dt_raw + dt_bias);  cs = inclusive
//      cumsum of dt*A within the chunk;
//   2. for each row t:  w_s = (C_t . B_s) exp(cs_t - cs_s) dt_s  (s <= t)
//        y_t = sum_s w_s x_s + exp(cs_t) C_t . S_prev + D x_t,  y_t *= SiLU(z_t)
//   3. S <- exp(cs_last) S + sum_s exp(cs_last - cs_s) dt_s x_s (outer) B_s.
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kP = 64;

template <int N, int Q>
struct SimtSmem {
    static constexpr int NB = N + 1;  // padded B / state rows: lanes walking s (or p) hit distinct banks
    static constexpr size_t floats = (size_t)Q * NB  // sB
                                     + (size_t)Q * N   // sC
                                     + (size_t)Q * kP  // sX
                                     + (size_t)kP * NB // sS
                                     + (size_t)kWarps * Q + 3 * (size_t)Q;
    static constexpr size_t bytes = floats * sizeof(float);
};

template <typename T>
__device__ __forceinline__ float raw_at(const PrefillArgs& a, int64_t b, int64_t row0, int64_t s, int c) {
    // pre-conv value of channel c at token s of sequence b (whose rows start at row0); s < 0 reads the history
    if (s < 0) {
        if (!a.init_conv_state) return 0.f;
        return to_f32(static_cast<const T*>(a.init_conv_state)[((size_t)b * a.conv_dim + c) * 3 + (s + 3)]);
    }
    const size_t row = (size_t)(row0 + s);
    if (c < a.HP) return to_f32(static_cast<const T*>(a.x)[row * a.rs_x + c]);
    if (c < a.HP + a.GN) return to_f32(static_cast<const T*>(a.B)[row * a.rs_B + (c - a.HP)]);
    return to_f32(static_cast<const T*>(a.C)[row * a.rs_C + (c - a.HP - a.GN)]);
}

template <typename T, typename TY, int N, int Q>
__global__ void __launch_bounds__(kThreads, 1) prefill_simt_kernel(PrefillArgs a) {
    using SM = SimtSmem<N, Q>;
    constexpr int NB = SM::NB;
    extern __shared__ float4 smem_f4[];
    float* sB = reinterpret_cast<float*>(smem_f4);
    float* sC = sB + Q * NB;
    float* sX = sC + Q * N;
    float* sS = sX + Q * kP;
    float* sW = sS + kP * NB;
    float* sDt = sW + kWarps * Q;
    float* sCs = sDt + Q;
    float* sE = sCs + Q;  // exp(cs_last - cs_s) * dt_s

    const int b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int g = h / a.hpg;
    const SeqSpan span = seq_span(a, b);  // rows of sequence b and its length
    if (!span.ok && threadIdx.x == 0 && a.err) atomicOr(a.err, kErrBadSeqlens);
    const int64_t Ls = span.len, nchunks = (Ls + Q - 1) / Q;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float A = a.A[h], Dh = a.D[h], dtb = a.dt_bias[h];
    const int cx = h * kP, cb = a.HP + g * N, cc = a.HP + a.GN + g * N;

    for (int i = tid; i < kP * N; i += kThreads) {
        const int p = i / N, n = i % N;
        sS[p * NB + n] = a.init_state ? a.init_state[((size_t)b * a.H + h) * kP * N + i] : 0.f;
    }

    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t t0 = c * Q;
        const int Qc = (int)(Ls - t0 < Q ? Ls - t0 : Q);
        __syncthreads();  // previous chunk fully consumed

        // 1. conv + SiLU of the head's channels, dt and the in-chunk cumsum.  Channel-major: a thread slides
        //    a 4-tap window down its channel's rows, the loads of kRowBlk rows issued before their FMAs
        //    (neighbouring threads read neighbouring channels of a row).
        constexpr int CH = kP + 2 * N;
        constexpr int kRowBlk = 8;
        for (int j = tid; j < CH; j += kThreads) {
            const int ch = j < kP ? cx + j : (j < kP + N ? cb + (j - kP) : cc + (j - kP - N));
            const float4 w = *reinterpret_cast<const float4*>(a.conv_w + (size_t)ch * 4);
            const float bias = a.conv_b[ch];
            float h0 = raw_at<T>(a, b, span.row0, t0 - 3, ch), h1 = raw_at<T>(a, b, span.row0, t0 - 2, ch),
                  h2 = raw_at<T>(a, b, span.row0, t0 - 1, ch);
            for (int tb = 0; tb < Qc; tb += kRowBlk) {
                float r[kRowBlk];
#pragma unroll
                for (int k = 0; k < kRowBlk; ++k) r[k] = tb + k < Qc ? raw_at<T>(a, b, span.row0, t0 + tb + k, ch) : 0.f;
#pragma unroll
                for (int k = 0; k < kRowBlk; ++k) {
                    const int t = tb + k;
                    const float u = silu_f(bias + w.x * h0 + w.y * h1 + w.z * h2 + w.w * r[k]);
                    h0 = h1;
                    h1 = h2;
                    h2 = r[k];
                    if (t < Qc) {
                        if (j < kP) sX[t * kP + j] = u;
                        else if (j < kP + N) sB[t * NB + (j - kP)] = u;
                        else sC[t * N + (j - kP - N)] = u;
                    }
                }
            }
        }
        if (warp == 0) {
            constexpr int PER = Q / 32;
            float v[PER];
            float run = 0.f;
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                const int t = lane * PER + k;
                float dA = 0.f;
                if (t < Qc) {
                    const float dtv = softplus_f(to_f32(static_cast<const T*>(a.dt)[((size_t)span.row0 + t0 + t) * a.rs_dt + h]) + dtb);
                    sDt[t] = dtv;
                    dA = dtv * A;
                } else {
                    sDt[t] = 0.f;
                }
                run += dA;
                v[k] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float up = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += up;
            }
            const float excl = incl - run;
#pragma unroll
            for (int k = 0; k < PER; ++k) sCs[lane * PER + k] = v[k] + excl;
        }
        __syncthreads();
        const float cs_last = sCs[Qc - 1];
        for (int s = tid; s < Q; s += kThreads) sE[s] = s < Qc ? __expf(cs_last - sCs[s]) * sDt[s] : 0.f;

        // 2. outputs, one row t per warp at a time (state S is the previous chunk's); the dot products run
        //    four independent partial sums so that their shared-memory loads overlap
        float* wrow = sW + warp * Q;
        for (int t = warp; t < Qc; t += kWarps) {
            const float cst = sCs[t];
            for (int s = lane; s < Q; s += 32) {
                float gsum = 0.f;
                if (s <= t) {
                    float g4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                    for (int n = 0; n < N; n += 4) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) g4[e] += sC[t * N + n + e] * sB[s * NB + n + e];
                    }
                    gsum = ((g4[0] + g4[1]) + (g4[2] + g4[3])) * (__expf(cst - sCs[s]) * sDt[s]);
                }
                wrow[s] = gsum;
            }
            __syncwarp();
            const float dec = __expf(cst);
            for (int p = lane; p < kP; p += 32) {
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
                int s = 0;
                for (; s + 3 <= t; s += 4) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) a4[e] += wrow[s + e] * sX[(s + e) * kP + p];
                }
                for (; s <= t; ++s) a4[0] += wrow[s] * sX[s * kP + p];
                const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
                float o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int n = 0; n < N; n += 4) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) o4[e] += sC[t * N + n + e] * sS[p * NB + n + e];
                }
                const float off = (o4[0] + o4[1]) + (o4[2] + o4[3]);
                const float yv = acc + dec * off + Dh * sX[t * kP + p];
                const size_t row = (size_t)span.row0 + t0 + t;
                const size_t o = row * a.HP + cx + p;
                const float zv = to_f32(static_cast<const T*>(a.z)[row * a.rs_z + cx + p]);
                static_cast<TY*>(a.y)[o] = from_f32<TY>(yv * silu_f(zv));
            }
            __syncwarp();
        }
        __syncthreads();

        // 3. state passing: S <- exp(cs_last) S + sum_s e_s x_s (outer) B_s
        const float dl = __expf(cs_last);
        for (int i = tid; i < kP * N; i += kThreads) {
            const int p = i / N, n = i % N;
            float a4[4] = {0.f, 0.f, 0.f, 0.f};
            int s = 0;
            for (; s + 4 <= Qc; s += 4) {
#pragma unroll
                for (int e = 0; e < 4; ++e) a4[e] += sE[s + e] * sX[(s + e) * kP + p] * sB[(s + e) * NB + n];
            }
            for (; s < Qc; ++s) a4[0] += sE[s] * sX[s * kP + p] * sB[s * NB + n];
            sS[p * NB + n] = dl * sS[p * NB + n] + ((a4[0] + a4[1]) + (a4[2] + a4[3]));
        }
    }
    __syncthreads();
    for (int i = tid; i < kP * N; i += kThreads) {
        const int p = i / N, n = i % N;
        a.final_state[((size_t)b * a.H + h) * kP * N + i] = sS[p * NB + n];
    }
    // conv tail: this head's x channels; the group's B/C channels by its first head
    const bool owns_bc = (h % a.hpg) == 0;
    const int nch = kP + (owns_bc ? 2 * N : 0);
    for (int i = tid; i < nch * 3; i += kThreads) {
        const int j = i / 3, k = i % 3;
        const int ch = j < kP ? cx + j : (j < kP + N ? cb + (j - kP) : cc + (j - kP - N));
        const float v = raw_at<T>(a, b, span.row0, Ls - 3 + k, ch);
        static_cast<T*>(a.conv_state)[((size_t)b * a.conv_dim + ch) * 3 + k] = from_f32<T>(v);
    }
}

template <typename T, typename TY, int N, int Q>
cudaError_t launch_simt_t(const PrefillArgs& a, cudaStream_t st, const TimingHook& hook) {
    const size_t smem = SimtSmem<N, Q>::bytes;
    cudaError_t e = cudaFuncSetAttribute(prefill_simt_kernel<T, TY, N, Q>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    hook.before(st);
    prefill_simt_kernel<T, TY, N, Q><<<(unsigned)(a.batch * a.H), kThreads, smem, st>>>(a);
    hook.after(st);
    return cudaGetLastError();
}

template <typename T, typename TY, int Q>
cudaError_t launch_simt_q(const PrefillArgs& a, cudaStream_t st, const TimingHook& hook) {
    switch (a.N) {
        case 16: return launch_simt_t<T, TY, 16, Q>(a, st, hook);
        case 32: return launch_simt_t<T, TY, 32, Q>(a, st, hook);
        case 64: return launch_simt_t<T, TY, 64, Q>(a, st, hook);
        case 128: return launch_simt_t<T, TY, 128, Q>(a, st, hook);
        default: return cudaErrorInvalidValue;
    }
}

template <typename T, typename TY>
cudaError_t launch_simt_dt(const PrefillArgs& a, cudaStream_t st, const TimingHook& hook) {
    return a.Q == 64 ? launch_simt_q<T, TY, 64>(a, st, hook) : launch_simt_q<T, TY, 128>(a, st, hook);
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a, ActKind kind, cudaStream_t st, const TimingHook& hook) {
    using bf16 = __nv_bfloat16;
    switch (kind) {
        case ActKind::BF16: return launch_simt_dt<bf16, bf16>(a, st, hook);
        case ActKind::BF16_YF32: return launch_simt_dt<bf16, float>(a, st, hook);
        default: return launch_simt_dt<float, float>(a, st, hook);
    }
}

}  // namespace ssd
