// ssd_cp.cu -- helpers for splitting one sequence across ranks (context parallelism).
//
// With the scalar-times-identity transition the state after a segment of
// tokens is affine in the state before it: S_out = Gamma * S_in + S_loc, where
// Gamma = exp(A * sum_t dt_t) (per sequence and head) and S_loc is the state the
// segment reaches from zero.  So W ranks holding consecutive segments of a
// sequence need one exchange: each scans its segment from zero (S_loc), the
// (S_loc, sum dt) of all ranks are gathered, every rank folds those of the
// ranks before it into its own initial state, and scans its segment again from
// that state (the chunked-prefill state passing of "EP6. 트랜스포머 대체 신경망 연구"
// §7-§8, carried across devices instead of across chunks).  The causal conv
// needs the 3 pre-conv tokens before a segment, which the previous rank
// provides.  This file holds the three small kernels of that scheme; the
// exchange itself is the caller's (NCCL all-gather).
#include "ssd.h"
#include "ssd_common.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

// conv_state[b][c][k] = pre-conv value of channel c at token L-3+k (history or zero before token 0).
template <typename T>
__global__ void conv_window_kernel(int64_t batch, int64_t L, int HP, int GN, const T* x, const T* Bm, const T* Cm,
                                   const T* hist, T* out) {
    const int conv_dim = HP + 2 * GN;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= batch * conv_dim * 3) return;
    const int k = (int)(e % 3);
    const int c = (int)((e / 3) % conv_dim);
    const int64_t b = e / (3 * (int64_t)conv_dim);
    const int64_t t = L - 3 + k;
    T v;
    if (t >= 0) {
        const size_t row = (size_t)(b * L + t);
        if (c < HP) v = x[row * HP + c];
        else if (c < HP + GN) v = Bm[row * GN + (c - HP)];
        else v = Cm[row * GN + (c - HP - GN)];
    } else {
        v = hist ? hist[((size_t)b * conv_dim + c) * 3 + (t + 3)] : from_f32<T>(0.f);
    }
    out[e] = v;
}

// dt_sum[b][h] = sum over the L tokens of softplus(dt_raw + dt_bias[h]).  Block (b, 32-head slice):
// lane = head, the 8 warps take every 8th token; the 8 partial sums are added in a fixed order.
template <typename T>
__global__ void __launch_bounds__(256) dt_sum_kernel(int64_t L, int H, const T* dt, const float* dt_bias,
                                                     float* dt_sum) {
    __shared__ float part[8][32];
    const int b = blockIdx.x, h = blockIdx.y * 32 + (threadIdx.x & 31), w = threadIdx.x >> 5;
    float s = 0.f;
    if (h < H) {
        const float bias = dt_bias[h];
        for (int64_t t = w; t < L; t += 8) s += softplus_f(to_f32(dt[((size_t)b * L + t) * H + h]) + bias);
    }
    part[w][threadIdx.x & 31] = s;
    __syncthreads();
    if (w == 0 && h < H) {
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) tot += part[k][threadIdx.x];
        dt_sum[(size_t)b * H + h] = tot;
    }
}

// state_in = fold of segments 0 .. upto-1 over init: S <- exp(A_h dt_sum[q]) S + seg_state[q].
__global__ void cp_combine_kernel(int64_t batch, int H, int PN, int upto, const float* A, const float* dt_sums,
                                  const float* seg_states, const float* init_state, float* state_in) {
    const int64_t per_seg = batch * H * (int64_t)PN;
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= per_seg) return;
    const int64_t bh = e / PN;
    const int h = (int)(bh % H);
    float s = init_state ? init_state[e] : 0.f;
    for (int q = 0; q < upto; ++q) s = __expf(A[h] * dt_sums[(size_t)q * batch * H + bh]) * s + seg_states[q * per_seg + e];
    state_in[e] = s;
}

}  // namespace
}  // namespace ssd

namespace {
bool al16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ssd_status check_core(const ssd_dims* d, ssd_dtype dtype) {
    if (!d) return SSD_ERR_NULL;
    if (dtype != SSD_F32 && dtype != SSD_BF16 && dtype != SSD_BF16_YF32) return SSD_ERR_DTYPE;
    if (d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->ngroups <= 0 || d->nheads % d->ngroups != 0)
        return SSD_ERR_SHAPE;
    if (d->headdim != 64 || !(d->d_state == 16 || d->d_state == 32 || d->d_state == 64 || d->d_state == 128))
        return SSD_ERR_SHAPE;
    return SSD_OK;
}
}  // namespace

extern "C" {

ssd_status ssd_conv_window(const ssd_dims* d, ssd_dtype dtype, const void* x, const void* B, const void* C,
                           const void* init_conv_state, void* conv_state, void* stream) {
    ssd_status st = check_core(d, dtype);
    if (st != SSD_OK) return st;
    const bool tokens = d->batch > 0 && d->seqlen > 0;
    if ((tokens && (!x || !B || !C)) || (d->batch > 0 && !conv_state)) return SSD_ERR_NULL;
    if (!al16(x) || !al16(B) || !al16(C) || !al16(init_conv_state) || !al16(conv_state)) return SSD_ERR_ALIGN;
    if (init_conv_state && init_conv_state == conv_state) return SSD_ERR_UNSUPPORTED;
    if (d->batch == 0) return SSD_OK;
    const ssd::Shape s = ssd::make_shape(*d);
    const int64_t n = s.batch * s.conv_dim * 3;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const unsigned blocks = (unsigned)((n + 255) / 256);
    if (dtype == SSD_F32)
        ssd::conv_window_kernel<float><<<blocks, 256, 0, cs>>>(s.batch, s.seqlen, s.HP, s.GN, (const float*)x,
                                                               (const float*)B, (const float*)C,
                                                               (const float*)init_conv_state, (float*)conv_state);
    else
        ssd::conv_window_kernel<__nv_bfloat16><<<blocks, 256, 0, cs>>>(
            s.batch, s.seqlen, s.HP, s.GN, (const __nv_bfloat16*)x, (const __nv_bfloat16*)B, (const __nv_bfloat16*)C,
            (const __nv_bfloat16*)init_conv_state, (__nv_bfloat16*)conv_state);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_dt_sum(const ssd_dims* d, ssd_dtype dtype, const float* dt_bias, const void* dt, float* dt_sum,
                      void* stream) {
    ssd_status st = check_core(d, dtype);
    if (st != SSD_OK) return st;
    if (!dt_bias || (d->batch > 0 && !dt_sum) || (d->batch > 0 && d->seqlen > 0 && !dt)) return SSD_ERR_NULL;
    if (!al16(dt) || !al16(dt_bias) || !al16(dt_sum)) return SSD_ERR_ALIGN;
    if (d->batch == 0) return SSD_OK;
    if (d->batch > 65535 * 64) return SSD_ERR_SHAPE;
    const dim3 grid((unsigned)d->batch, (unsigned)((d->nheads + 31) / 32));
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (dtype == SSD_F32)
        ssd::dt_sum_kernel<float><<<grid, 256, 0, cs>>>(d->seqlen, d->nheads, (const float*)dt, dt_bias, dt_sum);
    else
        ssd::dt_sum_kernel<__nv_bfloat16><<<grid, 256, 0, cs>>>(d->seqlen, d->nheads, (const __nv_bfloat16*)dt,
                                                                 dt_bias, dt_sum);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_cp_combine(const ssd_dims* d, int nseg, int upto, const float* A, const float* dt_sums,
                          const float* seg_states, const float* init_state, float* state_in, void* stream) {
    ssd_status st = check_core(d, SSD_F32);
    if (st != SSD_OK) return st;
    if (nseg < 1 || upto < 0 || upto > nseg) return SSD_ERR_SHAPE;
    if (!A || (d->batch > 0 && !state_in) || (upto > 0 && (!dt_sums || !seg_states))) return SSD_ERR_NULL;
    if (!al16(A) || !al16(dt_sums) || !al16(seg_states) || !al16(init_state) || !al16(state_in)) return SSD_ERR_ALIGN;
    if (init_state == state_in && init_state) return SSD_ERR_UNSUPPORTED;
    if (d->batch == 0) return SSD_OK;
    const int64_t n = d->batch * (int64_t)d->nheads * d->headdim * d->d_state;
    ssd::cp_combine_kernel<<<(unsigned)((n + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        d->batch, d->nheads, d->headdim * d->d_state, upto, A, dt_sums, seg_states, init_state, state_in);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // extern "C"
