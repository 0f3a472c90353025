// ssd_common.cuh -- small device helpers shared by the SSD kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Host-side view of the sizes, with the derived quantities every kernel needs.
struct Shape {
    int64_t batch, seqlen;
    int H, P, N, G, Q;
    int HP, GN, conv_dim, heads_per_group;
    int64_t nchunks;
};

inline Shape make_shape(const ssd_dims& d) {
    Shape s;
    s.batch = d.batch;
    s.seqlen = d.seqlen;
    s.H = d.nheads;
    s.P = d.headdim;
    s.N = d.d_state;
    s.G = d.ngroups;
    s.Q = d.chunk;
    s.HP = s.H * s.P;
    s.GN = s.G * s.N;
    s.conv_dim = s.HP + 2 * s.GN;
    s.heads_per_group = s.G > 0 ? s.H / s.G : 0;
    s.nchunks = s.Q > 0 ? (d.seqlen + s.Q - 1) / s.Q : 0;
    return s;
}

// ---- activation types --------------------------------------------------------
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// ---- scalar math (CUDA's own functions; no re-implementations) ---------------
// softplus(v) = log(1 + e^v); above 20 the correction log1p(e^-v) < 2.1e-9 is dropped.
__device__ __forceinline__ float softplus_f(float v) { return v > 20.f ? v : log1pf(__expf(v)); }
// SiLU(v) = v / (1 + e^-v) with the fast exponential and divide.
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.f + __expf(-v)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace ssd
