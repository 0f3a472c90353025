// ssd_norm.cu -- RMSNorm of the gated SSD output over contiguous channel groups.
//
// Mamba-2 blocks normalise the gated output y * SiLU(z) before their output
// projection; the "Mamba-3: 추론을 우선한 상태 공간 모델" page (정규화 section)
// keeps that norm in hybrid models and names its variants (before or after the
// gate, grouped or over all channels).  Here: after the gate (on the y that
// ssd_prefill / ssd_decode_step return), over norm_groups contiguous groups of
// each token's H*P channels:
//   out = v * rsqrt(mean_group(v^2) + eps) * weight[c]
// One warp per (token, group): the squares are summed in fp32 (each lane over
// its elements in order, then a fixed butterfly across lanes), the group is
// scaled and written.  HBM-bound: one read and one write of y.
#include "ssd.h"
#include "ssd_common.cuh"

namespace ssd {
namespace {

__device__ __forceinline__ void unpack8(const uint4 w, float (&v)[8]) {
    const uint32_t r[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(r[k] << 16);
        v[2 * k + 1] = __uint_as_float(r[k] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    unpack8(*reinterpret_cast<const uint4*>(p), v);
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t r[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        r[k] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(r[0], r[1], r[2], r[3]);
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Groups of up to kCache * 256 channels are read once and kept in registers (bf16 as the packed words
// loaded, unpacked twice, so that a thread holds 16 registers of data and more warps fit an SM); larger
// groups are read twice (the second time from L2).
constexpr int kCache = 4;

template <typename T>
__global__ void __launch_bounds__(256) group_rmsnorm_kernel(int64_t units, int channels, int group, float eps,
                                                            const T* in, const float* weight, T* out) {
    const int64_t u = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (row, group) of this warp
    const int lane = threadIdx.x & 31;
    if (u >= units) return;
    const int ngroups = channels / group;
    const int64_t row = u / ngroups;
    const int c0 = (int)(u % ngroups) * group;
    const T* src = in + (size_t)row * channels + c0;
    T* dst = out + (size_t)row * channels + c0;
    constexpr bool kPacked = sizeof(T) == 2;
    const bool cached = group <= kCache * 256;
    uint4 raw[kPacked ? kCache : 1];
    float v[kPacked ? 1 : kCache][8];
    float ss = 0.f;
    if (cached) {
#pragma unroll
        for (int it = 0; it < kCache; ++it) {
            const int c = lane * 8 + it * 256;
            if (c < group) {
                if constexpr (kPacked) raw[it] = *reinterpret_cast<const uint4*>(src + c);
                else load8(src + c, v[it]);
            }
        }
#pragma unroll
        for (int it = 0; it < kCache; ++it) {
            const int c = lane * 8 + it * 256;
            if (c < group) {
                float t[8];
                if constexpr (kPacked) unpack8(raw[it], t);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float x = kPacked ? t[k] : v[kPacked ? 0 : it][k];
                    ss = fmaf(x, x, ss);
                }
            }
        }
    } else {
        for (int c = lane * 8; c < group; c += 256) {
            float t[8];
            load8(src + c, t);
#pragma unroll
            for (int k = 0; k < 8; ++k) ss = fmaf(t[k], t[k], ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / (float)group + eps);
    auto scale_store = [&](int c, float (&t)[8]) {
        const float4 wa = *reinterpret_cast<const float4*>(weight + c0 + c);
        const float4 wb = *reinterpret_cast<const float4*>(weight + c0 + c + 4);
        const float w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = t[k] * r * w[k];
        store8(dst + c, t);
    };
    if (cached) {
#pragma unroll
        for (int it = 0; it < kCache; ++it) {
            const int c = lane * 8 + it * 256;
            if (c < group) {
                if constexpr (kPacked) {
                    float t[8];
                    unpack8(raw[it], t);
                    scale_store(c, t);
                } else {
                    scale_store(c, v[kPacked ? 0 : it]);
                }
            }
        }
    } else {
        for (int c = lane * 8; c < group; c += 256) {
            float t[8];
            load8(src + c, t);
            scale_store(c, t);
        }
    }
}

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_gated_rmsnorm(int64_t rows, int32_t channels, int32_t norm_groups, float eps,
                                        ssd_dtype dtype, const void* y, const float* weight, void* out,
                                        void* stream) {
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (rows < 0 || channels <= 0 || norm_groups <= 0 || channels % norm_groups != 0) return SSD_ERR_SHAPE;
    const int group = channels / norm_groups;
    if (group % 8 != 0 || !(eps >= 0.f)) return SSD_ERR_SHAPE;
    if (rows > 0 && (!y || !weight || !out)) return SSD_ERR_NULL;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(weight) |
                           reinterpret_cast<uintptr_t>(out)) & 15u;
    if (mis) return SSD_ERR_ALIGN;
    if (rows == 0) return SSD_OK;
    const int64_t units = rows * norm_groups;
    if (units > (int64_t)0x7fffffff * 8) return SSD_ERR_SHAPE;  // one warp per unit, 8 per block
    const unsigned blocks = (unsigned)((units * 32 + 255) / 256);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (dtype == SSD_F32)
        ssd::group_rmsnorm_kernel<float><<<blocks, 256, 0, cs>>>(units, channels, group, eps, (const float*)y, weight,
                                                                 (float*)out);
    else
        ssd::group_rmsnorm_kernel<__nv_bfloat16><<<blocks, 256, 0, cs>>>(units, channels, group, eps,
                                                                         (const __nv_bfloat16*)y, weight,
                                                                         (__nv_bfloat16*)out);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
