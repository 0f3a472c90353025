// emu_cuda.h -- a host emulation of the parts of the CUDA execution model that
// the backward kernels use, so that their exact source runs on the CPU under
// AddressSanitizer (tests only; never part of the library).
//
// A launch runs the grid's blocks one after another.  Each block gets one
// std::thread per CUDA thread, its own dynamic shared memory (filled with
// 0xFF bytes, a NaN pattern for floats, so reads of unwritten shared memory
// show up in the results) and a std::barrier that __syncthreads() waits on.
// threadIdx and blockIdx are per-thread; blockDim and gridDim per launch.
#pragma once

#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <barrier>
#include <memory>
#include <thread>
#include <vector>

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)

typedef int cudaError_t;
typedef void* cudaStream_t;
static constexpr cudaError_t cudaSuccess = 0;
inline cudaError_t cudaGetLastError() { return cudaSuccess; }

struct dim3 {
    unsigned x, y, z;
    dim3(unsigned a = 1, unsigned b = 1, unsigned c = 1) : x(a), y(b), z(c) {}
};

namespace emu {

struct Ctx {
    dim3 tid, bid;
    std::barrier<>* bar = nullptr;
    std::atomic<int>* or_flag = nullptr;  // __syncthreads_or's slot of this block
    unsigned char* smem = nullptr;
    std::barrier<>* warp_bar = nullptr;  // the 32 threads of this thread's warp
    float* warp_buf = nullptr;           // 32 exchange slots of this warp
    unsigned lane = 0;
};
inline thread_local Ctx ctx;
inline dim3 g_grid, g_block;
inline int g_error = 0;  // a kernel's device error word (set by an emulated bounded wait that gave up)

inline unsigned char* smem() { return ctx.smem; }

template <class F>
void launch(dim3 grid, dim3 block, size_t smem_bytes, F&& body) {
    g_grid = grid;
    g_block = block;
    const unsigned nt = block.x * block.y * block.z;
    for (unsigned bz = 0; bz < grid.z; ++bz)
        for (unsigned by = 0; by < grid.y; ++by)
            for (unsigned bx = 0; bx < grid.x; ++bx) {
                std::unique_ptr<unsigned char[]> sm(new unsigned char[smem_bytes ? smem_bytes : 1]);
                memset(sm.get(), 0xFF, smem_bytes ? smem_bytes : 1);
                std::barrier<> bar(nt);
                std::atomic<int> or_flag(0);
                const unsigned nw = (nt + 31) / 32;
                std::vector<std::unique_ptr<std::barrier<>>> wbar;
                for (unsigned w = 0; w < nw; ++w)
                    wbar.emplace_back(new std::barrier<>(static_cast<ptrdiff_t>(w + 1 < nw ? 32 : nt - 32 * w)));
                std::unique_ptr<float[]> wbuf(new float[32 * nw]);
                std::vector<std::thread> th;
                th.reserve(nt);
                for (unsigned t = 0; t < nt; ++t)
                    th.emplace_back([&, t]() {
                        ctx.tid = dim3(t % block.x, (t / block.x) % block.y, t / (block.x * block.y));
                        ctx.bid = dim3(bx, by, bz);
                        ctx.bar = &bar;
                        ctx.or_flag = &or_flag;
                        ctx.smem = sm.get();
                        ctx.warp_bar = wbar[t / 32].get();
                        ctx.warp_buf = wbuf.get() + 32 * (t / 32);
                        ctx.lane = t % 32;
                        body();
                        // a thread that returns early leaves the barriers' later phases to the others
                        bar.arrive_and_drop();
                        ctx.warp_bar->arrive_and_drop();
                    });
                for (auto& x : th) x.join();
            }
}

}  // namespace emu

#define threadIdx (::emu::ctx.tid)
#define blockIdx (::emu::ctx.bid)
#define blockDim (::emu::g_block)
#define gridDim (::emu::g_grid)

inline void __syncthreads() { ::emu::ctx.bar->arrive_and_wait(); }
// Block-wide OR of v: every thread of the block calls it (three barrier phases, so the slot can be
// reset before any thread can reach the next call).
inline int __syncthreads_or(int v) {
    ::emu::Ctx& c = ::emu::ctx;
    c.bar->arrive_and_wait();
    if (v) c.or_flag->store(1);
    c.bar->arrive_and_wait();
    const int r = c.or_flag->load();
    c.bar->arrive_and_wait();
    if (c.tid.x == 0 && c.tid.y == 0 && c.tid.z == 0) c.or_flag->store(0);
    return r;
}

// mbarriers and untiled bulk copies: a bulk copy is a plain copy made when it is issued, so every
// wait on its barrier succeeds at once (the copies' bounds are still checked by AddressSanitizer).
inline void mbar_init(uint64_t*, unsigned) {}
inline void fence_mbar_init() {}
inline void mbar_arrive_expect_tx(uint64_t*, unsigned) {}
inline bool mbar_wait(uint64_t*, unsigned, volatile int*, uint64_t = 0) { return true; }
inline void bulk_load(void* dst, const void* src, unsigned bytes, uint64_t*) { memcpy(dst, src, bytes); }
inline void bulk_store(void* dst, const void* src, unsigned bytes) { memcpy(dst, src, bytes); }
inline void bulk_commit() {}
inline void bulk_wait_read_all() {}
inline void fence_async_smem() {}

// Vector accesses must be aligned to their size on the GPU; the host would not fault, so check here.
inline void emu_check_aligned(const void* p, unsigned bytes) {
    if (reinterpret_cast<uintptr_t>(p) % bytes) {
        fprintf(stderr, "emu: misaligned %u-byte access at %p\n", bytes, p);
        abort();
    }
}
inline float __uint_as_float(unsigned u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}

// 16-byte vector, streaming loads and stores (plain accesses here)
struct float4 {
    float x, y, z, w;
};
struct float2 {
    float x, y;
};
inline float4 make_float4(float a, float b, float c, float d) { return float4{a, b, c, d}; }
inline float2 make_float2(float a, float b) { return float2{a, b}; }

inline float4 __ldcs(const float4* p) { return *p; }
inline void __stcs(float4* p, float4 v) { *p = v; }
inline float __expf(float v) { return expf(v); }
inline float __fdividef(float a, float b) { return a / b; }
// Blackwell's packed fp32 arithmetic, lane by lane
inline float2 __ffma2_rn(float2 x, float2 y, float2 z) { return make_float2(fmaf(x.x, y.x, z.x), fmaf(x.y, y.y, z.y)); }
inline float2 __fmul2_rn(float2 x, float2 y) { return make_float2(x.x * y.x, x.y * y.y); }
inline float2 __fadd2_rn(float2 x, float2 y) { return make_float2(x.x + y.x, x.y + y.y); }

// bf16 storage: round to nearest, ties to even, on the 16 dropped bits (NaN kept quiet)
struct __nv_bfloat16 {
    unsigned short bits;
};
inline __nv_bfloat16 __float2bfloat16_rn(float f) {
    unsigned u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return __nv_bfloat16{(unsigned short)((u >> 16) | 0x40u)};
    u += 0x7fffu + ((u >> 16) & 1u);
    return __nv_bfloat16{(unsigned short)(u >> 16)};
}

// Warp broadcast: every lane of the warp posts its value and reads lane src's (all 32 lanes call it).
inline float __shfl_sync(unsigned, float v, int src) {
    ::emu::Ctx& c = ::emu::ctx;
    c.warp_buf[c.lane] = v;
    c.warp_bar->arrive_and_wait();
    const float r = c.warp_buf[static_cast<unsigned>(src) & 31u];
    c.warp_bar->arrive_and_wait();
    return r;
}

// Warp shift: lane l reads lane l - delta's value (its own below delta); all 32 lanes call it.
inline float __shfl_up_sync(unsigned, float v, int delta) {
    ::emu::Ctx& c = ::emu::ctx;
    c.warp_buf[c.lane] = v;
    c.warp_bar->arrive_and_wait();
    const float r = c.lane >= static_cast<unsigned>(delta) ? c.warp_buf[c.lane - delta] : v;
    c.warp_bar->arrive_and_wait();
    return r;
}

// Warp shuffle: every lane of the warp posts its value, waits for the others, reads its partner's.
// All 32 lanes must call it (the kernels only shuffle in warp-uniform code).
inline float __shfl_xor_sync(unsigned, float v, int lanemask) {
    ::emu::Ctx& c = ::emu::ctx;
    c.warp_buf[c.lane] = v;
    c.warp_bar->arrive_and_wait();
    const float r = c.warp_buf[c.lane ^ static_cast<unsigned>(lanemask)];
    c.warp_bar->arrive_and_wait();
    return r;
}
