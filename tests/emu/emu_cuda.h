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
#include <string.h>

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
    unsigned char* smem = nullptr;
};
inline thread_local Ctx ctx;
inline dim3 g_grid, g_block;

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
                std::vector<std::thread> th;
                th.reserve(nt);
                for (unsigned t = 0; t < nt; ++t)
                    th.emplace_back([&, t]() {
                        ctx.tid = dim3(t % block.x, (t / block.x) % block.y, t / (block.x * block.y));
                        ctx.bid = dim3(bx, by, bz);
                        ctx.bar = &bar;
                        ctx.smem = sm.get();
                        body();
                        // a thread that returns early leaves the barrier's later phases to the others
                        bar.arrive_and_drop();
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
inline float __uint_as_float(unsigned u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}
