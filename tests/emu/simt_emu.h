// Host emulation of the SIMT subset the decode kernels use, for CPU tests.
//
// Each CUDA thread of a CTA runs as a std::thread; CTAs run one after
// another, so function-level `static` stands in for `__shared__` memory.
// Warp shuffles exchange through a per-warp slot array between two warp
// barriers; __syncthreads is a CTA barrier.  Built with AddressSanitizer and
// UndefinedBehaviorSanitizer, every global and shared access of the kernel
// source is bounds- and alignment-checked against exactly sized host
// buffers.  No tensor cores, TMA or mbarriers: only plain SIMT kernels.
#pragma once

#include <barrier>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <memory>
#include <stdexcept>
#include <thread>
#include <vector>

struct uint3_ {
  unsigned x = 0, y = 0, z = 0;
};
struct dim3 {
  unsigned x = 1, y = 1, z = 1;
  dim3(unsigned a = 1, unsigned b = 1, unsigned c = 1) : x(a), y(b), z(c) {}
};
// vector types with CUDA's alignment, so that UBSan checks the same
// alignment the device needs
struct alignas(8) uint2 {
  unsigned x, y;
};
struct alignas(16) uint4 {
  unsigned x, y, z, w;
};
struct alignas(8) float2 {
  float x, y;
};
struct alignas(16) float4 {
  float x, y, z, w;
};

#define __global__
#define __device__
#define __host__
#define __forceinline__ inline
#define __launch_bounds__(...)
#define __shared__ static
#define __restrict__

namespace emu {

struct Cta {
  unsigned nthreads = 0;
  std::unique_ptr<std::barrier<>> cta_bar;
  std::vector<std::unique_ptr<std::barrier<>>> warp_bar;
  std::vector<float> slots;  // [warp][32] exchange slots for shuffles
};

inline thread_local uint3_ t_thread, t_block;
inline thread_local dim3 t_bdim, t_gdim;
inline thread_local Cta* t_cta = nullptr;

}  // namespace emu

#define threadIdx (emu::t_thread)
#define blockIdx (emu::t_block)
#define blockDim (emu::t_bdim)
#define gridDim (emu::t_gdim)

inline void __syncthreads() { emu::t_cta->cta_bar->arrive_and_wait(); }

// warp barrier (full warps only, like the shuffles)
inline void __syncwarp(unsigned mask = 0xffffffffu) {
  if (mask != 0xffffffffu) throw std::logic_error("only full-warp __syncwarp is emulated");
  emu::t_cta->warp_bar[threadIdx.x / 32]->arrive_and_wait();
}

inline float __shfl_xor_sync(unsigned mask, float v, int lane_mask) {
  if (mask != 0xffffffffu) throw std::logic_error("only full-warp shuffles are emulated");
  emu::Cta* c = emu::t_cta;
  const unsigned tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (32 * (warp + 1) > c->nthreads) throw std::logic_error("shuffle in a partial warp");
  float* s = c->slots.data() + warp * 32;
  c->warp_bar[warp]->arrive_and_wait();
  s[lane] = v;
  c->warp_bar[warp]->arrive_and_wait();
  const float r = s[lane ^ static_cast<unsigned>(lane_mask)];
  return r;
}

using std::exp2f;
using std::fmaf;
using std::fmaxf;
using std::log2f;
inline int min(int a, int b) { return a < b ? a : b; }

namespace emu {

// Runs kernel(args...) over grid x block, one CTA at a time (1-D blocks).
template <typename K, typename... A>
void launch(dim3 grid, unsigned threads, K kernel, A... args) {
  if (threads == 0 || threads > 1024) throw std::logic_error("block size out of range");
  for (unsigned bz = 0; bz < grid.z; ++bz)
    for (unsigned by = 0; by < grid.y; ++by)
      for (unsigned bx = 0; bx < grid.x; ++bx) {
        Cta cta;
        cta.nthreads = threads;
        cta.cta_bar = std::make_unique<std::barrier<>>(threads);
        // a last, partial warp gets a barrier of its own size (its lanes
        // may not shuffle: only full-warp shuffles are emulated)
        for (unsigned w = 0; w < (threads + 31) / 32; ++w)
          cta.warp_bar.push_back(std::make_unique<std::barrier<>>(
              static_cast<std::ptrdiff_t>(threads - 32 * w < 32 ? threads - 32 * w : 32)));
        cta.slots.assign((threads + 31) / 32 * 32, 0.f);
        std::vector<std::thread> ts;
        ts.reserve(threads);
        for (unsigned t = 0; t < threads; ++t)
          ts.emplace_back([&, t] {
            t_thread = uint3_{t, 0, 0};
            t_block = uint3_{bx, by, bz};
            t_bdim = dim3(threads);
            t_gdim = grid;
            t_cta = &cta;
            kernel(args...);
          });
        for (auto& th : ts) th.join();
      }
}

}  // namespace emu
