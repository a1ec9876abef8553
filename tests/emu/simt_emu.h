// Host emulation of the SIMT subset the decode kernel uses, for CPU tests.
//
// Each CUDA thread of a CTA runs as a std::thread.  The CTAs of one thread
// block cluster run together (their threads at once), clusters one after
// another; each CTA gets its own exactly sized dynamic shared-memory
// buffer.  Warp-collective operations (shuffles, and the warp-level
// instructions of decode_ptx_emu.h) exchange through per-warp slot arrays
// between two warp barriers; __syncthreads is a CTA barrier and the cluster
// barrier one over the cluster's threads.  Built with AddressSanitizer and
// UndefinedBehaviorSanitizer, every global and shared access of the kernel
// source is bounds- and alignment-checked against exactly sized host
// buffers.  No TMA, tcgen05 or mbarriers.
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

struct Cluster;

struct Cta {
  unsigned nthreads = 0;
  std::unique_ptr<std::barrier<>> cta_bar;
  std::vector<std::unique_ptr<std::barrier<>>> warp_bar;
  std::vector<float> slots;     // [warp][32] exchange slots for shuffles
  std::vector<uint64_t> words;  // [warp][32][kWords] for warp-level instructions
  uint8_t* dsmem = nullptr;     // dynamic shared memory, dsmem_bytes long
  size_t dsmem_bytes = 0;
  Cluster* cluster = nullptr;
  unsigned rank = 0;            // within the cluster
};
constexpr int kWords = 8;

struct Cluster {
  std::unique_ptr<std::barrier<>> bar;  // all threads of all its CTAs
  std::vector<Cta*> ctas;               // by rank
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

namespace emu {
// Each lane of the calling warp contributes n <= kWords words; returns the
// warp's table [32][kWords], valid until the warp's next exchange.
inline const uint64_t* warp_exchange(const uint64_t* mine, int n) {
  Cta* c = t_cta;
  const unsigned tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (32 * (warp + 1) > c->nthreads) throw std::logic_error("warp-level op in a partial warp");
  if (n > kWords) throw std::logic_error("exchange too wide");
  uint64_t* w = c->words.data() + static_cast<size_t>(warp) * 32 * kWords;
  c->warp_bar[warp]->arrive_and_wait();  // the previous exchange's readers are done
  for (int i = 0; i < n; ++i) w[lane * kWords + i] = mine[i];
  c->warp_bar[warp]->arrive_and_wait();
  return w;
}

// `bytes` at p must lie in this CTA's dynamic shared memory, `align`-aligned.
inline void check_smem(const void* p, size_t bytes, size_t align) {
  const Cta* c = t_cta;
  const uint8_t* q = static_cast<const uint8_t*>(p);
  if (q < c->dsmem || q + bytes > c->dsmem + c->dsmem_bytes)
    throw std::logic_error("shared-memory access outside the CTA's dynamic shared memory");
  if (reinterpret_cast<uintptr_t>(q) % align != 0)
    throw std::logic_error("misaligned shared-memory access");
}
}  // namespace emu

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

// Runs kernel(args...) over a 1-D grid of `grid_x` CTAs of `threads`
// threads (1-D blocks) with `smem_bytes` of dynamic shared memory each, in
// clusters of `cluster` consecutive CTAs (cluster rank = x % cluster): the
// threads of a cluster's CTAs run together, clusters one after another.
template <typename K, typename... A>
void launch_ex(unsigned grid_x, unsigned threads, size_t smem_bytes, unsigned cluster, K kernel,
               A... args) {
  if (threads == 0 || threads > 1024) throw std::logic_error("block size out of range");
  if (cluster == 0 || cluster > 8 || grid_x % cluster != 0)
    throw std::logic_error("cluster size must be 1..8 and divide the grid");
  for (unsigned c0 = 0; c0 < grid_x; c0 += cluster) {
    std::vector<std::unique_ptr<Cta>> ctas;
    std::vector<std::unique_ptr<uint8_t[]>> smem;
    Cluster cl;
    cl.bar = std::make_unique<std::barrier<>>(static_cast<std::ptrdiff_t>(threads * cluster));
    for (unsigned r = 0; r < cluster; ++r) {
      auto cta = std::make_unique<Cta>();
      cta->nthreads = threads;
      cta->cta_bar = std::make_unique<std::barrier<>>(threads);
      // a last, partial warp gets a barrier of its own size (its lanes
      // may not shuffle: only full-warp collectives are emulated)
      for (unsigned w = 0; w < (threads + 31) / 32; ++w)
        cta->warp_bar.push_back(std::make_unique<std::barrier<>>(
            static_cast<std::ptrdiff_t>(threads - 32 * w < 32 ? threads - 32 * w : 32)));
      cta->slots.assign((threads + 31) / 32 * 32, 0.f);
      cta->words.assign(static_cast<size_t>((threads + 31) / 32) * 32 * kWords, 0u);
      if (smem_bytes) {
        smem.emplace_back(new uint8_t[smem_bytes]);  // exact size: ASan bounds
        std::memset(smem.back().get(), 0xa5, smem_bytes);  // not zero: no free zero fill
        cta->dsmem = smem.back().get();
        cta->dsmem_bytes = smem_bytes;
      }
      cta->cluster = &cl;
      cta->rank = r;
      cl.ctas.push_back(cta.get());
      ctas.push_back(std::move(cta));
    }
    std::vector<std::thread> ts;
    ts.reserve(threads * cluster);
    for (unsigned r = 0; r < cluster; ++r)
      for (unsigned t = 0; t < threads; ++t)
        ts.emplace_back([&, r, t] {
          t_thread = uint3_{t, 0, 0};
          t_block = uint3_{c0 + r, 0, 0};
          t_bdim = dim3(threads);
          t_gdim = dim3(grid_x);
          t_cta = ctas[r].get();
          kernel(args...);
        });
    for (auto& th : ts) th.join();
  }
}

}  // namespace emu
