// Work-item dealing for the persistent forward grid (the backward keeps
// plain alternating passes).
//
// Items are numbered longest first.  A grid of G CTAs takes them in passes:
// pass k deals items k*G .. k*G + G-1, one per CTA.  Which CTA gets which
// item of a pass is given by the pass's code: bit 15 the direction d, bits
// 0..14 a rotation r; item k*G + j goes to CTA (r + j) mod G (d = 0) or
// (r - j) mod G (d = 1).  Every pass is a bijection between its items and
// the CTAs, so every item is dealt exactly once whatever the codes.
//
// The host plans the codes once per shape (plan_passes): pass by pass it
// takes the direction and rotation that leave the lowest maximum CTA load
// (then the lowest sum of squared loads), with an item's load the number of
// tiles it works through, which puts the longest items of each pass on the
// least-loaded CTAs (longest-processing-time scheduling, one pass at a
// time).  Passes past the codes, or all passes when there are more than
// kMaxPassCodes, alternate direction without rotation (pass k even: item
// k*G + b to CTA b; odd: k*G + G-1-b).
#pragma once

#include <cstdint>

namespace cattn {

constexpr int kMaxPassCodes = 64;

struct PassCodes {
  uint32_t code2[kMaxPassCodes / 2];  // pass k's code in bits 16 (k & 1) .. + 15 of code2[k / 2]
  int n;                              // passes with a code (0: all alternate)
};

__host__ __device__ inline uint32_t pass_code(const PassCodes& pc, int k) {
  return (pc.code2[k >> 1] >> (16 * (k & 1))) & 0xffffu;
}

// The forward copies the codes into shared memory once (kPassSmemBytes at
// a 4-byte aligned address, before its start-up barrier) and looks them up
// there; the copy reads the kernel parameter at compile-time indices only.
constexpr int kPassSmemBytes = 2 * kMaxPassCodes;

// The item of pass k for CTA b, or -1 past the last item; `code` is pass
// k's code when k < n_codes.
__host__ __device__ inline int pass_item_coded(int k, int b, int G, int n_items, int n_codes,
                                               uint32_t code) {
  int j;
  if (k < n_codes) {
    const int r = static_cast<int>(code & 0x7fffu);
    j = (code >> 15) ? r - b : b - r;
    if (j < 0) j += G;  // |r - b| < G
  } else {
    j = (k & 1) ? G - 1 - b : b;
  }
  const long long u = static_cast<long long>(k) * G + j;
  return u < n_items ? static_cast<int>(u) : -1;
}

__host__ __device__ inline int pass_item(int k, int b, int G, int n_items, const PassCodes& pc) {
  return pass_item_coded(k, b, G, n_items, pc.n, k < pc.n ? pass_code(pc, k) : 0u);
}

#ifdef __CUDACC__
// The copy into shared memory (thread 0, fully unrolled), and the lookup
// from there.
__device__ __forceinline__ void pass_codes_to_smem(const PassCodes& pc, uint16_t* codes_s) {
  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < kMaxPassCodes / 2; ++i)
      reinterpret_cast<uint32_t*>(codes_s)[i] = pc.code2[i];
  }
}
__device__ __forceinline__ int pass_item_smem(int k, int b, int G, int n_items, int n_codes,
                                              const uint16_t* codes_s) {
  return pass_item_coded(k, b, G, n_items, n_codes, k < n_codes ? codes_s[k] : 0u);
}
#endif

}  // namespace cattn
