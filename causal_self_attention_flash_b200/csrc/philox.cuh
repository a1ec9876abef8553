// Attention dropout mask bits from the Philox4x32-10 counter-based generator.
//
// "nanoGPT: a real GPT in two 300-line files", section 2 "How the code
// works" (model.py, CausalSelfAttention) hands the model's dropout rate to
// the fused attention while training; section 3 "Run it, tested" uses 0.2
// for the Shakespeare model.  The dropout is inverted dropout on the
// attention probabilities after the softmax: each P_ij is kept with
// probability 1 - p and the kept ones are scaled by 1 / (1 - p).
//
// Generator: Philox4x32 with 10 rounds (J. K. Salmon, M. A. Moraes,
// R. O. Dror, D. E. Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC 2011): a 4-word counter and a 2-word key; each round multiplies
// counter words 0 and 2 by two fixed 32-bit constants, keeps both halves of
// the 64-bit products and mixes the high halves with the other two words
// and the key; the key advances by two Weyl constants between rounds.
//
// Mask element (b, h, i, j), query i and key j, takes 16 bits of the block
// with counter (j >> 3, i, b*H + h, offset) and key (seed low, seed high):
// word (j & 7) >> 1, low half for even j and high half for odd j.  It is
// dropped iff those bits are below t = round(p * 65536), so the keep scale is
// 65536 / (65536 - t) (the drop probability is t / 65536, p to within 2^-17).
// The mask therefore does not depend on how the kernels tile the work: the
// forward (thread = query row) and the backward (thread = key row) derive
// the same bits.
#pragma once

#include <cstdint>

namespace cattn {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

struct DropParams {
  uint32_t t16x;    // drop threshold t shifted left by 16 (t = round(p * 65536))
  uint32_t k0, k1;  // seed, low and high word
  uint32_t offset;  // counter word 3
  float inv_keep;   // 65536 / (65536 - t)
};

__device__ __forceinline__ void philox4x32_10(uint32_t& c0, uint32_t& c1, uint32_t& c2,
                                              uint32_t& c3, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += kPhiloxW0;
      k1 += kPhiloxW1;
    }
    const uint32_t lo0 = c0 * kPhiloxM0, hi0 = __umulhi(c0, kPhiloxM0);
    const uint32_t lo1 = c2 * kPhiloxM1, hi1 = __umulhi(c2, kPhiloxM1);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
}

// Keep bits of keys 8*jg .. 8*jg + 7 for query i of head bh: bit e set iff
// key 8*jg + e is kept.  A 16-bit half h of word w is >= t exactly when
// (w << 16) (low half) or w (high half) is >= t << 16.
__device__ __forceinline__ uint32_t keep_byte(uint32_t jg, uint32_t i, uint32_t bh,
                                              const DropParams& d) {
  uint32_t c0 = jg, c1 = i, c2 = bh, c3 = d.offset;
  philox4x32_10(c0, c1, c2, c3, d.k0, d.k1);
  const uint32_t w[4] = {c0, c1, c2, c3};
  uint32_t b = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    b |= static_cast<uint32_t>((w[k] << 16) >= d.t16x) << (2 * k);
    b |= static_cast<uint32_t>(w[k] >= d.t16x) << (2 * k + 1);
  }
  return b;
}

}  // namespace cattn
