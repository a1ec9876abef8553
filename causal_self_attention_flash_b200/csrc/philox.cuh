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
  uint32_t* mask;   // the keep bits kept between forward and backward, or null
};

// Keep-bit cache: one block of 128 x 4 words per (head bh, query tile qt,
// key tile kt <= qt) of 128 x 128, at block bh * n_pairs + qt (qt + 1) / 2
// + kt (n_pairs = n_tiles (n_tiles + 1) / 2); word [kr][w] of a block holds
// bit c = keep bit of query 128 qt + 32 w + c, key 128 kt + kr.  Keys and
// queries past T hold generator bits too; nothing reads them.  The forward
// (thread = query row) writes it, the backward (thread = key row) reads one
// word per 32 queries.
__host__ __device__ constexpr size_t keep_cache_block(long long bh, int n_tiles, int qt, int kt) {
  return (static_cast<size_t>(bh) * (static_cast<size_t>(n_tiles) * (n_tiles + 1) / 2) +
          static_cast<size_t>(qt) * (qt + 1) / 2 + kt) * 512;
}

// The calling warp holds 32 consecutive query rows (32 w .. 32 w + 31 of a
// tile), each lane its row's keep bits for 128 keys (bit c of kw[c / 32]);
// stores them transposed into cache block `blk`: word [kr][w] gets bit
// `lane` from lane's key kr.  Each 32 x 32 bit block is transposed across
// the warp in five exchange rounds: at round j the off-diagonal j x j
// sub-blocks of every 2j x 2j block swap between lanes l and l ^ j.
__device__ __forceinline__ void store_keep_block(const uint32_t (&kw)[4], uint32_t* blk, int w,
                                                 int lane) {
#pragma unroll
  for (int kb = 0; kb < 4; ++kb) {
    uint32_t x = kw[kb];
#pragma unroll
    for (int j = 16, i = 0; j > 0; j >>= 1, ++i) {
      const uint32_t m = i == 0 ? 0x0000FFFFu : i == 1 ? 0x00FF00FFu : i == 2 ? 0x0F0F0F0Fu
                                                : i == 3 ? 0x33333333u : 0x55555555u;
      const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
      x = (lane & j) ? ((x & ~m) | ((y >> j) & m)) : ((x & m) | ((y & m) << j));
    }
    blk[(32 * kb + lane) * 4 + w] = x;
  }
}

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
