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
// Mask element (b, h, i, j), query i and key j, takes 8 bits of the block
// with counter (j >> 4, i, b*H + h, offset) and key (seed low, seed high):
// byte j & 3 of word (j & 15) >> 2.  It is dropped iff that byte is below
// t = round(p * 256), so the keep scale is 256 / (256 - t) (the drop
// probability is t / 256, p to within 2^-9).  One block serves 16 keys of
// one query.  The mask does not depend on how the kernels tile the work:
// the forward (thread = query row) and the backward (thread = key row)
// derive the same bits.
#pragma once

#include <cstdint>

namespace cattn {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

constexpr int kPhiloxRounds = 10;

// DropParams{} is "no dropout".
struct DropParams {
  uint32_t t = 0;              // drop threshold round(p * 256); 0 = no dropout
  uint32_t t_lo = 0;           // (t & 0x7F) in every byte
  uint32_t t_maj = 0;          // all ones when t < 128, else 0 (see keep_flags)
  uint32_t offset = 0;         // counter word 3
  // the key of every round: rk[2r] = seed low + r * W0, rk[2r + 1] =
  // seed high + r * W1 (mod 2^32), set on the host so that the rounds read
  // them as kernel parameters
  uint32_t rk[2 * kPhiloxRounds] = {};
  float inv_keep = 1.f;        // 256 / (256 - t)
  uint32_t* mask = nullptr;    // the keep bits kept between forward and backward, or null
};

// The round keys of seed (k0 low, k1 high word).
__host__ __device__ inline void philox_round_keys(uint32_t k0, uint32_t k1, uint32_t* rk) {
  for (int r = 0; r < kPhiloxRounds; ++r) {
    rk[2 * r] = k0;
    rk[2 * r + 1] = k1;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
}

// Keep-bit cache: one block of 128 x 4 words per (head bh, query tile qt,
// key tile kt <= qt) of 128 x 128, at block bh * n_pairs + qt (qt + 1) / 2
// + kt (n_pairs = n_tiles (n_tiles + 1) / 2); word [kr][w] of a block holds
// the keep bit of query 128 qt + 32 w + c, key 128 kt + kr, at bit
// il_pos(c) (the interleaved order below).  Keys and queries past T hold
// generator bits too; nothing reads them.  The forward (thread = query
// row) writes it, the backward (thread = key row) reads one word per 32
// queries.
__host__ __device__ constexpr size_t keep_cache_block(long long bh, int n_tiles, int qt, int kt) {
  return (static_cast<size_t>(bh) * (static_cast<size_t>(n_tiles) * (n_tiles + 1) / 2) +
          static_cast<size_t>(qt) * (qt + 1) / 2 + kt) * 512;
}

// 32 x 32 bit transpose across a warp: on entry lane l holds row l (bit c
// = element (l, c)), on return column l (bit c = element (c, l)).  Five
// exchange rounds: at round j the off-diagonal j x j sub-blocks of every
// 2j x 2j block swap between lanes l and l ^ j.
__device__ __forceinline__ uint32_t warp_transpose32(uint32_t x, int lane) {
#pragma unroll
  for (int j = 16, i = 0; j > 0; j >>= 1, ++i) {
    const uint32_t m = i == 0 ? 0x0000FFFFu : i == 1 ? 0x00FF00FFu : i == 2 ? 0x0F0F0F0Fu
                                              : i == 3 ? 0x33333333u : 0x55555555u;
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, j);
    x = (lane & j) ? ((x & ~m) | ((y >> j) & m)) : ((x & m) | ((y & m) << j));
  }
  return x;
}

// Interleaved order of a 32-element keep word (keys in the forward's
// keep32_il, queries in the cache and the backward): element 16 h + 4 v + k
// sits at bit 8 k + 4 h + v, so that shifting the word left by 7 - 4 h - v
// puts the flags of elements 16 h + 4 v .. + 3 on the top bits of bytes
// 0 .. 3 (for prmt_sign).  il_key(position) inverts it.
__host__ __device__ constexpr int il_pos(int key) {
  return 8 * (key & 3) + 4 * ((key >> 4) & 1) + ((key >> 2) & 3);
}
__host__ __device__ constexpr int il_key(int pos) {
  return 16 * ((pos >> 2) & 1) + 4 * (pos & 3) + (pos >> 3);
}

// The calling warp holds 32 consecutive query rows (32 w .. 32 w + 31 of a
// tile), each lane its row's keep bits for 128 keys, key 32 kb + c at bit
// il_pos(c) of kw[kb]; stores them transposed into cache block `blk`: word
// [kr][w] gets query 32 w + c's bit for key kr at bit il_pos(c).  Lane p
// first takes the row of query il_key(p), so that the transpose puts the
// queries in the interleaved order; lane p then holds key il_key(p).
__device__ __forceinline__ void store_keep_block(const uint32_t (&kw)[4], uint32_t* blk, int w,
                                                 int lane) {
  const int kr = il_key(lane);
#pragma unroll
  for (int kb = 0; kb < 4; ++kb)
    blk[(32 * kb + kr) * 4 + w] = warp_transpose32(__shfl_sync(0xffffffffu, kw[kb], kr), lane);
}

// One round: both 32 x 32 -> 64-bit products as single widening multiplies.
__device__ __forceinline__ void philox4x32_10(uint32_t& c0, uint32_t& c1, uint32_t& c2,
                                              uint32_t& c3, const uint32_t (&rk)[2 * kPhiloxRounds]) {
#pragma unroll
  for (int r = 0; r < kPhiloxRounds; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(c0) * kPhiloxM0;
    const uint64_t p1 = static_cast<uint64_t>(c2) * kPhiloxM1;
    const uint32_t n0 = static_cast<uint32_t>(p1 >> 32) ^ c1 ^ rk[2 * r];
    const uint32_t n2 = static_cast<uint32_t>(p0 >> 32) ^ c3 ^ rk[2 * r + 1];
    c0 = n0;
    c1 = static_cast<uint32_t>(p1);
    c2 = n2;
    c3 = static_cast<uint32_t>(p0);
  }
}

// Bit k (k < 4) set iff byte k of w is >= t, all four bytes at once.
// r = (w | 0x80 in every byte) - (t & 0x7F in every byte) borrows across
// no byte boundary, and its top bit in byte k says whether the byte's low
// seven bits reach t's.  byte >= t iff its top bit beats t's, or the top
// bits are equal and the low seven bits reach t's: the majority of the
// byte's top bit, r's top bit and (t < 128).  The four top bits are then
// gathered by one multiplication (the partial products land on distinct
// bits, so nothing carries into bits 28..31).
__device__ __forceinline__ uint32_t keep_flags(uint32_t w, const DropParams& d) {
  const uint32_t r = (w | 0x80808080u) - d.t_lo;
  return ((w & r) | (d.t_maj & (w | r))) & 0x80808080u;
}
__device__ __forceinline__ uint32_t keep_nibble(uint32_t w, const DropParams& d) {
  return (keep_flags(w, d) * 0x00204081u) >> 28;
}

// Keep bits of keys 16*jg .. 16*jg + 15 for query i of head bh: bit e set
// iff key 16*jg + e is kept.
__device__ __forceinline__ uint32_t keep16(uint32_t jg, uint32_t i, uint32_t bh,
                                           const DropParams& d) {
  uint32_t c0 = jg, c1 = i, c2 = bh, c3 = d.offset;
  philox4x32_10(c0, c1, c2, c3, d.rk);
  return keep_nibble(c0, d) | keep_nibble(c1, d) << 4 | keep_nibble(c2, d) << 8 |
         keep_nibble(c3, d) << 12;
}

// Keep bits of keys 32*jp .. 32*jp + 31 for query i in the interleaved
// order (il_pos): the four flag words of a block need only a shift each.
__device__ __forceinline__ uint32_t keep32_il(uint32_t jp, uint32_t i, uint32_t bh,
                                              const DropParams& d) {
  uint32_t x = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t c0 = 2 * jp + h, c1 = i, c2 = bh, c3 = d.offset;
    philox4x32_10(c0, c1, c2, c3, d.rk);
    x |= keep_flags(c0, d) >> (7 - 4 * h) | keep_flags(c1, d) >> (6 - 4 * h) |
         keep_flags(c2, d) >> (5 - 4 * h) | keep_flags(c3, d) >> (4 - 4 * h);
  }
  return x;
}

// Byte-wise sign replication: byte n of the result is 0xFF iff the top
// bit of the byte of x chosen by selector nibble n (its low 3 bits) is set.
__device__ __forceinline__ uint32_t prmt_sign(uint32_t x, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(x), "r"(sel));
  return r;
}

}  // namespace cattn
