// Decode attention: the last Tq query rows of a sequence against a cache of
// its L keys and values.
//
// "nanoGPT: a real GPT in two 300-line files", section 2 "How the code
// works" describes generate() as a loop that runs the model and keeps the
// last position's scores; nanochat ("Karpathy's nano lineage: nanoGPT,
// llm.c, and nanochat") serves the same loop with a key/value cache.  Each
// step then needs causal attention for only the Tq newest positions
// (usually 1): query r sits at position L - Tq + r and sees keys
// 0 .. L - Tq + r.  That is the same softmax(scale q k^T) v as the full
// forward, for a few rows.
//
// There is almost no arithmetic per byte (2 * Tq flops per key element), so
// the work is bound by reading K and V once from HBM.  The keys of each head
// are split into chunks of kDecodeChunk, one CTA per (head, chunk), so even a
// batch of one sequence spreads over the SMs ("split-K"):
//   decode_partial_kernel<D, TQ>  per CTA: 4 warps stream the chunk's K and
//                          V rows, 16 bytes per lane and several keys per
//                          warp load, kDecodeUnroll loads per lane in flight
//                          (enough bytes in flight per SM to cover the DRAM
//                          latency); each lane group keeps an online softmax
//                          (running max m, sum l, output o) per query row,
//                          updated once per batch of keys; the groups are
//                          merged in shared memory and the CTA writes its
//                          (m, l, o) to the workspace.
//   decode_combine_kernel  per (head, query): merges the chunks' (m, l, o)
//                          (o = sum 2^(m_c - M) o_c / sum 2^(m_c - M) l_c)
//                          and writes O (bf16) and LSE (natural log).
// Scores are kept in log2 units (scale * log2(e) folded into q), so the
// exponentials are exp2; exp2f keeps them accurate, as the kernel is not
// bound by arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace cattn {

constexpr int kDecodeMaxTq = 8;     // query rows per call
constexpr int kDecodeChunk = 256;   // keys per CTA
constexpr int kDecodeWarps = 4;
constexpr int kDecodeUnroll = 4;    // key rows in flight per lane group

struct DecodeParams {
  const __nv_bfloat16* q;  // (B, H, Tq, D), element strides q_sb, q_sh, q_st
  const __nv_bfloat16* k;  // (B, H, >= L, D)
  const __nv_bfloat16* v;
  long long q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  float* part_ml;          // [BH][n_split][Tq][2]: m (log2 units), l
  float* part_o;           // [BH][n_split][Tq][D]
  __nv_bfloat16* o;        // (B, H, Tq, D), element strides o_sb, o_sh, o_st
  long long o_sb, o_sh, o_st;
  float* lse;              // (B, H, Tq) contiguous, natural log
  int H, Tq, L, n_split;
  float scale_log2;        // scale * log2(e)
};

// Lane layout: 8 consecutive elements (one 16-byte load) per lane, LPK
// lanes per key row, KPW keys side by side in a warp.
template <int D>
struct DecodeCfg {
  static constexpr int EPL = 8;
  static constexpr int LPK = D / EPL;                 // 2, 4, 8, 16 lanes per row
  static constexpr int KPW = 32 / LPK;                // 16, 8, 4, 2 keys per warp load
  static constexpr int SLOTS = kDecodeWarps * KPW;    // lane groups per CTA
  static constexpr int STEP = SLOTS * kDecodeUnroll;  // keys per CTA iteration
  static_assert(LPK * EPL == D && KPW * LPK == 32, "lane layout");
  static_assert(kDecodeChunk % STEP == 0, "chunk");
};

// 8 bf16 (one 16-byte load) -> 8 floats
__device__ __forceinline__ void unpack8(const uint4& t, float (&x)[8]) {
  const unsigned w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// TQ: query rows held per thread (Tq rounded up to 1, 2, 4 or 8; rows at or
// past Tq are idle).  Per iteration every lane group loads kDecodeUnroll
// keys' K and V rows at once (4 x 2 x 16 bytes per lane in flight), forms
// their scores, and then updates its online softmax once for the batch:
// m' = max(m, s_1..s_U), l' = l 2^(m - m') + sum 2^(s_u - m'),
// o' = o 2^(m - m') + sum 2^(s_u - m') v_u.
template <int D, int TQ>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_partial_kernel(const DecodeParams p) {
  using C = DecodeCfg<D>;
  constexpr int EPL = C::EPL, LPK = C::LPK, KPW = C::KPW, U = kDecodeUnroll;
  __shared__ float s_ml[C::SLOTS][TQ][2];
  __shared__ float s_o[C::SLOTS][TQ][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kslot = lane / LPK, sub = lane % LPK;   // key slot in the warp, lane in the row
  const int slot = warp * KPW + kslot;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int Tq = p.Tq;
  const int k0 = split * kDecodeChunk;
  const int k1 = min(p.L, k0 + kDecodeChunk);

  float qr[TQ][EPL];
  float m[TQ], l[TQ], o[TQ][EPL];
#pragma unroll
  for (int r = 0; r < TQ; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      o[r][e] = 0.f;
      qr[r][e] = 0.f;
    }
    if (r < Tq) {
      const uint4 t = *reinterpret_cast<const uint4*>(p.q + b * p.q_sb + h * p.q_sh +
                                                      r * p.q_st + sub * EPL);
      unpack8(t, qr[r]);
#pragma unroll
      for (int e = 0; e < EPL; ++e) qr[r][e] *= p.scale_log2;
    }
  }
  const __nv_bfloat16* kbase = p.k + b * p.k_sb + h * p.k_sh + sub * EPL;
  const __nv_bfloat16* vbase = p.v + b * p.v_sb + h * p.v_sh + sub * EPL;
  const int pos0 = p.L - Tq;  // position of query row 0

  // warp-uniform trip count: every lane runs every iteration (the shuffles
  // below take the full warp); keys past the chunk are masked, not skipped
  for (int base = k0; base < k1; base += C::STEP) {
    uint4 kraw[U], vraw[U];
    int key[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      key[u] = base + (u * kDecodeWarps + warp) * KPW + kslot;
      if (key[u] < k1) {
        kraw[u] = *reinterpret_cast<const uint4*>(kbase + static_cast<long long>(key[u]) * p.k_st);
        vraw[u] = *reinterpret_cast<const uint4*>(vbase + static_cast<long long>(key[u]) * p.v_st);
      } else {
        kraw[u] = vraw[u] = uint4{0u, 0u, 0u, 0u};
      }
    }
    // scores of the batch: s[r][u], -inf where not visible
    float s[TQ][U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float kx[EPL];
      unpack8(kraw[u], kx);
#pragma unroll
      for (int r = 0; r < TQ; ++r) {
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) d = fmaf(qr[r][e], kx[e], d);
#pragma unroll
        for (int off = LPK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        s[r][u] = (key[u] < k1 && key[u] <= pos0 + r) ? d : -INFINITY;
      }
    }
    // one online-softmax update per row for the whole batch; the scores
    // become the batch's weights 2^(s - m') in place
#pragma unroll
    for (int r = 0; r < TQ; ++r) {
      float mn = m[r];
#pragma unroll
      for (int u = 0; u < U; ++u) mn = fmaxf(mn, s[r][u]);
      // nothing visible yet: keep everything at zero (and avoid -inf - -inf)
      const float mu = mn == -INFINITY ? 0.f : mn;
      const float alpha = exp2f(m[r] - mu);  // 0 while m is -inf
      float lsum = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        s[r][u] = exp2f(s[r][u] - mu);         // 0 for a masked key
        lsum += s[r][u];
      }
      l[r] = fmaf(l[r], alpha, lsum);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[r][e] *= alpha;
      m[r] = mn;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float vx[EPL];
      unpack8(vraw[u], vx);
#pragma unroll
      for (int r = 0; r < TQ; ++r)
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[r][e] = fmaf(s[r][u], vx[e], o[r][e]);
    }
  }

  // lane groups -> shared memory -> one (m, l, o) per query for the CTA
#pragma unroll
  for (int r = 0; r < TQ; ++r) {
    if (r >= Tq) break;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s_o[slot][r][sub * EPL + e] = o[r][e];
    if (sub == 0) {
      s_ml[slot][r][0] = m[r];
      s_ml[slot][r][1] = l[r];
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < Tq * D; t += blockDim.x) {
    const int r = t / D, d = t - (t / D) * D;
    float M = -INFINITY;
    for (int sl = 0; sl < C::SLOTS; ++sl) M = fmaxf(M, s_ml[sl][r][0]);
    float lsum = 0.f, osum = 0.f;
    if (M > -INFINITY) {  // otherwise no key of this chunk is visible to the row
      for (int sl = 0; sl < C::SLOTS; ++sl) {
        const float w = exp2f(s_ml[sl][r][0] - M);  // 0 for a slot that saw nothing
        lsum = fmaf(s_ml[sl][r][1], w, lsum);
        osum = fmaf(s_o[sl][r][d], w, osum);
      }
    }
    const size_t row = (static_cast<size_t>(bh) * p.n_split + split) * Tq + r;
    p.part_o[row * D + d] = osum;
    if (d == 0) {
      p.part_ml[row * 2] = M;
      p.part_ml[row * 2 + 1] = lsum;
    }
  }
}

// One CTA of D threads per (head, query row): thread d merges column d of
// the chunks.  Key 0 is in chunk 0 and visible to every row, so the merged
// maximum is finite.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const DecodeParams p) {
  const int row = blockIdx.x;  // bh * Tq + r
  const int bh = row / p.Tq, r = row - (row / p.Tq) * p.Tq;
  const int b = bh / p.H, h = bh - b * p.H;
  const int d = threadIdx.x;
  const size_t first = static_cast<size_t>(bh) * p.n_split * p.Tq + r;  // chunk 0's row
  float M = -INFINITY;
  for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, p.part_ml[(first + static_cast<size_t>(s) * p.Tq) * 2]);
  float lsum = 0.f, osum = 0.f;
  for (int s = 0; s < p.n_split; ++s) {
    const size_t pr = first + static_cast<size_t>(s) * p.Tq;
    const float w = exp2f(p.part_ml[pr * 2] - M);
    lsum = fmaf(p.part_ml[pr * 2 + 1], w, lsum);
    osum = fmaf(p.part_o[pr * D + d], w, osum);
  }
  p.o[b * p.o_sb + h * p.o_sh + r * p.o_st + d] = __float2bfloat16_rn(osum / lsum);
  if (d == 0) p.lse[row] = (M + log2f(lsum)) * 0.69314718055994531f;
}

}  // namespace cattn
