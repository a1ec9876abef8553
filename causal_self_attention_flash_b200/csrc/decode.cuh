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
// the work is bound by reading K and V once from HBM, and the design is
// about keeping enough of that read in flight on every SM:
//   decode_kernel<D>, one launch:
//     - a head's keys are cut into chunks of decode_chunk(D) keys (4 KB of
//       K and 4 KB of V) and dealt to a thread-block cluster of n_split CTAs
//       (a contiguous run of chunks each), so that even a few heads spread
//       over the SMs ("split-K");
//     - inside a CTA, chunk j of the run goes to warp j % kDecodeWarps, and
//       every warp streams its own chunks through a private ring of
//       kDecodeStages shared-memory slots with cp.async (16-byte pieces,
//       swizzled by row so that the ldmatrix reads below are free of bank
//       conflicts): kDecodeStages chunks per warp are always on their way;
//     - per chunk, the warp computes s = q k^T on the tensor cores
//       (mma.sync m16n8k16: the query rows, zero-padded to 16, are the A
//       operand, held in registers for the whole run; K by ldmatrix), the
//       running maximum m, the weights p = 2^(s scale log2(e) - m) and
//       running sum l in registers (online softmax), then o += p v (p as
//       bf16 A fragments straight from the score accumulators, V by
//       transposed ldmatrix);
//     - at the end the warps' (m, l, o) are merged through shared memory,
//       then the cluster's CTAs' through distributed shared memory
//       (o = sum 2^(m_c - M) o_c / sum 2^(m_c - M) l_c), and O (bf16) and
//       LSE (natural log) are written.  No workspace and no second kernel.
// Exponentials are exp2f: the kernel is not bound by arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#ifndef CATTN_HOST_EMULATION
#include "decode_ptx.cuh"
#endif

namespace cattn {

constexpr int kDecodeMaxTq = 8;                        // query rows per call
constexpr int kDecodeWarps = 4;                        // warps per CTA
constexpr int kDecodeThreads = 32 * kDecodeWarps;
constexpr int kDecodeStages = 3;                       // chunks in flight per warp
constexpr int kDecodeMaxCluster = 8;                   // portable cluster size

// Bytes of K and V per chunk: 4 KB of K and 4 KB of V.
__host__ __device__ constexpr int decode_chunk_bytes(int D) { return (void)D, 8192; }
// Keys per chunk (128, 64, 32, 16 for D = 16 .. 128).
__host__ __device__ constexpr int decode_chunk(int D) { return decode_chunk_bytes(D) / 4 / D; }
// Dynamic shared memory per CTA: every warp's ring (96 KB).
__host__ __device__ constexpr int decode_smem_bytes(int D) {
  return kDecodeWarps * kDecodeStages * decode_chunk_bytes(D);
}
// Resident CTAs per SM (2 x 96 KB of shared memory).
__host__ __device__ constexpr int decode_ctas_per_sm(int D) { return (void)D, 2; }

// CTAs per head (the cluster size): enough to fill `slots` resident CTAs
// (SMs x decode_ctas_per_sm(D)), at most kDecodeMaxCluster and at most one per
// chunk; then the number of CTAs that a run of equal length leaves work
// for.
__host__ __device__ constexpr int decode_splits_for(long long BH, int L, int D, int slots) {
  const int n_chunks = (L + decode_chunk(D) - 1) / decode_chunk(D);
  long long want = BH > 0 ? slots / BH : 1;
  if (want > kDecodeMaxCluster) want = kDecodeMaxCluster;
  if (want > n_chunks) want = n_chunks;
  if (want < 1) want = 1;
  const int cpc = (n_chunks + static_cast<int>(want) - 1) / static_cast<int>(want);
  return (n_chunks + cpc - 1) / cpc;
}
__host__ __device__ constexpr int decode_chunks_per_cta(long long BH, int L, int D, int slots) {
  const int n_chunks = (L + decode_chunk(D) - 1) / decode_chunk(D);
  const int s = decode_splits_for(BH, L, D, slots);
  return (n_chunks + s - 1) / s;
}

struct DecodeParams {
  const __nv_bfloat16* q;  // (B, H, Tq, D), element strides q_sb, q_sh, q_st
  const __nv_bfloat16* k;  // (B, H, >= L, D)
  const __nv_bfloat16* v;
  long long q_sb, q_sh, q_st, k_sb, k_sh, k_st, v_sb, v_sh, v_st;
  __nv_bfloat16* o;        // (B, H, Tq, D), element strides o_sb, o_sh, o_st
  long long o_sb, o_sh, o_st;
  float* lse;              // (B, H, Tq) contiguous, natural log
  int H, Tq, L;
  int n_split;             // CTAs per head = cluster size
  int chunks_per_cta;      // chunks of a CTA's run (the last run shorter)
  float scale_log2;        // scale * log2(e)
};

// Byte offset of 16-byte piece `pc` of row `row` in a chunk tile of D-wide
// rows.  The 8 rows an ldmatrix reads (consecutive rows, same piece) land
// in 8 different 16-byte bank groups: the piece index is XORed with the
// row's position among the rows that share a 128-byte line span.
template <int D>
__host__ __device__ constexpr int dec_swz(int row, int pc) {
  constexpr int P = D / 8;                  // pieces per row
  constexpr int RPL = P >= 8 ? 1 : 8 / P;   // rows per 128 bytes
  constexpr int MASK = (P >= 8 ? 8 : P) - 1;
  return (row * P + (pc ^ ((row / RPL) & MASK))) * 16;
}

// Grid: BH * n_split CTAs of kDecodeThreads, clusters of n_split along x
// (CTA x: head x / n_split, cluster rank x % n_split), decode_smem_bytes(D)
// of dynamic shared memory.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads, decode_ctas_per_sm(D))
    decode_kernel(const DecodeParams p) {
  constexpr int CK = decode_chunk(D);  // keys per chunk
  constexpr int P = D / 8;             // 16-byte pieces per row
  constexpr int NS = CK / 8;           // score n-tiles per chunk
  constexpr int KS = D / 16;           // k-steps of q k^T
  constexpr int NO = D / 8;            // output n-tiles
  constexpr int TILE = CK * D * 2;     // bytes of K (of V) per chunk
  constexpr int NW = kDecodeWarps;
  constexpr int CB = decode_chunk_bytes(D);
  static_assert(2 * TILE == CB && TILE / 16 % 32 == 0, "chunk");
  static_assert(NS % 2 == 0 && D % 16 == 0, "tiles");
  static_assert((2 * NW * 8 + NW * 8 * D + 16 + 8 * D) * 4 <= decode_smem_bytes(D), "merge area");

  // launched as a programmatic dependent: the previous kernel (say, the one
  // that appends to the cache) has finished and its writes are visible
  // after this; the next call may then take SMs as this grid drains
  dec_grid_dep_wait();
  dec_grid_dep_launch();
  uint8_t* smem = dec_dynamic_smem();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;  // fragment row, column pair
  const int split = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.n_split));
  const long long bh = blockIdx.x / static_cast<unsigned>(p.n_split);
  const long long b = bh / p.H, h = bh - b * p.H;
  const int Tq = p.Tq, L = p.L, pos0 = L - Tq;  // position of query row 0
  const int n_chunks = (L + CK - 1) / CK;
  const int c_begin = split * p.chunks_per_cta;
  const int c_end = min(n_chunks, c_begin + p.chunks_per_cta);
  const __nv_bfloat16* kb = p.k + b * p.k_sb + h * p.k_sh;
  const __nv_bfloat16* vb = p.v + b * p.v_sb + h * p.v_sh;

  // this warp's chunks: first, first + NW, ... below c_end
  const int first = c_begin + warp;
  const int n_my = first < c_end ? (c_end - first + NW - 1) / NW : 0;
  uint8_t* ring = smem + warp * (kDecodeStages * CB);

  // chunk i of this warp into ring slot i % kDecodeStages; keys past the
  // cache are zero-filled (and masked below)
  auto issue = [&](int i) {
    const int k0 = (first + NW * i) * CK;
    uint8_t* sk = ring + (i % kDecodeStages) * CB;
    uint8_t* sv = sk + TILE;
#pragma unroll
    for (int u = 0; u < TILE / 16 / 32; ++u) {
      const int piece = lane + 32 * u, row = piece / P, pc = piece - (piece / P) * P;
      const int key = k0 + row;
      const bool ok = key < L;
      const long long kr = ok ? key : 0;
      dec_cp_async16(sk + dec_swz<D>(row, pc), kb + kr * p.k_st + pc * 8, ok);
      dec_cp_async16(sv + dec_swz<D>(row, pc), vb + kr * p.v_st + pc * 8, ok);
    }
  };
  // one commit group per ring slot, empty when the warp has fewer chunks,
  // so that "all but the newest kDecodeStages - 1 groups done" is always
  // "chunk i has landed"
#pragma unroll
  for (int i = 0; i < kDecodeStages; ++i) {
    if (i < n_my) issue(i);
    dec_cp_async_commit();
  }

  // the query rows as mma A fragments (rows g >= Tq and 8 .. 15 zero):
  // qa[kk][0] = q[g][16kk + 2 t4 ..+1], qa[kk][1] = q[g][16kk + 8 + 2 t4 ..+1]
  uint32_t qa[KS][2];
  {
    const __nv_bfloat16* qr = p.q + b * p.q_sb + h * p.q_sh + static_cast<long long>(g) * p.q_st;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = g < Tq ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 2 * t4) : 0u;
      qa[kk][1] = g < Tq ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 8 + 2 * t4) : 0u;
    }
  }

  // running state of row g (lanes of a quad share it; l is the lane's part)
  float o[NO][4];
#pragma unroll
  for (int j = 0; j < NO; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const float sl2 = p.scale_log2;
  // last key row g sees (padding rows >= Tq: every key of the cache)
  const int last_visible = min(pos0 + g, L - 1);

  for (int i = 0; i < n_my; ++i) {
    dec_cp_async_wait<kDecodeStages - 1>();
    __syncwarp();  // every lane's pieces of chunk i are in shared memory
    const uint8_t* sk = ring + (i % kDecodeStages) * CB;
    const uint8_t* sv = sk + TILE;
    const int k0 = (first + NW * i) * CK;

    // s = q k^T: n-tile nt holds keys k0 + 8nt .. +7; lane's c0, c1 are
    // row g, keys 8nt + 2t4, +1
    float s[NS][4];
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      if constexpr (P >= 4) {
#pragma unroll
        for (int x = 0; x < P / 4; ++x) {
          uint32_t r[4];
          dec_ldsm_x4(r, sk + dec_swz<D>(nt * 8 + (lane & 7), 4 * x + (lane >> 3)));
          dec_mma(s[nt], qa[2 * x][0], 0u, qa[2 * x][1], 0u, r[0], r[1]);
          dec_mma(s[nt], qa[2 * x + 1][0], 0u, qa[2 * x + 1][1], 0u, r[2], r[3]);
        }
      } else {  // D = 16: one k-step, two matrices
        uint32_t r[2];
        dec_ldsm_x2(r, sk + dec_swz<D>(nt * 8 + (lane & 7), (lane >> 3) & 1));
        dec_mma(s[nt], qa[0][0], 0u, qa[0][1], 0u, r[0], r[1]);
      }
    }
    // keys past the cache, and keys after the row's position
    if (k0 + CK - 1 > pos0) {
#pragma unroll
      for (int nt = 0; nt < NS; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          if (k0 + nt * 8 + 2 * t4 + c > last_visible) s[nt][c] = -INFINITY;
    }

    // online softmax of row g over this chunk
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) mx = fmaxf(mx, fmaxf(s[nt][0], s[nt][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx * sl2);
    const float mu = m_new == -INFINITY ? 0.f : m_new;  // no visible key yet
    const float alpha = exp2f(m_run - mu);               // 0 while m_run is -inf
    m_run = m_new;
    uint32_t pk[NS];  // the weights as bf16 pairs (A fragments of p v)
    float ls = 0.f;
#pragma unroll
    for (int nt = 0; nt < NS; ++nt) {
      const float p0 = exp2f(fmaf(s[nt][0], sl2, -mu));
      const float p1 = exp2f(fmaf(s[nt][1], sl2, -mu));
      ls += p0 + p1;
      pk[nt] = dec_pack_bf16(p0, p1);
    }
    l_run = fmaf(l_run, alpha, ls);
#pragma unroll
    for (int j = 0; j < NO; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }

    // o += p v over the chunk's 16-key steps; one transposed x4 covers 16
    // keys x 16 columns (two output n-tiles)
#pragma unroll
    for (int kk = 0; kk < CK / 16; ++kk) {
#pragma unroll
      for (int jj = 0; jj < D / 16; ++jj) {
        const int mi = lane >> 3;
        uint32_t r[4];
        dec_ldsm_x4_t(r, sv + dec_swz<D>(kk * 16 + (mi & 1) * 8 + (lane & 7), 2 * jj + (mi >> 1)));
        dec_mma(o[2 * jj], pk[2 * kk], 0u, pk[2 * kk + 1], 0u, r[0], r[1]);
        dec_mma(o[2 * jj + 1], pk[2 * kk], 0u, pk[2 * kk + 1], 0u, r[2], r[3]);
      }
    }
    __syncwarp();  // every lane has read the slot: refill it
    if (i + kDecodeStages < n_my) issue(i + kDecodeStages);
    dec_cp_async_commit();
  }
  dec_cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();  // every warp is done with its ring: reuse it

  // merge area: per warp (m, l, o) of its 8 fragment rows, then the CTA's
  float* wm = reinterpret_cast<float*>(smem);  // [NW][8]
  float* wl = wm + NW * 8;                      // [NW][8]
  float* wo = wl + NW * 8;                      // [NW][8][D]
  float* cm = wo + NW * 8 * D;                  // [8]
  float* cl = cm + 8;                           // [8]
  float* co = cl + 8;                           // [8][D]
  if (t4 == 0) {
    wm[warp * 8 + g] = m_run;
    wl[warp * 8 + g] = l_run;
  }
#pragma unroll
  for (int j = 0; j < NO; ++j)
    *reinterpret_cast<float2*>(wo + (warp * 8 + g) * D + j * 8 + 2 * t4) = float2{o[j][0], o[j][1]};
  __syncthreads();

  __nv_bfloat16* ob = p.o + b * p.o_sb + h * p.o_sh;
  float* lseb = p.lse + bh * Tq;
  for (int e = tid; e < Tq * D; e += kDecodeThreads) {
    const int r = e / D, d = e - (e / D) * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, wm[w * 8 + r]);
    float Ls = 0.f, Os = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = wm[w * 8 + r];
      const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);  // warp without a visible key
      Ls = fmaf(f, wl[w * 8 + r], Ls);
      Os = fmaf(f, wo[(w * 8 + r) * D + d], Os);
    }
    if (p.n_split == 1) {  // key 0 is in this CTA: M is finite, Ls > 0
      ob[r * p.o_st + d] = __float2bfloat16_rn(Os / Ls);
      if (d == 0) lseb[r] = (M + log2f(Ls)) * 0.69314718055994531f;
    } else {
      co[r * D + d] = Os;
      if (d == 0) {
        cm[r] = M;
        cl[r] = Ls;
      }
    }
  }
  if (p.n_split > 1) {
    dec_cluster_sync();  // every CTA's partial is in its shared memory
    const unsigned ns = static_cast<unsigned>(p.n_split);
    for (int e = split * kDecodeThreads + tid; e < Tq * D; e += p.n_split * kDecodeThreads) {
      const int r = e / D, d = e - (e / D) * D;
      float M = -INFINITY;
      for (unsigned c = 0; c < ns; ++c) M = fmaxf(M, dec_cluster_ld(cm + r, c));
      float Ls = 0.f, Os = 0.f;  // key 0 is visible to every row: M is finite
      for (unsigned c = 0; c < ns; ++c) {
        const float mc = dec_cluster_ld(cm + r, c);
        const float f = mc == -INFINITY ? 0.f : exp2f(mc - M);
        Ls = fmaf(f, dec_cluster_ld(cl + r, c), Ls);
        Os = fmaf(f, dec_cluster_ld(co + r * D + d, c), Os);
      }
      ob[r * p.o_st + d] = __float2bfloat16_rn(Os / Ls);
      if (d == 0) lseb[r] = (M + log2f(Ls)) * 0.69314718055994531f;
    }
    dec_cluster_sync();  // no CTA leaves while its shared memory is read
  }
}

}  // namespace cattn
