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
// are split into chunks of DecodeCfg<D>::CHUNK (16 KB of K and 16 KB of V),
// one CTA per (head, chunk), so even a batch of one sequence spreads over
// the SMs ("split-K"):
//   decode_partial_kernel<D, TQ>  per CTA (256 threads), over a run of
//   chunks of one head:
//     1. every thread's 16-byte loads of a chunk's K and V rows go out at
//        once (the whole chunk in flight, while the previous chunk is
//        computed), then into shared memory, 16-byte pieces swizzled by row
//        so that the reads below are free of bank conflicts;
//     2. scores s[r][key] = q_r . k_key in log2 units (scale * log2(e)
//        folded into q), one (key, query row) pair per thread, -inf where
//        the key is not visible to the row or past the cache;
//     3. one warp per query row: the running maximum m, the weights
//        2^(s - m) and the running sum l (warp shuffles);
//     4. o[r][d] = 2^(m_old - m) o[r][d] + sum_key w[r][key] v[key][d],
//        threads over (part of the keys, r, d);
//     5. after its last chunk, the CTA's (m, l, o) to the workspace (the
//        key parts summed through shared memory).
//   decode_combine_kernel  per (head, query): merges the chunks' (m, l, o)
//                          (o = sum 2^(m_c - M) o_c / sum 2^(m_c - M) l_c)
//                          and writes O (bf16) and LSE (natural log).
// Scores are kept in log2 units, so the exponentials are exp2; exp2f keeps
// them accurate, as the kernel is not bound by arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace cattn {

constexpr int kDecodeMaxTq = 8;      // query rows per call
constexpr int kDecodeThreads = 256;  // threads per partial CTA

// Keys per chunk: 16 KB of K (and of V), at most 256 keys.
__host__ __device__ constexpr int decode_chunk(int D) { return 8192 / D < 256 ? 8192 / D : 256; }

// Resident partial CTAs per SM: 4 for up to 2 query rows (the launch bounds
// then hold a thread to 64 registers, and the shared memory fits 4), 3 for
// more rows (left unbounded: their accumulators would spill at 64).
__host__ __device__ constexpr int decode_ctas_per_sm(int Tq) { return Tq <= 2 ? 4 : 3; }

// Partial CTAs per head: one wave of CTAs on a 148-SM B200, at most one per
// chunk.
__host__ __device__ constexpr int decode_splits_for(long long BH, int L, int D, int Tq) {
  const int n_chunks = (L + decode_chunk(D) - 1) / decode_chunk(D);
  const long long want = BH > 0 ? 148LL * decode_ctas_per_sm(Tq) / BH : 1;
  const int s = want < 1 ? 1 : (want > n_chunks ? n_chunks : static_cast<int>(want));
  // chunks per CTA, then the CTAs that actually have chunks
  const int cpc = (n_chunks + s - 1) / s;
  return (n_chunks + cpc - 1) / cpc;
}
__host__ __device__ constexpr int decode_chunks_per_cta(long long BH, int L, int D, int Tq) {
  const int n_chunks = (L + decode_chunk(D) - 1) / decode_chunk(D);
  const int s = decode_splits_for(BH, L, D, Tq);
  return (n_chunks + s - 1) / s;
}

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
  int chunks_per_cta;      // chunks of CHUNK keys each partial CTA takes
  float scale_log2;        // scale * log2(e)
};

template <int D>
struct DecodeCfg {
  static constexpr int CHUNK = decode_chunk(D);        // keys per CTA
  static constexpr int VPR = D / 8;                    // 16-byte pieces per row
  static constexpr int PIECES = CHUNK * VPR;           // per tensor per chunk
  static constexpr int LOADS = PIECES / kDecodeThreads;  // per thread per tensor
  static constexpr int TPK = kDecodeThreads / CHUNK;   // threads per key (scores)
  static_assert(LOADS * kDecodeThreads == PIECES && TPK * CHUNK == kDecodeThreads, "chunk");
};

// 8 bf16 (one 16-byte piece) -> 8 floats
__device__ __forceinline__ void unpack8(const uint4& t, float (&x)[8]) {
  const unsigned w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

// Shared-memory position of 16-byte piece c of chunk row `row`: pieces are
// rotated by the row so that consecutive rows' piece c fall in different
// banks (a thread per row reads its row piece by piece).
template <int VPR>
__device__ __forceinline__ int dec_swz(int row, int c) {
  return row * VPR + (c ^ (row % VPR));
}

// TQ: query rows the CTA is compiled for (Tq rounded up to 1, 2, 4 or 8;
// rows at or past Tq compute nothing useful and are not written).
// CTA (bh, split) takes the chunks split*cpc .. split*cpc + cpc - 1 of head
// bh (cpc = p.chunks_per_cta, the last CTA fewer), so that the grid is one
// wave.  While it computes a chunk from shared memory, the next chunk's
// loads are already in flight into registers; a running (m, l, o) per row
// merges the chunks as the online softmax does.
template <int D, int TQ>
__global__ void __launch_bounds__(kDecodeThreads, TQ <= 2 ? 4 : 1)
    decode_partial_kernel(const DecodeParams p) {
  using C = DecodeCfg<D>;
  constexpr int VPR = C::VPR, CH = C::CHUNK, NT = kDecodeThreads;
  __shared__ uint4 sK[C::PIECES];  // uint4: 16-byte aligned by its type
  __shared__ uint4 sV[C::PIECES];
  __shared__ float sQ[TQ][D];         // q rows * scale * log2(e)
  __shared__ float sW[TQ][CH];        // scores, then weights 2^(s - M)
  __shared__ float sML[TQ][2];        // running M and l per row
  __shared__ float sAlpha[TQ];        // this chunk's rescale of the running o
  constexpr int OUTS = TQ * D;        // outputs per CTA
  constexpr int PARTS = OUTS >= NT ? 1 : NT / OUTS;  // key parts of the sum
  constexpr int OPT = OUTS >= NT ? OUTS / NT : 1;    // outputs per thread
  __shared__ float sO[PARTS][OUTS];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x, split = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int Tq = p.Tq;
  const int pos0 = p.L - Tq;          // position of query row 0
  const int n_chunks = (p.L + CH - 1) / CH;
  const int c_begin = split * p.chunks_per_cta;
  const int c_end = min(n_chunks, c_begin + p.chunks_per_cta);
  const __nv_bfloat16* kb = p.k + b * p.k_sb + h * p.k_sh;
  const __nv_bfloat16* vb = p.v + b * p.v_sb + h * p.v_sh;

  // loads of chunk c into registers (zero past the cache)
  uint4 kr[C::LOADS], vr[C::LOADS];
  auto load_chunk = [&](int c) {
    const int k0 = c * CH, n = min(CH, p.L - k0);
#pragma unroll
    for (int u = 0; u < C::LOADS; ++u) {
      const int i = tid + NT * u, row = i / VPR, pc = i - (i / VPR) * VPR;
      kr[u] = vr[u] = uint4{0u, 0u, 0u, 0u};
      if (row < n) {
        const long long key = k0 + row;
        kr[u] = *reinterpret_cast<const uint4*>(kb + key * p.k_st + pc * 8);
        vr[u] = *reinterpret_cast<const uint4*>(vb + key * p.v_st + pc * 8);
      }
    }
  };
  load_chunk(c_begin);
  for (int i = tid; i < TQ * D; i += NT) {
    const int r = i / D, d = i - (i / D) * D;
    float x = 0.f;
    if (r < Tq) x = __bfloat162float(p.q[b * p.q_sb + h * p.q_sh + r * p.q_st + d]) * p.scale_log2;
    sQ[r][d] = x;
  }
  if (tid < TQ) {
    sML[tid][0] = -INFINITY;
    sML[tid][1] = 0.f;
  }
  float o_run[OPT];
#pragma unroll
  for (int j = 0; j < OPT; ++j) o_run[j] = 0.f;

  for (int c = c_begin; c < c_end; ++c) {
    const int k0 = c * CH, n = min(CH, p.L - k0);
    // 1. the chunk (loaded into registers) into shared memory; then the
    //    next chunk's loads go out while this one is computed
#pragma unroll
    for (int u = 0; u < C::LOADS; ++u) {
      const int i = tid + NT * u, row = i / VPR, pc = i - (i / VPR) * VPR;
      sK[dec_swz<VPR>(row, pc)] = kr[u];
      sV[dec_swz<VPR>(row, pc)] = vr[u];
    }
    __syncthreads();
    if (c + 1 < c_end) load_chunk(c + 1);

    // 2. scores: thread -> key tid % CH, rows tid / CH, + TPK, ...
    {
      const int key = tid % CH;
      for (int r = tid / CH; r < TQ; r += C::TPK) {
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int pc = 0; pc < VPR; ++pc) {
          float x[8];
          unpack8(sK[dec_swz<VPR>(key, pc)], x);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            d0 = fmaf(sQ[r][pc * 8 + e], x[e], d0);
            d1 = fmaf(sQ[r][pc * 8 + e + 1], x[e + 1], d1);
          }
        }
        const bool visible = key < n && k0 + key <= pos0 + r;
        sW[r][key] = visible ? d0 + d1 : -INFINITY;
      }
    }
    __syncthreads();

    // 3. one warp per query row: the new running maximum M, the weights
    //    2^(s - M), the running sum, and alpha = 2^(M_old - M) for o
    for (int r = warp; r < TQ; r += NT / 32) {
      float m = -INFINITY;
      for (int j = lane; j < CH; j += 32) m = fmaxf(m, sW[r][j]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float m_old = sML[r][0];
      const float M = fmaxf(m_old, m);
      // no key visible to the row yet: everything stays zero
      const float mu = M == -INFINITY ? 0.f : M;
      float l = 0.f;
      for (int j = lane; j < CH; j += 32) {
        const float w = exp2f(sW[r][j] - mu);  // 0 for a masked key
        sW[r][j] = w;
        l += w;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      __syncwarp();
      if (lane == 0) {
        const float alpha = exp2f(m_old - mu);  // 0 while m_old is -inf
        sAlpha[r] = alpha;
        sML[r][0] = M;
        sML[r][1] = sML[r][1] * alpha + l;
      }
    }
    __syncthreads();

    // 4. o[r][d] = alpha o[r][d] + sum_key w[r][key] v[key][d]: thread ->
    //    outputs (tid % OUTS) + NT j over key part tid / OUTS
    {
      const __nv_bfloat16* sVh = reinterpret_cast<const __nv_bfloat16*>(sV);
      const int part = OUTS >= NT ? 0 : tid / OUTS;
      const int kb0 = part * (CH / PARTS), ke = kb0 + CH / PARTS;
#pragma unroll
      for (int j = 0; j < OPT; ++j) {
        const int out = (OUTS >= NT ? tid + NT * j : tid % OUTS);
        const int r = out / D, d = out - (out / D) * D;
        float a0 = 0.f, a1 = 0.f;
        for (int key = kb0; key < ke; key += 2) {
          a0 = fmaf(sW[r][key], __bfloat162float(sVh[dec_swz<VPR>(key, d / 8) * 8 + (d & 7)]), a0);
          a1 = fmaf(sW[r][key + 1],
                    __bfloat162float(sVh[dec_swz<VPR>(key + 1, d / 8) * 8 + (d & 7)]), a1);
        }
        o_run[j] = fmaf(o_run[j], sAlpha[r], a0 + a1);
      }
    }
    __syncthreads();  // shared K, V and W are rewritten by the next chunk
  }

  // 5. the CTA's (M, l, o) to the workspace: the key parts summed
  {
    const int part = OUTS >= NT ? 0 : tid / OUTS;
#pragma unroll
    for (int j = 0; j < OPT; ++j) sO[part][OUTS >= NT ? tid + NT * j : tid % OUTS] = o_run[j];
  }
  __syncthreads();
  for (int out = tid; out < Tq * D; out += NT) {
    const int r = out / D, d = out - (out / D) * D;
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < PARTS; ++q) acc += sO[q][out];
    const size_t row = (static_cast<size_t>(bh) * p.n_split + split) * Tq + r;
    p.part_o[row * D + d] = acc;
    if (d == 0) {
      p.part_ml[row * 2] = sML[r][0];
      p.part_ml[row * 2 + 1] = sML[r][1];
    }
  }
}

// One CTA of kCombineThreads per (head, query row) merges the chunks:
// first M = max_c m_c (the threads read the chunks' m in parallel, then a
// block reduction), then per column d the sums over the chunks of
// 2^(m_c - M) o_c[d] and 2^(m_c - M) l_c, the chunks dealt to
// kCombineThreads / D thread groups so that every thread has few,
// independent loads, then the groups' sums added.  Key 0 is in chunk 0 and
// visible to every row, so M is finite.
constexpr int kCombineThreads = 128;

template <int D>
__global__ void __launch_bounds__(kCombineThreads) decode_combine_kernel(const DecodeParams p) {
  constexpr int NT = kCombineThreads;
  constexpr int PARTS = NT / D;  // thread groups over the chunks (D <= 128)
  __shared__ float sRed[NT / 32];
  __shared__ float sO[PARTS][D];
  __shared__ float sL[PARTS];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;  // bh * Tq + r
  const int bh = row / p.Tq, r = row - (row / p.Tq) * p.Tq;
  const int b = bh / p.H, h = bh - b * p.H;
  const size_t first = static_cast<size_t>(bh) * p.n_split * p.Tq + r;  // chunk 0's row
  float m = -INFINITY;
  for (int c = tid; c < p.n_split; c += NT)
    m = fmaxf(m, p.part_ml[(first + static_cast<size_t>(c) * p.Tq) * 2]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) sRed[warp] = m;
  __syncthreads();
  float M = sRed[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) M = fmaxf(M, sRed[i]);
  const int d = tid % D, part = tid / D;
  float o = 0.f, l = 0.f;
#pragma unroll 4
  for (int c = part; c < p.n_split; c += PARTS) {
    const size_t pr = first + static_cast<size_t>(c) * p.Tq;
    const float w = exp2f(p.part_ml[pr * 2] - M);
    o = fmaf(w, p.part_o[pr * D + d], o);
    l = fmaf(p.part_ml[pr * 2 + 1], w, l);
  }
  sO[part][d] = o;
  if (d == 0) sL[part] = l;
  __syncthreads();
  if (part == 0) {
    float os = 0.f, ls = 0.f;
#pragma unroll
    for (int q = 0; q < PARTS; ++q) {
      os += sO[q][d];
      ls += sL[q];
    }
    p.o[b * p.o_sb + h * p.o_sh + r * p.o_st + d] = __float2bfloat16_rn(os / ls);
    if (d == 0) p.lse[row] = (M + log2f(ls)) * 0.69314718055994531f;
  }
}

}  // namespace cattn
