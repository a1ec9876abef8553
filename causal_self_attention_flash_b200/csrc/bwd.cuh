// Backward kernels for causal attention: gradients of a scalar loss L with
// dL/dO = dO through O = softmax(scale * Q K^T + causal mask) V.
//
// The pages leave the gradient to autograd ("nanoGPT: a real GPT in two
// 300-line files", section 1 "Summary": "Autograd does the calculus"); it
// is the chain rule through the written-out attention of section 2:
//     dV = P^T dO,  dP = dO V^T,  Delta_i = sum_d dO_id O_id,
//     dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q,
// with P recomputed from Q, K and the forward's LSE (P = exp(S - LSE)), so
// no T x T matrix is ever stored.
//
// Three kernels:
//   bwd_pre_kernel   Delta = rowsum(dO * O) with 16-byte loads (O + O_lo when
//                    the forward's bf16 residual O_lo = O - bf16(O) is given,
//                    which makes Delta exact to fp32 rounding), LSE * log2(e)
//                    into a tile-padded vector, and zeroing of the fp32 dQ
//                    accumulator.
//   bwd_kernel       one CTA per (head, 128-key tile); loops over the query
//                    tiles at or after it (causal), accumulating dK and dV in
//                    TMEM and adding each dQ tile into the fp32 accumulator
//                    with a TMA reduce-add.
//   dq_convert_kernel dQ = bf16(scale * accumulator), or fp32 when the caller
//                    asks for fp32 gradients.
//
// Precision: P enters the dV MMA as a bf16 hi/lo pair (x = hi + lo to ~14
// bits).  dS enters the dK and dQ MMAs as bf16 (SLO = false, the usual mixed
// precision) or also as a hi/lo pair (SLO = true, used with the forward's
// O_lo residual or with fp32 gradient outputs, where the aim is gradients
// accurate to ~fp32).
//
// Instances bwd_kernel<D, SLO, DROP, FLAT>:
//   DROP   attention dropout with the forward's mask (philox.cuh): a compute
//          thread owns one key and 32 queries, so each lane draws the bits
//          of 8 keys for one query and a warp shuffle per query hands every
//          lane its own bit; dV takes the dropped P^T (the keep scale is
//          applied in the epilogue) and dS = P * (dP~ * mask / (1 - p) -
//          Delta).
//   FLAT   Q, K, V, dO, dK and dV address (b, h) as one b*H + h index (3-D
//          tensor maps); otherwise 4-D maps take any element strides.
// bwd_pre_kernel<D, CONTIG> and the dQ convert have contiguous and strided
// forms too.
#pragma once

#include "philox.cuh"
#include "sm100.cuh"

namespace cattn {

// ---------------------------------------------------------------------------
// Preprocess
// ---------------------------------------------------------------------------

struct PreParams {
  const __nv_bfloat16* o;     // (B, H, T, D), element strides o_sb, o_sh, o_st
  const __nv_bfloat16* o_lo;  // may be null; the strides of o
  const __nv_bfloat16* dout;  // element strides do_sb, do_sh, do_st
  long long o_sb, o_sh, o_st, do_sb, do_sh, do_st;
  int H;
  const float* lse;      // may be null (no lse2 output)
  float* delta;          // (BH, row_stride)
  float* lse2;           // (BH, row_stride) or null
  float4* zero;          // buffer to clear, or null
  size_t zero_n4;        // its length in float4
  unsigned int* status;  // the call's {code, where} words, cleared here (or null)
  int T;
  int row_stride;        // T (public preprocess) or T rounded up to 128
  long long n_rows;      // BH * row_stride
};

// Threads per row: each handles 8 bf16 (16 bytes) of O and of dO.
// CONTIG: O and dO are contiguous (B, H, T, D), addressed as rows of D.
template <int D, bool CONTIG>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const PreParams p) {
  // the previous kernel's O, dO, LSE.  (The main kernel is not released
  // early: its CTAs, resident while this grid drained, made the GPT-2
  // layer's backward call 168.6 against 165.9 us.)
  grid_dep_wait();
  constexpr int TPR = D / 8;
  constexpr int RPW = 32 / TPR;  // rows per warp per step
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPR;
  const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  constexpr float kLog2e = 1.4426950408889634f;

  // the backward call's status words start clear (this kernel runs first)
  if (p.status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
    p.status[0] = 0u;
    p.status[1] = 0u;
  }

  // two row groups per step, their loads issued before either is reduced
  constexpr int U = 2;
  const bool small = p.n_rows <= 0x7fffffffLL;  // 32-bit index arithmetic
  for (long long base = warp_global * (RPW * U); base < p.n_rows; base += n_warps * (RPW * U)) {
    long long pr[U];
    long long bh[U];
    int t[U];
    bool valid[U];
    uint4 a[U], bb[U], c[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      pr[u] = base + u * RPW + lane / TPR;
      bh[u] = 0;
      t[u] = 0;
      if (pr[u] < p.n_rows) {
        if (small) {
          const unsigned q = static_cast<unsigned>(pr[u]) / static_cast<unsigned>(p.row_stride);
          bh[u] = q;
          t[u] = static_cast<int>(static_cast<unsigned>(pr[u]) - q * static_cast<unsigned>(p.row_stride));
        } else {
          bh[u] = pr[u] / p.row_stride;
          t[u] = static_cast<int>(pr[u] - bh[u] * p.row_stride);
        }
      }
      valid[u] = pr[u] < p.n_rows && t[u] < p.T;
      a[u] = bb[u] = c[u] = make_uint4(0u, 0u, 0u, 0u);
      if (valid[u]) {
        long long off, doff;
        if constexpr (CONTIG) {
          off = doff = (static_cast<long long>(bh[u]) * p.T + t[u]) * D + sub * 8;
        } else {
          // (B*H < 2^31: a 32-bit division)
          const unsigned hb = static_cast<unsigned>(bh[u]) / static_cast<unsigned>(p.H);
          const long long b_ = hb, h_ = static_cast<long long>(bh[u]) - b_ * p.H;
          off = b_ * p.o_sb + h_ * p.o_sh + t[u] * p.o_st + sub * 8;
          doff = b_ * p.do_sb + h_ * p.do_sh + t[u] * p.do_st + sub * 8;
        }
        a[u] = *reinterpret_cast<const uint4*>(p.o + off);
        bb[u] = *reinterpret_cast<const uint4*>(p.dout + doff);
        if (p.o_lo != nullptr) c[u] = *reinterpret_cast<const uint4*>(p.o_lo + off);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = 0.f;
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bb[u]);
      const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fb = __bfloat1622float2(b2[e]);
        const float2 fc = __bfloat1622float2(c2[e]);
        acc = fmaf(fa.x + fc.x, fb.x, acc);
        acc = fmaf(fa.y + fc.y, fb.y, acc);
      }
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (pr[u] < p.n_rows && sub == 0) {
        p.delta[pr[u]] = acc;  // 0 on padding rows
        if (p.lse2 != nullptr)  // stored negated: P = 2^(s * scale_log2 + lse2)
          p.lse2[pr[u]] =
              valid[u] ? -(p.lse[static_cast<size_t>(bh[u]) * p.T + t[u]] * kLog2e) : -INFINITY;
      }
    }
  }
  if (p.zero != nullptr) {
    const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const size_t nth = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t i = tid; i < p.zero_n4; i += nth) p.zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// ---------------------------------------------------------------------------
// dQ convert
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) dq_convert_f32_kernel(const float4* __restrict__ acc,
                                                             float4* __restrict__ dq, size_t n4,
                                                             float scale) {
  grid_dep_wait();  // the main kernel's accumulator
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nth = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = tid; i < n4; i += nth) {
    const float4 a = acc[i];
    dq[i] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
  }
}

__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ acc,
                                                         uint4* __restrict__ dq, size_t n8,
                                                         float scale) {
  grid_dep_wait();  // the main kernel's accumulator
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nth = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t i = tid; i < n8; i += nth) {
    const float4 a = acc[2 * i];
    const float4 b = acc[2 * i + 1];
    uint4 r;
    r.x = pack_bf16(a.x * scale, a.y * scale);
    r.y = pack_bf16(a.z * scale, a.w * scale);
    r.z = pack_bf16(b.x * scale, b.y * scale);
    r.w = pack_bf16(b.z * scale, b.w * scale);
    dq[i] = r;
  }
}

// dQ into an output with any (b, h, t) element strides: one thread per 8
// elements, the accumulator (B*H, T, D) read contiguously.
template <int D, bool F32>
__global__ void __launch_bounds__(256) dq_convert_strided_kernel(const float4* __restrict__ acc,
                                                                 void* __restrict__ dq, int H,
                                                                 int T, long long n8,
                                                                 long long sb, long long sh,
                                                                 long long st, float scale) {
  grid_dep_wait();  // the main kernel's accumulator
  constexpr int C8 = D / 8;  // 8-element chunks per row
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nth = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = tid; i < n8; i += nth) {
    const long long row = i / C8;  // C8 is a power of two: a shift
    const int c8 = static_cast<int>(i - row * C8);
    const long long bh = row <= 0xffffffffLL
                             ? static_cast<long long>(static_cast<unsigned>(row) / static_cast<unsigned>(T))
                             : row / T;
    const long long t = row - bh * T;
    const long long b = static_cast<unsigned>(bh) / static_cast<unsigned>(H), h = bh - b * H;
    const long long off = b * sb + h * sh + t * st + c8 * 8;
    const float4 a = acc[2 * i];
    const float4 c = acc[2 * i + 1];
    if constexpr (F32) {
      float4* out = reinterpret_cast<float4*>(static_cast<float*>(dq) + off);
      out[0] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
      out[1] = make_float4(c.x * scale, c.y * scale, c.z * scale, c.w * scale);
    } else {
      uint4 r;
      r.x = pack_bf16(a.x * scale, a.y * scale);
      r.y = pack_bf16(a.z * scale, a.w * scale);
      r.z = pack_bf16(c.x * scale, c.y * scale);
      r.w = pack_bf16(c.z * scale, c.w * scale);
      reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dq) + off)[0] = r;
    }
  }
}

// ---------------------------------------------------------------------------
// Main backward kernel
// ---------------------------------------------------------------------------
//
// Work item: (head, 128-key tile j).  For each query tile i >= j:
//   S^T  = K_j Q_i^T               (TMEM, fp32; lane = key)
//   P^T  = exp2(S^T*scale*log2e - LSE2_i); masked on the diagonal tile;
//          written back over S^T as bf16 hi/lo pairs
//   dP^T = V_j dO_i^T              (TMEM, fp32)
//   dS^T = P^T * (dP^T - Delta_i); written back over dP^T (bf16, or hi/lo
//          pairs), and (as dS) to shared memory for the dQ MMA
//   dV  += P^T_hi dO_i + P^T_lo dO_i        (A from TMEM)
//   dK  += dS^T_hi Q_i (+ dS^T_lo Q_i)      (A from TMEM; DK_SMEM: from the
//                                            shared dS, K-major)
//   dQ_i = dS_hi K_j (+ dS_lo K_j)          (A from shared, MN-major),
//          drained to shared memory and added into the fp32 accumulator
//          with a TMA reduce-add.
//
// Warp roles (640 threads):
//   warps 0-15 compute: warp w serves TMEM lanes 32*(w%4).. (key rows) and
//              query columns 32*(w/4) .. +32 of the tile (four warps per SM
//              sub-partition, to hide the latency of the exponentials and
//              tensor-memory loads); they also drain dQ and write dK, dV.
//   warp 16    TMA producer: per work item K, V (double-buffered where
//              shared memory allows); Q_t with the LSE2 and Delta vectors
//              through a 2-stage ring, dO_t through a 2-stage (D <= 64) or
//              1-stage ring, both running on across items.
//   warp 17    MMA issuer A and TMEM owner: S(t+1) as soon as dV(t) has read
//              P^T(t), dQ(t), dP(t+1) once dK(t) has read dS^T(t) (and, with
//              dQ in dP^T's columns, once dQ(t) has been drained).
//   warp 18    MMA issuer B: dV(t) (P^T_hi part), dK(t).
//   warp 19    MMA issuer C: the P^T_lo part of dV(t), into dV' (where TMEM
//              holds a separate dV' accumulator; otherwise warp 18 does it).
// The kernel is persistent: CTA b loops over work items (key tiles).

struct BwdParams {
  const float* lse2;   // (BH, T_pad) -LSE * log2(e); -inf on padding rows
  const float* delta;  // (BH, T_pad); 0 on padding rows
  float* dk_f32;       // fp32 gradient outputs (BH, T, D), or null
  float* dv_f32;
  __nv_bfloat16* dk_bf16;  // bf16 gradient outputs, used when dk_f32 is null
  __nv_bfloat16* dv_bf16;
  // element strides (b, h, t) of the dK and dV outputs (either type)
  long long dk_sb, dk_sh, dk_st, dv_sb, dv_sh, dv_st;
  int H;
  int T;
  int T_pad;
  int n_tiles;
  int BH;
  float scale;
  float scale_log2;
  uint64_t timeout_ns;
  DropParams drop;  // attention dropout (kernels instantiated with DROP only)
  unsigned int* status;  // the call's {code, where} words in its workspace
};

template <int D, bool SLO>
struct BwdCfg {
  static constexpr int CB = D < 64 ? D : 64;       // bf16 columns per swizzle block
  static constexpr int RB = CB * 2;
  static constexpr int NCB = D / CB;
  static constexpr int BLOCK_BYTES = 128 * RB;
  static constexpr int TILE_BYTES = 128 * D * 2;
  // Q ring depth (a third stage, where shared memory allows it, measured no
  // faster on the GPT-2 layer)
  static constexpr int QST = 2;
  static constexpr int DOST = D <= 64 ? 2 : 1;      // dO ring depth
  static constexpr uint32_t SW = swizzle_code(RB);
  // fp32 dQ staging in the dS buffers (CTA-wide drain): blocks of
  // [128 rows][CBQ floats]
  static constexpr int CBQ = D < 32 ? D : 32;
  static constexpr int RBQ = CBQ * 4;
  // WARP_DQ (D <= 64): every compute warp drains its own [32 rows][D/4]
  // slice of dQ through its own fp32 staging tile and TMA reduce, so no
  // CTA-wide barrier is needed; otherwise the CTA stages all of dQ in the dS
  // buffers and one thread issues the reduce.
  static constexpr bool WARP_DQ = D <= 64;
  static constexpr int RBW = D;                                // (D/4) floats per row
  static constexpr int WARP_STAGE = (32 * RBW + 1023) / 1024 * 1024;
  // dS lo buffer: with SLO, and as the second half of the CTA dQ staging
  static constexpr int DSL_BYTES = (SLO || !WARP_DQ) ? 32768 : 0;
  // shared memory map; KVB = 2 K/V buffers (the next work item's K, V load
  // while the current one finishes) where they fit
  static constexpr int layout_end(int kvb) {
    return ((kvb * 2 * TILE_BYTES + (QST + DOST) * TILE_BYTES + 32768 + DSL_BYTES +
             QST * 1024 + 1023) / 1024 * 1024) +
           (WARP_DQ ? 16 * WARP_STAGE : 0) + 40 * 8 + 64;
  }
  static constexpr int KVB = layout_end(2) + 1024 <= kMaxDynSmem ? 2 : 1;
  static constexpr int OFF_KV = 0;                             // [KVB][K, V]
  static constexpr int OFF_Q = OFF_KV + KVB * 2 * TILE_BYTES;
  static constexpr int OFF_DO = OFF_Q + QST * TILE_BYTES;
  static constexpr int OFF_DSH = OFF_DO + DOST * TILE_BYTES;  // [2][128 keys][64 q] bf16
  static constexpr int OFF_DSL = OFF_DSH + 32768;
  static constexpr int OFF_LSE = OFF_DSL + DSL_BYTES;         // [QST][128] fp32
  static constexpr int OFF_DELTA = OFF_LSE + QST * 512;       // [QST][128] fp32
  static constexpr int OFF_DQW = (OFF_DELTA + QST * 512 + 1023) / 1024 * 1024;
  static constexpr int OFF_BAR = WARP_DQ ? OFF_DQW + 16 * WARP_STAGE : OFF_DELTA + QST * 512;
  static constexpr int NUM_BARS = 33;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_USED = OFF_MISC + 64;
  static constexpr int SMEM_BYTES =
      SMEM_USED + 1024 <= kMaxDynSmem ? SMEM_USED + 1024 : SMEM_USED;
  static_assert(SMEM_USED <= kMaxDynSmem, "shared memory layout too large");
  static_assert(WARP_DQ || 128 * D * 4 <= 32768 + DSL_BYTES, "dQ staging must fit the dS buffers");
  // TMEM columns.  MMAs that accumulate into one TMEM tile run back to back
  // at about half the rate of independent ones, so where columns allow, the
  // P_lo products of dV get their own accumulator dV' (summed at the end)
  // and dK, dQ are issued interleaved.
  static constexpr bool ALIAS_DQ = 256 + 3 * D > 512;
  static constexpr bool SPLIT_DV = 256 + 4 * D <= 512;
  // CTA-wide dQ staging (D = 128) over the dS hi buffer (HI_BLOCKS blocks)
  // and the lo buffer: with bf16 dS the dS phase rewrites the hi buffer
  // only, so it need not wait for the reduce to read the lo part.
  static constexpr int HI_BLOCKS = 32768 / (128 * RBQ);
  static constexpr bool STAGE_SPLIT = !WARP_DQ && !SLO && HI_BLOCKS < D / CBQ;
  // DK_SMEM (D = 128, bf16 dS): dK takes dS^T from the shared-memory copy
  // of dS that the dQ product reads (the [2][128 keys][64 queries] 128-byte
  // swizzled blocks are dS^T in K-major order), so the compute warps store
  // dS to shared memory only, and dQ (whose TMEM columns are dP^T's) need
  // not wait for dK; the CTA-wide staging then waits for dK before it
  // overwrites the dS blocks.
  static constexpr bool DK_SMEM = !WARP_DQ && !SLO;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = ALIAS_DQ ? COL_DP : 256 + 2 * D;
  static constexpr uint32_t COL_DVL = SPLIT_DV ? 256 + 3 * D : COL_DV;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 640;
  // Registers: 96 per thread at launch (65536 / 640, rounded down to 8);
  // setmaxnreg then gives the compute warpgroups REGS_COMP and the fifth
  // warpgroup (producer and MMA issuers) REGS_OTHER, within the launch total.
  static constexpr bool REBALANCE = D <= 64 && !SLO;
  static constexpr int LAUNCH_REGS = 96, REGS_COMP = 104, REGS_OTHER = 64;
  static_assert(!REBALANCE || 512 * REGS_COMP + 128 * REGS_OTHER <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
  static constexpr int NCOMP = 512;   // compute threads
};

// barrier indices (two of each K/V buffer barrier, QST of the Q ring's,
// DOST (<= 2) of the dO ring's)
// (room for up to 4 Q stages and 4 dO stages)
enum : int {
  BB_KVFULL = 0, BB_KVFREE = 2, BB_QFULL = 4, BB_QEMPTY = 8, BB_DOFULL = 12, BB_DOEMPTY = 16,
  BB_SFULL = 20, BB_DPFULL = 21, BB_PFULL = 22, BB_DSFULL = 23, BB_DQFULL = 24,
  BB_DQEMPTY = 25, BB_ACCFREE = 26, BB_PTDONE = 27, BB_DKDONE = 28,
  BB_DRAIN = 29,  // + issuer 0, 1, 2
  BB_PFULL2 = 32  // second half of P^T (BB_PFULL is the first)
};

// Work items: key tiles (kt, bh), numbered longest first (u = 0 ..
// BH*n_tiles-1: kt = u / BH, bh = u % BH; key tile kt meets n_tiles - kt
// query tiles).  The grid is persistent (at most one CTA per SM); CTA b
// takes items in passes over the grid, alternating direction: pass k takes
// item k*G + b (k even) or k*G + G-1-b (k odd).  Returns -1 past the end.
__device__ __forceinline__ int bwd_item(int k, int b, int G, int n_items) {
  const int u = k * G + ((k & 1) ? G - 1 - b : b);
  return u < n_items ? u : -1;
}

// FLAT: Q, K, V, dO, dK and dV address (b, h) as one b*H + h axis (3-D
// tensor maps, dK/dV offsets bh * d?_sh); otherwise 4-D maps with (h, b)
// coordinates.
template <int D, bool SLO, bool DROP, bool FLAT>
__global__ void __launch_bounds__(640, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
           const __grid_constant__ CUtensorMap tmDQacc, const BwdParams p) {
  using C = BwdCfg<D, SLO>;
  static_assert(BB_PFULL2 + 1 <= C::NUM_BARS, "barrier count");
  static_assert(C::QST <= 4 && C::DOST <= 4, "barrier map");
  // launched behind the preprocess, which writes Delta, LSE, the cleared
  // accumulator and status words: nothing before this line touches memory
  grid_dep_wait();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw, C::SMEM_USED, p.status);
  if (smem == nullptr) return;  // uniform over the CTA: nothing touched yet
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sDSH = sbase + C::OFF_DSH, sDSL = sbase + C::OFF_DSL;
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * i; };
  auto sK = [&](int kvb) { return sbase + C::OFF_KV + kvb * 2 * C::TILE_BYTES; };
  auto sV = [&](int kvb) { return sbase + C::OFF_KV + kvb * 2 * C::TILE_BYTES + C::TILE_BYTES; };
  // misc: [0] TMEM address, [1] abort flag, [2..3] the call's status address
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = p.BH * p.n_tiles;
  const int G = gridDim.x, b = blockIdx.x;

  WaitCtx w{p.timeout_ns, abort_flag, 2u, true};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *reinterpret_cast<unsigned int**>(misc + 2) = p.status;
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BB_KVFULL + s), 1);
      mbar_init(bar(BB_KVFREE + s), 1);
    }
    for (int s = 0; s < C::QST; ++s) {
      mbar_init(bar(BB_QFULL + s), 1);
      mbar_init(bar(BB_QEMPTY + s), 1);
    }
    for (int s = 0; s < C::DOST; ++s) {
      mbar_init(bar(BB_DOFULL + s), 1);
      // released by dP (warp 17) and dV (warp 18, and 19 with a dV' accumulator)
      mbar_init(bar(BB_DOEMPTY + s), C::SPLIT_DV ? 3 : 2);
    }
    mbar_init(bar(BB_SFULL), 1);
    mbar_init(bar(BB_DPFULL), 1);
    mbar_init(bar(BB_PFULL), C::NCOMP);
    mbar_init(bar(BB_PFULL2), C::NCOMP);
    mbar_init(bar(BB_DSFULL), C::NCOMP);
    mbar_init(bar(BB_DQFULL), 1);
    mbar_init(bar(BB_DQEMPTY), C::NCOMP);
    mbar_init(bar(BB_ACCFREE), C::NCOMP);
    mbar_init(bar(BB_PTDONE), C::SPLIT_DV ? 2 : 1);  // dV by warps 18 (and 19)
    mbar_init(bar(BB_DKDONE), 1);
    mbar_init(bar(BB_DRAIN), 1);
    mbar_init(bar(BB_DRAIN + 1), 1);
    mbar_init(bar(BB_DRAIN + 2), 1);
    fence_mbar_init();
  }
  if (warp == 17) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  // Running counters across the CTA's items: t = query tiles processed so
  // far (one per iteration: the phase of the per-iteration barriers and the
  // position in the Q and dO rings), n = items so far (K/V buffer n % KVB).
  if (warp >= 16) {
  // fifth warpgroup: the producer and the MMA issuers
  if constexpr (C::REBALANCE) regs_dec<C::REGS_OTHER>();
  if (warp == 16) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      int tq = 0, tdo = 0, n = 0;  // loads issued
      // one [128][CB] box at column x, row y of head bh: a 4-D map takes
      // (h, b) coordinates, a 3-D map (the (B*H, T, D) layout) takes bh
      auto load_tile = [&](uint32_t dst, const CUtensorMap* m, int bit, uint32_t mbar, int x,
                           int y, int bh) {
        (void)bit;
        if constexpr (FLAT)
          tma_load_3d(dst, m, mbar, x, y, bh);
        else
          tma_load_4d(dst, m, mbar, x, y, bh % p.H, bh / p.H);
      };
      auto load_q = [&](int qi, int bh) {
        const int qs = tq % C::QST;
        if (tq >= C::QST) wait1(w, bar(BB_QEMPTY + qs), ((tq / C::QST) - 1) & 1, 1);
        if (*abort_flag) return;
        const size_t vec = static_cast<size_t>(bh) * p.T_pad + static_cast<size_t>(qi) * 128;
        const uint32_t sQ = sbase + C::OFF_Q + qs * C::TILE_BYTES;
        mbar_arrive_expect_tx(bar(BB_QFULL + qs), C::TILE_BYTES + 1024);
        for (int bb = 0; bb < C::NCB; ++bb)
          load_tile(sQ + bb * C::BLOCK_BYTES, &tmQ, 1, bar(BB_QFULL + qs), bb * C::CB, qi * 128,
                    bh);
        bulk_load(sbase + C::OFF_LSE + qs * 512, p.lse2 + vec, 512, bar(BB_QFULL + qs));
        bulk_load(sbase + C::OFF_DELTA + qs * 512, p.delta + vec, 512, bar(BB_QFULL + qs));
        ++tq;
      };
      auto load_do = [&](int qi, int bh) {
        const int ds = tdo % C::DOST;
        if (tdo >= C::DOST) wait1(w, bar(BB_DOEMPTY + ds), ((tdo / C::DOST) - 1) & 1, 2);
        if (*abort_flag) return;
        const uint32_t sDO = sbase + C::OFF_DO + ds * C::TILE_BYTES;
        mbar_arrive_expect_tx(bar(BB_DOFULL + ds), C::TILE_BYTES);
        for (int bb = 0; bb < C::NCB; ++bb)
          load_tile(sDO + bb * C::BLOCK_BYTES, &tmDO, 8, bar(BB_DOFULL + ds), bb * C::CB,
                    qi * 128, bh);
        ++tdo;
      };
      for (int k = 0;; ++k) {
        const int u = bwd_item(k, b, G, n_items);
        if (u < 0 || *abort_flag) break;
        const int kt = u / p.BH, bh = u % p.BH;
        const int n_iter = p.n_tiles - kt;
        // in the order the MMAs consume them: Q_0 (S), K and V, dO_0 (dP)
        load_q(kt, bh);
        const int kvb = n % C::KVB;
        if (n >= C::KVB) wait1(w, bar(BB_KVFREE + kvb), ((n / C::KVB) - 1) & 1, 3);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(bar(BB_KVFULL + kvb), 2 * C::TILE_BYTES);
        for (int bb = 0; bb < C::NCB; ++bb) {
          load_tile(sK(kvb) + bb * C::BLOCK_BYTES, &tmK, 2, bar(BB_KVFULL + kvb), bb * C::CB,
                    kt * 128, bh);
          load_tile(sV(kvb) + bb * C::BLOCK_BYTES, &tmV, 4, bar(BB_KVFULL + kvb), bb * C::CB,
                    kt * 128, bh);
        }
        ++n;
        load_do(kt, bh);
        for (int i = 1; i < n_iter && !*abort_flag; ++i) {
          load_q(kt + i, bh);
          load_do(kt + i, bh);
        }
      }
      if (*abort_flag) {
        // wait (bounded, ignoring the abort flag) for the last loads issued,
        // which nobody may consume, before the CTA exits
        int zero = 0;
        WaitCtx wd{p.timeout_ns, &zero, 2u, false};
        for (int j = (n > C::KVB ? n - C::KVB : 0); j < n; ++j)
          wait1(wd, bar(BB_KVFULL + j % C::KVB), (j / C::KVB) & 1, 20);
        for (int j = (tq > C::QST ? tq - C::QST : 0); j < tq; ++j)
          wait1(wd, bar(BB_QFULL + j % C::QST), (j / C::QST) & 1, 21);
        for (int j = (tdo > C::DOST ? tdo - C::DOST : 0); j < tdo; ++j)
          wait1(wd, bar(BB_DOFULL + j % C::DOST), (j / C::DOST) & 1, 22);
      }
    }
  } else {
    // -------------------------------------------------- MMA issuers
    // warp 17 (A): S, dP, dQ -- the products that read K and V;
    // warps 18, 19 (B, C): dV, dK -- the accumulations.  One thread issues
    // an N = 64 MMA only every ~50 cycles, so several issuers keep the
    // tensor core busier.  What one issuer's in-order execution guaranteed is now
    // explicit: S(t+1) waits for dV(t) (PTDONE), dP(t+1) for dK(t) (DKDONE).
    if (lane == 0 && (warp != 19 || C::SPLIT_DV)) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idKD = idesc_bf16(128, D, 0, 1);    // dV, dK: B MN-major
      constexpr uint32_t idQ = idesc_bf16(128, D, 1, 1);     // dQ: A (dS) MN-major
      if (warp == 17) {
        auto issue_s = [&](int t, uint32_t k_s) {  // S^T = K Q_t^T
          const int qs = t % C::QST;
          wait1(w, bar(BB_QFULL + qs), (t / C::QST) & 1, 4);
          // S overwrites P^T(t-1), which dV(t-1) reads
          if (t >= 1) wait1(w, bar(BB_PTDONE), (t - 1) & 1, 24);
          tc_fence_after();
          const uint32_t sQ = sbase + C::OFF_Q + qs * C::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int blk = (kk * 16) / C::CB;
            const int off = ((kk * 16) % C::CB) * 2;
            mma_ss(tbase + C::COL_S,
                   smem_desc(k_s + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW),
                   smem_desc(sQ + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW), idSS,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(BB_SFULL));
        };
        auto issue_dp = [&](int t, uint32_t v_s) {  // dP^T = V dO_t^T
          const int ds = t % C::DOST;
          wait1(w, bar(BB_DOFULL + ds), (t / C::DOST) & 1, 5);
          // dP overwrites dS^T(t-1), which dK(t-1) reads, and, aliased,
          // dQ(t-1), which the compute warps must have drained
          // (DK_SMEM: dS^T(t-1) is not in TMEM; the compute warps loaded
          // dP^T(t-1) before draining dQ(t-1), which the wait below covers)
          if (!C::DK_SMEM && t >= 1) wait1(w, bar(BB_DKDONE), (t - 1) & 1, 25);
          if (C::ALIAS_DQ && t >= 1) wait1(w, bar(BB_DQEMPTY), (t - 1) & 1, 12);
          tc_fence_after();
          const uint32_t sDO = sbase + C::OFF_DO + ds * C::TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int blk = (kk * 16) / C::CB;
            const int off = ((kk * 16) % C::CB) * 2;
            mma_ss(tbase + C::COL_DP,
                   smem_desc(v_s + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW),
                   smem_desc(sDO + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW), idSS,
                   kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(BB_DPFULL));
          mma_commit(bar(BB_DOEMPTY + ds));  // one of the slot's two releases
        };
        // a flat walk over the CTA's (item, query tile) pairs, one ahead:
        // S and dP of the next pair are issued as early as their operands
        // and buffers allow, across item boundaries when the next item's
        // K, V have their own buffer
        int k = 0, u = bwd_item(0, b, G, n_items);
        if (u >= 0) {
          int kt = u / p.BH, n_iter = p.n_tiles - kt, i = 0, n = 0, t = 0;
          wait1(w, bar(BB_KVFULL + 0), 0, 6);
          issue_s(0, sK(0));
          issue_dp(0, sV(0));
          while (true) {
            // the pair after (n, i)
            int u2 = u, i2 = i + 1, n2 = n;
            if (i2 == n_iter) {
              u2 = bwd_item(k + 1, b, G, n_items);
              i2 = 0;
              n2 = n + 1;
            }
            const bool has_next = u2 >= 0;
            const bool new_item = has_next && n2 != n;
            const int kvb2 = n2 % C::KVB;
            const bool early = has_next && (!new_item || C::KVB == 2);
            if (early) {
              if (new_item) wait1(w, bar(BB_KVFULL + kvb2), (n2 / C::KVB) & 1, 6);
              issue_s(t + 1, sK(kvb2));
            }
            // dQ_t = dS K (A = dS hi/lo in shared, MN-major; K = 128 keys)
            wait1(w, bar(BB_DSFULL), t & 1, 9);
            if (!C::ALIAS_DQ && t >= 1) wait1(w, bar(BB_DQEMPTY), (t - 1) & 1, 10);
            if (C::ALIAS_DQ && !C::DK_SMEM)
              wait1(w, bar(BB_DKDONE), t & 1, 26);  // dQ overwrites dS^T
            tc_fence_after();
            {
              const uint64_t dkk = smem_desc(sK(n % C::KVB), C::BLOCK_BYTES, 8 * C::RB, C::SW);
              const uint64_t dsh = smem_desc(sDSH, 16384, 1024, 2);
              const uint64_t dsl = smem_desc(sDSL, 16384, 1024, 2);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                mma_ss(tbase + C::COL_DQ, dsh + ((kk * 2048) >> 4), dkk + ((kk * 16 * C::RB) >> 4),
                       idQ, kk > 0 ? 1u : 0u);
                if (SLO)
                  mma_ss(tbase + C::COL_DQ, dsl + ((kk * 2048) >> 4),
                         dkk + ((kk * 16 * C::RB) >> 4), idQ, 1u);
              }
            }
            mma_commit(bar(BB_DQFULL));
            // every MMA that reads this item's K, V has been issued
            if (!has_next || new_item) mma_commit(bar(BB_KVFREE + n % C::KVB));
            if (!has_next) break;
            if (!early) {
              wait1(w, bar(BB_KVFULL + kvb2), (n2 / C::KVB) & 1, 6);
              issue_s(t + 1, sK(kvb2));
            }
            issue_dp(t + 1, sV(kvb2));
            if (new_item) {
              k = k + 1;
              u = u2;
              kt = u / p.BH;
              n_iter = p.n_tiles - kt;
            }
            i = i2;
            n = n2;
            ++t;
          }
        }
      } else {
        int t = 0, n = 0;
        for (int k = 0;; ++k) {
          const int u = bwd_item(k, b, G, n_items);
          if (u < 0) break;
          const int n_iter = p.n_tiles - u / p.BH;
          for (int i = 0; i < n_iter; ++i, ++t) {
            const int qs = t % C::QST;
            const int ds = t % C::DOST;
            const uint32_t sQ = sbase + C::OFF_Q + qs * C::TILE_BYTES;
            const uint32_t sDO = sbase + C::OFF_DO + ds * C::TILE_BYTES;
            // dV += P^T dO_t  (A = P^T hi/lo in TMEM over S^T; K = 128 queries),
            // in two halves as the compute warps hand P^T over: MMA kk
            // reads queries 16kk.., i.e. half kk % 2 of query block kk / 2.
            // Warp 18 adds P^T_hi (and, without a dV' accumulator, P^T_lo),
            // warp 19 adds P^T_lo into dV'.
            const bool lo_role = warp == 19;
            // the first dV, dK of an item overwrite the accumulators: the
            // previous item's epilogue must have read them
            if (i == 0 && n > 0) wait1(w, bar(BB_ACCFREE), (n - 1) & 1, 8);
            wait1(w, bar(BB_DOFULL + ds), (t / C::DOST) & 1, 27);  // (visibility)
            const uint64_t ddo = smem_desc(sDO, C::BLOCK_BYTES, 8 * C::RB, C::SW);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              wait1(w, bar(h ? BB_PFULL2 : BB_PFULL), t & 1, 7);
              tc_fence_after();
#pragma unroll
              for (int g4 = 0; g4 < 4; ++g4) {
                const int kk = 2 * g4 + h;
                const uint32_t acol = C::COL_S + g4 * 32 + h * 8;
                const uint64_t bd = ddo + ((kk * 16 * C::RB) >> 4);
                const uint32_t first = (i > 0 || kk > 0) ? 1u : 0u;
                if (!lo_role) mma_ts(tbase + C::COL_DV, tbase + acol, bd, idKD, first);
                if (lo_role || !C::SPLIT_DV)
                  mma_ts(tbase + C::COL_DVL, tbase + acol + 16, bd, idKD, C::SPLIT_DV ? first : 1u);
              }
            }
            mma_commit(bar(BB_PTDONE));
            mma_commit(bar(BB_DOEMPTY + ds));  // one of the slot's releases
            if (lo_role) continue;
            // dK += dS^T Q_t (A = dS^T hi/lo in TMEM over dP^T; DK_SMEM: A =
            // the shared dS hi blocks, K-major, 16 queries = 32 bytes a step)
            wait1(w, bar(BB_DSFULL), t & 1, 9);
            wait1(w, bar(BB_QFULL + qs), (t / C::QST) & 1, 28);  // (visibility)
            tc_fence_after();
            const uint64_t dqq = smem_desc(sQ, C::BLOCK_BYTES, 8 * C::RB, C::SW);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
              if constexpr (C::DK_SMEM) {
                const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_ss(tbase + C::COL_DK, smem_desc(sDSH + aoff, 16, 1024, 2),
                       dqq + ((kk * 16 * C::RB) >> 4), idKD, acc);
              } else {
                const uint32_t acol = C::COL_DP + (kk >> 1) * 32 + (kk & 1) * 8;
                mma_ts(tbase + C::COL_DK, tbase + acol, dqq + ((kk * 16 * C::RB) >> 4), idKD,
                       acc);
                if (SLO)
                  mma_ts(tbase + C::COL_DK, tbase + acol + 16, dqq + ((kk * 16 * C::RB) >> 4),
                         idKD, 1u);
              }
            }
            mma_commit(bar(BB_DKDONE));
            mma_commit(bar(BB_QEMPTY + qs));  // S(t), which also read Q_t, completed long ago
          }
          ++n;
        }
      }
      mma_commit(bar(BB_DRAIN + (warp - 17)));
      int zero = 0;
      WaitCtx wd{p.timeout_ns, &zero, 2u, false};
      wait1(wd, bar(BB_DRAIN + (warp - 17)), 0, 13);
    }
  }
  } else {
    if constexpr (C::REBALANCE) regs_inc<C::REGS_COMP>();
    // ------------------------------------------- compute warps (row = key)
    // Thread (warp w, lane l): key row r = 32*(w%4) + l, query columns
    // [32g, 32g+32) of each tile with g = w/4.  In tensor memory, P^T and
    // dS^T of query block g sit in columns 32g .. 32g+31 of their regions:
    // 16 columns of bf16 pairs (hi), then 16 (lo).
    const int quarter = warp & 3;
    const int grp = warp >> 2;                   // query column group 0..3
    const int r = quarter * 32 + lane;           // key row == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    const bool leader = threadIdx.x == 0;
    constexpr int NQ = D / 4;                    // dQ / dK / dV columns per thread

    auto load_cols = [&](uint32_t col, float (&x)[NQ]) {
      if constexpr (NQ == 32) {
        uint32_t v[32];
        tmem_ld32(col, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(v[e]);
      } else if constexpr (NQ == 16) {
        uint32_t v[16];
        tmem_ld16(col, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(v[e]);
      } else if constexpr (NQ == 8) {
        uint32_t v[8];
        tmem_ld8(col, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(v[e]);
      } else {
        uint32_t v[4];
        tmem_ld4(col, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = __uint_as_float(v[e]);
      }
    };

    // dQ(t) drain: TMEM (lane = query row) -> fp32 staging -> TMA
    // reduce-add into the accumulator, rows q0 .. q0+127 of head bh
    auto drain_dq = [&](int t, int q0, int bh) {
      wait_warp(w, bar(BB_DQFULL), t & 1, 14);
      tc_fence_after();
      float acc[NQ];
      load_cols(tbase + lane_base + C::COL_DQ + grp * NQ, acc);
      tc_fence_before();
      mbar_arrive(bar(BB_DQEMPTY));
      if constexpr (C::WARP_DQ) {
        // this warp's tile [32 rows][NQ floats]; its previous reduce must
        // have finished reading it
        const uint32_t sW = sbase + C::OFF_DQW + warp * C::WARP_STAGE;
        if (lane == 0) bulk_wait_read0();
        __syncwarp();
#pragma unroll
        for (int e = 0; e < NQ; e += 4)
          st_shared_v4(sW + swz<C::RBW>(lane * C::RBW + e * 4), __float_as_uint(acc[e]),
                       __float_as_uint(acc[e + 1]), __float_as_uint(acc[e + 2]),
                       __float_as_uint(acc[e + 3]));
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && !*abort_flag) {
          tma_reduce_add_3d(&tmDQacc, sW, grp * NQ, q0 + quarter * 32, bh);
          bulk_commit();
        }
      } else {
        // staging: blocks of [128 rows][CBQ floats], swizzled.  The
        // previous drain's reduce may still be reading its second group
        // (the blocks in the dS lo buffer, see staging_free): wait for it.
        if constexpr (C::DK_SMEM) {  // dK(t) reads the dS blocks the staging overwrites
          wait_warp(w, bar(BB_DKDONE), t & 1, 34);
          tc_fence_after();
        }
        if constexpr (C::STAGE_SPLIT) {
          if (leader) bulk_wait_read0();
          named_bar_sync(1, C::NCOMP);
        }
#pragma unroll
        for (int e = 0; e < NQ; e += 4) {
          const int f = grp * NQ + e;
          const int blk = f / C::CBQ;
          const int within = (f % C::CBQ) * 4;
          st_shared_v4(sDSH + blk * 128 * C::RBQ + swz<C::RBQ>(r * C::RBQ + within),
                       __float_as_uint(acc[e]), __float_as_uint(acc[e + 1]),
                       __float_as_uint(acc[e + 2]), __float_as_uint(acc[e + 3]));
        }
        fence_async_smem();
        // A hardware named barrier over the 512 compute threads: every
        // compute thread executes the same sequence of these (drain_dq and
        // staging_free are called at the same points of a loop whose trip
        // counts are uniform over the CTA, whatever any wait returned), so
        // each barrier is reached by all 512 and cannot hang.  A bounded
        // mbarrier in its place measured 14 % slower on the long-context
        // backward.
        named_bar_sync(1, C::NCOMP);
        if (leader && !*abort_flag) {
          // two commit groups: the blocks in the dS hi buffer, then the rest
          // (STAGE_SPLIT: the next dS phase waits for the first only)
          constexpr int NB = D / C::CBQ, NH = C::STAGE_SPLIT ? C::HI_BLOCKS : NB;
#pragma unroll
          for (int blk = 0; blk < NH; ++blk)
            tma_reduce_add_3d(&tmDQacc, sDSH + blk * 128 * C::RBQ, blk * C::CBQ, q0, bh);
          bulk_commit();
          if constexpr (NH < NB) {
#pragma unroll
            for (int blk = NH; blk < NB; ++blk)
              tma_reduce_add_3d(&tmDQacc, sDSH + blk * 128 * C::RBQ, blk * C::CBQ, q0, bh);
            bulk_commit();
          }
        }
      }
    };
    // the dS buffers may be rewritten once the reduce has read them (CTA
    // staging only; STAGE_SPLIT: the dS phase writes the hi buffer only, so
    // it waits for the first commit group, and the next drain for the rest)
    auto staging_free = [&]() {
      if constexpr (!C::WARP_DQ) {
        if (leader) {
          if constexpr (C::STAGE_SPLIT) bulk_wait_read1();
          else bulk_wait_read0();
        }
        named_bar_sync(1, C::NCOMP);
      }
    };

    // dK, dV epilogue of key tile kt of head bh, whose last query tile was
    // t_last: this thread's NQ columns of its key row, straight from TMEM
    // to global memory, once dK(t_last) (and so every dV, dK) is complete
    auto epilogue = [&](int kt, int bh, int t_last) {
      wait_warp(w, bar(BB_DKDONE), t_last & 1, 29);
      wait_warp(w, bar(BB_PTDONE), t_last & 1, 30);  // dV' (warp 19) complete too
      tc_fence_after();
      const int key = kt * 128 + r;
      const long long kb = FLAT ? 0 : bh / p.H, kh = FLAT ? 0 : bh % p.H;
      const long long kr = key < p.T ? key : 0;
      // which = 0: dV (+ dV'), 1: dK * scale; the accumulators are released
      // after the last TMEM load
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        float x[NQ];
        load_cols(tbase + lane_base + (which ? C::COL_DK : C::COL_DV) + grp * NQ, x);
        if (C::SPLIT_DV && which == 0) {
          float x2[NQ];
          load_cols(tbase + lane_base + C::COL_DVL + grp * NQ, x2);
#pragma unroll
          for (int e = 0; e < NQ; ++e) x[e] += x2[e];
        }
        if (which == 1) {
          tc_fence_before();
          mbar_arrive(bar(BB_ACCFREE));
        }
        const float mul = which ? p.scale : (DROP ? p.drop.inv_keep : 1.f);
#pragma unroll
        for (int e = 0; e < NQ; ++e) x[e] *= mul;
        if (key >= p.T) continue;
        const long long off =
            FLAT ? (which ? bh * p.dk_sh + kr * p.dk_st : bh * p.dv_sh + kr * p.dv_st) + grp * NQ
                 : (which ? kb * p.dk_sb + kh * p.dk_sh + kr * p.dk_st
                          : kb * p.dv_sb + kh * p.dv_sh + kr * p.dv_st) + grp * NQ;
        if (p.dk_f32 != nullptr) {
          float* out = (which ? p.dk_f32 : p.dv_f32) + off;
#pragma unroll
          for (int e = 0; e < NQ; e += 4)
            reinterpret_cast<float4*>(out + e)[0] = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        } else if constexpr (NQ >= 8) {
          __nv_bfloat16* out = (which ? p.dk_bf16 : p.dv_bf16) + off;
#pragma unroll
          for (int e = 0; e < NQ; e += 8)
            reinterpret_cast<uint4*>(out + e)[0] =
                make_uint4(pack_bf16(x[e], x[e + 1]), pack_bf16(x[e + 2], x[e + 3]),
                           pack_bf16(x[e + 4], x[e + 5]), pack_bf16(x[e + 6], x[e + 7]));
        } else {
          __nv_bfloat16* out = (which ? p.dk_bf16 : p.dv_bf16) + off;
          reinterpret_cast<uint2*>(out)[0] =
              make_uint2(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]));
        }
      }
    };

    // kLateDrain (own dQ staging, dQ not aliased): drain dQ(t-1) after the
    // dS phase of tile t rather than after its P phase, so that dS(t) (and
    // dK(t), dQ(t) after it) come earlier and the drain fills the wait for
    // S(t+1).
    constexpr bool kLateDrain = C::WARP_DQ && !C::ALIAS_DQ;
    float pv[32];
    int t = 0;
    // the previous query tile (its dQ is drained in the next iteration) and
    // the previous item (its epilogue follows the first P phase of the next)
    int prev_q0 = 0, prev_bh = 0, prev_kt = -1;
    for (int k = 0;; ++k) {
      const int u = bwd_item(k, b, G, n_items);
      if (u < 0) break;
      const int kt = u / p.BH, bh = u % p.BH;
      const int n_iter = p.n_tiles - kt;
      for (int i = 0; i < n_iter; ++i, ++t) {
        const int qs = t % C::QST;
        // ---- dropout keep bits (DROP), while S is on its way: bit
        // il_pos(c) of keepm is this key row's bit for query column 32g + c.
        // Lane l draws query 32g + il_key(l)'s bits for the warp's 32 keys
        // (two generator blocks), and a 32 x 32 warp transpose hands every
        // lane its own key's bits for the 32 queries.
        [[maybe_unused]] uint32_t keepm = 0u;
        if (DROP && p.drop.mask != nullptr) {  // the forward's copy: one word
          keepm = p.drop.mask[keep_cache_block(bh, p.n_tiles, kt + i, kt) + r * 4 + grp];
        } else if constexpr (DROP) {
          const uint32_t jg = static_cast<uint32_t>((kt * 128 + quarter * 32) / 16);
          const uint32_t qi = static_cast<uint32_t>((kt + i) * 128 + grp * 32 + il_key(lane));
          const uint32_t bhu = static_cast<uint32_t>(bh);
          keepm = warp_transpose32(keep16(jg, qi, bhu, p.drop) | keep16(jg + 1, qi, bhu, p.drop) << 16,
                                   lane);
        }
        // ---- P phase
        wait_warp(w, bar(BB_SFULL), t & 1, 15);
        tc_fence_after();
        {
          uint32_t v[32];
          tmem_ld32(tbase + lane_base + C::COL_S + grp * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) pv[e] = __uint_as_float(v[e]);
        }
        wait_warp(w, bar(BB_QFULL + qs), (t / C::QST) & 1, 16);  // LSE2 visibility
        const uint32_t sL = sbase + C::OFF_LSE + qs * 512 + grp * 128;
        // in two halves of 16 queries, each handed to the dV MMAs as soon
        // as it is in TMEM (hi at columns 32g + 8h, lo at 32g + 16 + 8h)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int c = 16 * h; c < 16 * h + 16; c += 4) {
            float l0, l1, l2, l3;  // -LSE * log2(e) of four queries
            ld_shared_v4f(sL + c * 4, l0, l1, l2, l3);
            float x0, x1, x2, x3;
            f2_split(fma2(f2(pv[c], pv[c + 1]), f2(sl2, sl2), f2(l0, l1)), x0, x1);
            f2_split(fma2(f2(pv[c + 2], pv[c + 3]), f2(sl2, sl2), f2(l2, l3)), x2, x3);
            pv[c] = ex2(x0);
            pv[c + 1] = ex2(x1);
            pv[c + 2] = ex2(x2);
            pv[c + 3] = ex2(x3);
          }
          if (i == 0) {  // diagonal tile: query (32g + c) sees key r only if r <= query
            const int lim = r - grp * 32;
#pragma unroll
            for (int c = 16 * h; c < 16 * h + 16; ++c)
              if (c < lim) pv[c] = 0.f;
          }
          uint32_t hi[8], lo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            split_bf16x2_p(f2(pv[16 * h + 2 * e], pv[16 * h + 2 * e + 1]), hi[e], lo[e]);
            if constexpr (DROP) {  // dV takes the dropped P (scaled in the epilogue)
              const uint32_t m =
                  prmt_sign(keepm << (7 - 4 * h - (e >> 1)), (e & 1) ? 0xBBAAu : 0x9988u);
              hi[e] &= m;
              lo[e] &= m;
            }
          }
          tmem_st8(tbase + lane_base + C::COL_S + grp * 32 + 8 * h, hi);
          tmem_st8(tbase + lane_base + C::COL_S + grp * 32 + 16 + 8 * h, lo);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(h ? BB_PFULL2 : BB_PFULL));
        }

        // ---- dQ of the previous query tile (its MMA ran during this P phase)
        // (kLateDrain: after the dS phase instead, see there)
        if (!kLateDrain && t >= 1) drain_dq(t - 1, prev_q0, prev_bh);
        // ---- the previous item's dK, dV
        if (i == 0 && prev_kt >= 0) epilogue(prev_kt, prev_bh, t - 1);

        // ---- dS phase
        wait_warp(w, bar(BB_DPFULL), t & 1, 17);
        tc_fence_after();
        // (the Delta vector arrived with Q_t, whose barrier was waited above)
        const uint32_t sD = sbase + C::OFF_DELTA + qs * 512 + grp * 128;
        uint32_t hi[16], lo[16];
        {
          uint32_t v[32];
          tmem_ld32(tbase + lane_base + C::COL_DP + grp * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float d0, d1, d2, d3;
            ld_shared_v4f(sD + e * 4, d0, d1, d2, d3);
            float s0, s1, s2, s3;
            float g0 = __uint_as_float(v[e]), g1 = __uint_as_float(v[e + 1]);
            float g2 = __uint_as_float(v[e + 2]), g3 = __uint_as_float(v[e + 3]);
            if constexpr (DROP) {  // dP = dP~ * mask / (1 - p)
              const float kp = p.drop.inv_keep;
              f2_split(mul2(f2(g0, g1), f2(kp, kp)), g0, g1);
              f2_split(mul2(f2(g2, g3), f2(kp, kp)), g2, g3);
              // queries 32g + e .. + 3 are at the byte tops of y
              const uint32_t y = keepm << (7 - 4 * (e >> 4) - ((e >> 2) & 3));
              g0 = __uint_as_float(__float_as_uint(g0) & prmt_sign(y, 0x8888u));
              g1 = __uint_as_float(__float_as_uint(g1) & prmt_sign(y, 0x9999u));
              g2 = __uint_as_float(__float_as_uint(g2) & prmt_sign(y, 0xAAAAu));
              g3 = __uint_as_float(__float_as_uint(g3) & prmt_sign(y, 0xBBBBu));
            }
            const uint64_t a01 = mul2(f2(pv[e], pv[e + 1]), sub2(f2(g0, g1), f2(d0, d1)));
            const uint64_t a23 = mul2(f2(pv[e + 2], pv[e + 3]), sub2(f2(g2, g3), f2(d2, d3)));
            f2_split(a01, s0, s1);
            f2_split(a23, s2, s3);
            if (SLO) {
              split_bf16x2_p(f2(s0, s1), hi[e / 2], lo[e / 2]);
              split_bf16x2_p(f2(s2, s3), hi[e / 2 + 1], lo[e / 2 + 1]);
            } else {
              hi[e / 2] = pack_bf16(s0, s1);
              hi[e / 2 + 1] = pack_bf16(s2, s3);
            }
          }
        }
        if constexpr (!C::DK_SMEM) {
          tmem_st16(tbase + lane_base + C::COL_DP + grp * 32, hi);
          if (SLO) tmem_st16(tbase + lane_base + C::COL_DP + grp * 32 + 16, lo);
        }
        // dS (hi, lo) -> shared for the dQ MMA: [2][128 keys][64 queries];
        // query block g is half g/2, chunks 4*(g%2) .. +3 of the row.  (dQ(t-1),
        // which read the previous dS, is complete: drained above.)
        // the previous dQ MMA, which read the previous dS, must be complete
        if (kLateDrain && t >= 1) {
          wait_warp(w, bar(BB_DQFULL), (t - 1) & 1, 31);
          tc_fence_after();
        }
        if (t >= 1) staging_free();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint32_t off = (grp >> 1) * 16384 + swz<128>(r * 128 + ((grp & 1) * 4 + ch) * 16);
          st_shared_v4(sDSH + off, hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
          if (SLO)
            st_shared_v4(sDSL + off, lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
        }
        fence_async_smem();
        if constexpr (!C::DK_SMEM) tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(BB_DSFULL));
        // ---- kLateDrain: the previous query tile's dQ, while the next S is
        // computed (the compute warps would otherwise wait for it)
        if (kLateDrain && t >= 1) drain_dq(t - 1, prev_q0, prev_bh);
        prev_q0 = (kt + i) * 128;
        prev_bh = bh;
      }
      prev_kt = kt;
    }
    if (t >= 1) {
      drain_dq(t - 1, prev_q0, prev_bh);  // waits for the last MMAs: everything is complete
      epilogue(prev_kt, prev_bh, t - 1);
    }
    // before the CTA exits, its bulk copies must have read their shared
    // memory sources (their global writes complete on their own; the next
    // kernel on the stream sees them)
    if (C::WARP_DQ) {
      if (lane == 0) bulk_wait_read0();
    } else if (leader) {
      bulk_wait_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace cattn
