// Forward kernel: O = softmax(scale * Q K^T + causal mask) V and LSE, one
// CTA per (head, 128-row query tile), never materialising the T x T matrix.
//
// Definition ("nanoGPT: a real GPT in two 300-line files", section 2 "How
// the code works", CausalSelfAttention, the written-out attention): scores
// q.k times 1/sqrt(head size), future keys filled with -inf, softmax, then
// a weighted sum of v.  The online softmax below is an exact rewrite of
// that softmax: a running maximum m and running sum l per row, with the
// partial output rescaled whenever m moves.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile, which is TMEM
//              lane t.  Reads S from TMEM, masks the diagonal tile, updates
//              m and l, writes P (bf16) to shared memory, rescales O in
//              TMEM when needed; at the end normalises O and writes O, LSE.
//   warp 4     TMA producer: Q once, then K_j, V_j through a 2-stage ring.
//   warp 5     MMA issuer (one thread) and TMEM owner:
//              S_j = Q K_j^T into one of two TMEM buffers, then
//              O += P_{j-1} V_{j-1}, so S_j overlaps the softmax of j-1.
//
// Causal tile skipping: tile i only visits key tiles 0..i (BM = BN = 128);
// only the last (diagonal) one is masked.
//
// Lazy rescaling: m is only moved when the new tile maximum exceeds it by
// more than 8 (log2 units).  The exponentials then stay below 2^8, and
// because O and l are accumulated against the same m the final O / l is
// unchanged: it is still exactly the softmax, as the online rewrite is.
#pragma once

#include "sm100.cuh"

namespace cattn {

struct FwdParams {
  float* lse;          // (BH, T) fp32 out
  int write_o_lo;      // also write O_lo = bf16(O - bf16(O)) through tmOlo
  int T;
  int n_qtiles;
  float scale_log2;    // scale * log2(e)
  uint64_t timeout_ns;
};

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int CB = D < 64 ? D : 64;      // columns per swizzle block
  static constexpr int RB = CB * 2;               // bytes per row of a block
  static constexpr int NCB = D / CB;              // column blocks
  static constexpr int BLOCK_BYTES = 128 * RB;    // one [128][CB] block
  static constexpr int TILE_BYTES = 128 * D * 2;  // [128][D] bf16
  static constexpr int STAGES = 2;
  static constexpr uint32_t SW = swizzle_code(RB);
  // shared memory map (all tiles 1024-aligned)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * TILE_BYTES;   // [2][128][64] bf16
  static constexpr int OFF_BAR = OFF_P + 128 * 128 * 2;
  static constexpr int NUM_BARS = 16;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_USED = OFF_MISC + 64;
  // keep one CTA per SM: the TMEM allocation below takes all 512 columns
  static constexpr int SMEM_BYTES = (SMEM_USED < 120 * 1024 ? 120 * 1024 : SMEM_USED) + 1024;
  static_assert(SMEM_BYTES <= kMaxDynSmem, "shared memory layout too large");
  // TMEM columns
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 192;
};

// barrier indices
enum : int {
  FB_Q = 0, FB_KFULL = 1, FB_VFULL = 3, FB_KVEMPTY = 5, FB_SFULL = 7, FB_SEMPTY = 9,
  FB_PFULL = 11, FB_OFULL = 12, FB_DRAIN = 13
};

template <int D>
__global__ void __launch_bounds__(192, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
           const __grid_constant__ CUtensorMap tmOlo, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte align the working area (swizzle atoms)
  uint8_t* smem = aligned_smem(smem_raw, C::SMEM_USED);
  if (smem == nullptr) return;  // uniform over the CTA: nothing touched yet
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sP = sbase + C::OFF_P;
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int qt = p.n_qtiles - 1 - blockIdx.y;  // longest (most key tiles) first
  const int n_kv = qt + 1;

  WaitCtx w{p.timeout_ns, abort_flag, 1u};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(FB_Q), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(FB_KFULL + s), 1);
      mbar_init(bar(FB_VFULL + s), 1);
      mbar_init(bar(FB_KVEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(FB_SFULL + b), 1);
      mbar_init(bar(FB_SEMPTY + b), 128);
    }
    mbar_init(bar(FB_PFULL), 128);
    mbar_init(bar(FB_OFULL), 1);
    mbar_init(bar(FB_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int q0 = qt * C::BM;
      mbar_arrive_expect_tx(bar(FB_Q), C::TILE_BYTES);
      for (int b = 0; b < C::NCB; ++b)
        tma_load_3d(sQ + b * C::BLOCK_BYTES, &tmQ, bar(FB_Q), b * C::CB, q0, bh);
      int n_issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::STAGES;
        if (j >= C::STAGES) wait1(w, bar(FB_KVEMPTY + st), ((j / C::STAGES) - 1) & 1, 1);
        if (*abort_flag) break;
        n_issued = j + 1;
        const uint32_t sK = sbase + C::OFF_K + st * C::TILE_BYTES;
        const uint32_t sV = sbase + C::OFF_V + st * C::TILE_BYTES;
        mbar_arrive_expect_tx(bar(FB_KFULL + st), C::TILE_BYTES);
        for (int b = 0; b < C::NCB; ++b)
          tma_load_3d(sK + b * C::BLOCK_BYTES, &tmK, bar(FB_KFULL + st), b * C::CB, j * C::BN, bh);
        mbar_arrive_expect_tx(bar(FB_VFULL + st), C::TILE_BYTES);
        for (int b = 0; b < C::NCB; ++b)
          tma_load_3d(sV + b * C::BLOCK_BYTES, &tmV, bar(FB_VFULL + st), b * C::CB, j * C::BN, bh);
      }
      if (*abort_flag) {
        // abort path: wait (bounded, ignoring the abort flag) for the loads
        // this thread issued that nobody consumed, before the CTA exits
        int zero = 0;
        WaitCtx wd{p.timeout_ns, &zero, 1u};
        for (int j = (n_issued > C::STAGES ? n_issued - C::STAGES : 0); j < n_issued; ++j) {
          const int st = j % C::STAGES;
          wait1(wd, bar(FB_KFULL + st), (j / C::STAGES) & 1, 11);
          wait1(wd, bar(FB_VFULL + st), (j / C::STAGES) & 1, 12);
        }
        wait1(wd, bar(FB_Q), 0, 13);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);    // P K-major, V MN-major
      auto issue_pv = [&](int jj) {
        const int st = jj % C::STAGES;
        wait1(w, bar(FB_PFULL), jj & 1, 2);
        wait1(w, bar(FB_VFULL + st), (jj / C::STAGES) & 1, 3);
        tc_fence_after();
        const uint32_t sV = sbase + C::OFF_V + st * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per MMA
          const uint64_t a = smem_desc(sP + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t b = smem_desc(sV + kk * 16 * C::RB, C::BLOCK_BYTES, 8 * C::RB, C::SW);
          mma_ss(tbase + C::COL_O, a, b, idO, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(FB_OFULL));
        mma_commit(bar(FB_KVEMPTY + st));
      };
      wait1(w, bar(FB_Q), 0, 4);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::STAGES;
        const int sb = j & 1;
        wait1(w, bar(FB_KFULL + st), (j / C::STAGES) & 1, 5);
        if (j >= 2) wait1(w, bar(FB_SEMPTY + sb), ((j >> 1) - 1) & 1, 6);
        tc_fence_after();
        const uint32_t sK = sbase + C::OFF_K + st * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int blk = (kk * 16) / C::CB;
          const int off = ((kk * 16) % C::CB) * 2;
          const uint64_t a = smem_desc(sQ + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW);
          const uint64_t b = smem_desc(sK + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW);
          mma_ss(tbase + (sb ? C::COL_S1 : C::COL_S0), a, b, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(FB_SFULL + sb));
        if (j >= 1) issue_pv(j - 1);
      }
      issue_pv(n_kv - 1);
      // drain: everything issued above has completed before TMEM is freed
      mma_commit(bar(FB_DRAIN));
      int zero = 0;
      WaitCtx wd{p.timeout_ns, &zero, 1u};  // the drain wait ignores the abort flag
      wait1(wd, bar(FB_DRAIN), 0, 7);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;            // 0..127 == TMEM lane
    const uint32_t lane_base = (warp * 32) << 16;
    const int q_row = qt * C::BM + row;
    const float sl2 = p.scale_log2;
    float m_used = -INFINITY;  // running max, scaled log2 units
    float l = 0.f;
    float s[128];
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      wait_warp(w, bar(FB_SFULL + sb), (j >> 1) & 1, 8);
      tc_fence_after();
      const uint32_t scol = tbase + lane_base + (sb ? C::COL_S1 : C::COL_S0);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(scol + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
      }
      tc_fence_before();
      mbar_arrive(bar(FB_SEMPTY + sb));

      if (j == n_kv - 1) {  // diagonal tile: key index > query index is future
        const int lim = q_row - j * C::BN;  // keys c <= lim are visible
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_tile = mx * sl2;
      float alpha = 1.f;
      const bool move = (j == 0) || (m_tile > m_used + 8.f);
      if (move) {
        const float m_new = fmaxf(m_used, m_tile);
        alpha = ex2(m_used - m_new);  // 0 on the first tile (m_used = -inf)
        m_used = m_new;
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = ex2(fmaf(s[c], sl2, -m_used));
        sum += s[c];
      }
      l = l * alpha + sum;

      if (j > 0) {
        // P buffer and O accumulator are free once PV_{j-1} has completed
        wait_warp(w, bar(FB_OFULL), (j - 1) & 1, 9);
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          const uint32_t ocol = tbase + lane_base + C::COL_O;
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            uint32_t r[16];
            tmem_ld16(ocol + c * 16, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16(ocol + c * 16, r);
          }
          tmem_wait_st();
        }
      }
      // P (bf16) -> shared, K-major 128B-swizzled [2][128 rows][64 keys]
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int c0 = ch * 8;
        const uint32_t addr = sP + (c0 >> 6) * 16384 + swz<128>(row * 128 + ((c0 & 63) >> 3) * 16);
        st_shared_v4(addr, pack_bf16(s[c0], s[c0 + 1]), pack_bf16(s[c0 + 2], s[c0 + 3]),
                     pack_bf16(s[c0 + 4], s[c0 + 5]), pack_bf16(s[c0 + 6], s[c0 + 7]));
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(FB_PFULL));
    }

    // ---------------------------------------------------------- epilogue
    wait_warp(w, bar(FB_OFULL), (n_kv - 1) & 1, 10);
    tc_fence_after();
    const float inv_l = 1.f / l;
    const uint32_t ocol = tbase + lane_base + C::COL_O;
    // O staging reuses the Q tile and O_lo staging the first K stage: every
    // MMA that read them has completed and no load is in flight.
    const uint32_t sOlo = sbase + C::OFF_K;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      uint32_t r[16];
      tmem_ld16(ocol + c * 16, r);
      tmem_wait_ld();
      uint32_t pk[8], lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        split_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l,
                     pk[e], lo[e]);
      const int d0 = c * 16;
      const int blk = d0 / C::CB;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int dd = (d0 % C::CB) + h * 8;
        const uint32_t off = blk * C::BLOCK_BYTES + swz<C::RB>(row * C::RB + dd * 2);
        st_shared_v4(sQ + off, pk[4 * h], pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
        if (p.write_o_lo)
          st_shared_v4(sOlo + off, lo[4 * h], lo[4 * h + 1], lo[4 * h + 2], lo[4 * h + 3]);
      }
    }
    tc_fence_before();
    fence_async_smem();
    named_bar_sync(1, 128);
    if (threadIdx.x == 0 && !*abort_flag) {
      for (int b = 0; b < C::NCB; ++b) {
        tma_store_3d(&tmO, sQ + b * C::BLOCK_BYTES, b * C::CB, qt * C::BM, bh);
        if (p.write_o_lo)
          tma_store_3d(&tmOlo, sOlo + b * C::BLOCK_BYTES, b * C::CB, qt * C::BM, bh);
      }
      bulk_commit();
      bulk_wait_read0();
    }
    if (q_row < p.T) {
      // natural-log LSE: m_used is in log2 units of the scaled score
      p.lse[static_cast<size_t>(bh) * p.T + q_row] = m_used * 0.69314718055994531f + logf(l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace cattn
