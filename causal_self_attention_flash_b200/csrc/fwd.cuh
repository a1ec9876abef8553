// Forward kernel: O = softmax(scale * Q K^T + causal mask) V and LSE,
// never materialising the T x T matrix.
//
// Definition ("nanoGPT: a real GPT in two 300-line files", section 2 "How
// the code works", CausalSelfAttention, the written-out attention): scores
// q.k times 1/sqrt(head size), future keys filled with -inf, softmax, then
// a weighted sum of v.  The online softmax below is an exact rewrite of
// that softmax: a running maximum m and running sum l per row, with the
// partial output rescaled whenever m moves.
//
// The kernel is persistent: one CTA per SM loops over work items, each a
// pair of 128-row query tiles (2c, 2c+1) of one head.  The two tiles go to
// two softmax warpgroups, so the tensor core alternates between them: while
// one warpgroup works on its scores, the MMAs of the other run.  The next
// item's Q and K/V are loaded while the current item finishes.
//
// Warp roles (352 threads; 384 with D = 128):
//   warps 0-3, 4-7  softmax warpgroups g = 0, 1, one query tile each per item;
//              thread t of a group owns query row t, which is TMEM lane t.
//              It reads S_g from TMEM, masks the diagonal tile, updates m
//              and l, and writes P to TMEM: as bf16 (PLO = false, the usual
//              mixed precision), or as bf16 hi/lo pairs (PLO = true, P = hi +
//              lo to ~14 bits, used when the caller wants the O_lo residual,
//              whose purpose is an O accurate to ~fp32); at the end it
//              normalises O_g and writes O (bf16), with PLO also
//              O_lo = bf16(O - bf16(O)), and LSE, each thread its own row
//              straight from registers.
//   warp 8     TMA producer: per item each group's Q tile (once the previous
//              item's S MMAs are done with the buffer), then K_j, V_j through
//              a ring that runs on across items.
//   warp 11    (D = 128 only) idle; it completes the third warpgroup
//              (warps 8-11), whose registers go to the softmax warpgroups.
//   warps 9, 10  MMA issuers for groups 0, 1 (warp 9 also owns TMEM).  Two
//              issuing threads keep the tensor core fed where one thread's
//              issue rate would not (N = D <= 64 MMAs).  Per key tile j:
//              O_g += P_hi V_j (A from TMEM), with PLO also O'_g += P_lo V_j
//              (for D <= 64 into a second accumulator, summed at the end,
//              because MMAs that accumulate into one TMEM tile run back to
//              back at about half the rate of independent ones), and
//              S_g(j+1) = Q_g K_{j+1}^T.
//
// Where P lives decides when S_g(j+1) can start (the MMAs one thread issues
// execute in issue order):
//   EARLY (bf16 P, D <= 64): P_g has its own TMEM columns.  S_g(j+1) is
//              issued as soon as the softmax has loaded S_g(j) into registers,
//              so it runs during the softmax of tile j; the softmax waits for
//              PV_g(j-1) before it rescales O_g or overwrites P_g.
//   otherwise  P_g is written over S_g (TMEM holds no room for separate P
//              columns), and S_g(j+1) is issued right behind PV_g(j).
//
// Causal tile skipping: query tile t visits key tiles 0..t only
// (BM = BN = 128); only the last (diagonal) one is masked.
//
// Lazy rescaling: m is only moved when the new tile maximum exceeds it by
// more than 8 (log2 units).  The exponentials then stay below 2^8, and
// because O and l are accumulated against the same m the final O / l is
// unchanged: it is still exactly the softmax, as the online rewrite is.
//
// Instances fwd_kernel<D, PLO, DROP, FLAT>:
//   DROP   attention dropout (philox.cuh): each softmax thread draws its
//          row's keep bits for a key tile before that tile's scores arrive,
//          writes the dropped P entries as 0 (the row sum l still takes
//          every entry) and folds the keep scale 1 / (1 - p) into 1 / l.
//   FLAT   Q, K, V and O address (b, h) as one b*H + h index (3-D tensor
//          maps); otherwise 4-D maps {d, t, h, b} take any element strides,
//          e.g. q, k, v as views into one fused (B, T, 3C) projection.
#pragma once

#include "philox.cuh"
#include "sched.cuh"
#include "sm100.cuh"

namespace cattn {

struct FwdParams {
  __nv_bfloat16* o;     // (B, H, T, D) bf16 out, element strides o_sb, o_sh, o_st
  __nv_bfloat16* o_lo;  // O_lo = bf16(O - bf16(O)) out (same strides), or null
  long long o_sb, o_sh, o_st;
  float* lse;          // (B, H, T) fp32 out, contiguous
  int H;
  int T;
  int BH;
  int n_qtiles;
  float scale_log2;    // scale * log2(e)
  uint64_t timeout_ns;
  DropParams drop;     // attention dropout (kernels instantiated with DROP only)
  PassCodes passes;    // how the work items are dealt to the CTAs (sched.cuh)
};

template <int D, bool PLO, bool DROP = false>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int CB = D < 64 ? D : 64;      // columns per swizzle block
  static constexpr int RB = CB * 2;               // bytes per row of a block
  static constexpr int NCB = D / CB;              // column blocks
  static constexpr int BLOCK_BYTES = 128 * RB;    // one [128][CB] block
  static constexpr int TILE_BYTES = 128 * D * 2;  // [128][D] bf16
  // K/V ring depth (measured on the GPT-2 layer: 3 stages 65.9 us, 4 stages
  // 66.6 us, 5 stages 69.5 us)
  static constexpr int STAGES = D <= 64 ? 3 : 2;
  static constexpr uint32_t SW = swizzle_code(RB);
  // shared memory map (all tiles 1024-aligned)
  static constexpr int OFF_Q = 0;                              // [2] query tiles
  static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
  static constexpr int NUM_BARS = 47;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_PASS = OFF_MISC + 64;  // the pass codes (sched.cuh)
  static constexpr int SMEM_USED = OFF_PASS + kPassSmemBytes;
  // at least 116 KB so that one CTA holds an SM (it takes all 512 TMEM columns)
  static constexpr int SMEM_WANT = SMEM_USED + 1024 < 116 * 1024 ? 116 * 1024 : SMEM_USED + 1024;
  static constexpr int SMEM_BYTES = SMEM_WANT <= kMaxDynSmem ? SMEM_WANT : SMEM_USED;
  static_assert(SMEM_USED <= kMaxDynSmem, "shared memory layout too large");
  // EARLY (bf16 P, D <= 64): P_g has its own 64 TMEM columns, so S_g(j+1)
  // can be computed while the softmax still works on tile j.  Otherwise P
  // (bf16, or hi/lo pairs) is written over S_g.
  static constexpr bool EARLY = !PLO && D <= 64;
  // TMEM columns: S_0, S_1, [P_0, P_1 if EARLY], O_0, O_1, and with P hi/lo
  // for D <= 64 the second accumulators O'_0, O'_1 of the P_lo products
  static constexpr bool SPLIT = PLO && 256 + 4 * D <= 512;
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128;
  static constexpr uint32_t COL_P0 = EARLY ? 256 : COL_S0, COL_P1 = EARLY ? 320 : COL_S1;
  static constexpr uint32_t COL_O0 = EARLY ? 384 : 256, COL_O1 = COL_O0 + D;
  static constexpr uint32_t COL_OL0 = SPLIT ? 256 + 2 * D : COL_O0;
  static constexpr uint32_t COL_OL1 = SPLIT ? 256 + 3 * D : COL_O1;
  static constexpr uint32_t TMEM_COLS = 512;
  // Two softmax warpgroups, then the producer and two MMA issuers.  With
  // D >= 64 (REBALANCE) a twelfth, idle warp completes the third warpgroup
  // so that its registers can be handed to the softmax warps (setmaxnreg
  // acts on whole warpgroups): at launch every thread holds LAUNCH_REGS
  // (65536 / 384, rounded down to 8); the third warpgroup then drops to
  // REGS_OTHER and the softmax warpgroups rise to REGS_SOFTMAX, within the
  // launch total.  That removed the D = 128 softmax's spills (3.6 % faster
  // on the long-context workload, at 216 and 64; 208 and 80 measured 2-4 %
  // faster still, 224 and 48 between them).  D = 64 takes 200 and 88 (1 %
  // faster than 168 throughout; 208 and 72 the same; 216 and 64 measured
  // 4 % slower); D <= 32 keeps 11 warps and 168 registers.  With dropout
  // the softmax threads draw the keep bits themselves: at 200 registers
  // that measured faster than a fourth warpgroup drawing them into a
  // shared-memory ring (145 against 167 us on the GPT-2 layer).
  static constexpr bool REBALANCE = D >= 64;
  static constexpr int THREADS = REBALANCE ? 384 : 352;
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int REGS_SOFTMAX = D == 128 ? 208 : 200;
  static constexpr int REGS_OTHER = D == 128 ? 80 : 88;
  static_assert(!REBALANCE ||
                    256 * REGS_SOFTMAX + (THREADS - 256) * REGS_OTHER <= THREADS * LAUNCH_REGS,
                "register split exceeds the launch allocation");
};

// barrier indices
// (KVEMPTY: one per group and stage, index FB_KVEMPTY + kMaxStages * g + stage; the
// other per-group barriers at base + g)
constexpr int kMaxStages = 6;
enum : int {
  FB_KFULL = 0, FB_VFULL = kMaxStages, FB_KVEMPTY = 2 * kMaxStages, FB_QFULL = 4 * kMaxStages,
  FB_QFREE = FB_QFULL + 2, FB_SFULL = FB_QFULL + 4, FB_ODONE = FB_QFULL + 6,
  FB_OFREE = FB_QFULL + 8, FB_SFREE = FB_QFULL + 10, FB_DRAIN = FB_QFULL + 12,
  FB_PFULL = FB_QFULL + 14,  // FB_PFULL + 4 * g + part
  FB_OFFSET = FB_PFULL + 8   // the one-time start offset of the two groups
};

// Pairs of score columns whose exponential is taken by exp2_poly2 on the FMA
// pipes instead of the ex2 unit, as a bit mask over the pair index within a
// 16-column chunk.  The ex2 unit does 16 per clock per SM; with D = 128 a
// tile's MMAs take as long as its exponentials, and moving 2 of 8 pairs to
// the FMA pipes measured 4 % faster (long-context workload).  With D <= 64
// the softmax warps have no issue slots to spare and the share measured
// slower, so it is 0 there.  Only used on tiles without masked entries
// (exp2_poly2 has no exact zero).
__host__ __device__ constexpr uint32_t fwd_poly_pairs(int D) { return D == 128 ? 0x11u : 0x00u; }

// Exponential-phase turns: the two softmax warps of a sub-partition (warp
// q of group 0 and warp 4 + q of group 1) share its ex2 unit.  When both
// run their exponential phases at once, each takes twice as long and their
// other work (score loads, maxima, waits) then overlaps nothing; so a warp
// about to start its phase first waits, for a bounded number of short
// sleeps, while its partner's busy flag (shared memory) is set.  Only a
// scheduling hint: a warp that gives up, or that races its partner past the
// check, just runs its phase alongside, and no result depends on it.
// Measured: 4-5 % faster forward with D = 128 (long-context workload, 16
// polls; 64 and 256 polls gained less), 5 % slower with D = 64, whose
// phases are short against the waits between them: only D = 128 takes
// turns.
__host__ __device__ constexpr bool fwd_exp_turns(int D) { return D == 128; }
constexpr int kFwdTurnPolls = 16;  // sleeps of ~32 ns before giving up

// P_g(j) is handed to the MMA warp in kPvParts parts (of 128 / kPvParts
// keys each), so PV_g(j) starts while the later exponentials are computed.
constexpr int kPvParts = 2;

// P = 2^(s * scale_log2 - m) for one row of a 128-column tile: written to
// TMEM as bf16 (or bf16 hi/lo), the row sum accumulated in sum2.
// DROP: P entries whose bit in keep (column c at bit il_pos(c % 32) of
// keep[c / 32]) is clear are written as 0; the row sum still takes every
// entry.  A pair's two bits become a bf16x2 AND mask with one prmt.
template <int D, bool POLY, bool PLO, bool DROP>
__device__ __forceinline__ void fwd_exp_row(const float (&s)[128], uint64_t sl2x2, uint64_t negm2,
                                            uint32_t scol, uint64_t (&sum2)[2], uint32_t pfull0,
                                            const uint32_t* keep) {
#pragma unroll
  for (int ch = 0; ch < 8; ++ch) {  // 16 columns per chunk
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint64_t x2 = fma2(f2(s[ch * 16 + 2 * e], s[ch * 16 + 2 * e + 1]), sl2x2, negm2);
      uint64_t p2;
      if (POLY && ((fwd_poly_pairs(D) >> e) & 1u)) {
        float x0, x1;
        f2_split(x2, x0, x1);
        p2 = exp2_poly2(x0, x1);
      } else {
        float x0, x1;
        f2_split(x2, x0, x1);
        p2 = f2(ex2(x0), ex2(x1));
      }
      sum2[e & 1] = add2(sum2[e & 1], p2);
      if (PLO) {
        split_bf16x2_p(p2, hi[e], lo[e]);
      } else {
        float p0, p1;
        f2_split(p2, p0, p1);
        hi[e] = pack_bf16(p0, p1);
      }
      if constexpr (DROP) {
        // columns 16 ch + 2 e, + 1: keys 16 h + 4 v + k, k = 2 (e & 1) and
        // 2 (e & 1) + 1, of word ch / 2; the shift moves their flags to the
        // top of bytes k
        const uint32_t y = keep[ch >> 1] << (7 - 4 * (ch & 1) - (e >> 1));
        const uint32_t m = prmt_sign(y, (e & 1) ? 0xBBAAu : 0x9988u);
        hi[e] &= m;
        if (PLO) lo[e] &= m;
      }
    }
    tmem_st8(scol + ch * 8, hi);
    if (PLO) tmem_st8(scol + 64 + ch * 8, lo);
    if ((ch + 1) % (8 / kPvParts) == 0) {  // a part of P is complete: the MMA may read it
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(pfull0 + 8u * ((ch + 1) / (8 / kPvParts) - 1));
    }
  }
}

// Work items: pairs (c, bh) of query tiles 2c, 2c+1 of head bh, numbered
// longest first (u = 0 .. BH*n_pairs-1: c = n_pairs-1 - u / BH, bh = u % BH).
// The grid is persistent (at most one CTA per SM); CTA b takes items in
// passes over the grid, one item per pass, dealt by the call's pass codes
// (sched.cuh) so that every CTA gets a similar total.  Returns -1 past the
// last item.
__device__ __forceinline__ int fwd_item(int k, int b, int G, int n_items, int n_codes,
                                         const uint16_t* codes_s) {
  return pass_item_smem(k, b, G, n_items, n_codes, codes_s);
}

// An item's two query tiles go to the two softmax groups, the longer one
// (one key tile more) to group 1 on even passes k and to group 0 on odd
// ones, so that over its items a CTA's groups carry about equal work.
struct FwdItem {
  int bh;
  int tile[2];  // query tile of group g
  int n[2];     // key tiles group g visits (0: no tile)
  int n_kv;     // key tiles loaded for the item
};

__device__ __forceinline__ FwdItem fwd_item_info(int u, int k, int BH, int n_pairs,
                                                  int n_qtiles) {
  FwdItem it;
  const int c = n_pairs - 1 - u / BH;
  it.bh = u % BH;
  const int t0 = 2 * c;
  const int nlo = t0 + 1;                           // tile t0
  const int nhi = t0 + 1 < n_qtiles ? t0 + 2 : 0;   // tile t0 + 1, if any
  const int s = k & 1;
  it.tile[s] = t0 + 1;
  it.n[s] = nhi;
  it.tile[s ^ 1] = t0;
  it.n[s ^ 1] = nlo;
  it.n_kv = nhi ? nhi : nlo;
  return it;
}

// FLAT: Q, K, V and O address (b, h) as one b*H + h axis (3-D tensor
// maps, O offsets bh * o_sh); otherwise 4-D maps with (h, b) coordinates.
template <int D, bool PLO, bool DROP, bool FLAT>
__global__ void __launch_bounds__(FwdCfg<D, PLO, DROP>::THREADS, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, PLO, DROP>;
  static_assert(FB_OFFSET + 1 <= C::NUM_BARS, "barrier count");
  static_assert(C::STAGES <= kMaxStages, "barrier map");
  // launched as a programmatic dependent of the previous kernel: its
  // writes (Q, K, V) are visible after this
  grid_dep_wait();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = aligned_smem(smem_raw, C::SMEM_USED, nullptr);
  if (smem == nullptr) return;  // uniform over the CTA: nothing touched yet
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_pairs = (p.n_qtiles + 1) >> 1;
  const int n_items = p.BH * n_pairs;
  const int G = gridDim.x, b = blockIdx.x;

  WaitCtx w{p.timeout_ns, abort_flag, 1u, false};

  volatile int* exp_busy = reinterpret_cast<volatile int*>(misc + 8);  // [8 softmax warps]
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 8; ++i) exp_busy[i] = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(FB_KFULL + s), 1);
      mbar_init(bar(FB_VFULL + s), 1);
      mbar_init(bar(FB_KVEMPTY + s), 1);
      mbar_init(bar(FB_KVEMPTY + kMaxStages + s), 1);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(bar(FB_QFULL + g), 1);
      mbar_init(bar(FB_QFREE + g), 1);
      mbar_init(bar(FB_SFULL + g), 1);
      for (int h = 0; h < kPvParts; ++h) mbar_init(bar(FB_PFULL + 4 * g + h), 128);
      mbar_init(bar(FB_ODONE + g), 1);
      mbar_init(bar(FB_OFREE + g), 128);
      mbar_init(bar(FB_SFREE + g), 128);
      mbar_init(bar(FB_DRAIN + g), 1);
    }
    mbar_init(bar(FB_OFFSET), 128);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  uint16_t* const pass_s = reinterpret_cast<uint16_t*>(smem + C::OFF_PASS);
  pass_codes_to_smem(p.passes, pass_s);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  if (warp >= 8) {
  // third warpgroup: producer, MMA issuers (and with REBALANCE an idle
  // warp)
  if constexpr (C::REBALANCE) regs_dec<C::REGS_OTHER>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Per item: Q_g once the previous item no longer needs the Q_g buffer,
    // then K_j, V_j through a ring that runs on across items (tk counts the
    // CTA's K/V tiles).
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int tk = 0, aq[2] = {0, 0};
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
      for (int k = 0;; ++k) {
        const int u = fwd_item(k, b, G, n_items, p.passes.n, pass_s);
        if (u < 0 || *abort_flag) break;
        const FwdItem it = fwd_item_info(u, k, p.BH, n_pairs, p.n_qtiles);
        for (int g = 0; g < 2; ++g) {
          if (it.n[g] == 0) continue;
          if (aq[g] > 0) wait1(w, bar(FB_QFREE + g), (aq[g] - 1) & 1, 1);
          mbar_arrive_expect_tx(bar(FB_QFULL + g), C::TILE_BYTES);
          for (int bb = 0; bb < C::NCB; ++bb)
            load_tile(sbase + C::OFF_Q + g * C::TILE_BYTES + bb * C::BLOCK_BYTES, &tmQ, 1,
                      bar(FB_QFULL + g), bb * C::CB, it.tile[g] * C::BM, it.bh);
          ++aq[g];
        }
        for (int j = 0; j < it.n_kv; ++j, ++tk) {
          const int st = tk % C::STAGES;
          if (tk >= C::STAGES) {  // both groups have released the tile this stage held
            const uint32_t ph = ((tk / C::STAGES) - 1) & 1;
            wait1(w, bar(FB_KVEMPTY + st), ph, 1);
            wait1(w, bar(FB_KVEMPTY + kMaxStages + st), ph, 1);
          }
          if (*abort_flag) break;
          const uint32_t sK = sbase + C::OFF_K + st * C::TILE_BYTES;
          const uint32_t sV = sbase + C::OFF_V + st * C::TILE_BYTES;
          mbar_arrive_expect_tx(bar(FB_KFULL + st), C::TILE_BYTES);
          for (int bb = 0; bb < C::NCB; ++bb)
            load_tile(sK + bb * C::BLOCK_BYTES, &tmK, 2, bar(FB_KFULL + st), bb * C::CB,
                      j * C::BN, it.bh);
          mbar_arrive_expect_tx(bar(FB_VFULL + st), C::TILE_BYTES);
          for (int bb = 0; bb < C::NCB; ++bb)
            load_tile(sV + bb * C::BLOCK_BYTES, &tmV, 4, bar(FB_VFULL + st), bb * C::CB,
                      j * C::BN, it.bh);
        }
      }
      if (*abort_flag) {
        // abort path: wait (bounded, ignoring the abort flag) for the last
        // loads this thread issued, which may not have been consumed, before
        // the CTA exits
        int zero = 0;
        WaitCtx wd{p.timeout_ns, &zero, 1u, false};
        for (int t = (tk > C::STAGES ? tk - C::STAGES : 0); t < tk; ++t) {
          const int st = t % C::STAGES;
          wait1(wd, bar(FB_KFULL + st), (t / C::STAGES) & 1, 11);
          wait1(wd, bar(FB_VFULL + st), (t / C::STAGES) & 1, 12);
        }
        for (int g = 0; g < 2; ++g)
          if (aq[g] > 0) wait1(wd, bar(FB_QFULL + g), (aq[g] - 1) & 1, 13);
      }
    }
  } else if (warp <= 10) {
    // ------------------------------------------------- MMA issuers (one per group)
    // Running counters across items: tg = tiles of this group so far (the
    // phase of its S/P/O barriers), aq = items of this group so far (Q and
    // O hand-over), tk = K/V ring position.
    const int g = warp - 9;
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);  // Q K-major, K K-major
      constexpr uint32_t idO = idesc_bf16(128, D, 0, 1);    // P (TMEM), V MN-major
      const uint64_t dq = smem_desc(sbase + C::OFF_Q + g * C::TILE_BYTES, 16, 8 * C::RB, C::SW);
      const uint32_t scol_t = tbase + (g ? C::COL_S1 : C::COL_S0);
      const uint32_t pcol_t = tbase + (g ? C::COL_P1 : C::COL_P0);
      const uint32_t ocol_t = tbase + (g ? C::COL_O1 : C::COL_O0);
      const uint32_t olcol_t = tbase + (g ? C::COL_OL1 : C::COL_OL0);
      int tg = 0, aq = 0, tk = 0;
      auto issue_s = [&](int j, int tkj) {  // S_g = Q_g K_j^T
        const int st = tkj % C::STAGES;
        wait1(w, bar(FB_KFULL + st), (tkj / C::STAGES) & 1, 2);
        tc_fence_after();
        const uint64_t dk = smem_desc(sbase + C::OFF_K + st * C::TILE_BYTES, 16, 8 * C::RB, C::SW);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int blk = (kk * 16) / C::CB;
          const uint32_t off = (blk * C::BLOCK_BYTES + ((kk * 16) % C::CB) * 2) >> 4;
          mma_ss(scol_t, dq + off, dk + off, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(FB_SFULL + g));
      };
      auto issue_pv = [&](int j, int tkj, int tgj) {  // O_g += (P_hi + P_lo) V_j
        const int st = tkj % C::STAGES;
        wait1(w, bar(FB_VFULL + st), (tkj / C::STAGES) & 1, 4);
        const uint64_t dv = smem_desc(sbase + C::OFF_V + st * C::TILE_BYTES, C::BLOCK_BYTES,
                                      8 * C::RB, C::SW);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 128 keys, 16 per MMA
          if (kk % (8 / kPvParts) == 0) {  // the next part of P_g(j) is in TMEM
            wait1(w, bar(FB_PFULL + 4 * g + kk / (8 / kPvParts)), tgj & 1, 3);
            tc_fence_after();
          }
          const uint64_t bdesc = dv + ((kk * 16 * C::RB) >> 4);
          const uint32_t first = (j > 0 || kk > 0) ? 1u : 0u;
          mma_ts(ocol_t, pcol_t + kk * 8, bdesc, idO, first);
          if (PLO) mma_ts(olcol_t, pcol_t + 64 + kk * 8, bdesc, idO, C::SPLIT ? first : 1u);
        }
        mma_commit(bar(FB_ODONE + g));
      };
      for (int k = 0;; ++k) {
        const int u = fwd_item(k, b, G, n_items, p.passes.n, pass_s);
        if (u < 0) break;
        const FwdItem it = fwd_item_info(u, k, p.BH, n_pairs, p.n_qtiles);
        const int ng = it.n[g];
        if (ng > 0) {
          wait1(w, bar(FB_QFULL + g), aq & 1, 5);
          // EARLY: S_g is read by the softmax before S_g(0) may overwrite it
          if (C::EARLY && tg > 0) wait1(w, bar(FB_SFREE + g), (tg - 1) & 1, 6);
          issue_s(0, tk);
          if (ng == 1) mma_commit(bar(FB_QFREE + g));  // last read of Q_g issued
          for (int j = 0; j < ng; ++j) {
            if (C::EARLY && j + 1 < ng) {
              // S_g(j+1) as soon as the softmax has S_g(j) in registers
              wait1(w, bar(FB_SFREE + g), (tg + j) & 1, 6);
              issue_s(j + 1, tk + j + 1);
              if (j + 2 == ng) mma_commit(bar(FB_QFREE + g));
            }
            // O_g is overwritten by PV_g(0): the epilogue of the previous
            // item must have read it
            if (j == 0 && aq > 0) wait1(w, bar(FB_OFREE + g), (aq - 1) & 1, 8);
            issue_pv(j, tk + j, tg + j);
            // P over S: S_g(j+1) goes in order behind PV_g(j), which reads P_g(j)
            if (!C::EARLY && j + 1 < ng) {
              issue_s(j + 1, tk + j + 1);
              if (j + 2 == ng) mma_commit(bar(FB_QFREE + g));
            }
            mma_commit(bar(FB_KVEMPTY + kMaxStages * g + (tk + j) % C::STAGES));
          }
          tg += ng;
          ++aq;
        }
        // K/V tiles of this item that this group does not use: released once
        // loaded (never earlier: a release of a tile not yet loaded would
        // complete two phases of the stage's barrier before the producer
        // waits, and its parity wait would then not see them)
        for (int j = ng; j < it.n_kv; ++j) {
          const int t = tk + j;
          wait1(w, bar(FB_KFULL + t % C::STAGES), (t / C::STAGES) & 1, 2);
          mma_commit(bar(FB_KVEMPTY + kMaxStages * g + t % C::STAGES));
        }
        tk += it.n_kv;
      }
      // drain: everything issued above has completed before TMEM is freed
      mma_commit(bar(FB_DRAIN + g));
      int zero = 0;
      WaitCtx wd{p.timeout_ns, &zero, 1u, false};  // the drain wait ignores the abort flag
      wait1(wd, bar(FB_DRAIN + g), 0, 7);
    }
  }
  } else {
    if constexpr (C::REBALANCE) regs_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax
    const int g = warp >> 2;                 // warpgroup: one query tile per item
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;     // query row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t scol = tbase + lane_base + (g ? C::COL_S1 : C::COL_S0);
    const uint32_t pcol = tbase + lane_base + (g ? C::COL_P1 : C::COL_P0);
    const uint32_t ocol = tbase + lane_base + (g ? C::COL_O1 : C::COL_O0);
    const uint32_t olcol = tbase + lane_base + (g ? C::COL_OL1 : C::COL_OL0);
    const float sl2 = p.scale_log2;
    int tg = 0;
    float s[128];
    // Once per CTA, group 1 starts only after group 0's first exponential
    // phase: the two groups then stay out of step, so their exponential
    // phases overlap less on the ex2 unit.  Exactly one phase of the
    // FB_OFFSET barrier per CTA: group 0's 128 threads arrive once (after
    // the exponentials of the first tile of the first item), group 1 waits
    // once, here (bounded, like every wait), and both take it only when both
    // groups have a tile in the first item.  Waiting before the loop keeps
    // the wait out of the loop body.
    {
      const int u0 = fwd_item(0, b, G, n_items, p.passes.n, pass_s);
      if (u0 >= 0 && g == 1) {
        const FwdItem it0 = fwd_item_info(u0, 0, p.BH, n_pairs, p.n_qtiles);
        if (it0.n[0] > 0 && it0.n[1] > 0) wait_warp(w, bar(FB_OFFSET), 0, 11);
      }
    }
    for (int k = 0;; ++k) {
      const int u = fwd_item(k, b, G, n_items, p.passes.n, pass_s);
      if (u < 0) break;
      const FwdItem it = fwd_item_info(u, k, p.BH, n_pairs, p.n_qtiles);
      const int ng = it.n[g];
      if (ng == 0) continue;
      float m_used = -INFINITY;  // running max, scaled log2 units
      float l = 0.f;
      for (int j = 0; j < ng; ++j) {
        const int tgj = tg + j;
        // dropout keep bits of this row's 128 keys of tile j, computed while
        // the scores are still on their way
        [[maybe_unused]] uint32_t keep[4] = {0u, 0u, 0u, 0u};
        if constexpr (DROP) {
          const uint32_t qi = static_cast<uint32_t>(it.tile[g] * C::BM + row);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            keep[c4] = keep32_il(static_cast<uint32_t>(j * 4 + c4), qi, static_cast<uint32_t>(it.bh),
                                 p.drop);
          if (p.drop.mask != nullptr)  // the backward's copy
            store_keep_block(keep, p.drop.mask + keep_cache_block(it.bh, p.n_qtiles, it.tile[g], j),
                             quarter, lane);
        }
        wait_warp(w, bar(FB_SFULL + g), tgj & 1, 8);
        tc_fence_after();
        {
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(scol, r0);
          tmem_ld32(scol + 32, r1);
          tmem_ld32(scol + 64, r2);
          tmem_ld32(scol + 96, r3);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            s[e] = __uint_as_float(r0[e]);
            s[32 + e] = __uint_as_float(r1[e]);
            s[64 + e] = __uint_as_float(r2[e]);
            s[96 + e] = __uint_as_float(r3[e]);
          }
        }
        if (C::EARLY) {  // S_g may now be overwritten by the next score tile
          tc_fence_before();
          mbar_arrive(bar(FB_SFREE + g));
        }
        if (j == ng - 1) {  // diagonal tile: key column > query row is future
#pragma unroll
          for (int cc = 0; cc < 128; ++cc)
            if (cc > row) s[cc] = -INFINITY;
        }
        float mx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmax3(s[i], s[4 + i], s[8 + i]);
#pragma unroll
        for (int cc = 12; cc < 124; cc += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = fmax3(mx[i], s[cc + i], s[cc + 4 + i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], s[124 + i]);
        const float mxa = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
        const float m_tile = mxa * sl2;
        float alpha = 1.f;
        const bool move = (j == 0) || (m_tile > m_used + 8.f);
        if (move) {
          const float m_new = fmaxf(m_used, m_tile);
          alpha = ex2(m_used - m_new);  // 0 on the first tile (m_used = -inf)
          m_used = m_new;
        }
        // O_g must be stable before it is rescaled, and P_g(j-1) read before
        // P_g(j) is written.  Over S (not EARLY): S_g(j), whose completion
        // was just observed, was issued after PV_g(j-1), and MMAs complete
        // in issue order.  EARLY: wait for PV_g(j-1) itself.  (For j = 0,
        // the previous item's epilogue waited for its last PV.)
        if (C::EARLY && j > 0) {
          wait_warp(w, bar(FB_ODONE + g), (tgj - 1) & 1, 9);
          tc_fence_after();
        }
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int acc = 0; acc < (C::SPLIT ? 2 : 1); ++acc) {
            const uint32_t col = acc ? olcol : ocol;
#pragma unroll
            for (int cc = 0; cc < D / 16; ++cc) {
              uint32_t r[16];
              tmem_ld16(col + cc * 16, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
              tmem_st16(col + cc * 16, r);
            }
          }
        }
        const uint64_t sl2x2 = f2(sl2, sl2);
        const uint64_t negm2 = f2(-m_used, -m_used);
        uint64_t sum2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
        // Group 0's side of the one-time offset (see before the item loop).
        const bool offset = k == 0 && j == 0 && it.n[0] > 0 && it.n[1] > 0;
        if constexpr (fwd_exp_turns(D)) {
          if (lane == 0) {
            for (int i = 0; i < kFwdTurnPolls && exp_busy[warp ^ 4]; ++i) __nanosleep(32);
            exp_busy[warp] = 1;
          }
          __syncwarp();
        }
        if (j == ng - 1)
          fwd_exp_row<D, false, PLO, DROP>(s, sl2x2, negm2, pcol, sum2, bar(FB_PFULL + 4 * g),
                                           DROP ? keep : nullptr);
        else
          fwd_exp_row<D, true, PLO, DROP>(s, sl2x2, negm2, pcol, sum2, bar(FB_PFULL + 4 * g),
                                          DROP ? keep : nullptr);
        if constexpr (fwd_exp_turns(D)) {
          __syncwarp();
          if (lane == 0) exp_busy[warp] = 0;
        }
        if (offset && g == 0) mbar_arrive(bar(FB_OFFSET));
        float sa, sb, sc2, sd;
        f2_split(sum2[0], sa, sb);
        f2_split(sum2[1], sc2, sd);
        l = l * alpha + ((sa + sb) + (sc2 + sd));
      }

      // -------------------------------------------------------- epilogue
      wait_warp(w, bar(FB_ODONE + g), (tg + ng - 1) & 1, 10);
      tc_fence_after();
      // (DROP: O = P~ V with P~ = P * mask / (1 - p): the keep scale is
      // applied here, once per row)
      const float inv_l = DROP ? p.drop.inv_keep / l : 1.f / l;
      // O (and O') into registers; then TMEM is free for the next item
      uint32_t o_all[D / 2], lo_all[PLO ? D / 2 : 1];
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) {
        uint32_t r[16];
        tmem_ld16(ocol + cc * 16, r);
        if (C::SPLIT) {
          uint32_t r2[16];
          tmem_ld16(olcol + cc * 16, r2);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            r[e] = __float_as_uint(__uint_as_float(r[e]) + __uint_as_float(r2[e]));
        } else {
          tmem_wait_ld();
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x0 = __uint_as_float(r[2 * e]) * inv_l;
          const float x1 = __uint_as_float(r[2 * e + 1]) * inv_l;
          if constexpr (PLO) split_bf16x2(x0, x1, o_all[cc * 8 + e], lo_all[cc * 8 + e]);
          else o_all[cc * 8 + e] = pack_bf16(x0, x1);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(FB_OFREE + g));
      // each thread writes its own row (D contiguous bf16) straight to
      // global memory: no staging, no barrier, no wait
      const int tile = it.tile[g];
      const int q_row = tile * C::BM + row;
      if (q_row < p.T) {
        const long long off =
            FLAT ? static_cast<long long>(it.bh) * p.o_sh + static_cast<long long>(q_row) * p.o_st
                 : static_cast<long long>(it.bh / p.H) * p.o_sb +
                       static_cast<long long>(it.bh % p.H) * p.o_sh +
                       static_cast<long long>(q_row) * p.o_st;
        uint4* orow = reinterpret_cast<uint4*>(p.o + off);
#pragma unroll
        for (int e = 0; e < D / 8; ++e)
          orow[e] = make_uint4(o_all[4 * e], o_all[4 * e + 1], o_all[4 * e + 2], o_all[4 * e + 3]);
        if (PLO && p.o_lo != nullptr) {
          uint4* lrow = reinterpret_cast<uint4*>(p.o_lo + off);
#pragma unroll
          for (int e = 0; e < D / 8; ++e)
            lrow[e] = make_uint4(lo_all[4 * e], lo_all[4 * e + 1], lo_all[4 * e + 2],
                                 lo_all[4 * e + 3]);
        }
        // natural-log LSE: m_used is in log2 units of the scaled score
        p.lse[static_cast<size_t>(it.bh) * p.T + q_row] = m_used * 0.69314718055994531f + logf(l);
      }
      tg += ng;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace cattn
