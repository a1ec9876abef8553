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
//   bwd_pre_kernel   Delta = rowsum(dO * O) with 16-byte loads, LSE * log2(e)
//                    into a tile-padded vector, and zeroing of the fp32 dQ
//                    accumulator.
//   bwd_kernel       one CTA per (head, 128-key tile); loops over the query
//                    tiles at or after it (causal), accumulating dK and dV in
//                    TMEM and adding each dQ tile into the fp32 accumulator
//                    with a TMA reduce-add.
//   dq_convert_kernel dQ = bf16(scale * accumulator).
#pragma once

#include "sm100.cuh"

namespace cattn {

// ---------------------------------------------------------------------------
// Preprocess
// ---------------------------------------------------------------------------

struct PreParams {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;      // may be null (no lse2 output)
  float* delta;          // (BH, row_stride)
  float* lse2;           // (BH, row_stride) or null
  float4* zero;          // buffer to clear, or null
  size_t zero_n4;        // its length in float4
  int T;
  int row_stride;        // T (public preprocess) or T rounded up to 128
  long long n_rows;      // BH * row_stride
};

// Threads per row: each handles 8 bf16 (16 bytes) of O and of dO.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const PreParams p) {
  constexpr int TPR = D / 8;
  constexpr int RPW = 32 / TPR;  // rows per warp per step
  const int lane = threadIdx.x & 31;
  const int sub = lane % TPR;
  const long long warp_global = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  constexpr float kLog2e = 1.4426950408889634f;

  for (long long base = warp_global * RPW; base < p.n_rows; base += n_warps * RPW) {
    const long long pr = base + lane / TPR;
    const bool in_range = pr < p.n_rows;
    long long bh = 0;
    int t = 0;
    if (in_range) {
      bh = pr / p.row_stride;
      t = static_cast<int>(pr - bh * p.row_stride);
    }
    const bool valid = in_range && t < p.T;
    float acc = 0.f;
    if (valid) {
      const size_t off = (static_cast<size_t>(bh) * p.T + t) * D + sub * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(p.o + off);
      const uint4 b = *reinterpret_cast<const uint4*>(p.dout + off);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(a2[e]);
        const float2 fb = __bfloat1622float2(b2[e]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (in_range && sub == 0) {
      p.delta[pr] = acc;  // 0 on padding rows
      if (p.lse2 != nullptr)
        p.lse2[pr] = valid ? p.lse[static_cast<size_t>(bh) * p.T + t] * kLog2e : INFINITY;
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

__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ acc,
                                                         uint4* __restrict__ dq, size_t n8,
                                                         float scale) {
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

// ---------------------------------------------------------------------------
// Main backward kernel
// ---------------------------------------------------------------------------

struct BwdParams {
  const float* lse2;   // (BH, T_pad) LSE * log2(e); +inf on padding rows
  const float* delta;  // (BH, T_pad); 0 on padding rows
  int T;
  int T_pad;
  int n_tiles;
  float scale;
  float scale_log2;
  uint64_t timeout_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int CB = D < 64 ? D : 64;       // bf16 columns per swizzle block
  static constexpr int RB = CB * 2;
  static constexpr int NCB = D / CB;
  static constexpr int BLOCK_BYTES = 128 * RB;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int ST = D <= 64 ? 2 : 1;        // Q/dO ring depth
  static constexpr uint32_t SW = swizzle_code(RB);
  // fp32 dQ staging: blocks of [128 rows][CBQ floats], swizzled by row bytes
  static constexpr int CBQ = D < 32 ? D : 32;
  static constexpr int RBQ = CBQ * 4;
  static constexpr int QCHUNK = D < 64 ? D : 64;    // dQ columns staged at a time
  static constexpr int QCHUNK_BYTES = 128 * QCHUNK * 4;
  // shared memory map
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + TILE_BYTES;
  static constexpr int OFF_DO = OFF_Q + ST * TILE_BYTES;
  static constexpr int OFF_PT = OFF_DO + ST * TILE_BYTES;   // [2][128 keys][64 queries] bf16
  static constexpr int OFF_DST = OFF_PT + 32768;            // same layout, dS^T
  static constexpr int OFF_DQ = OFF_DST + 32768;
  static constexpr int OFF_LSE = OFF_DQ + QCHUNK_BYTES;     // [ST][128] fp32
  static constexpr int OFF_DELTA = OFF_LSE + ST * 512;
  static constexpr int OFF_BAR = OFF_DELTA + ST * 512;
  static constexpr int NUM_BARS = 24;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  // TMEM columns
  static constexpr bool ALIAS_DQ = 256 + 3 * D > 512;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t COL_DQ = ALIAS_DQ ? COL_DP : 256 + 2 * D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 320;
};

enum : int {
  BB_KV = 0, BB_QFULL = 1, BB_DOFULL = 3, BB_QDOEMPTY = 5, BB_SFULL = 7, BB_STFREE = 8,
  BB_DPFULL = 9, BB_DPTFREE = 10, BB_PTFULL = 11, BB_PTFREE = 12, BB_DSFULL = 13,
  BB_DSFREE = 14, BB_DQFULL = 15, BB_DQEMPTY = 16, BB_DRAIN = 17
};

template <int D>
__global__ void __launch_bounds__(320, 1)
bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
           const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
           const __grid_constant__ CUtensorMap tmDQacc, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  const uint32_t sPt = sbase + C::OFF_PT, sdSt = sbase + C::OFF_DST, sDQ = sbase + C::OFF_DQ;
  auto bar = [&](int i) { return sbase + C::OFF_BAR + 8u * i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int kt = blockIdx.y;            // key tile; tile 0 has the most work
  const int n_iter = p.n_tiles - kt;    // query tiles kt .. n_tiles-1

  WaitCtx w{p.timeout_ns, abort_flag, 2u};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(BB_KV), 1);
    for (int s = 0; s < C::ST; ++s) {
      mbar_init(bar(BB_QFULL + s), 1);
      mbar_init(bar(BB_DOFULL + s), 1);
      mbar_init(bar(BB_QDOEMPTY + s), 1);
    }
    mbar_init(bar(BB_SFULL), 1);
    mbar_init(bar(BB_STFREE), 128);
    mbar_init(bar(BB_DPFULL), 1);
    mbar_init(bar(BB_DPTFREE), 128);
    mbar_init(bar(BB_PTFULL), 128);
    mbar_init(bar(BB_PTFREE), 1);
    mbar_init(bar(BB_DSFULL), 128);
    mbar_init(bar(BB_DSFREE), 1);
    mbar_init(bar(BB_DQFULL), 1);
    mbar_init(bar(BB_DQEMPTY), 128);
    mbar_init(bar(BB_DRAIN), 1);
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(sbase + C::OFF_MISC, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = misc[0];

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(bar(BB_KV), 2 * C::TILE_BYTES);
      for (int b = 0; b < C::NCB; ++b) {
        tma_load_3d(sK + b * C::BLOCK_BYTES, &tmK, bar(BB_KV), b * C::CB, kt * 128, bh);
        tma_load_3d(sV + b * C::BLOCK_BYTES, &tmV, bar(BB_KV), b * C::CB, kt * 128, bh);
      }
      int n_issued = 0;
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % C::ST;
        const int qi = kt + i;
        if (i >= C::ST) wait1(w, bar(BB_QDOEMPTY + st), ((i / C::ST) - 1) & 1, 1);
        if (*abort_flag) break;
        n_issued = i + 1;
        const uint32_t sQ = sbase + C::OFF_Q + st * C::TILE_BYTES;
        const uint32_t sDO = sbase + C::OFF_DO + st * C::TILE_BYTES;
        const size_t vec = static_cast<size_t>(bh) * p.T_pad + static_cast<size_t>(qi) * 128;
        mbar_arrive_expect_tx(bar(BB_QFULL + st), C::TILE_BYTES + 512);
        for (int b = 0; b < C::NCB; ++b)
          tma_load_3d(sQ + b * C::BLOCK_BYTES, &tmQ, bar(BB_QFULL + st), b * C::CB, qi * 128, bh);
        bulk_load(sbase + C::OFF_LSE + st * 512, p.lse2 + vec, 512, bar(BB_QFULL + st));
        mbar_arrive_expect_tx(bar(BB_DOFULL + st), C::TILE_BYTES + 512);
        for (int b = 0; b < C::NCB; ++b)
          tma_load_3d(sDO + b * C::BLOCK_BYTES, &tmDO, bar(BB_DOFULL + st), b * C::CB, qi * 128, bh);
        bulk_load(sbase + C::OFF_DELTA + st * 512, p.delta + vec, 512, bar(BB_DOFULL + st));
      }
      if (*abort_flag) {
        int zero = 0;
        WaitCtx wd{p.timeout_ns, &zero, 2u};
        wait1(wd, bar(BB_KV), 0, 20);
        for (int i = (n_issued > C::ST ? n_issued - C::ST : 0); i < n_issued; ++i) {
          const int st = i % C::ST;
          wait1(wd, bar(BB_QFULL + st), (i / C::ST) & 1, 21);
          wait1(wd, bar(BB_DOFULL + st), (i / C::ST) & 1, 22);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idKD = idesc_bf16(128, D, 0, 1);    // dV, dK: A K-major, B MN-major
      constexpr uint32_t idQ = idesc_bf16(128, D, 1, 1);     // dQ: A (dS) MN-major
      wait1(w, bar(BB_KV), 0, 2);
      for (int i = 0; i < n_iter; ++i) {
        const int st = i % C::ST;
        const uint32_t ph = (i / C::ST) & 1;
        const uint32_t sQ = sbase + C::OFF_Q + st * C::TILE_BYTES;
        const uint32_t sDO = sbase + C::OFF_DO + st * C::TILE_BYTES;
        // S^T = K Q^T  (M = keys, N = queries, K = D)
        wait1(w, bar(BB_QFULL + st), ph, 3);
        if (i >= 1) wait1(w, bar(BB_STFREE), (i - 1) & 1, 4);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int blk = (kk * 16) / C::CB;
          const int off = ((kk * 16) % C::CB) * 2;
          mma_ss(tbase + C::COL_S,
                 smem_desc(sK + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW),
                 smem_desc(sQ + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW), idSS,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BB_SFULL));
        // dP^T = V dO^T
        wait1(w, bar(BB_DOFULL + st), ph, 5);
        if (i >= 1) wait1(w, bar(BB_DPTFREE), (i - 1) & 1, 6);
        if (C::ALIAS_DQ && i >= 1) wait1(w, bar(BB_DQEMPTY), (i - 1) & 1, 7);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int blk = (kk * 16) / C::CB;
          const int off = ((kk * 16) % C::CB) * 2;
          mma_ss(tbase + C::COL_DP,
                 smem_desc(sV + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW),
                 smem_desc(sDO + blk * C::BLOCK_BYTES + off, 16, 8 * C::RB, C::SW), idSS,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BB_DPFULL));
        // dV += P^T dO  (M = keys, K = queries, N = D)
        wait1(w, bar(BB_PTFULL), i & 1, 8);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_ss(tbase + C::COL_DV, smem_desc(sPt + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, 2),
                 smem_desc(sDO + kk * 16 * C::RB, C::BLOCK_BYTES, 8 * C::RB, C::SW), idKD,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(BB_PTFREE));
        // dK += dS^T Q ; dQ = dS K
        wait1(w, bar(BB_DSFULL), i & 1, 9);
        if (!C::ALIAS_DQ && i >= 1) wait1(w, bar(BB_DQEMPTY), (i - 1) & 1, 10);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_ss(tbase + C::COL_DK,
                 smem_desc(sdSt + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024, 2),
                 smem_desc(sQ + kk * 16 * C::RB, C::BLOCK_BYTES, 8 * C::RB, C::SW), idKD,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 keys, 16 per MMA
          mma_ss(tbase + C::COL_DQ, smem_desc(sdSt + kk * 2048, 16384, 1024, 2),
                 smem_desc(sK + kk * 16 * C::RB, C::BLOCK_BYTES, 8 * C::RB, C::SW), idQ,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BB_DQFULL));
        mma_commit(bar(BB_DSFREE));
        mma_commit(bar(BB_QDOEMPTY + st));
      }
      mma_commit(bar(BB_DRAIN));
      int zero = 0;
      WaitCtx wd{p.timeout_ns, &zero, 2u};
      wait1(wd, bar(BB_DRAIN), 0, 11);
    }
  } else if (warp < 4) {
    // ------------------------------------------------- P and dS (row = key)
    const int r = threadIdx.x;                   // key row in tile == TMEM lane
    const uint32_t lane_base = (warp * 32) << 16;
    const float sl2 = p.scale_log2;
    float pr[128];
    for (int i = 0; i < n_iter; ++i) {
      const int st = i % C::ST;
      const uint32_t ph = (i / C::ST) & 1;
      wait_warp(w, bar(BB_SFULL), i & 1, 12);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tbase + lane_base + C::COL_S + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) pr[c * 32 + e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
      mbar_arrive(bar(BB_STFREE));
      wait_warp(w, bar(BB_QFULL + st), ph, 13);  // makes the LSE vector visible
      const uint32_t sL = sbase + C::OFF_LSE + st * 512;
#pragma unroll
      for (int c = 0; c < 128; c += 4) {
        float l0, l1, l2, l3;
        ld_shared_v4f(sL + c * 4, l0, l1, l2, l3);
        pr[c] = ex2(fmaf(pr[c], sl2, -l0));
        pr[c + 1] = ex2(fmaf(pr[c + 1], sl2, -l1));
        pr[c + 2] = ex2(fmaf(pr[c + 2], sl2, -l2));
        pr[c + 3] = ex2(fmaf(pr[c + 3], sl2, -l3));
      }
      if (i == 0) {  // diagonal tile: query c sees key r only if r <= c
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c < r) pr[c] = 0.f;
      }
      if (i >= 1) wait_warp(w, bar(BB_PTFREE), (i - 1) & 1, 14);
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int c0 = ch * 8;
        st_shared_v4(sPt + (c0 >> 6) * 16384 + swz<128>(r * 128 + ((c0 & 63) >> 3) * 16),
                     pack_bf16(pr[c0], pr[c0 + 1]), pack_bf16(pr[c0 + 2], pr[c0 + 3]),
                     pack_bf16(pr[c0 + 4], pr[c0 + 5]), pack_bf16(pr[c0 + 6], pr[c0 + 7]));
      }
      fence_async_smem();
      mbar_arrive(bar(BB_PTFULL));

      wait_warp(w, bar(BB_DPFULL), i & 1, 15);
      tc_fence_after();
      wait_warp(w, bar(BB_DOFULL + st), ph, 16);  // makes the Delta vector visible
      if (i >= 1) wait_warp(w, bar(BB_DSFREE), (i - 1) & 1, 17);
      const uint32_t sD = sbase + C::OFF_DELTA + st * 512;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        tmem_ld32(tbase + lane_base + C::COL_DP + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int c0 = c * 32 + ch * 8;
          float d[8];
          ld_shared_v4f(sD + c0 * 4, d[0], d[1], d[2], d[3]);
          ld_shared_v4f(sD + c0 * 4 + 16, d[4], d[5], d[6], d[7]);
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = pr[c0 + 2 * e] * (__uint_as_float(v[ch * 8 + 2 * e]) - d[2 * e]);
            const float a1 =
                pr[c0 + 2 * e + 1] * (__uint_as_float(v[ch * 8 + 2 * e + 1]) - d[2 * e + 1]);
            pk[e] = pack_bf16(a0, a1);
          }
          st_shared_v4(sdSt + (c0 >> 6) * 16384 + swz<128>(r * 128 + ((c0 & 63) >> 3) * 16),
                       pk[0], pk[1], pk[2], pk[3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(BB_DPTFREE));
      fence_async_smem();
      mbar_arrive(bar(BB_DSFULL));
    }

    // ------------------------------------------------ dK, dV epilogue
    wait_warp(w, bar(BB_DQFULL), (n_iter - 1) & 1, 18);  // every MMA has completed
    tc_fence_after();
#pragma unroll
    for (int which = 0; which < 2; ++which) {  // 0: dV -> sPt, 1: dK -> sdSt
      const uint32_t col = tbase + lane_base + (which ? C::COL_DK : C::COL_DV);
      const uint32_t dst = which ? sdSt : sPt;
      const float mul = which ? p.scale : 1.f;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {
        uint32_t v[16];
        tmem_ld16(col + c * 16, v);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          pk[e] = pack_bf16(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
        const int d0 = c * 16;
        const int blk = d0 / C::CB;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int dd = (d0 % C::CB) + h * 8;
          st_shared_v4(dst + blk * C::BLOCK_BYTES + swz<C::RB>(r * C::RB + dd * 2), pk[4 * h],
                       pk[4 * h + 1], pk[4 * h + 2], pk[4 * h + 3]);
        }
      }
    }
    tc_fence_before();
    fence_async_smem();
    named_bar_sync(1, 128);
    if (threadIdx.x == 0 && !*abort_flag) {
      for (int b = 0; b < C::NCB; ++b) {
        tma_store_3d(&tmDV, sPt + b * C::BLOCK_BYTES, b * C::CB, kt * 128, bh);
        tma_store_3d(&tmDK, sdSt + b * C::BLOCK_BYTES, b * C::CB, kt * 128, bh);
      }
      bulk_commit();
      bulk_wait0();
    }
  } else {
    // ------------------------------------------------ dQ drain (row = query)
    const int r = threadIdx.x - 128;
    const uint32_t lane_base = ((warp - 4) * 32) << 16;
    const bool leader = (r == 0);
    for (int i = 0; i < n_iter; ++i) {
      const int qi = kt + i;
      wait_warp(w, bar(BB_DQFULL), i & 1, 19);
      tc_fence_after();
      float acc[D];
      if constexpr (D >= 32) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tbase + lane_base + C::COL_DQ + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[c * 32 + e] = __uint_as_float(v[e]);
        }
      } else {
        uint32_t v[16];
        tmem_ld16(tbase + lane_base + C::COL_DQ, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
      mbar_arrive(bar(BB_DQEMPTY));
#pragma unroll
      for (int ch = 0; ch < D / C::QCHUNK; ++ch) {
        // stage [128][QCHUNK] fp32 as QCHUNK/CBQ swizzled blocks
#pragma unroll
        for (int e = 0; e < C::QCHUNK; e += 4) {
          const int blk = e / C::CBQ;
          const int within = (e % C::CBQ) * 4;
          const float* a = &acc[ch * C::QCHUNK + e];
          st_shared_v4(sDQ + blk * 128 * C::RBQ + swz<C::RBQ>(r * C::RBQ + within),
                       __float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                       __float_as_uint(a[3]));
        }
        fence_async_smem();
        named_bar_sync(2, 128);
        if (leader && !*abort_flag) {
#pragma unroll
          for (int blk = 0; blk < C::QCHUNK / C::CBQ; ++blk)
            tma_reduce_add_3d(&tmDQacc, sDQ + blk * 128 * C::RBQ,
                              ch * C::QCHUNK + blk * C::CBQ, qi * 128, bh);
          bulk_commit();
          bulk_wait_read0();
        }
        named_bar_sync(2, 128);
      }
    }
    if (leader) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace cattn
