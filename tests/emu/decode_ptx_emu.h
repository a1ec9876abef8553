// Host definitions of the decode kernel's device primitives (the functions
// of decode_ptx.cuh), for the CPU emulator.  Each follows the documented
// semantics of its PTX instruction, written independently of the kernel:
//   cp.async 16 bytes (src-size 0: zero fill, nothing read), completed at
//     once (commit/wait are then no-ops);
//   ldmatrix .m8n8 .x2/.x4 [.trans] .b16: lane 8m + i gives row i of matrix
//     m; without .trans lane l receives elements (l/4, 2(l%4)) and
//     (l/4, 2(l%4)+1) of each matrix, with .trans elements (2(l%4), l/4) and
//     (2(l%4)+1, l/4), the first in the low half;
//   mma.sync .m16n8k16 .row.col bf16 -> f32 with g = l/4, t = l%4:
//     A: a0 (g, 2t..2t+1), a1 (g+8, 2t..), a2 (g, 2t+8..), a3 (g+8, 2t+8..);
//     B: b0 (k 2t..2t+1, n g), b1 (k 2t+8.., n g);
//     C/D: c0 (g, 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1);
//     products summed in double, then added to the fp32 accumulator;
//   barrier.cluster: a barrier over all threads of the cluster's CTAs;
//   mapa + ld.shared::cluster: the same offset in another CTA's shared
//     memory.
// Every shared-memory address is checked to lie in the CTA's own dynamic
// shared memory with the instruction's alignment (a logic_error otherwise).
#pragma once

#include <cstdint>
#include <cstring>
#include <stdexcept>

#include "simt_emu.h"
#include "cuda_bf16.h"

namespace cattn {

inline uint8_t* dec_dynamic_smem() { return emu::t_cta->dsmem; }

inline void dec_cp_async16(void* dst, const void* src, bool valid) {
  emu::check_smem(dst, 16, 16);
  if (valid) {
    if (reinterpret_cast<uintptr_t>(src) % 16 != 0)
      throw std::logic_error("cp.async from a misaligned global address");
    std::memcpy(dst, src, 16);
  } else {
    std::memset(dst, 0, 16);
  }
}
inline void dec_cp_async_commit() {}
template <int N>
inline void dec_cp_async_wait() {}

namespace emu_detail {
inline uint16_t ld16(const uint8_t* p) {
  uint16_t v;
  std::memcpy(&v, p, 2);
  return v;
}

// nmat matrices; lanes 0 .. 8 nmat - 1 give row addresses
inline void ldsm(uint32_t* r, int nmat, bool trans, const void* row) {
  const unsigned lane = threadIdx.x % 32, g = lane / 4, t = lane % 4;
  const uint64_t mine = reinterpret_cast<uintptr_t>(row);
  const uint64_t* all = emu::warp_exchange(&mine, 1);
  auto addr = [&](unsigned l) {
    const uint8_t* p = reinterpret_cast<const uint8_t*>(static_cast<uintptr_t>(all[l * emu::kWords]));
    emu::check_smem(p, 16, 16);
    return p;
  };
  for (int m = 0; m < nmat; ++m) {
    if (!trans) {
      std::memcpy(&r[m], addr(8 * m + g) + 4 * t, 4);
    } else {
      const uint32_t lo = ld16(addr(8 * m + 2 * t) + 2 * g);
      const uint32_t hi = ld16(addr(8 * m + 2 * t + 1) + 2 * g);
      r[m] = lo | (hi << 16);
    }
  }
}

inline double bf(uint32_t w, int half) {
  __nv_bfloat16 h{static_cast<uint16_t>(half ? w >> 16 : w & 0xffffu)};
  return __bfloat162float(h);
}
}  // namespace emu_detail

inline void dec_ldsm_x4(uint32_t (&r)[4], const void* row) {
  emu_detail::ldsm(r, 4, false, row);
}
inline void dec_ldsm_x4_t(uint32_t (&r)[4], const void* row) {
  emu_detail::ldsm(r, 4, true, row);
}
inline void dec_ldsm_x2(uint32_t (&r)[2], const void* row) {
  emu_detail::ldsm(r, 2, false, row);
}

inline void dec_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                    uint32_t b0, uint32_t b1) {
  using emu_detail::bf;
  const uint64_t mine[6] = {a0, a1, a2, a3, b0, b1};
  const uint64_t* all = emu::warp_exchange(mine, 6);
  double A[16][16], Bm[16][8];
  for (unsigned l = 0; l < 32; ++l) {
    const unsigned g = l / 4, t = l % 4;
    const uint64_t* f = all + l * emu::kWords;
    for (int e = 0; e < 2; ++e) {
      A[g][2 * t + e] = bf(static_cast<uint32_t>(f[0]), e);
      A[g + 8][2 * t + e] = bf(static_cast<uint32_t>(f[1]), e);
      A[g][2 * t + 8 + e] = bf(static_cast<uint32_t>(f[2]), e);
      A[g + 8][2 * t + 8 + e] = bf(static_cast<uint32_t>(f[3]), e);
      Bm[2 * t + e][g] = bf(static_cast<uint32_t>(f[4]), e);
      Bm[2 * t + 8 + e][g] = bf(static_cast<uint32_t>(f[5]), e);
    }
  }
  const unsigned lane = threadIdx.x % 32, g = lane / 4, t = lane % 4;
  const unsigned rows[4] = {g, g, g + 8, g + 8}, cols[4] = {2 * t, 2 * t + 1, 2 * t, 2 * t + 1};
  for (int i = 0; i < 4; ++i) {
    double acc = 0.0;
    for (int k = 0; k < 16; ++k) acc += A[rows[i]][k] * Bm[k][cols[i]];
    c[i] = static_cast<float>(static_cast<double>(c[i]) + acc);
  }
}

inline uint32_t dec_pack_bf16(float lo, float hi) {
  return static_cast<uint32_t>(__float2bfloat16_rn(lo).bits) |
         (static_cast<uint32_t>(__float2bfloat16_rn(hi).bits) << 16);
}

inline void dec_cluster_sync() { emu::t_cta->cluster->bar->arrive_and_wait(); }

// One grid at a time: nothing to wait for, nothing to release.
inline void dec_grid_dep_wait() {}
inline void dec_grid_dep_launch() {}

inline float dec_cluster_ld(const float* local, unsigned rank) {
  emu::check_smem(local, 4, 4);
  const emu::Cta* c = emu::t_cta;
  if (rank >= c->cluster->ctas.size()) throw std::logic_error("cluster rank out of range");
  const size_t off = reinterpret_cast<const uint8_t*>(local) - c->dsmem;
  float v;
  std::memcpy(&v, c->cluster->ctas[rank]->dsmem + off, 4);
  return v;
}

}  // namespace cattn
