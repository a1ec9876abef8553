// Device primitives of the decode kernel, as inline PTX:
//   - cp.async 16-byte global -> shared copies (zero fill past the cache)
//     with commit / wait groups: each warp streams its own key chunks;
//   - ldmatrix (plain and transposed) and mma.sync m16n8k16 bf16 -> fp32:
//     the decode's products q k^T and p v have at most 8 query rows and are
//     bound by reading K and V, so the warp-level tensor-core instructions
//     (one warp, registers in and out) fit them better than tcgen05's
//     128-row tiles and TMEM;
//   - thread-block cluster rank, barrier and distributed-shared-memory
//     loads, through which the CTAs of one head merge their partial results
//     on chip.
// The CPU emulator (tests/emu) defines the same functions on the host with
// the instructions' documented semantics, so the kernel source runs
// unchanged under AddressSanitizer.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace cattn {

__device__ __forceinline__ uint32_t dec_smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The kernel's dynamic shared memory.
__device__ __forceinline__ uint8_t* dec_dynamic_smem() {
  extern __shared__ __align__(128) uint8_t dec_smem_base[];
  return dec_smem_base;
}

// 16 bytes from global `src` to shared `dst` (both 16-byte aligned),
// asynchronously; with valid == false nothing is read and dst is zeroed.
__device__ __forceinline__ void dec_cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dec_smem_addr(dst)),
               "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
// Programmatic dependent launch (as grid_dep_wait of the main kernels):
// wait for the grid launched before this one to complete and its writes to
// be visible; let the next grid be scheduled once every CTA of this one
// has executed dec_grid_dep_launch (or exited).
__device__ __forceinline__ void dec_grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void dec_grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void dec_cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// Until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void dec_cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Four 8x8 b16 matrices; lane 8m + i gives the address of row i of matrix
// m, and r[m] receives row lane/4, columns 2(lane%4) and 2(lane%4)+1.
__device__ __forceinline__ void dec_ldsm_x4(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(dec_smem_addr(row))
               : "memory");
}
// As dec_ldsm_x4 with each matrix transposed: r[m] receives rows 2(lane%4)
// and 2(lane%4)+1 of column lane/4.
__device__ __forceinline__ void dec_ldsm_x4_t(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(dec_smem_addr(row))
               : "memory");
}
// Two matrices (addresses from lanes 0-15).
__device__ __forceinline__ void dec_ldsm_x2(uint32_t (&r)[2], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(dec_smem_addr(row))
               : "memory");
}

// c += A B for a 16x16 bf16 A (row-major fragments a0..a3) and a 16x8 bf16
// B (column fragments b0, b1), fp32 accumulators c0..c3.
__device__ __forceinline__ void dec_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two floats as bf16 (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t dec_pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Every thread of every CTA of the cluster arrives, then waits for all;
// release/acquire order the shared-memory writes before it with the
// cluster's reads after it.  A hardware barrier (all CTAs of a cluster are
// resident together), reached by every thread unconditionally.
__device__ __forceinline__ void dec_cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n"
      "barrier.cluster.wait.acquire.aligned;\n" ::
          : "memory");
}

// The float at the same shared-memory offset as `local`, in the CTA of
// cluster rank `rank`.
__device__ __forceinline__ float dec_cluster_ld(const float* local, unsigned rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n"
               : "=r"(remote)
               : "r"(dec_smem_addr(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

}  // namespace cattn
