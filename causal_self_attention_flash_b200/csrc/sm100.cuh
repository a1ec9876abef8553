// Device-side building blocks for sm_100a: mbarriers with bounded waits,
// TMA tile copies, tcgen05 tensor-core MMAs accumulating in tensor memory
// (TMEM), TMEM loads/stores and the shared-memory matrix descriptors the
// MMAs read.  Everything is inline PTX written from the PTX ISA's
// definitions of these instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace cattn {

// ---------------------------------------------------------------------------
// Status word and hang guard
// ---------------------------------------------------------------------------

// Status words.  g_status is the library-global device status: 0 = OK,
// else the first error code any kernel recorded since it was last cleared;
// g_status_where names the wait that gave up (kernel id << 8 | barrier id).
// The library is one translation unit, which defines them here.  A call
// that has a caller-owned workspace (the backward) also records into the
// two words {code, where} at the start of that workspace, so that calls on
// different workspaces (and streams) keep separate records.
__device__ unsigned int g_status = 0;
__device__ unsigned int g_status_where = 0;

constexpr unsigned int kStatusTimeout = 4;  // == CATTN_ERR_TIMEOUT

// Record `code` (first error wins) in the global word and, if given, in a
// call's own words.
__device__ __forceinline__ void record_status(unsigned int* call, unsigned int code,
                                              unsigned int where) {
  if (atomicCAS(&g_status, 0u, code) == 0u) g_status_where = where;
  if (call != nullptr && atomicCAS(call, 0u, code) == 0u) call[1] = where;
}

constexpr unsigned int kStatusUnsupported = 2;  // == CATTN_ERR_UNSUPPORTED
constexpr int kMaxDynSmem = 232448;              // 227 KB opt-in limit per CTA

// Shared-memory layouts assume 1024-byte aligned tiles.  The host asks for
// `used + 1024` bytes when that fits, else exactly `used`; here the kernel
// finds the aligned start and checks it fits what it was given.  Returns
// nullptr (after recording CATTN_ERR_UNSUPPORTED) if not: the caller must
// then return before touching any barrier, copy or tensor memory.
__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw, uint32_t used,
                                                 unsigned int* call_status) {
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  if (pad + used > dyn) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0)
      record_status(call_status, kStatusUnsupported, 0u);
    return nullptr;
  }
  return raw + pad;
}

// ---------------------------------------------------------------------------
// Shared-memory addresses
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

// Programmatic dependent launch: wait until the grid this one was launched
// behind has completed and its memory writes are visible (returns at once
// for a launch without that dependency).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Make barrier initialisation visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA wait context: a time limit and a shared abort flag.  Once any
// thread of the CTA gives up, every later wait returns at once, so all
// warps run to the end of the kernel (where TMEM is freed and copies in
// flight are drained) instead of hanging.  With `call_slot`, the 8 bytes
// after the abort flag (shared memory) hold the address of the call's own
// status words (or null), read only when a wait gives up: the hot loops
// carry no extra register for it.
//
// The limit is counted in SM clock cycles (clock64, cheap to read) at 2.1
// cycles per ns: at or below the 1965 MHz maximum SM clock the real limit
// is at least the requested time.
struct WaitCtx {
  uint64_t timeout_ns;
  volatile int* abort;  // in shared memory
  unsigned int kernel_id;
  bool call_slot;        // the call's status address follows *abort
};

// The call's status address kept in the 8 bytes after the abort flag.
__device__ __forceinline__ unsigned int* call_status_of(const WaitCtx& w) {
  if (!w.call_slot) return nullptr;
  return *reinterpret_cast<unsigned int* const volatile*>(
      reinterpret_cast<const volatile char*>(w.abort) + 8);
}

__device__ __forceinline__ uint64_t cycles_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
  return t;
}

// What a wait that gives up does, out of line: one copy serves every wait
// site.  Inlined at each of the kernels' ~30 sites, this cold code measured
// 10 % slower on the backward (instruction-cache pressure in its hot loops).
__device__ __noinline__ void record_timeout_of(const WaitCtx& w, unsigned int where) {
  *w.abort = 1;
  record_status(call_status_of(w), kStatusTimeout, where);
}

// Single-thread bounded wait.  Returns false on timeout/abort.
__device__ __forceinline__ bool wait1(const WaitCtx& w, uint32_t bar, uint32_t parity,
                                      unsigned int bar_id) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = cycles_now();
  const uint64_t limit = w.timeout_ns * 21 / 10;
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (cycles_now() - t0 > limit) {
      record_timeout_of(w, (w.kernel_id << 8) | bar_id);
      return false;
    }
  }
}

// Warp-uniform bounded wait: every lane returns the same value, so the
// warp stays converged for the .sync.aligned tcgen05 instructions after it.
__device__ __forceinline__ bool wait_warp(const WaitCtx& w, uint32_t bar, uint32_t parity,
                                          unsigned int bar_id) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait1(w, bar, parity, bar_id);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  return ok;
}

// ---------------------------------------------------------------------------
// Proxy fences
// ---------------------------------------------------------------------------

// Generic-proxy shared-memory writes -> visible to the async proxy (the
// tensor core reading an operand, or a TMA store reading a staging tile).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}


// Hardware named barrier over nthreads threads (a multiple of 32).  Used
// only where every participating thread provably reaches it.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), 3-D tensor maps {x = d, y = t, z = b*H + h}
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 4-D tensor maps {x = d, y = t, z = h, w = b} over (B, H, T, D) tensors
// with any strides (the d stride is 1)
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on an mbarrier's transaction count.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int x, int y,
                                             int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Element-wise fp32 add of a shared tile into global memory.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, uint32_t src, int x,
                                                  int y, int z) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the bulk stores have finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Until at most one committed bulk group is still reading its source.
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Wait until the bulk stores have completed (writes performed).
__device__ __forceinline__ void bulk_wait0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}


// ---------------------------------------------------------------------------
// Tensor memory (TMEM) and tcgen05
// ---------------------------------------------------------------------------

// Allocate `ncols` (power of two, >= 32) TMEM columns; whole warp executes.
// The TMEM address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
               "r"(ncols)
               : "memory");
}

// Per-warpgroup register re-balancing (all four warps of a warpgroup run
// the same one).  The totals must stay within what the block was launched
// with: threads x registers per thread at launch.
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T-ish per the descriptors; one thread issues.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// A operand from TMEM, B from shared memory.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when all tcgen05 operations this thread has
// issued so far are complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread (lane l of the warp)
// receives row (lane base + l), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
      " [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32"
      " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
      " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::
                   "r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32"
      " [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// TMEM address of (lane, column): lane in bits [31:16], column in [15:0].
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// ---------------------------------------------------------------------------
// UMMA shared-memory matrix descriptor and instruction descriptor
// ---------------------------------------------------------------------------
//
// Shared-memory descriptor (64 bit):
//   [0,14)  start address >> 4        [16,30) leading-dimension byte offset >> 4
//   [32,46) stride-dimension byte offset >> 4
//   [46,48) version = 1 (sm_100)      [49,52) base offset = 0 (1024-B aligned atoms)
//   [52]    LBO mode = 0              [61,64) layout: 0 none, 2 = 128B swizzle,
//                                             4 = 64B swizzle, 6 = 32B swizzle
//
// Canonical layouts used here (16-byte units, bf16):
//   K-major, swizzle W bytes: 8-row groups of rows W bytes long; SBO = 8*W
//     bytes between 8-row groups; the K offset inside the swizzle row is
//     selected by advancing the start address (LBO unused).
//   MN-major, swizzle W bytes: each K row holds W bytes of consecutive M/N
//     elements; SBO = 8*W bytes between 8-row groups of K; LBO = bytes
//     between consecutive W-byte column blocks of M/N.

__host__ __device__ constexpr uint32_t swizzle_code(uint32_t row_bytes) {
  return row_bytes == 128 ? 2u : row_bytes == 64 ? 4u : row_bytes == 32 ? 6u : 0u;
}

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator.
//   [4,6) D format (1 = f32)  [7,10) A format (1 = bf16)  [10,13) B format
//   [15] A major (0 K, 1 MN)  [16] B major  [17,23) N >> 3  [24,29) M >> 4
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t a_mn_major,
                                                  uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Shared-memory swizzle, the pattern TMA writes and the MMA expects:
// 16-byte chunk index (address bits [4,7)) XOR row-group bits [7,10),
// masked to the swizzle width.  Tiles are 1024-byte aligned.
// ---------------------------------------------------------------------------
template <uint32_t kRowBytes>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  constexpr uint32_t mask = kRowBytes / 16 - 1;  // 7, 3 or 1
  return off ^ (((off >> 7) & mask) << 4);
}

// ---------------------------------------------------------------------------
// Small numeric helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max of three (sm_100 three-input form)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Packed pairs of fp32 in one 64-bit register: sm_100 executes add, mul
// and fma on both halves with one instruction.
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a packed pair on the FMA pipes (no ex2 unit): 2^x = 2^j * p(f)
// with j = round(x) and f = x - j in [-1/2, 1/2]; p is the degree-4 minimax
// fit of 2^f for relative error (Remez exchange; gen_exp2_poly.py prints
// these coefficients), max relative error 2.7e-6.  j is formed by adding
// 1.5 * 2^23, which leaves round(x) in the low mantissa bits; those bits
// shifted into the exponent field scale p by 2^j.  Inputs are clamped to
// x >= -126 (results below 2^-126 come out as 2^-126 instead of 0: callers
// that need exact zeros, e.g. masked scores, must not use this).
constexpr float kExp2C0 = 0.9999992847442627f;
constexpr float kExp2C1 = 0.6931217908859253f;
constexpr float kExp2C2 = 0.240247443318367f;
constexpr float kExp2C3 = 0.05591785907745361f;
constexpr float kExp2C4 = 0.009570102207362652f;

__device__ __forceinline__ uint64_t exp2_poly2(float x0, float x1) {
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  const uint64_t magic = f2(12582912.f, 12582912.f);
  const uint64_t x = f2(x0, x1);
  const uint64_t t = add2(x, magic);
  const uint64_t f = sub2(x, sub2(t, magic));
  uint64_t p = fma2(f2(kExp2C4, kExp2C4), f, f2(kExp2C3, kExp2C3));
  p = fma2(p, f, f2(kExp2C2, kExp2C2));
  p = fma2(p, f, f2(kExp2C1, kExp2C1));
  p = fma2(p, f, f2(kExp2C0, kExp2C0));
  float t0, t1, p0, p1;
  f2_split(t, t0, t1);
  f2_split(p, p0, p1);
  return f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
            __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// hi/lo split of a packed pair without conversion instructions: hi is the
// top half of each fp32 word (bf16 rounded toward zero), lo = x - hi, which
// is exact in fp32, likewise truncated to bf16.  |x - hi - lo| < 2^-7 |lo|
// < 2^-14 |x|.  Each bf16x2 word is assembled with one byte permute.
__device__ __forceinline__ uint32_t top_halves(uint32_t a, uint32_t b) {
  uint32_t d;  // low half = a's top 16 bits, high half = b's top 16 bits
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void split_bf16x2_p(uint64_t x, uint32_t& hi, uint32_t& lo) {
  float x0, x1;
  f2_split(x, x0, x1);
  const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
  hi = top_halves(b0, b1);
  const uint64_t h = f2(__uint_as_float(b0 & 0xffff0000u), __uint_as_float(b1 & 0xffff0000u));
  float r0, r1;
  f2_split(sub2(x, h), r0, r1);
  lo = top_halves(__float_as_uint(r0), __float_as_uint(r1));
}

// bf16 hi/lo split of two floats: hi = bf16(x) (round to nearest even) and
// lo = bf16(x - hi), packed as bf16x2 (first element in the low half).
// hi + lo carries x to about 16 significant bits.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(x0, x1);
  const float h0 = __uint_as_float(hi << 16);
  const float h1 = __uint_as_float(hi & 0xffff0000u);
  lo = pack_bf16(x0 - h0, x1 - h1);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void ld_shared_v4f(uint32_t addr, float& a, float& b, float& c,
                                              float& d) {
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(a), "=f"(b), "=f"(c), "=f"(d)
               : "r"(addr));
}

}  // namespace cattn
