// C ABI of libcattn: argument checks, TMA tensor maps, launches.
// The operations are declared and documented in include/cattn.h.

#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <array>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "cattn.h"
#include "bwd.cuh"
#include "decode.cuh"
#include "fwd.cuh"

// Scratch of attn_bwd_noalloc: one fixed array per device, owned by the
// library for the process's lifetime.  Host code must not use this name as
// a device address (on the host it is only a stand-in for the symbol); the
// address is looked up with cudaGetSymbolAddress per device.
static __device__ __align__(256) unsigned char cattn_noalloc_scratch[CATTN_NOALLOC_SCRATCH_BYTES];

namespace cattn {
namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
uint64_t g_timeout_ns = kDefaultTimeoutNs;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
thread_local int g_last_cuda_error = 0;  // cudaError_t / CUresult of the last failure

cattn_status cuda_fail(int code) {
  g_last_cuda_error = code;
  return CATTN_ERR_CUDA;
}
int g_dev_ok[kMaxDevices];           // 0 unknown, 1 sm_100, -1 other
uint64_t g_attr_done[kMaxDevices][2];  // bit per kernel instance (128)
int g_sm_count[kMaxDevices];         // multiprocessors (persistent grids)

cattn_status init_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return CATTN_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    return cuda_fail(cudaGetLastError());
  }
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return CATTN_OK;
}

thread_local int g_bound_device = -1;  // device whose primary context this thread holds

cattn_status check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail(cudaGetLastError());
  // A host thread that has made no runtime call yet (an autograd worker, a
  // fresh std::thread) has no current context, and the driver's tensor-map
  // encoder needs one: bind the device's primary context once per thread.
  if (g_bound_device != dev) {
    if (cudaSetDevice(dev) != cudaSuccess) return cuda_fail(cudaGetLastError());
    g_bound_device = dev;
  }
  if (dev < 0 || dev >= kMaxDevices) return CATTN_ERR_UNSUPPORTED;
  if (g_dev_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      return cuda_fail(cudaGetLastError());
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return cuda_fail(cudaGetLastError());
    g_sm_count[dev] = sms > 0 ? sms : 1;
    g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  if (g_dev_ok[dev] != 1) return CATTN_ERR_UNSUPPORTED;
  *dev_out = dev;
  return init_encode();
}

// Set the dynamic shared-memory limit of a kernel once per device.  A
// kernel that re-balances registers between its warpgroups (setmaxnreg)
// assumes it is launched with `launch_regs` registers per thread: with
// fewer, its increase would wait forever, so a build where the compiler
// chose another count is refused (CATTN_ERR_UNSUPPORTED) instead of run.
template <typename K>
cattn_status ensure_smem(int dev, unsigned bit, K kernel, int bytes, int launch_regs = 0) {
  if (g_attr_done[dev][bit >> 6] & (1ull << (bit & 63))) return CATTN_OK;
  if (launch_regs > 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return cuda_fail(cudaGetLastError());
    if (fa.numRegs != launch_regs) return CATTN_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    return cuda_fail(cudaGetLastError());
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_attr_done[dev][bit >> 6] |= 1ull << (bit & 63);
  return CATTN_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Pass codes for items of the given costs (numbered longest first) on G
// CTAs, planned greedily pass by pass (sched.cuh): each pass takes the
// direction and rotation that leave the lowest maximum CTA load, then the
// lowest sum of squared loads.  More than kMaxPassCodes passes: none
// (every pass alternates).
void plan_passes(const std::vector<int>& cost, int G, PassCodes* pc) {
  pc->n = 0;
  for (uint32_t& w : pc->code2) w = 0u;
  const long long n = static_cast<long long>(cost.size());
  if (G < 2 || n == 0) return;
  const long long passes = (n + G - 1) / G;
  if (passes > kMaxPassCodes) return;
  std::vector<long long> load(G, 0), trial(G);
  for (int k = 0; k < passes; ++k) {
    const long long first = static_cast<long long>(k) * G;
    const int m = static_cast<int>(n - first < G ? n - first : G);
    long long best_mx = -1, best_sq = 0;
    int best = 0;
    for (int d = 0; d < 2; ++d)
      for (int r = 0; r < G; ++r) {
        trial = load;
        for (int j = 0; j < m; ++j) {
          int b = (d ? r - j : r + j) % G;
          if (b < 0) b += G;
          trial[b] += cost[first + j];
        }
        long long mx = 0, sq = 0;
        for (long long x : trial) {
          mx = x > mx ? x : mx;
          sq += x * x;
        }
        if (best_mx < 0 || mx < best_mx || (mx == best_mx && sq < best_sq)) {
          best_mx = mx;
          best_sq = sq;
          best = (d << 15) | r;
        }
      }
    for (int j = 0; j < m; ++j) {
      const int r = best & 0x7fff;
      int b = ((best >> 15) ? r - j : r + j) % G;
      if (b < 0) b += G;
      load[b] += cost[first + j];
    }
    pc->code2[k >> 1] = (pc->code2[k >> 1] & (0xffffu << (16 * (1 - (k & 1))))) |
                        (static_cast<uint32_t>(best) << (16 * (k & 1)));
  }
  pc->n = static_cast<int>(passes);
}

// The pass codes of a persistent launch, planned once per (kernel kind,
// B*H, tiles, grid size): kind 0 deals the forward's items (query-tile
// pairs, an item's load its two groups' key tiles).  The backward (kind 1)
// keeps alternating passes: every variant of it that looked its items up
// through pass codes (from the parameters or from shared memory) measured
// slower (GPT-2 layer backward call 180-187 against 170 us), even with all
// passes alternating.
PassCodes pass_plan(int kind, int BH, int n_tiles, int G) {
  static std::map<std::array<int, 4>, PassCodes> cache;
  const std::array<int, 4> key{kind, BH, n_tiles, G};
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  PassCodes pc{};
  const long long items = kind == 0 ? static_cast<long long>(BH) * ((n_tiles + 1) / 2)
                                    : static_cast<long long>(BH) * n_tiles;
  if (kind != 0 || G < 2 || (items + G - 1) / G > kMaxPassCodes) {  // every pass alternates
    cache.emplace(key, pc);
    return pc;
  }
  const int n_pairs = (n_tiles + 1) / 2;
  std::vector<int> cost(static_cast<size_t>(BH) * n_pairs);
  for (size_t u = 0; u < cost.size(); ++u) {
    const int c = n_pairs - 1 - static_cast<int>(u / BH);
    const int nlo = 2 * c + 1, nhi = 2 * c + 1 < n_tiles ? 2 * c + 2 : 0;
    cost[u] = nlo + nhi;
  }
  plan_passes(cost, G, &pc);
  cache.emplace(key, pc);
  return pc;
}

// Launch `kernel` on stream s; with `dependent`, behind the previous kernel
// as a programmatic dependent: its CTAs may be scheduled while that kernel
// drains.  Every kernel launched so starts with grid_dep_wait, before its
// first access to global memory, so whatever kernel precedes it on the
// stream has completed and its writes are visible.  (55 against 60 us for
// the 64x6x256x64 backward, 172 against 173 us on the GPT-2 layer; with
// dropout, 206 against 212 us for the GPT-2 layer's backward and 59
// against 67 us for the 64x6x256x64 one.)
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(bool dependent, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                             size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool d_supported(int D) { return D == 16 || D == 32 || D == 64 || D == 128; }

// Common shape checks. Returns CATTN_OK, or INVALID_ARG / UNSUPPORTED.
cattn_status check_shape(int B, int H, int T, int D) {
  if (B < 0 || H < 0 || T < 0 || D < 0) return CATTN_ERR_INVALID_ARG;
  if (!d_supported(D)) return CATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return CATTN_ERR_INVALID_ARG;
  if (T > (1 << 20)) return CATTN_ERR_INVALID_ARG;
  return CATTN_OK;
}

bool empty_shape(int B, int H, int T) { return B == 0 || H == 0 || T == 0; }

// 3-D tensor map {x = d, y = t, z = b*H + h} with element strides t_stride
// and bh_stride (0: the contiguous D and T*D).
cattn_status make_tmap(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elem_bytes,
                       int D, int T, long long BH, int box_x, int box_y, long long t_stride = 0,
                       long long bh_stride = 0) {
  if (t_stride == 0) t_stride = D;
  if (bh_stride == 0) bh_stride = static_cast<long long>(T) * D;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(t_stride) * elem_bytes,
                                 static_cast<cuuint64_t>(bh_stride) * elem_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_x), static_cast<cuuint32_t>(box_y), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const int row_bytes = box_x * elem_bytes;
  CUtensorMapSwizzle sw = row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = g_encode(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CATTN_OK : cuda_fail(10000 + static_cast<int>(r));
}

cattn_layout contiguous_layout(int H, int T, int D) {
  cattn_layout l;
  l.b = static_cast<long long>(H) * T * D;
  l.h = static_cast<long long>(T) * D;
  l.t = D;
  return l;
}

bool is_contiguous(cattn_layout l, int H, int T, int D) {
  const cattn_layout c = contiguous_layout(H, T, D);
  return l.b == c.b && l.h == c.h && l.t == c.t;
}

// Element strides the kernels accept: positive multiples of 8 (rows start
// on 16-byte boundaries, as the TMA and the 16-byte stores need), each below
// 2^38 so that byte offsets stay far inside the TMA's 2^40 stride limit.
bool layout_ok(cattn_layout l) {
  const long long lim = 1LL << 38;
  return l.b > 0 && l.h > 0 && l.t > 0 && l.b % 8 == 0 && l.h % 8 == 0 && l.t % 8 == 0 &&
         l.b < lim && l.h < lim && l.t < lim;
}

// An output layout must not make two of its own elements share an address
// (16-byte stores from different threads would race).  Sufficient test:
// with the axes of extent > 1 taken in increasing stride order (d first,
// stride 1), every stride must exceed the span the smaller ones cover.
// This admits the contiguous layout, padded rows and head-interleaved
// (B, T, C) outputs alike.
bool output_layout_ok(cattn_layout l, int B, int H, int T, int D) {
  struct Ax { long long stride, extent; } ax[3] = {{l.t, T}, {l.h, H}, {l.b, B}};
  for (int i = 0; i < 3; ++i)      // sort by stride (three elements)
    for (int j = i + 1; j < 3; ++j)
      if (ax[j].stride < ax[i].stride) { Ax x = ax[i]; ax[i] = ax[j]; ax[j] = x; }
  long long span = D;  // the d axis: elements 0 .. D-1
  for (int i = 0; i < 3; ++i) {
    if (ax[i].extent <= 1) continue;
    if (ax[i].stride < span) return false;
    span += ax[i].stride * (ax[i].extent - 1);
  }
  return true;
}

// 4-D tensor map {x = d, y = t, z = h, w = b} over a bf16 (B, H, T, D)
// tensor with element strides lay (the d stride is 1); boxes of
// [128 rows][min(D, 64) columns], swizzled by the box's row bytes.
// A (B, H, T, D) layout whose batch stride is H head strides: (b, h) then
// address like the single index b*H + h.
bool collapses(cattn_layout l, int H) { return l.b == static_cast<long long>(H) * l.h; }

cattn_status make_bf16_map(CUtensorMap* m, const void* ptr, int D, int T, int H, int B,
                           cattn_layout lay, bool flat) {
  const int cb = D < 64 ? D : 64;
  if (flat)  // a layout that collapses: 3-D over the b*H + h axis
    return make_tmap(m, ptr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, T,
                     static_cast<long long>(B) * H, cb, 128, lay.t, lay.h);
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(T),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(lay.t) * 2,
                                 static_cast<cuuint64_t>(lay.h) * 2,
                                 static_cast<cuuint64_t>(lay.b) * 2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(cb), 128, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const int row_bytes = cb * 2;
  CUtensorMapSwizzle sw = row_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                          : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : row_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? CATTN_OK : cuda_fail(10000 + static_cast<int>(r));
}

cattn_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? CATTN_OK : cuda_fail(e);
}

// A non-sticky error left in this thread's runtime state by an earlier call
// of the caller's (e.g. a not-ready query) must not be taken for a failure
// of our launches: clear it before launching.
void clear_stale_error() { (void)cudaGetLastError(); }

int grid_for(size_t work_items, int per_block) {
  size_t g = (work_items + per_block - 1) / per_block;
  const size_t cap = 148 * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

// ------------------------------------------------------------ kernel timer
// Optional CUDA-event timing of each launch, on the launching stream (a
// benchmarking aid; off by default, and then it costs nothing).

enum KernelId {
  K_FWD = 0, K_BWD_PRE = 1, K_BWD_MAIN = 2, K_DQ_CONVERT = 3, K_DECODE = 4, K_COUNT = 5
};

bool g_timing = false;
struct TimingRec {
  cudaEvent_t a, b;
  int kernel;
};
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

struct LaunchTimer {
  cudaEvent_t a = nullptr, b = nullptr;
  cudaStream_t s;
  int kernel;
  LaunchTimer(int k, cudaStream_t st) : s(st), kernel(k) {
    if (!g_timing) return;
    std::lock_guard<std::mutex> lk(g_mu);
    a = take_event();
    b = take_event();
    if (a) cudaEventRecord(a, s);
  }
  ~LaunchTimer() {
    if (!g_timing || !a || !b) return;
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_mu);
    g_recs.push_back({a, b, kernel});
  }
};

// ------------------------------------------------------------------ forward

unsigned d_index(int D) { return D == 16 ? 0 : D == 32 ? 1 : D == 64 ? 2 : 3; }

template <int D, bool PLO, bool DROP, bool FLAT>
cattn_status fwd_impl(int dev, const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                      const void* v, cattn_layout lv, float scale, int B, int H, int T, void* o,
                      cattn_layout lo, float* lse, void* o_lo, const DropParams& dp,
                      cudaStream_t s) {
  const int BH = B * H;
  using C = FwdCfg<D, PLO, DROP>;
  clear_stale_error();
  cattn_status st = ensure_smem(dev, (FLAT ? 32 : 0) + (DROP ? 16 : 0) + 2 * d_index(D) + PLO,
                                fwd_kernel<D, PLO, DROP, FLAT>, C::SMEM_BYTES,
                                C::REBALANCE ? C::LAUNCH_REGS : 0);
  if (st != CATTN_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_bf16_map(&mq, q, D, T, H, B, lq, FLAT)) != CATTN_OK) return st;
  if ((st = make_bf16_map(&mk, k, D, T, H, B, lk, FLAT)) != CATTN_OK) return st;
  if ((st = make_bf16_map(&mv, v, D, T, H, B, lv, FLAT)) != CATTN_OK) return st;
  FwdParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_lo = static_cast<__nv_bfloat16*>(o_lo);
  p.o_sb = lo.b;
  p.o_sh = lo.h;
  p.o_st = lo.t;
  p.lse = lse;
  p.H = H;
  p.T = T;
  p.BH = BH;
  p.n_qtiles = (T + 127) / 128;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns;
  p.drop = dp;
  // persistent: one CTA per SM (it holds all of an SM's TMEM), each looping
  // over work items of two query tiles
  const long long n_items = static_cast<long long>(BH) * ((p.n_qtiles + 1) / 2);
  if (n_items > 0x7fffffffLL) return CATTN_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(n_items < g_sm_count[dev] ? n_items : g_sm_count[dev]));
  p.passes = pass_plan(0, BH, p.n_qtiles, static_cast<int>(grid.x));
  cudaError_t e;
  {
    LaunchTimer t(K_FWD, s);
    e = launch_dependent(true, fwd_kernel<D, PLO, DROP, FLAT>, grid, dim3(C::THREADS),
                         C::SMEM_BYTES, s, mq, mk, mv, p);
  }
  return e == cudaSuccess ? CATTN_OK : cuda_fail(e);
}

// One forward instance per (PLO, DROP, FLAT); each line picks exactly one.
template <int D>
cattn_status fwd_dispatch(bool plo, bool drop, bool flat, int dev, const void* q, cattn_layout lq,
                          const void* k, cattn_layout lk, const void* v, cattn_layout lv,
                          float scale, int B, int H, int T, void* o, cattn_layout lo, float* lse,
                          void* o_lo, const DropParams& dp, cudaStream_t s) {
#define CATTN_FWD(PL, DR, FL) \
  fwd_impl<D, PL, DR, FL>(dev, q, lq, k, lk, v, lv, scale, B, H, T, o, lo, lse, o_lo, dp, s)
  if (plo && drop) return flat ? CATTN_FWD(true, true, true) : CATTN_FWD(true, true, false);
  if (plo) return flat ? CATTN_FWD(true, false, true) : CATTN_FWD(true, false, false);
  if (drop) return flat ? CATTN_FWD(false, true, true) : CATTN_FWD(false, true, false);
  return flat ? CATTN_FWD(false, false, true) : CATTN_FWD(false, false, false);
#undef CATTN_FWD
}

// ----------------------------------------------------------------- backward

// Workspace of a backward call: the call's status words {code, where}
// (CATTN_OK = 0, else the first error a kernel recorded; read back by
// cattn_last_device_status), then the fp32 dQ accumulator and the
// LSE * log2(e) and Delta vectors; every part 256-byte aligned.
struct WsLayout {
  size_t status_off, dq_off, lse2_off, delta_off, total;
  int T_pad;
};

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(long long BH, int T, int D) {
  WsLayout L;
  L.T_pad = (T + 127) / 128 * 128;
  L.status_off = 0;
  L.dq_off = 256;
  L.lse2_off = L.dq_off + round256(static_cast<size_t>(BH) * T * D * 4);
  L.delta_off = L.lse2_off + round256(static_cast<size_t>(BH) * L.T_pad * 4);
  L.total = L.delta_off + round256(static_cast<size_t>(BH) * L.T_pad * 4);
  return L;
}

template <int D>
cattn_status pre_impl(const void* o, cattn_layout lo, const void* o_lo, const void* dout,
                      cattn_layout ldo, const float* lse, float* delta, float* lse2, float4* zero,
                      size_t zero_n4, int B, int H, int T, int row_stride,
                      unsigned int* status, cudaStream_t s, bool dependent = true) {
  clear_stale_error();
  const long long BH = static_cast<long long>(B) * H;
  PreParams p;
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.o_lo = static_cast<const __nv_bfloat16*>(o_lo);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.o_sb = lo.b;
  p.o_sh = lo.h;
  p.o_st = lo.t;
  p.do_sb = ldo.b;
  p.do_sh = ldo.h;
  p.do_st = ldo.t;
  p.H = H;
  p.lse = lse;
  p.delta = delta;
  p.lse2 = lse2;
  p.zero = zero;
  p.zero_n4 = zero_n4;
  p.status = status;
  p.T = T;
  p.row_stride = row_stride;
  p.n_rows = BH * row_stride;
  constexpr int rows_per_block = 256 / (D / 8);
  const size_t work = static_cast<size_t>(p.n_rows);
  cudaError_t e;
  {
    LaunchTimer t(K_BWD_PRE, s);
    const dim3 g(grid_for(work > zero_n4 / 64 ? work : zero_n4 / 64, rows_per_block));
    if (is_contiguous(lo, H, T, D) && is_contiguous(ldo, H, T, D))
      e = launch_dependent(dependent, bwd_pre_kernel<D, true>, g, dim3(256), 0, s, p);
    else
      e = launch_dependent(dependent, bwd_pre_kernel<D, false>, g, dim3(256), 0, s, p);
  }
  return e == cudaSuccess ? CATTN_OK : cuda_fail(e);
}

// The strides of one backward call (element strides of each tensor).
struct BwdLayouts {
  cattn_layout q, k, v, o, dout, dq, dk, dv;
};

BwdLayouts contiguous_bwd_layouts(int H, int T, int D) {
  const cattn_layout c = contiguous_layout(H, T, D);
  return BwdLayouts{c, c, c, c, c, c, c, c};
}

template <int D, bool SLO, bool DROP, bool FLAT>
cattn_status bwd_impl(int dev, const void* q, const void* k, const void* v, const void* o,
                      const void* o_lo, const float* lse, const void* dout, float scale, int B,
                      int H, int T, void* dq, void* dk, void* dv, const BwdLayouts& ly,
                      bool grad_f32, void* ws, const DropParams& dp, cudaStream_t s) {
  using C = BwdCfg<D, SLO>;
  const int BH = B * H;
  clear_stale_error();
  cattn_status st = ensure_smem(dev, (FLAT ? 32 : 0) + (DROP ? 24 : 8) + 2 * d_index(D) + SLO,
                                bwd_kernel<D, SLO, DROP, FLAT>, C::SMEM_BYTES,
                                C::REBALANCE ? C::LAUNCH_REGS : 0);
  if (st != CATTN_OK) return st;
  const WsLayout L = ws_layout(BH, T, D);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  float* dq_acc = reinterpret_cast<float*>(wb + L.dq_off);
  float* lse2 = reinterpret_cast<float*>(wb + L.lse2_off);
  float* delta = reinterpret_cast<float*>(wb + L.delta_off);
  unsigned int* status = reinterpret_cast<unsigned int*>(wb + L.status_off);
  const size_t n_dq = static_cast<size_t>(BH) * T * D;

  CUtensorMap mq, mk, mv, mdo, mdq;
  if ((st = make_bf16_map(&mq, q, D, T, H, B, ly.q, FLAT)) != CATTN_OK) return st;
  if ((st = make_bf16_map(&mk, k, D, T, H, B, ly.k, FLAT)) != CATTN_OK) return st;
  if ((st = make_bf16_map(&mv, v, D, T, H, B, ly.v, FLAT)) != CATTN_OK) return st;
  if ((st = make_bf16_map(&mdo, dout, D, T, H, B, ly.dout, FLAT)) != CATTN_OK) return st;
  if ((st = make_tmap(&mdq, dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, T, BH,
                      C::WARP_DQ ? D / 4 : C::CBQ, C::WARP_DQ ? 32 : 128)) !=
      CATTN_OK)
    return st;

  st = pre_impl<D>(o, ly.o, o_lo, dout, ly.dout, lse, delta, lse2,
                   reinterpret_cast<float4*>(dq_acc), n_dq / 4, B, H, T, L.T_pad, status, s);
  if (st != CATTN_OK) return st;

  BwdParams p;
  p.lse2 = lse2;
  p.delta = delta;
  p.dk_f32 = grad_f32 ? static_cast<float*>(dk) : nullptr;
  p.dv_f32 = grad_f32 ? static_cast<float*>(dv) : nullptr;
  p.dk_bf16 = grad_f32 ? nullptr : static_cast<__nv_bfloat16*>(dk);
  p.dv_bf16 = grad_f32 ? nullptr : static_cast<__nv_bfloat16*>(dv);
  p.dk_sb = ly.dk.b;
  p.dk_sh = ly.dk.h;
  p.dk_st = ly.dk.t;
  p.dv_sb = ly.dv.b;
  p.dv_sh = ly.dv.h;
  p.dv_st = ly.dv.t;
  p.H = H;
  p.BH = BH;
  p.T = T;
  p.T_pad = L.T_pad;
  p.n_tiles = L.T_pad / 128;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns;
  p.drop = dp;
  p.status = status;
  // persistent: one CTA per SM, each looping over key tiles
  const long long n_items = static_cast<long long>(BH) * p.n_tiles;
  if (n_items > 0x7fffffffLL) return CATTN_ERR_INVALID_ARG;
  dim3 grid(static_cast<unsigned>(n_items < g_sm_count[dev] ? n_items : g_sm_count[dev]));
  cudaError_t e;
  constexpr bool dep = true;  // programmatic dependents (see launch_dependent)
  {
    LaunchTimer t(K_BWD_MAIN, s);
    e = launch_dependent(dep, bwd_kernel<D, SLO, DROP, FLAT>, grid, dim3(C::THREADS),
                         C::SMEM_BYTES, s, mq, mk, mv, mdo, mdq, p);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  {
    LaunchTimer t(K_DQ_CONVERT, s);
    const float4* acc = reinterpret_cast<const float4*>(dq_acc);
    if (!is_contiguous(ly.dq, H, T, D)) {
      const long long n8 = static_cast<long long>(n_dq / 8);
      const dim3 g(grid_for(static_cast<size_t>(n8), 256));
      if (grad_f32)
        e = launch_dependent(dep, dq_convert_strided_kernel<D, true>, g, dim3(256), 0, s, acc, dq,
                             H, T, n8, ly.dq.b, ly.dq.h, ly.dq.t, scale);
      else
        e = launch_dependent(dep, dq_convert_strided_kernel<D, false>, g, dim3(256), 0, s, acc, dq,
                             H, T, n8, ly.dq.b, ly.dq.h, ly.dq.t, scale);
    } else if (grad_f32)
      e = launch_dependent(dep, dq_convert_f32_kernel, dim3(grid_for(n_dq / 4, 256)), dim3(256), 0,
                           s, acc, static_cast<float4*>(dq), n_dq / 4, scale);
    else
      e = launch_dependent(dep, dq_convert_kernel, dim3(grid_for(n_dq / 8, 256)), dim3(256), 0, s,
                           acc, static_cast<uint4*>(dq), n_dq / 8, scale);
  }
  return e == cudaSuccess ? CATTN_OK : cuda_fail(e);
}

template <int D>
cattn_status bwd_dispatch(bool slo, int dev, const void* q, const void* k, const void* v,
                          const void* o, const void* o_lo, const float* lse, const void* dout,
                          float scale, int B, int H, int T, void* dq, void* dk, void* dv,
                          const BwdLayouts& ly, bool f32, void* ws, const DropParams& dp,
                          cudaStream_t s) {
  // FLAT: every tensor the main kernel addresses by (b, h) collapses to one
  // b*H + h axis (the contiguous layout among others): 3-D tensor maps and
  // no division by H in the kernel
  const bool flat = collapses(ly.q, H) && collapses(ly.k, H) && collapses(ly.v, H) &&
                    collapses(ly.dout, H) && collapses(ly.dk, H) && collapses(ly.dv, H);
  // one instance per (SLO, DROP, FLAT); each line picks exactly one
  const bool drop = dp.t != 0;
#define CATTN_BWD(SS, DR, FL) \
  bwd_impl<D, SS, DR, FL>(dev, q, k, v, o, o_lo, lse, dout, scale, B, H, T, dq, dk, dv, ly, f32, ws, dp, s)
  if (slo && drop) return flat ? CATTN_BWD(true, true, true) : CATTN_BWD(true, true, false);
  if (slo) return flat ? CATTN_BWD(true, false, true) : CATTN_BWD(true, false, false);
  if (drop) return flat ? CATTN_BWD(false, true, true) : CATTN_BWD(false, true, false);
  return flat ? CATTN_BWD(false, false, true) : CATTN_BWD(false, false, false);
#undef CATTN_BWD
}

// Dropout parameters of a call: t = round(p * 256) (the drop threshold on
// 8 random bits), 1 / (1 - t / 256) as the keep scale; false for a
// probability outside [0, 1).  t = 0 (no dropout, p < 2^-9) selects the
// kernels without the mask, whose result is then the same.
bool drop_params(const cattn_dropout* d, DropParams* out) {
  *out = DropParams{};
  if (d == nullptr) return true;
  if (!(d->p >= 0.f) || !(d->p < 1.f)) return false;
  if (!aligned(d->mask, 16)) return false;
  out->mask = static_cast<uint32_t*>(d->mask);
  long t = lrint(static_cast<double>(d->p) * 256.0);
  if (t > 255) t = 255;
  out->t = static_cast<uint32_t>(t);
  out->t_lo = (out->t & 0x7Fu) * 0x01010101u;
  out->t_maj = out->t < 128u ? 0xFFFFFFFFu : 0u;
  philox_round_keys(static_cast<uint32_t>(d->seed & 0xffffffffull),
                    static_cast<uint32_t>(d->seed >> 32), out->rk);
  out->offset = d->offset;
  out->inv_keep = static_cast<float>(256.0 / (256.0 - static_cast<double>(t)));
  return true;
}

// ---------------------------------------------------------- hang-guard test

__global__ void selftest_wait_kernel(uint64_t timeout_ns, unsigned int* call_status) {
  __shared__ __align__(8) uint64_t mbar;
  // the abort flag, then (8 bytes on) the call's status address, as in the
  // backward kernel
  __shared__ __align__(8) int abort_and_call[4];
  int& abort_flag = abort_and_call[0];
  if (threadIdx.x == 0) {
    abort_flag = 0;
    *reinterpret_cast<unsigned int**>(&abort_and_call[2]) = call_status;
    mbar_init(smem_u32(&mbar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{timeout_ns, &abort_flag, 15u, true};
    wait1(w, smem_u32(&mbar), 0, 1);  // nothing ever arrives
  }
  __syncthreads();
}

// ------------------------------------------------------------------ decode

// Resident decode CTAs on the device: its SMs x decode_ctas_per_sm(D).
int decode_slots(int dev, int D) { return g_sm_count[dev] * decode_ctas_per_sm(D); }

template <int D>
cattn_status decode_impl(const DecodeParams& p, long long BH, int dev, cudaStream_t s) {
  cattn_status st = ensure_smem(dev, 64 + d_index(D), decode_kernel<D>, decode_smem_bytes(D));
  if (st != CATTN_OK) return st;
  clear_stale_error();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH * p.n_split));
  cfg.blockDim = dim3(kDecodeThreads);
  cfg.dynamicSmemBytes = decode_smem_bytes(D);
  cfg.stream = s;
  // a programmatic dependent of the previous kernel (see launch_dependent),
  // and a cluster of the n_split CTAs of one (b, h) where it splits
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(p.n_split);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.n_split > 1 ? 2 : 1;
  LaunchTimer t(K_DECODE, s);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_kernel<D>, p);
  return e == cudaSuccess ? CATTN_OK : cuda_fail(e);
}

}  // namespace
}  // namespace cattn

using namespace cattn;

extern "C" {

cattn_status attn_fwd_dropout(const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                              const void* v, cattn_layout lv, float scale, int B, int H, int T,
                              int D, const cattn_dropout* dropout, void* o, cattn_layout lo,
                              float* lse, void* o_lo, void* stream) {
  cattn_status st = check_shape(B, H, T, D);
  if (st != CATTN_OK) return st;
  if (!(scale > 0.f) || !isfinite(scale)) return CATTN_ERR_INVALID_ARG;
  DropParams dp;
  if (!drop_params(dropout, &dp)) return CATTN_ERR_INVALID_ARG;
  if (empty_shape(B, H, T)) return CATTN_OK;
  if (!q || !k || !v || !o || !lse) return CATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(o_lo, 16))
    return CATTN_ERR_INVALID_ARG;
  if (!layout_ok(lq) || !layout_ok(lk) || !layout_ok(lv) || !layout_ok(lo))
    return CATTN_ERR_INVALID_ARG;
  if (!output_layout_ok(lo, B, H, T, D)) return CATTN_ERR_INVALID_ARG;
  int dev;
  if ((st = check_device(&dev)) != CATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // FLAT: q, k, v and o all collapse to one b*H + h axis (see bwd_dispatch)
  const bool flat = collapses(lq, H) && collapses(lk, H) && collapses(lv, H) && collapses(lo, H);
  const bool plo = o_lo != nullptr, drop = dp.t != 0;
  switch (D) {
    case 16: return fwd_dispatch<16>(plo, drop, flat, dev, q, lq, k, lk, v, lv, scale, B, H, T, o, lo, lse, o_lo, dp, s);
    case 32: return fwd_dispatch<32>(plo, drop, flat, dev, q, lq, k, lk, v, lv, scale, B, H, T, o, lo, lse, o_lo, dp, s);
    case 64: return fwd_dispatch<64>(plo, drop, flat, dev, q, lq, k, lk, v, lv, scale, B, H, T, o, lo, lse, o_lo, dp, s);
    case 128: return fwd_dispatch<128>(plo, drop, flat, dev, q, lq, k, lk, v, lv, scale, B, H, T, o, lo, lse, o_lo, dp, s);
  }
  return CATTN_ERR_UNSUPPORTED;
}

cattn_status attn_fwd_strided(const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                              const void* v, cattn_layout lv, float scale, int B, int H, int T,
                              int D, void* o, cattn_layout lo, float* lse, void* o_lo,
                              void* stream) {
  return attn_fwd_dropout(q, lq, k, lk, v, lv, scale, B, H, T, D, nullptr, o, lo, lse, o_lo,
                          stream);
}

cattn_status attn_fwd_ex(const void* q, const void* k, const void* v, float scale, int B, int H,
                         int T, int D, void* o, float* lse, void* o_lo, void* stream) {
  const cattn_layout c = contiguous_layout(H, T, D);
  return attn_fwd_strided(q, c, k, c, v, c, scale, B, H, T, D, o, c, lse, o_lo, stream);
}

cattn_status attn_fwd(const void* q, const void* k, const void* v, float scale, int B, int H,
                      int T, int D, void* o, float* lse, void* stream) {
  return attn_fwd_ex(q, k, v, scale, B, H, T, D, o, lse, nullptr, stream);
}

size_t attn_dropout_mask_bytes(int B, int H, int T) {
  if (B <= 0 || H <= 0 || T <= 0 || static_cast<long long>(B) * H > 0x7fffffffLL ||
      T > (1 << 20))
    return 0;
  const int n_tiles = (T + 127) / 128;
  return keep_cache_block(static_cast<long long>(B) * H, n_tiles, 0, 0) * sizeof(uint32_t);
}

size_t attn_decode_workspace_bytes(int B, int H, int Tq, int L, int D) {
  // the CTAs of a head merge their partial results on chip
  (void)B, (void)H, (void)Tq, (void)L, (void)D;
  return 0;
}

cattn_status attn_decode(const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                         const void* v, cattn_layout lv, float scale, int B, int H, int Tq, int L,
                         int D, void* o, cattn_layout lo, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream) {
  cattn_status st = check_shape(B, H, L, D);
  if (st != CATTN_OK) return st;
  if (!(scale > 0.f) || !isfinite(scale)) return CATTN_ERR_INVALID_ARG;
  if (Tq > kDecodeMaxTq) return CATTN_ERR_UNSUPPORTED;
  if (B == 0 || H == 0) return CATTN_OK;
  if (Tq < 1 || L < Tq) return CATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse) return CATTN_ERR_INVALID_ARG;
  (void)workspace, (void)workspace_bytes;  // none needed
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(lse, 4))
    return CATTN_ERR_INVALID_ARG;
  if (!layout_ok(lq) || !layout_ok(lk) || !layout_ok(lv) || !layout_ok(lo))
    return CATTN_ERR_INVALID_ARG;
  if (!output_layout_ok(lo, B, H, Tq, D)) return CATTN_ERR_INVALID_ARG;
  const long long BH = static_cast<long long>(B) * H;
  int dev;
  if ((st = check_device(&dev)) != CATTN_OK) return st;
  const int n_split = decode_splits_for(BH, L, D, decode_slots(dev, D));
  if (BH * n_split > 0x7fffffffLL) return CATTN_ERR_INVALID_ARG;
  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.q_sb = lq.b; p.q_sh = lq.h; p.q_st = lq.t;
  p.k_sb = lk.b; p.k_sh = lk.h; p.k_st = lk.t;
  p.v_sb = lv.b; p.v_sh = lv.h; p.v_st = lv.t;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = lo.b; p.o_sh = lo.h; p.o_st = lo.t;
  p.lse = lse;
  p.H = H;
  p.Tq = Tq;
  p.L = L;
  p.n_split = n_split;
  p.chunks_per_cta = decode_chunks_per_cta(BH, L, D, decode_slots(dev, D));
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (D) {
    case 16: return decode_impl<16>(p, BH, dev, s);
    case 32: return decode_impl<32>(p, BH, dev, s);
    case 64: return decode_impl<64>(p, BH, dev, s);
    case 128: return decode_impl<128>(p, BH, dev, s);
  }
  return CATTN_ERR_UNSUPPORTED;
}

size_t attn_bwd_workspace_bytes(int B, int H, int T, int D) {
  if (check_shape(B, H, T, D) != CATTN_OK) return 0;
  if (empty_shape(B, H, T)) return 0;
  return ws_layout(static_cast<long long>(B) * H, T, D).total;
}

cattn_status attn_bwd_preprocess(const void* o, const void* dout, int B, int H, int T, int D,
                                 float* delta, void* stream) {
  cattn_status st = check_shape(B, H, T, D);
  if (st != CATTN_OK) return st;
  if (empty_shape(B, H, T)) return CATTN_OK;
  if (!o || !dout || !delta) return CATTN_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(delta, 4)) return CATTN_ERR_INVALID_ARG;
  int dev;
  if ((st = check_device(&dev)) != CATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cattn_layout c = contiguous_layout(H, T, D);
  switch (D) {
    case 16: return pre_impl<16>(o, c, nullptr, dout, c, nullptr, delta, nullptr, nullptr, 0, B, H, T, T, nullptr, s);
    case 32: return pre_impl<32>(o, c, nullptr, dout, c, nullptr, delta, nullptr, nullptr, 0, B, H, T, T, nullptr, s);
    case 64: return pre_impl<64>(o, c, nullptr, dout, c, nullptr, delta, nullptr, nullptr, 0, B, H, T, T, nullptr, s);
    case 128: return pre_impl<128>(o, c, nullptr, dout, c, nullptr, delta, nullptr, nullptr, 0, B, H, T, T, nullptr, s);
  }
  return CATTN_ERR_UNSUPPORTED;
}

cattn_status attn_bwd_dropout(const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                              const void* v, cattn_layout lv, const void* o, cattn_layout lo,
                              const void* o_lo, const float* lse, const void* dout,
                              cattn_layout ldo, float scale, int B, int H, int T, int D,
                              const cattn_dropout* dropout, void* dq, cattn_layout ldq, void* dk,
                              cattn_layout ldk, void* dv, cattn_layout ldv, int grad_dtype,
                              void* workspace, size_t workspace_bytes, void* stream) {
  cattn_status st = check_shape(B, H, T, D);
  if (st != CATTN_OK) return st;
  if (!(scale > 0.f) || !isfinite(scale)) return CATTN_ERR_INVALID_ARG;
  DropParams dp;
  if (!drop_params(dropout, &dp)) return CATTN_ERR_INVALID_ARG;
  if (empty_shape(B, H, T)) return CATTN_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return CATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 256) || !aligned(o_lo, 16))
    return CATTN_ERR_INVALID_ARG;
  if (!layout_ok(lq) || !layout_ok(lk) || !layout_ok(lv) || !layout_ok(lo) || !layout_ok(ldo) ||
      !layout_ok(ldq) || !layout_ok(ldk) || !layout_ok(ldv))
    return CATTN_ERR_INVALID_ARG;
  if (!output_layout_ok(ldq, B, H, T, D) || !output_layout_ok(ldk, B, H, T, D) ||
      !output_layout_ok(ldv, B, H, T, D))
    return CATTN_ERR_INVALID_ARG;
  const int BH = B * H;
  if (workspace_bytes < ws_layout(BH, T, D).total) return CATTN_ERR_INVALID_ARG;
  if (grad_dtype != CATTN_DTYPE_BF16 && grad_dtype != CATTN_DTYPE_F32)
    return CATTN_ERR_INVALID_ARG;
  const bool f32 = grad_dtype == CATTN_DTYPE_F32;
  int dev;
  if ((st = check_device(&dev)) != CATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const BwdLayouts ly{lq, lk, lv, lo, ldo, ldq, ldk, ldv};
  // dS as a hi/lo pair when the caller asks for gradients accurate to ~fp32
  const bool slo = o_lo != nullptr || f32;
  switch (D) {
    case 16: return bwd_dispatch<16>(slo, dev, q, k, v, o, o_lo, lse, dout, scale, B, H, T, dq, dk, dv, ly, f32, workspace, dp, s);
    case 32: return bwd_dispatch<32>(slo, dev, q, k, v, o, o_lo, lse, dout, scale, B, H, T, dq, dk, dv, ly, f32, workspace, dp, s);
    case 64: return bwd_dispatch<64>(slo, dev, q, k, v, o, o_lo, lse, dout, scale, B, H, T, dq, dk, dv, ly, f32, workspace, dp, s);
    case 128: return bwd_dispatch<128>(slo, dev, q, k, v, o, o_lo, lse, dout, scale, B, H, T, dq, dk, dv, ly, f32, workspace, dp, s);
  }
  return CATTN_ERR_UNSUPPORTED;
}

cattn_status attn_bwd_strided(const void* q, cattn_layout lq, const void* k, cattn_layout lk,
                              const void* v, cattn_layout lv, const void* o, cattn_layout lo,
                              const void* o_lo, const float* lse, const void* dout,
                              cattn_layout ldo, float scale, int B, int H, int T, int D, void* dq,
                              cattn_layout ldq, void* dk, cattn_layout ldk, void* dv,
                              cattn_layout ldv, int grad_dtype, void* workspace,
                              size_t workspace_bytes, void* stream) {
  return attn_bwd_dropout(q, lq, k, lk, v, lv, o, lo, o_lo, lse, dout, ldo, scale, B, H, T, D,
                          nullptr, dq, ldq, dk, ldk, dv, ldv, grad_dtype, workspace,
                          workspace_bytes, stream);
}

cattn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                         const void* o_lo, const float* lse, const void* dout, float scale, int B,
                         int H, int T, int D, void* dq, void* dk, void* dv, int grad_dtype,
                         void* workspace, size_t workspace_bytes, void* stream) {
  const cattn_layout c = contiguous_layout(H, T, D);
  return attn_bwd_strided(q, c, k, c, v, c, o, c, o_lo, lse, dout, c, scale, B, H, T, D, dq, c,
                          dk, c, dv, c, grad_dtype, workspace, workspace_bytes, stream);
}

cattn_status attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const float* lse, const void* dout, float scale, int B, int H, int T, int D,
                      void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                      void* stream) {
  return attn_bwd_ex(q, k, v, o, nullptr, lse, dout, scale, B, H, T, D, dq, dk, dv,
                     CATTN_DTYPE_BF16, workspace, workspace_bytes, stream);
}

// Device addresses of cattn_noalloc_scratch, looked up once per device.
static void* g_noalloc_scratch_ptr[kMaxDevices];

cattn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                              const float* lse, const void* dout, float scale, int B, int H,
                              int T, int D, void* dq, void* dk, void* dv, void* stream) {
  cattn_status st = check_shape(B, H, T, D);
  if (st != CATTN_OK) return st;
  if (!(scale > 0.f) || !isfinite(scale)) return CATTN_ERR_INVALID_ARG;
  if (empty_shape(B, H, T)) return CATTN_OK;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return CATTN_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4))
    return CATTN_ERR_INVALID_ARG;
  const int BH = B * H;
  if (ws_layout(BH, T, D).total > CATTN_NOALLOC_SCRATCH_BYTES) return CATTN_ERR_TOO_LARGE;
  int dev;
  if ((st = check_device(&dev)) != CATTN_OK) return st;
  void* scratch = nullptr;
  {
    // set-up, once per device, with that device current (check_device
    // bound it to this thread): the array's device address
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_scratch_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, cattn_noalloc_scratch);
      if (e != cudaSuccess || ptr == nullptr) return cuda_fail(e != cudaSuccess ? e : cudaErrorUnknown);
      g_noalloc_scratch_ptr[dev] = ptr;
    }
    scratch = g_noalloc_scratch_ptr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the backward clears what must start at zero (the dQ accumulator) and
  // overwrites the rest on every call
  const BwdLayouts ly = contiguous_bwd_layouts(H, T, D);
  const DropParams no_drop{};
  switch (D) {
    case 16:
      return bwd_impl<16, false, false, true>(dev, q, k, v, o, nullptr, lse, dout, scale, B, H, T, dq, dk,
                                        dv, ly, false, scratch, no_drop, s);
    case 32:
      return bwd_impl<32, false, false, true>(dev, q, k, v, o, nullptr, lse, dout, scale, B, H, T, dq, dk,
                                        dv, ly, false, scratch, no_drop, s);
    case 64:
      return bwd_impl<64, false, false, true>(dev, q, k, v, o, nullptr, lse, dout, scale, B, H, T, dq, dk,
                                        dv, ly, false, scratch, no_drop, s);
    case 128:
      return bwd_impl<128, false, false, true>(dev, q, k, v, o, nullptr, lse, dout, scale, B, H, T, dq, dk,
                                        dv, ly, false, scratch, no_drop, s);
  }
  return CATTN_ERR_UNSUPPORTED;
}

cattn_status cattn_get_device_status(int clear, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_fail(cudaGetLastError());
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess)
    return cuda_fail(cudaGetLastError());
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_status, &z, sizeof(z)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_status_where, &z, sizeof(z)) != cudaSuccess) {
      return cuda_fail(cudaGetLastError());
    }
  }
  return v == 0 ? CATTN_OK : static_cast<cattn_status>(v);
}

cattn_status cattn_last_device_status(void* workspace, void* stream) {
  if (workspace == nullptr || !aligned(workspace, 256)) return CATTN_ERR_INVALID_ARG;
  int dev;
  cattn_status st = check_device(&dev);
  if (st != CATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_fail(cudaGetLastError());
  unsigned int v = 0;
  if (cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_fail(cudaGetLastError());
  return v == 0 ? CATTN_OK : static_cast<cattn_status>(v);
}

cattn_status cattn_selftest_wait_timeout_ws(uint32_t timeout_us, void* workspace, void* stream) {
  if (workspace == nullptr || !aligned(workspace, 256)) return CATTN_ERR_INVALID_ARG;
  int dev;
  cattn_status st = check_device(&dev);
  if (st != CATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int before = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess ||
      cudaMemcpyFromSymbol(&before, g_status, sizeof(before)) != cudaSuccess ||
      cudaMemsetAsync(workspace, 0, 8, s) != cudaSuccess)
    return cuda_fail(cudaGetLastError());
  clear_stale_error();
  selftest_wait_kernel<<<1, 32, 0, s>>>(static_cast<uint64_t>(timeout_us) * 1000ull,
                                        static_cast<unsigned int*>(workspace));
  if (launch_status() != CATTN_OK) return CATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return cuda_fail(cudaGetLastError());
  if (before == 0) {  // leave the global word as it was found
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_status, &z, sizeof(z)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_status_where, &z, sizeof(z)) != cudaSuccess)
      return cuda_fail(cudaGetLastError());
  }
  return cattn_last_device_status(workspace, stream);
}

void cattn_set_wait_timeout_us(uint32_t us) {
  g_timeout_ns = us == 0 ? kDefaultTimeoutNs : static_cast<uint64_t>(us) * 1000ull;
}

cattn_status cattn_selftest_wait_timeout(uint32_t timeout_us, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cattn_status st = cattn_get_device_status(1, stream);  // start from a clear word
  if (st != CATTN_OK && st != CATTN_ERR_TIMEOUT) return st;
  selftest_wait_kernel<<<1, 32, 0, s>>>(static_cast<uint64_t>(timeout_us) * 1000ull, nullptr);
  if (launch_status() != CATTN_OK) return CATTN_ERR_CUDA;
  st = cattn_get_device_status(1, stream);
  return st;
}

void cattn_timing_enable(int enable) { g_timing = enable != 0; }

cattn_status cattn_timing_read(float* total_ms, int* launches, int n) {
  if (!total_ms || !launches || n < 0) return CATTN_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    total_ms[i] = 0.f;
    launches[i] = 0;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  cattn_status st = CATTN_OK;
  for (const TimingRec& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess ||
        cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      st = cuda_fail(cudaGetLastError());
    } else if (r.kernel < n) {
      total_ms[r.kernel] += ms;
      launches[r.kernel] += 1;
    }
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_recs.clear();
  return st;
}

const char* cattn_status_string(cattn_status s) {
  switch (s) {
    case CATTN_OK: return "ok";
    case CATTN_ERR_INVALID_ARG: return "invalid argument";
    case CATTN_ERR_UNSUPPORTED: return "unsupported (head size or device)";
    case CATTN_ERR_CUDA: return "CUDA error";
    case CATTN_ERR_TIMEOUT: return "kernel wait timed out";
    case CATTN_ERR_TOO_LARGE: return "shape exceeds the fixed scratch of attn_bwd_noalloc";
  }
  return "unknown status";
}

int cattn_version(void) { return 100; }

int cattn_plan_passes(int kind, int BH, int n_tiles, int G, uint16_t* codes, int max_codes) {
  if ((kind != 0 && kind != 1) || BH < 1 || n_tiles < 1 || G < 1) return -1;
  const PassCodes pc = pass_plan(kind, BH, n_tiles, G);
  for (int k = 0; k < pc.n && k < max_codes; ++k) codes[k] = static_cast<uint16_t>(pass_code(pc, k));
  return pc.n;
}

int cattn_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
