// Runs the decode kernel of decode.cuh (the device source itself) on the
// host through simt_emu.h and decode_ptx_emu.h, for CPU tests: exactly
// sized buffers under AddressSanitizer and UBSan, so any out-of-bounds or
// misaligned access of the kernel fails the run.
//
//   decode_emu B H Tq L D Tmax layout scale in.bin out.bin [ctas_per_head]
//     layout 0: k, v stored (B, H, Tmax, D); 1: stored (B, Tmax, H, D)
//     in.bin:  q (B, H, Tq, D), k, v (stored layout) as bf16 bit patterns
//     out.bin: o (B, H, Tq, D) bf16 bit patterns, then lse (B, H, Tq) fp32
//     ctas_per_head: CTAs per head, the cluster size (default: attn_decode's
//     own choice on a 148-SM B200); fewer CTAs than chunks make each CTA,
//     and each of its warps, walk several chunks
// The host set-up (cluster size, chunks per CTA, strides) follows
// attn_decode in api.cu.
#define CATTN_HOST_EMULATION 1
#include "simt_emu.h"

#include <cstdio>
#include <cstdlib>

#include "decode_ptx_emu.h"
#include "decode.cuh"

using namespace cattn;

template <typename T>
static T* exact(size_t n) {
  return static_cast<T*>(std::calloc(n ? n : 1, sizeof(T)));
}

template <int D>
static void run(DecodeParams p, int BH) {
  emu::launch_ex(static_cast<unsigned>(BH * p.n_split), kDecodeThreads, decode_smem_bytes(D),
                 static_cast<unsigned>(p.n_split), decode_kernel<D>, p);
}

int main(int argc, char** argv) {
  if (argc != 11 && argc != 12) {
    std::fprintf(stderr, "usage: decode_emu B H Tq L D Tmax layout scale in out [ctas_per_head]\n");
    return 2;
  }
  const int B = std::atoi(argv[1]), H = std::atoi(argv[2]), Tq = std::atoi(argv[3]);
  const int L = std::atoi(argv[4]), D = std::atoi(argv[5]), Tmax = std::atoi(argv[6]);
  const int layout = std::atoi(argv[7]);
  const float scale = static_cast<float>(std::atof(argv[8]));
  const size_t nq = static_cast<size_t>(B) * H * Tq * D, nkv = static_cast<size_t>(B) * H * Tmax * D;
  auto* q = exact<__nv_bfloat16>(nq);
  auto* k = exact<__nv_bfloat16>(nkv);
  auto* v = exact<__nv_bfloat16>(nkv);
  FILE* f = std::fopen(argv[9], "rb");
  if (!f || std::fread(q, 2, nq, f) != nq || std::fread(k, 2, nkv, f) != nkv ||
      std::fread(v, 2, nkv, f) != nkv)
    return 3;
  std::fclose(f);
  const int BH = B * H;
  const int n_chunks = (L + decode_chunk(D) - 1) / decode_chunk(D);
  const int slots = 148 * decode_ctas_per_sm(D);
  int n_split = decode_splits_for(static_cast<long long>(B) * H, L, D, slots);
  int cpc = decode_chunks_per_cta(static_cast<long long>(B) * H, L, D, slots);
  if (argc == 12) {  // a chosen number of CTAs per head
    const int want = std::atoi(argv[11]);
    cpc = (n_chunks + want - 1) / want;
    n_split = (n_chunks + cpc - 1) / cpc;
  }
  auto* o = exact<__nv_bfloat16>(nq);
  auto* lse = exact<float>(static_cast<size_t>(BH) * Tq);
  DecodeParams p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.q_sb = static_cast<long long>(H) * Tq * D;
  p.q_sh = static_cast<long long>(Tq) * D;
  p.q_st = D;
  if (layout == 0) {
    p.k_sb = static_cast<long long>(H) * Tmax * D;
    p.k_sh = static_cast<long long>(Tmax) * D;
    p.k_st = D;
  } else {
    p.k_sb = static_cast<long long>(Tmax) * H * D;
    p.k_sh = D;
    p.k_st = static_cast<long long>(H) * D;
  }
  p.v_sb = p.k_sb;
  p.v_sh = p.k_sh;
  p.v_st = p.k_st;
  p.o = o;
  p.o_sb = p.q_sb;
  p.o_sh = p.q_sh;
  p.o_st = p.q_st;
  p.lse = lse;
  p.H = H;
  p.Tq = Tq;
  p.L = L;
  p.n_split = n_split;
  p.chunks_per_cta = cpc;
  p.scale_log2 = scale * 1.4426950408889634f;
  switch (D) {
    case 16: run<16>(p, BH); break;
    case 32: run<32>(p, BH); break;
    case 64: run<64>(p, BH); break;
    case 128: run<128>(p, BH); break;
    default: return 4;
  }
  f = std::fopen(argv[10], "wb");
  if (!f) return 5;
  std::fwrite(o, 2, nq, f);
  std::fwrite(lse, 4, static_cast<size_t>(BH) * Tq, f);
  std::fclose(f);
  std::free(q);
  std::free(k);
  std::free(v);
  std::free(o);
  std::free(lse);
  return 0;
}
