// The dropout mask code of csrc/philox.cuh compiled for the host: the
// generator, the byte-wise threshold compare and the interleaved keep-word
// order, as the kernels call them.  Test harness for tests/test_philox_host.py.
//
//   philox_host swar
//       every byte value at every byte position of a word against every
//       threshold: keep_flags / keep_nibble against a plain comparison;
//       prints "ok" or the first mismatch.
//   philox_host mask B H T seed offset p
//       the keep bits of every (b, h, i, j < T) as drawn by keep16 and by
//       keep32_il (mapped back through il_key): one line per (b*H + h, i),
//       "<bh> <i> <hex of keep16 bits> <hex of keep32_il bits>", key j at
//       bit j of the hex number (most significant digit first).
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#define __host__
#define __device__
#define __forceinline__ inline
// the warp shuffles are device code that the host never calls here
inline unsigned __shfl_xor_sync(unsigned, unsigned v, int) { std::abort(); return v; }
inline unsigned __shfl_sync(unsigned, unsigned v, int) { std::abort(); return v; }

#include "philox.cuh"

using cattn::DropParams;

static DropParams params(double p, unsigned long long seed, unsigned offset) {
  DropParams d;
  long t = std::lrint(p * 256.0);
  if (t > 255) t = 255;
  d.t = static_cast<uint32_t>(t);
  d.t_lo = (d.t & 0x7Fu) * 0x01010101u;
  d.t_maj = d.t < 128u ? 0xFFFFFFFFu : 0u;
  d.offset = offset;
  cattn::philox_round_keys(static_cast<uint32_t>(seed & 0xffffffffull),
                           static_cast<uint32_t>(seed >> 32), d.rk);
  d.inv_keep = static_cast<float>(256.0 / (256.0 - t));
  return d;
}

static int swar() {
  for (int t = 0; t < 256; ++t) {
    DropParams d = params(t / 256.0, 0, 0);
    if (static_cast<int>(d.t) != t) {
      std::printf("threshold %d -> %u\n", t, d.t);
      return 1;
    }
    for (int b = 0; b < 256; ++b)
      for (int pos = 0; pos < 4; ++pos) {
        // the byte under test at `pos`, its neighbours set so that a borrow
        // or carry across a byte boundary would show
        const uint32_t others[3] = {0x00000000u, 0xFFFFFFFFu, 0x807F01FEu};
        for (uint32_t o : others) {
          const uint32_t w = (o & ~(0xFFu << (8 * pos))) | (static_cast<uint32_t>(b) << (8 * pos));
          const uint32_t f = cattn::keep_flags(w, d);
          const uint32_t n = cattn::keep_nibble(w, d);
          for (int k = 0; k < 4; ++k) {
            const bool want = static_cast<int>((w >> (8 * k)) & 0xFFu) >= t;
            const bool got_f = (f >> (8 * k + 7)) & 1u;
            const bool got_n = (n >> k) & 1u;
            if (got_f != want || got_n != want || (f & ~0x80808080u) != 0 || (n >> 4) != 0) {
              std::printf("t %d word %08x byte %d: want %d flags %08x nibble %x\n", t, w, k,
                          int(want), f, n);
              return 1;
            }
          }
        }
      }
  }
  for (int c = 0; c < 32; ++c)
    if (cattn::il_key(cattn::il_pos(c)) != c) {
      std::printf("il_key(il_pos(%d)) = %d\n", c, cattn::il_key(cattn::il_pos(c)));
      return 1;
    }
  std::printf("ok\n");
  return 0;
}

static std::string hex_bits(const uint32_t* words, int n_words, int T) {
  // key j at bit j; printed most significant digit first, T bits
  std::string s;
  const int digits = (T + 3) / 4;
  for (int dgt = digits - 1; dgt >= 0; --dgt) {
    uint32_t v = 0;
    for (int b = 3; b >= 0; --b) {
      const int j = 4 * dgt + b;
      const uint32_t bit = j < T ? (words[j / 32] >> (j % 32)) & 1u : 0u;
      v = (v << 1) | bit;
    }
    s += "0123456789abcdef"[v];
  }
  (void)n_words;
  return s;
}

static int mask(int B, int H, int T, unsigned long long seed, unsigned offset, double p) {
  const DropParams d = params(p, seed, offset);
  const int n32 = (T + 31) / 32;
  uint32_t* a = static_cast<uint32_t*>(std::calloc(n32, 4));
  uint32_t* b = static_cast<uint32_t*>(std::calloc(n32, 4));
  for (int bh = 0; bh < B * H; ++bh)
    for (int i = 0; i < T; ++i) {
      for (int w = 0; w < n32; ++w) {
        a[w] = cattn::keep16(2 * w, i, bh, d) | cattn::keep16(2 * w + 1, i, bh, d) << 16;
        const uint32_t il = cattn::keep32_il(w, i, bh, d);
        b[w] = 0;
        for (int pos = 0; pos < 32; ++pos) b[w] |= ((il >> pos) & 1u) << cattn::il_key(pos);
      }
      std::printf("%d %d %s %s\n", bh, i, hex_bits(a, n32, T).c_str(), hex_bits(b, n32, T).c_str());
    }
  std::free(a);
  std::free(b);
  return 0;
}

int main(int argc, char** argv) {
  if (argc >= 2 && std::strcmp(argv[1], "swar") == 0) return swar();
  if (argc == 8 && std::strcmp(argv[1], "mask") == 0)
    return mask(std::atoi(argv[2]), std::atoi(argv[3]), std::atoi(argv[4]),
                std::strtoull(argv[5], nullptr, 0), static_cast<unsigned>(std::strtoul(argv[6], nullptr, 0)),
                std::atof(argv[7]));
  std::fprintf(stderr, "usage: philox_host swar | mask B H T seed offset p\n");
  return 2;
}
