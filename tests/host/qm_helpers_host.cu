// Host-side checks of the integer helpers of the mask/code passes (quant_mask.cuh),
// against their definitions written out independently here:
//   ternary code  = clamp(rint(fp32(w / gamma)), -1, 1)  (BitNet b1.58 2B4T article, section 一)
//   keep bits     = the N largest |w| of each group of M, the lower index winning ties
//                   (Sparse-BitNet article, sections 五 and 六)
//   2-bit packing = code j of a byte at bits 2j, +1 -> 01, -1 -> 11, 0 -> 00
//                   (BitNet b1.58 2B4T article, section 四)
//   byte permute  = the PTX prmt.b32 default mode (selector bit 3 replicates the sign)
// Prints "OK <checks>" and exits 0, or prints the first mismatches and exits 1.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>

#include "../../sparsity_step_b200/csrc/quant_mask.cuh"

static long g_bad = 0, g_checks = 0;
#define CHECK(cond, ...)                    \
  do {                                      \
    ++g_checks;                             \
    if (!(cond)) {                          \
      if (g_bad++ < 10) {                   \
        std::printf(__VA_ARGS__);           \
        std::printf("\n");                  \
      }                                     \
    }                                       \
  } while (0)

static uint32_t u_of(float f) { uint32_t u; std::memcpy(&u, &f, 4); return u; }

static int8_t ternary(float w, float gamma) {
  const float q = std::rint(w / gamma);   // IEEE fp32 division, round half to even
  return static_cast<int8_t>(q > 1.0f ? 1.0f : (q < -1.0f ? -1.0f : q));
}

static uint32_t prmt_ref(uint32_t x, uint32_t y, uint32_t sel) {
  uint8_t in[8];
  for (int i = 0; i < 4; ++i) { in[i] = (x >> (8 * i)) & 0xFF; in[4 + i] = (y >> (8 * i)) & 0xFF; }
  uint32_t r = 0;
  for (int k = 0; k < 4; ++k) {
    const unsigned s = (sel >> (4 * k)) & 0xF;
    uint8_t b = in[s & 7];
    if (s & 8) b = (b & 0x80) ? 0xFF : 0x00;
    r |= static_cast<uint32_t>(b) << (8 * k);
  }
  return r;
}

// keep bits by ranking: element j is kept when fewer than N others outrank it
static uint32_t keep_ref(const float* w, int M, int N) {
  uint32_t keep = 0;
  for (int j = 0; j < M; ++j) {
    int above = 0;
    for (int i = 0; i < M; ++i) {
      if (i == j) continue;
      const float ai = std::fabs(w[i]), aj = std::fabs(w[j]);
      if (ai > aj || (ai == aj && i < j)) ++above;
    }
    if (above < N) keep |= 1u << j;
  }
  return keep;
}

template <int M, int NK>
static void check_keep(std::mt19937& rng) {
  std::uniform_int_distribution<int> small(0, 3);
  std::normal_distribution<float> nd(0.0f, 0.02f);
  for (int it = 0; it < 20000; ++it) {
    float w[8];
    for (int j = 0; j < 8; ++j) {
      // many ties: values from a tiny set half of the time, either sign
      w[j] = (it & 1) ? nd(rng) : 0.25f * small(rng) * (small(rng) & 1 ? -1.0f : 1.0f);
    }
    uint32_t b[8];
    for (int j = 0; j < 8; ++j) b[j] = u_of(w[j]);
    const uint32_t got = bl::qm_keep8<M, NK>(b, NK);
    uint32_t ref = keep_ref(w, M, NK);
    if (M == 4) ref |= keep_ref(w + 4, M, NK) << 4;
    CHECK(got == ref, "keep %d:%d it %d: got %02x want %02x", NK, M, it, got, ref);
    if (M == 8 && NK == 6) {   // runtime-N path (NK = 0) agrees for every N
      for (int n = 1; n <= 8; ++n) {
        uint32_t a[8];
        for (int j = 0; j < 8; ++j) a[j] = b[j] & 0x7fffffffu;
        const uint32_t g2 = bl::group_keep<8, 0, 0>(a, n);
        CHECK(g2 == keep_ref(w, 8, n), "runtime keep %d:8 it %d", n, it);
      }
    }
  }
}

int main() {
  std::mt19937 rng(12345);
  // byte permute, every selector nibble value in every position
  for (int it = 0; it < 4096; ++it) {
    const uint32_t x = rng(), y = rng(), sel = rng() & 0xFFFFu;
    CHECK(bl::qm_prmt(x, y, sel) == prmt_ref(x, y, sel), "prmt %08x %08x %04x", x, y, sel);
  }
  // ternary code words: random weights around +-gamma/2, exact boundary values, large values
  std::normal_distribution<float> nd(0.0f, 0.05f);
  for (int it = 0; it < 200000; ++it) {
    const float gamma = std::fabs(nd(rng)) + 1e-5f;
    const float half = 0.5f * gamma;
    float w[4];
    for (int j = 0; j < 4; ++j) {
      switch ((it + j) % 6) {
        case 0: w[j] = half; break;
        case 1: w[j] = -half; break;
        case 2: w[j] = std::nextafter(half, 1.0f) * ((it & 1) ? -1.0f : 1.0f); break;
        case 3: w[j] = std::nextafter(half, 0.0f); break;
        case 4: w[j] = nd(rng) * 50.0f; break;
        default: w[j] = nd(rng); break;
      }
    }
    uint32_t b[4], a[4];
    for (int j = 0; j < 4; ++j) { b[j] = u_of(w[j]); a[j] = b[j] & 0x7fffffffu; }
    const uint32_t word = bl::qm_code_word(b, a, u_of(half));
    for (int j = 0; j < 4; ++j) {
      const int8_t got = static_cast<int8_t>((word >> (8 * j)) & 0xFF);
      CHECK(got == ternary(w[j], gamma), "code w=%a gamma=%a: got %d want %d", w[j], gamma, got, ternary(w[j], gamma));
    }
  }
  // 2-bit packing of every pair of code words over {+1, -1, 0}
  const uint8_t vals[3] = {0x00, 0x01, 0xFF};
  for (int c = 0; c < 6561; ++c) {   // 3^8
    uint32_t lo = 0, hi = 0, want = 0;
    int x = c;
    for (int j = 0; j < 8; ++j) {
      const int v = x % 3;
      x /= 3;
      (j < 4 ? lo : hi) |= static_cast<uint32_t>(vals[v]) << (8 * (j & 3));
      want |= static_cast<uint32_t>(v == 0 ? 0 : (v == 1 ? 1 : 3)) << (2 * j);
    }
    CHECK(bl::qm_pack16(lo, hi) == want, "pack %08x %08x: got %04x want %04x", lo, hi, bl::qm_pack16(lo, hi), want);
  }
  // 2:4 metadata nibble: the kept positions completed with the lowest unused ones
  for (uint32_t kb = 0; kb < 16; ++kb) {
    if (__builtin_popcount(kb) > 2) continue;
    uint32_t f = kb;
    for (int p = 0; p < 4 && __builtin_popcount(f) < 2; ++p) f |= (f >> p & 1u) ? 0u : (1u << p);
    int i0 = -1, i1 = -1;
    for (int p = 0; p < 4; ++p)
      if (f >> p & 1u) (i0 < 0 ? i0 : i1) = p;
    CHECK(bl::sp24_nibble(kb) == static_cast<uint32_t>(i0 | (i1 << 2)), "sp24 nibble %x", kb);
  }
  check_keep<8, 8>(rng); check_keep<8, 7>(rng); check_keep<8, 6>(rng); check_keep<8, 5>(rng);
  check_keep<8, 4>(rng); check_keep<8, 3>(rng); check_keep<8, 2>(rng); check_keep<8, 1>(rng);
  check_keep<4, 4>(rng); check_keep<4, 3>(rng); check_keep<4, 2>(rng); check_keep<4, 1>(rng);
  if (g_bad) {
    std::printf("FAIL %ld of %ld\n", g_bad, g_checks);
    return 1;
  }
  std::printf("OK %ld\n", g_checks);
  return 0;
}
