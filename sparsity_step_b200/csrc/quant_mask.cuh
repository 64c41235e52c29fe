// Steps a1 + a2 of the BitLinear path: absmean scale, N:M mask, ternary codes.
//
// Sparse-BitNet article (m.top168.com), section 三: the mask is recomputed at every
// training step; section 五: one threshold per group of 8 weights; section 六:
// quantise first, then sparsify, and rank on the full-precision latent weights.
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 一: absmean quantisation to
// {-1, 0, +1}; section 四: four ternary values packed per byte.
//
// Two launches, both streaming W (one thread = 8 contiguous weights = one group of 8 or
// two groups of 4; a warp covers 1 KB contiguous; two groups per thread in flight):
//   qm_sum_mask_kernel : exact integer sum of floor(|w| * 2^32) per block; when the
//                        caller wants the mask, also the top-N keep bits (knock-out
//                        tournaments; the mask needs no gamma), stored to the mask
//                        output. The last block adds the partials (128-bit), rounds
//                        S / (n * 2^32) once to fp32 and writes gamma = mean + 1e-5.
//   qm_codes_kernel    : walks W in reverse (pass 1's last lines, still in L2, first),
//                        reads the keep bits back (or ranks the group itself when no
//                        mask output is wanted), and writes the ternary codes (integer
//                        arithmetic on the bit patterns), their 2-bit packing, the
//                        optional int8 weights and the optional 2:4 form.
// Ranking in pass 1 puts the ALU-heavy tournaments in the pass that is otherwise bound
// by memory latency, and leaves pass 2 a short stream of loads, byte permutes and stores.
#pragma once

#include "common.cuh"

namespace bl {

// Workspace layout (bytes): [0,4) range flag, [4,8) status, [8,12) blocks done,
// [12,16) reserved, [256, 256 + 16 * blocks) per-block 128-bit partial sums (lo, hi).
// The first 16 bytes must be zero when a call starts (the host clears them).
constexpr size_t kQmWsHeader = 256;
constexpr int kQmThreads = 256;
constexpr int64_t kQmMaxElemsPerThread = 1 << 14;   // keeps a thread's u64 sum < 2^62

struct QmScratch {
  unsigned int* range_flag;
  int* status;
  unsigned int* done;
  unsigned long long* partials;
};


// 16-byte read-only loads without L1 allocation (W is read once per pass); `ok` false
// gives zeros without a load.
__device__ __forceinline__ uint4 ld_nc_u4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
struct QmPair {   // the 8 weights of one thread step (bit patterns)
  uint4 lo, hi;
};
__device__ __forceinline__ QmPair qm_load(const uint4* w4, int64_t g, bool ok) {
  QmPair v{make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
  if (ok) {
    v.lo = ld_nc_u4(w4 + 2 * g);
    v.hi = ld_nc_u4(w4 + 2 * g + 1);
  }
  return v;
}

// floor(|w| * 2^32) of 8 weights into the thread's sum: |w| * 2^32 is exact (a power-of-
// two scale, < 2^48 for |w| < 2^16) and truncation toward zero is the floor; the eight
// terms are added as a tree (short dependency chains). Range: |w| >= 2^16, inf and NaN
// are exactly the |w| patterns >= 0x47800000, i.e. those whose sum with 0x38800000
// reaches bit 31 (no overflow below 2^31 + 0x38800000); `bad` collects bit 31 of those
// sums, tested after the loop.
__device__ __forceinline__ void qm_accumulate8(const uint32_t (&b)[8], uint64_t& acc, uint32_t& bad) {
  uint64_t u[8];
  uint32_t r = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t a = b[j] & 0x7fffffffu;
    r |= a + 0x38800000u;
    u[j] = __float2ull_rz(__uint_as_float(a) * 4294967296.0f);
  }
  bad |= r;
  acc += ((u[0] + u[1]) + (u[2] + u[3])) + ((u[4] + u[5]) + (u[6] + u[7]));
}

__device__ float rn_f32_ratio_u128(uint64_t slo, uint64_t shi, int64_t numel);

// Block-reduce a 128-bit value held by every thread; the result is valid in thread 0.
__device__ __forceinline__ void block_sum_u128(uint64_t& lo, uint64_t& hi) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t lo2 = __shfl_xor_sync(0xffffffffu, lo, off);
    const uint64_t hi2 = __shfl_xor_sync(0xffffffffu, hi, off);
    add_u128(lo, hi, lo2, hi2);
  }
  __shared__ uint64_t s_lo[32], s_hi[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();   // s_lo/s_hi may be reused by a previous call in this block
  if (lane == 0) {
    s_lo[warp] = lo;
    s_hi[warp] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t blo = 0, bhi = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) add_u128(blo, bhi, s_lo[w], s_hi[w]);
    lo = blo;
    hi = bhi;
  }
}

// ---- exact rounding of S / D to fp32 (round to nearest, ties to even) ----------
// S, D are unsigned 128-bit integers with 0 < D < 2^100 and S < 2^100. Long
// division produces a 26..27-bit quotient plus a remainder (the sticky bit); the
// mantissa is then rounded half-to-even and scaled by an exact power of two.

struct U128 {
  uint64_t lo, hi;
};

__device__ __forceinline__ int bitlen_u128(U128 v) {
  if (v.hi) return 128 - __clzll(static_cast<long long>(v.hi));
  if (v.lo) return 64 - __clzll(static_cast<long long>(v.lo));
  return 0;
}
__device__ __forceinline__ U128 shl_u128(U128 v, int s) {
  if (s == 0) return v;
  if (s >= 64) return U128{0, v.lo << (s - 64)};
  return U128{v.lo << s, (v.hi << s) | (v.lo >> (64 - s))};
}
__device__ __forceinline__ bool ge_u128(U128 a, U128 b) { return a.hi > b.hi || (a.hi == b.hi && a.lo >= b.lo); }
__device__ __forceinline__ U128 sub_u128(U128 a, U128 b) {
  return U128{a.lo - b.lo, a.hi - b.hi - (a.lo < b.lo ? 1ull : 0ull)};
}

__device__ float rn_f32_ratio(U128 s, U128 d) {
  if (s.lo == 0 && s.hi == 0) return 0.0f;
  const int sh = 26 - (bitlen_u128(s) - bitlen_u128(d));   // s * 2^sh / d in [2^25, 2^27)
  U128 num = s, den = d;
  if (sh >= 0) num = shl_u128(num, sh);
  else den = shl_u128(den, -sh);
  // restoring long division; the quotient has at most 27 bits
  uint64_t q = 0;
  U128 rem = num;
  for (int b = 27; b >= 0; --b) {
    const U128 t = shl_u128(den, b);
    if (bitlen_u128(den) + b <= 127 && ge_u128(rem, t)) {
      rem = sub_u128(rem, t);
      q |= 1ull << b;
    }
  }
  const bool rem_nonzero = (rem.lo | rem.hi) != 0;
  const int drop = (q >= (1ull << 26)) ? 3 : 2;
  uint64_t m = q >> drop;
  const uint64_t guard = (q >> (drop - 1)) & 1ull;
  const bool sticky = ((q & ((1ull << (drop - 1)) - 1ull)) != 0) || rem_nonzero;
  if (guard && (sticky || (m & 1ull))) ++m;
  int e = drop - sh;
  if (m == (1ull << 24)) {
    m >>= 1;
    ++e;
  }
  return ldexpf(static_cast<float>(m), e);   // exact: 24-bit mantissa, normal range
}

// mean = S / (numel * 2^32), rounded once to fp32.
__device__ float rn_f32_ratio_u128(uint64_t slo, uint64_t shi, int64_t numel) {
  const U128 den = shl_u128(U128{static_cast<uint64_t>(numel), 0}, 32);
  return rn_f32_ratio(U128{slo, shi}, den);
}


// ---- integer helpers of the mask/code passes (host-callable, so that host tests can
// check them against brute force) ---------------------------------------------------

// Byte permute with the full PTX semantics: selector nibble bits 0-2 pick one of the
// eight bytes of {y, x} (x = bytes 0-3), bit 3 replicates the picked byte's sign bit
// over the result byte.
__host__ __device__ __forceinline__ uint32_t qm_prmt(uint32_t x, uint32_t y, uint32_t sel) {
#ifdef __CUDA_ARCH__
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(y), "r"(sel));
  return r;
#else
  const uint64_t v = (static_cast<uint64_t>(y) << 32) | x;
  uint32_t r = 0;
  for (int k = 0; k < 4; ++k) {
    const uint32_t s = (sel >> (4 * k)) & 0xFu;
    uint32_t byte = static_cast<uint32_t>((v >> (8 * (s & 7u))) & 0xFFu);
    if (s & 8u) byte = (byte & 0x80u) ? 0xFFu : 0x00u;
    r |= byte << (8 * k);
  }
  return r;
#endif
}
__host__ __device__ __forceinline__ int qm_popc(uint32_t x) {
#ifdef __CUDA_ARCH__
  return __popc(x);
#else
  return __builtin_popcount(x);
#endif
}
__host__ __device__ __forceinline__ uint32_t qm_lowest_bit(uint32_t x) {   // x != 0
#ifdef __CUDA_ARCH__
  return static_cast<uint32_t>(__ffs(x) - 1);
#else
  return static_cast<uint32_t>(__builtin_ctz(x));
#endif
}
__host__ __device__ __forceinline__ uint32_t qm_highest_bit(uint32_t x) {   // x != 0
#ifdef __CUDA_ARCH__
  return 31u - static_cast<uint32_t>(__clz(x));
#else
  return 31u - static_cast<uint32_t>(__builtin_clz(x));
#endif
}

// Index (0..M-1) of the weakest of M magnitudes (bit patterns of |w|): the smallest;
// among equal magnitudes the higher index is weaker (the lower index wins ties). A
// knock-out tournament: every comparison sets a lower-index subtree against a
// higher-index one, so letting the higher one win on "<=" applies the tie rule.
template <int M>
__host__ __device__ __forceinline__ int qm_weakest(const uint32_t (&g)[M]) {
  uint32_t v[M];
  int id[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    v[j] = g[j];
    id[j] = j;
  }
#pragma unroll
  for (int w = 1; w < M; w <<= 1) {
#pragma unroll
    for (int j = 0; j < M; j += 2 * w) {
      const bool upper = v[j + w] <= v[j];
      v[j] = upper ? v[j + w] : v[j];
      id[j] = upper ? id[j + w] : id[j];
    }
  }
  return id[0];
}

// Index of the strongest (largest; the lower index wins ties). Knocked-out entries
// hold -1, below every magnitude.
template <int M>
__host__ __device__ __forceinline__ int qm_strongest(const int32_t (&g)[M]) {
  int32_t v[M];
  int id[M];
#pragma unroll
  for (int j = 0; j < M; ++j) {
    v[j] = g[j];
    id[j] = j;
  }
#pragma unroll
  for (int w = 1; w < M; w <<= 1) {
#pragma unroll
    for (int j = 0; j < M; j += 2 * w) {
      const bool upper = v[j + w] > v[j];
      v[j] = upper ? v[j + w] : v[j];
      id[j] = upper ? id[j + w] : id[j];
    }
  }
  return id[0];
}

// Keep-mask of one group of M (weights [G0, G0+M) of the 8 held by the thread), bit
// G0 + j for element j. Element j outranks i when |w_j| > |w_i|, or they are equal and
// j < i. NK > 0: compile-time N; NK >= M/2 drops the M - NK weakest (one tournament
// each, the loser knocked out by setting bit 31, above every |w| pattern), NK < M/2
// keeps the NK strongest the same way. NK == 0: runtime N via rank counting.
template <int M, int NK, int G0>
__host__ __device__ __forceinline__ uint32_t group_keep(const uint32_t (&a)[8], int n_keep) {
  constexpr uint32_t all = (1u << M) - 1u;
  if (NK == M) return all << G0;
  if (NK > 0 && 2 * NK >= M) {
    uint32_t g[M];
#pragma unroll
    for (int j = 0; j < M; ++j) g[j] = a[G0 + j];
    uint32_t dropped = 0;
#pragma unroll
    for (int r = 0; r < M - NK; ++r) {
      const int d = qm_weakest<M>(g);
      dropped |= 1u << d;
      if (r + 1 < M - NK) {
#pragma unroll
        for (int j = 0; j < M; ++j) g[j] |= (j == d) ? 0x80000000u : 0u;
      }
    }
    return (all & ~dropped) << G0;
  }
  if (NK > 0) {
    int32_t g[M];
#pragma unroll
    for (int j = 0; j < M; ++j) g[j] = static_cast<int32_t>(a[G0 + j]);
    uint32_t kept = 0;
#pragma unroll
    for (int r = 0; r < NK; ++r) {
      const int k = qm_strongest<M>(g);
      kept |= 1u << k;
      if (r + 1 < NK) {
#pragma unroll
        for (int j = 0; j < M; ++j) g[j] = (j == k) ? -1 : g[j];
      }
    }
    return kept << G0;
  }
  uint32_t keep = 0;
#pragma unroll
  for (int j = 0; j < M; ++j) {
    int rank = 0;
#pragma unroll
    for (int t = 0; t < M; ++t) {
      if (t == j) continue;
      rank += (t < j) ? (a[G0 + t] >= a[G0 + j] ? 1 : 0) : (a[G0 + t] > a[G0 + j] ? 1 : 0);
    }
    keep |= (rank < n_keep ? 1u : 0u) << j;
  }
  return keep << G0;
}

// Ternary code of one weight. Equivalent, bit for bit, to
// clamp(rint(fp32(w / gamma)), -1, 1) for every finite w and normal gamma > 0:
// the correctly rounded quotient exceeds 0.5 exactly when |w| / gamma exceeds
// 0.5 * (1 + 2^-24) (0.5 + 2^-25 is the midpoint to the next float and ties go to
// the even 0.5), and no fp32 lies in (0.5 * gamma, 0.5 * gamma * (1 + 2^-24)] since
// the spacing just above 0.5 * gamma is at least 0.5 * gamma * 2^-23 ... 2^-24 with
// strict inequality (mantissa < 2^24). Quotients >= 1.5 round to 2 and clip to 1.
// So code = sign(w) when |w| > 0.5 * gamma (0.5 * gamma exact in fp32), else 0;
// on the bit patterns of non-negative floats the comparison is an unsigned compare.
//
// Four codes as int8 bytes (+1, -1, 0) of weights b[0..3] (bit patterns; a = |w|
// patterns): half - a is negative exactly when |w| > gamma/2 (both below 2^31); byte
// permutes with sign replication turn the four sign bits of (half - a) into a byte mask
// `mag` and the four sign bits of w into a byte mask `neg`; code = mag & (neg | 0x01).
__host__ __device__ __forceinline__ uint32_t qm_code_word(const uint32_t* b, const uint32_t* a, uint32_t half_bits) {
  const uint32_t t0 = half_bits - a[0], t1 = half_bits - a[1], t2 = half_bits - a[2], t3 = half_bits - a[3];
  const uint32_t mag = qm_prmt(qm_prmt(t0, t1, 0x00FBu), qm_prmt(t2, t3, 0xFB00u), 0x7610u);
  const uint32_t neg = qm_prmt(qm_prmt(b[0], b[1], 0x00FBu), qm_prmt(b[2], b[3], 0xFB00u), 0x7610u);
  return mag & (neg | 0x01010101u);
}

// Four keep bits -> a byte mask (0xFF for each kept byte): bit j moves to bit 8j
// (shifts 0, 7, 14, 21 of a 4-bit value never overlap), then 0x01 -> 0xFF per byte.
__host__ __device__ __forceinline__ uint32_t qm_keep_bytes(uint32_t k4) {
  return ((k4 * 0x00204081u) & 0x01010101u) * 0xFFu;
}

// Two int8 code words (bytes +1 / -1 / 0; lo = elements 0-3, hi = 4-7) -> their eight
// 2-bit codes (01 / 11 / 00), element j at bits 2j. The low two bits of each byte are
// the code; one multiply gathers the four fields of a word into its top byte (field k
// moves from bit 8k to bit 24 + 2k; every other partial product lands below bit 24 in a
// field of its own, so no carry reaches the top byte), and a byte permute joins the two.
__host__ __device__ __forceinline__ uint32_t qm_pack16(uint32_t lo, uint32_t hi) {
  const uint32_t x = (lo & 0x03030303u) * 0x01041040u;
  const uint32_t y = (hi & 0x03030303u) * 0x01041040u;
  return qm_prmt(x, y, 0x0073u) & 0xFFFFu;
}

// 2:4 storage of one group of four (keep nibble kb, at most two bits set): the two
// stored positions i0 < i1 are the kept ones, completed with the lowest unused
// positions. Returns i0 | i1 << 2 (the metadata nibble).
__host__ __device__ __forceinline__ uint32_t sp24_nibble(uint32_t kb) {
  uint32_t f = kb;
#pragma unroll
  for (int r = 0; r < 2; ++r)
    if (qm_popc(f) < 2) f |= ~f & (f + 1u);   // add the lowest clear position
  const uint32_t i0 = qm_lowest_bit(f), i1 = qm_highest_bit(f);
  return i0 | (i1 << 2);
}

// Keep bits of the thread's 8 weights (bit patterns b; |w| patterns are order-
// preserving): one group of 8, or two groups of 4.
template <int M, int NK>
__host__ __device__ __forceinline__ uint32_t qm_keep8(const uint32_t (&b)[8], int n_keep) {
  uint32_t a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = b[j] & 0x7fffffffu;
  uint32_t keep = group_keep<M, NK, 0>(a, n_keep);
  if (M == 4) keep |= group_keep<M, NK, 4>(a, n_keep);
  return keep;
}

// Everything pass 2 derives from 8 contiguous weights and their keep bits: the masked
// int8 codes (lo = elements 0-3, hi = 4-7), the packed 2-bit codes, and the 2:4 form
// (values word and metadata byte).
struct QmCodes8 {
  uint32_t lo, hi, packed, sp_values, sp_meta;
};

template <bool kSp>
__host__ __device__ __forceinline__ QmCodes8 qm_codes8(const uint32_t (&b)[8], uint32_t keep, uint32_t half_gamma_bits,
                                                       bool gamma_ok) {
  uint32_t a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = b[j] & 0x7fffffffu;
  QmCodes8 r;
  const uint32_t code_keep = gamma_ok ? keep : 0u;   // range error: all codes 0 (gamma is NaN)
  r.lo = qm_code_word(b, a, half_gamma_bits) & qm_keep_bytes(code_keep & 0xFu);
  r.hi = qm_code_word(b + 4, a + 4, half_gamma_bits) & qm_keep_bytes(code_keep >> 4);
  r.packed = qm_pack16(r.lo, r.hi);
  r.sp_values = r.sp_meta = 0;
  if (kSp) {
    // 2:4 form (meaningful for masks with at most two kept per aligned four): masked
    // codes are 0 at unkept positions, so one byte permute picks each group's two values
    const uint32_t n0 = sp24_nibble(keep & 0xFu), n1 = sp24_nibble((keep >> 4) & 0xFu);
    r.sp_values =
        qm_prmt(r.lo, r.hi, (n0 & 3u) | ((n0 >> 2) << 4) | ((4u + (n1 & 3u)) << 8) | ((4u + (n1 >> 2)) << 12));
    r.sp_meta = n0 | (n1 << 4);
  }
  return r;
}

// Optimizer step of the latent weights fused into pass 1 (kUpdate): W <- fp32(W - lr * G)
// with G the bf16 gradient, one fused multiply-add (a single rounding) per weight; the
// updated weights are stored back and summed and ranked in the same pass, so the mask
// recompute costs no extra read of W. Loads of W then use the coherent path (the kernel
// writes W). `step` holds the 8 weights of one thread step and their 8 gradients.
struct QmStepIn {
  QmPair w;
  uint4 g;
};
template <bool kUpdate>
__device__ __forceinline__ QmStepIn qm_load_step(const uint4* w4, const uint4* g4, int64_t g, bool ok) {
  QmStepIn v{{make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)}, make_uint4(0, 0, 0, 0)};
  if (!kUpdate) {
    v.w = qm_load(w4, g, ok);
  } else if (ok) {
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.w.lo.x), "=r"(v.w.lo.y), "=r"(v.w.lo.z), "=r"(v.w.lo.w)
                 : "l"(w4 + 2 * g));
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.w.hi.x), "=r"(v.w.hi.y), "=r"(v.w.hi.z), "=r"(v.w.hi.w)
                 : "l"(w4 + 2 * g + 1));
    v.g = ld_nc_u4(g4 + g);
  }
  return v;
}

// Pass 1: exact integer sum of floor(|w| * 2^32) and, with kMask, the keep bits of
// every group stored to `mask`. Each block stores its partial sum; the last block to
// finish (atomic ticket) adds all partials, rounds the mean once to fp32, writes
// gamma = mean + 1e-5 (NaN and status BL_ERR_RANGE on a range error) and clears the
// ticket and the flag for the next call. Two thread steps are in flight per thread
// (register double buffer; loads past the end give zeros, which add nothing). With
// kUpdate, `w4` is updated in place first (see above).
template <int M, int NK, bool kMask, bool kUpdate>
__global__ void __launch_bounds__(kQmThreads) qm_sum_mask_kernel(const uint4* w4, int64_t n8,
                                                                  int64_t numel, int n_keep, QmScratch ws,
                                                                  float* __restrict__ gamma_out,
                                                                  uint8_t* __restrict__ mask, uint4* w4_out,
                                                                  const uint4* __restrict__ g4, float lr) {
  static_assert(M == 4 || M == 8, "groups of 4 or 8");
  uint64_t acc = 0;
  uint32_t bad = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float neg_lr = -lr;
  auto step = [&](const QmStepIn& v, int64_t g) {
    uint32_t b[8] = {v.w.lo.x, v.w.lo.y, v.w.lo.z, v.w.lo.w, v.w.hi.x, v.w.hi.y, v.w.hi.z, v.w.hi.w};
    if (kUpdate) {
      const uint32_t gw[4] = {v.g.x, v.g.y, v.g.z, v.g.w};   // bf16 pairs: element 2i low, 2i+1 high
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float gj = __uint_as_float((j & 1) ? (gw[j >> 1] & 0xffff0000u) : (gw[j >> 1] << 16));
        b[j] = __float_as_uint(__fmaf_rn(neg_lr, gj, __uint_as_float(b[j])));
      }
      w4_out[2 * g] = make_uint4(b[0], b[1], b[2], b[3]);
      w4_out[2 * g + 1] = make_uint4(b[4], b[5], b[6], b[7]);
    }
    qm_accumulate8(b, acc, bad);
    if (kMask) {
      const uint32_t keep = qm_keep8<M, NK>(b, n_keep);
      if (M == 8) mask[g] = static_cast<uint8_t>(keep);
      else reinterpret_cast<uint16_t*>(mask)[g] = static_cast<uint16_t>((keep & 0xFu) | ((keep >> 4) << 8));
    }
  };
  int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  QmStepIn va = qm_load_step<kUpdate>(w4, g4, g, g < n8), vb;
  for (; g < n8; g += 2 * stride) {
    vb = qm_load_step<kUpdate>(w4, g4, g + stride, g + stride < n8);
    step(va, g);
    if (g + stride >= n8) break;
    va = qm_load_step<kUpdate>(w4, g4, g + 2 * stride, g + 2 * stride < n8);
    step(vb, g + stride);
  }
  if (bad & 0x80000000u) atomicOr(ws.range_flag, 1u);   // |w| >= 2^16, inf or NaN

  uint64_t lo = acc, hi = 0;
  block_sum_u128(lo, hi);
  __shared__ bool s_last;
  if (threadIdx.x == 0) {
    ws.partials[2 * blockIdx.x] = lo;
    ws.partials[2 * blockIdx.x + 1] = hi;
    __threadfence();   // the partial is visible before the ticket is taken
    s_last = atomicAdd(ws.done, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  lo = 0;
  hi = 0;
  for (int b = threadIdx.x; b < static_cast<int>(gridDim.x); b += blockDim.x)
    add_u128(lo, hi, __ldcg(ws.partials + 2 * b), __ldcg(ws.partials + 2 * b + 1));
  block_sum_u128(lo, hi);
  if (threadIdx.x != 0) return;
  const unsigned int flag = atomicAdd(ws.range_flag, 0u);
  *ws.range_flag = 0;   // leave the scratch ready for the next call
  *ws.done = 0;
  if (flag) {
    *ws.status = -4;   // BL_ERR_RANGE
    *gamma_out = __int_as_float(0x7fc00000);
    return;
  }
  *ws.status = 0;
  *gamma_out = __fadd_rn(rn_f32_ratio_u128(lo, hi, numel), 1e-5f);   // one fp32 add
}

// Pass 2 of steps a1 + a2. One thread = 8 contiguous weights. Walks W in reverse
// (grid-stride from the end) so that the lines pass 1 read last, still in L2, are read
// first. kMaskIn: the keep bits come from pass 1 through `mask`; otherwise (no mask
// output wanted) they are ranked here and `mask` is unused. kSp: also the 2:4 form
// (the host allows it only for 2:4-valid masks).
template <int M, int NK, bool kMaskIn, bool kSp>
__global__ void __launch_bounds__(kQmThreads) qm_codes_kernel(const uint4* __restrict__ w4, int64_t n8, int n_keep,
                                                              const float* __restrict__ gamma_ptr,
                                                              const uint8_t* __restrict__ mask,
                                                              uint16_t* __restrict__ codes_out,
                                                              uint2* __restrict__ w_i8_out,
                                                              uint32_t* __restrict__ sp_values_out,
                                                              uint8_t* __restrict__ sp_meta_out, int64_t k8,
                                                              int64_t meta_pitch) {
  static_assert(M == 4 || M == 8, "groups of 4 or 8");
  const float gamma = *gamma_ptr;
  const bool gamma_ok = isfinite(gamma) && gamma > 0.0f;
  const uint32_t half_gamma_bits = __float_as_uint(0.5f * gamma);   // 0.5 * gamma is exact
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  // the padded metadata has a row pitch of meta_pitch bytes: track this thread's (row,
  // column) of the k8 bytes per row, stepping back by `stride` without dividing
  int64_t mrow = 0, mcol = 0, sq = 0, sr = 0;
  if (kSp && tid < n8) {
    mrow = (n8 - 1 - tid) / k8;
    mcol = (n8 - 1 - tid) % k8;
    sq = stride / k8;
    sr = stride % k8;
  }
  auto load_keep = [&](int64_t i, bool ok) -> uint32_t {
    if (!kMaskIn || !ok) return 0u;
    if (M == 8) return mask[i];
    const uint32_t m2 = reinterpret_cast<const uint16_t*>(mask)[i];
    return (m2 & 0xFu) | ((m2 >> 8) << 4);
  };
  auto step = [&](const QmPair& v, uint32_t keep, int64_t i) {
    const uint32_t b[8] = {v.lo.x, v.lo.y, v.lo.z, v.lo.w, v.hi.x, v.hi.y, v.hi.z, v.hi.w};
    if (!kMaskIn) keep = qm_keep8<M, NK>(b, n_keep);
    const QmCodes8 c = qm_codes8<kSp>(b, keep, half_gamma_bits, gamma_ok);
    codes_out[i] = static_cast<uint16_t>(c.packed);
    if (w_i8_out != nullptr) w_i8_out[i] = make_uint2(c.lo, c.hi);
    if (kSp) {
      sp_values_out[i] = c.sp_values;
      sp_meta_out[mrow * meta_pitch + mcol] = static_cast<uint8_t>(c.sp_meta);
      mcol -= sr;
      mrow -= sq;
      if (mcol < 0) {
        mcol += k8;
        mrow -= 1;
      }
    }
  };
  // thread step r covers group index i = n8 - 1 - r; two steps in flight per thread
  int64_t r = tid;
  QmPair va = qm_load(w4, n8 - 1 - r, r < n8), vb;
  uint32_t ka = load_keep(n8 - 1 - r, r < n8), kb;
  for (; r < n8; r += 2 * stride) {
    const int64_t r1 = r + stride, r2 = r + 2 * stride;
    vb = qm_load(w4, n8 - 1 - r1, r1 < n8);
    kb = load_keep(n8 - 1 - r1, r1 < n8);
    step(va, ka, n8 - 1 - r);
    if (r1 >= n8) break;
    va = qm_load(w4, n8 - 1 - r2, r2 < n8);
    ka = load_keep(n8 - 1 - r2, r2 < n8);
    step(vb, kb, n8 - 1 - r1);
  }
}

}  // namespace bl
