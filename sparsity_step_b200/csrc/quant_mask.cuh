// Steps a1 + a2 of the BitLinear path: absmean scale, N:M mask, ternary codes.
//
// Sparse-BitNet article (m.top168.com), section 三: the mask is recomputed at every
// training step; section 五: one threshold per group of 8 weights; section 六:
// quantise first, then sparsify, and rank on the full-precision latent weights.
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 一: absmean quantisation to
// {-1, 0, +1}; section 四: four ternary values packed per byte.
//
// Two launches, both HBM-bound:
//   qm_abs_sum_kernel   : grid-stride read of W (four 16-byte loads in flight per
//                         thread), per-block exact integer sum of floor(|w| * 2^32);
//                         the last block adds the partials (128-bit), rounds
//                         S / (n * 2^32) once to fp32 and writes gamma = mean + 1e-5.
//   qm_mask_codes_kernel: one thread per 8 contiguous weights (two 16-byte loads,
//                         a warp covers 1 KB contiguous), walking W in reverse so
//                         that pass 1's last lines, still in L2, come first; top-N
//                         mask by knock-out tournaments, ternary codes by integer
//                         arithmetic on the bit patterns, 2-bit packing, optional
//                         int8 weights and 2:4 form.
#pragma once

#include "common.cuh"

namespace bl {

// Workspace layout (bytes): [0,4) range flag, [4,8) status, [8,12) blocks done,
// [12,16) reserved, [256, 256 + 16 * blocks) per-block 128-bit partial sums (lo, hi).
// The first 16 bytes must be zero when a call starts (the host clears them).
constexpr size_t kQmWsHeader = 256;
constexpr int kQmThreads = 256;
constexpr int kQmUnroll = 4;                        // 16-byte loads in flight per thread
constexpr int64_t kQmMaxElemsPerThread = 1 << 14;   // keeps a thread's u64 sum < 2^62
constexpr float kAbsLimit = 65536.0f;              // |w| < 2^16 is summed exactly

struct QmScratch {
  unsigned int* range_flag;
  int* status;
  unsigned int* done;
  unsigned long long* partials;
};

// 16-byte read-only loads without L1 allocation (W is read once per pass).
__device__ __forceinline__ float4 ld_nc_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_nc_u4(const float4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void qm_accumulate(const float4& v, uint64_t& acc, bool& bad) {
  const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = fabsf(e[j]);
    if (a < kAbsLimit) {
      // a * 2^32 is exact (power-of-two scale, < 2^48); truncation toward zero is floor
      acc += __float2ull_rz(a * 4294967296.0f);
    } else {
      bad = true;   // also catches NaN (the comparison is false)
    }
  }
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

// Pass 1: exact integer sum of floor(|w| * 2^32). Each block stores its partial; the
// last block to finish (atomic ticket) adds all partials, rounds the mean once to
// fp32, writes gamma = mean + 1e-5 (NaN and status BL_ERR_RANGE on a range error)
// and clears the ticket and the flag for the next call.
__global__ void __launch_bounds__(kQmThreads) qm_abs_sum_kernel(const float4* __restrict__ w4, int64_t n4, int64_t numel,
                                                                 QmScratch ws, float* __restrict__ gamma_out) {
  uint64_t acc = 0;
  bool bad = false;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + (kQmUnroll - 1) * stride < n4; i += kQmUnroll * stride) {
    float4 v[kQmUnroll];
#pragma unroll
    for (int u = 0; u < kQmUnroll; ++u) v[u] = ld_nc_f4(w4 + i + u * stride);
#pragma unroll
    for (int u = 0; u < kQmUnroll; ++u) qm_accumulate(v[u], acc, bad);
  }
  for (; i < n4; i += stride) qm_accumulate(ld_nc_f4(w4 + i), acc, bad);
  if (bad) atomicOr(ws.range_flag, 1u);

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


// ---- integer helpers of the mask/code pass (host-callable, so that host tests can
// check them against brute force) ---------------------------------------------------

__host__ __device__ __forceinline__ uint32_t qm_prmt(uint32_t x, uint32_t y, uint32_t sel) {
#ifdef __CUDA_ARCH__
  return __byte_perm(x, y, sel);
#else
  const uint64_t v = (static_cast<uint64_t>(y) << 32) | x;
  uint32_t r = 0;
  for (int k = 0; k < 4; ++k) r |= static_cast<uint32_t>((v >> (8 * ((sel >> (4 * k)) & 7u))) & 0xFFu) << (8 * k);
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
// patterns): m = -1 when |w| > gamma/2 (the sign of half - a, both below 2^31), s = -1
// for negative w, code byte = low byte of m & (s | 1); three byte permutes gather them.
__host__ __device__ __forceinline__ uint32_t qm_code_word(const uint32_t* b, const uint32_t* a, uint32_t half_bits) {
  uint32_t c[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t m = static_cast<uint32_t>(static_cast<int32_t>(half_bits - a[j]) >> 31);
    const uint32_t sg = static_cast<uint32_t>(static_cast<int32_t>(b[j]) >> 31);
    c[j] = m & (sg | 1u);
  }
  return qm_prmt(qm_prmt(c[0], c[1], 0x0040u), qm_prmt(c[2], c[3], 0x0040u), 0x5410u);
}

// Four keep bits -> a byte mask (0xFF for each kept byte): bit j moves to bit 8j
// (shifts 0, 7, 14, 21 of a 4-bit value never overlap), then 0x01 -> 0xFF per byte.
__host__ __device__ __forceinline__ uint32_t qm_keep_bytes(uint32_t k4) {
  return ((k4 * 0x00204081u) & 0x01010101u) * 0xFFu;
}

// int8 code word (bytes +1 / -1 / 0) -> its four 2-bit codes (01 / 11 / 00) in one byte,
// element j at bits 2j.
__host__ __device__ __forceinline__ uint32_t qm_pack2(uint32_t w) {
  uint32_t x = w & 0x03030303u;
  x |= x >> 6;
  x |= x >> 12;
  return x & 0xFFu;
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

// Everything the mask/code pass derives from 8 contiguous weights (one group of 8, or
// two groups of 4): the keep bits, the masked int8 codes (lo = elements 0-3, hi = 4-7),
// the packed 2-bit codes, and the 2:4 form (values word and metadata byte).
struct QmGroup8 {
  uint32_t keep, lo, hi, packed, sp_values, sp_meta;
};

template <int M, int NK>
__host__ __device__ __forceinline__ QmGroup8 qm_group8(const uint32_t (&b)[8], int n_keep, uint32_t half_gamma_bits,
                                                       bool gamma_ok) {
  uint32_t a[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) a[j] = b[j] & 0x7fffffffu;   // |w| bits: order-preserving
  QmGroup8 r;
  r.keep = group_keep<M, NK, 0>(a, n_keep);
  if (M == 4) r.keep |= group_keep<M, NK, 4>(a, n_keep);
  const uint32_t code_keep = gamma_ok ? r.keep : 0u;   // range error: all codes 0 (gamma is NaN)
  r.lo = qm_code_word(b, a, half_gamma_bits) & qm_keep_bytes(code_keep & 0xFu);
  r.hi = qm_code_word(b + 4, a + 4, half_gamma_bits) & qm_keep_bytes(code_keep >> 4);
  r.packed = qm_pack2(r.lo) | (qm_pack2(r.hi) << 8);
  // 2:4 form (meaningful for masks with at most two kept per aligned four): masked
  // codes are 0 at unkept positions, so one byte permute picks each group's two values
  const uint32_t n0 = sp24_nibble(r.keep & 0xFu), n1 = sp24_nibble((r.keep >> 4) & 0xFu);
  r.sp_values = qm_prmt(r.lo, r.hi, (n0 & 3u) | ((n0 >> 2) << 4) | ((4u + (n1 & 3u)) << 8) | ((4u + (n1 >> 2)) << 12));
  r.sp_meta = n0 | (n1 << 4);
  return r;
}

// Pass 2 of steps a1 + a2. One thread = 8 contiguous weights (one group of 8, or two
// groups of 4). Walks W in reverse (grid-stride from the end) so that the lines pass 1
// read last, still in L2, are read first (measured: 43 % of W from L2 for a 90 MB tensor).
template <int M, int NK>
__global__ void __launch_bounds__(kQmThreads) qm_mask_codes_kernel(const float4* __restrict__ w4, int64_t n8, int n_keep,
                                                                    const float* __restrict__ gamma_ptr,
                                                                    uint8_t* __restrict__ mask_out,
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
  if (sp_meta_out != nullptr && tid < n8) {
    mrow = (n8 - 1 - tid) / k8;
    mcol = (n8 - 1 - tid) % k8;
    sq = stride / k8;
    sr = stride % k8;
  }
  // the next iteration's 32 bytes are loaded before this one is processed
  uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
  if (tid < n8) {
    n0 = ld_nc_u4(w4 + 2 * (n8 - 1 - tid));
    n1 = ld_nc_u4(w4 + 2 * (n8 - 1 - tid) + 1);
  }
  for (int64_t r = tid; r < n8; r += stride) {
    const int64_t i = n8 - 1 - r;
    const uint4 v0 = n0, v1 = n1;
    if (r + stride < n8) {
      n0 = ld_nc_u4(w4 + 2 * (i - stride));
      n1 = ld_nc_u4(w4 + 2 * (i - stride) + 1);
    }
    const uint32_t b[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const QmGroup8 g = qm_group8<M, NK>(b, n_keep, half_gamma_bits, gamma_ok);
    codes_out[i] = static_cast<uint16_t>(g.packed);
    if (mask_out != nullptr) {
      if (M == 8) mask_out[i] = static_cast<uint8_t>(g.keep);
      else reinterpret_cast<uint16_t*>(mask_out)[i] = static_cast<uint16_t>((g.keep & 0xFu) | ((g.keep >> 4) << 8));
    }
    if (w_i8_out != nullptr) w_i8_out[i] = make_uint2(g.lo, g.hi);
    if (sp_values_out != nullptr) {   // the host allows it only for 2:4-valid masks
      sp_values_out[i] = g.sp_values;
      sp_meta_out[mrow * meta_pitch + mcol] = static_cast<uint8_t>(g.sp_meta);
      mcol -= sr;
      mrow -= sq;
      if (mcol < 0) {
        mcol += k8;
        mrow -= 1;
      }
    }
  }
}

}  // namespace bl
