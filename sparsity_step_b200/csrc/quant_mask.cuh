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
//                         a warp covers 1 KB contiguous); top-N mask by selection
//                         scans, ternary codes, 2-bit packing, optional int8 weights.
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
    for (int u = 0; u < kQmUnroll; ++u) v[u] = __ldcs(w4 + i + u * stride);   // read once: streamed
#pragma unroll
    for (int u = 0; u < kQmUnroll; ++u) qm_accumulate(v[u], acc, bad);
  }
  for (; i < n4; i += stride) qm_accumulate(__ldcs(w4 + i), acc, bad);
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


// Keep-mask of one group of M (weights [G0, G0+M) of the 8 held by the thread).
// Element j outranks i when |w_j| > |w_i|, or they are equal and j < i (lower index
// wins). NK > 0: compile-time N, found by selection scans: NK >= M/2 removes the
// (M - NK) weakest one at a time, NK < M/2 picks the NK strongest; each scan is one
// pass of compares in index order. NK == 0: runtime N via rank counting.
template <int M, int NK, int G0>
__device__ __forceinline__ uint32_t group_keep(const uint32_t (&a)[8], int n_keep) {
  constexpr uint32_t all = (1u << M) - 1u;
  if (NK == M) return all << G0;
  if (NK > 0 && 2 * NK >= M) {
    uint32_t dropped = 0;
#pragma unroll
    for (int r = 0; r < M - NK; ++r) {
      uint32_t best_a = 0xFFFFFFFFu;
      int best_j = 0;
#pragma unroll
      for (int j = 0; j < M; ++j) {
        // scanning in index order, a later equal element is weaker: <= picks it
        const bool take = !((dropped >> j) & 1u) && a[G0 + j] <= best_a;
        best_a = take ? a[G0 + j] : best_a;
        best_j = take ? j : best_j;
      }
      dropped |= 1u << best_j;
    }
    return (all & ~dropped) << G0;
  }
  if (NK > 0) {
    uint32_t kept = 0;
#pragma unroll
    for (int r = 0; r < NK; ++r) {
      int best_a = -1;
      int best_j = 0;
#pragma unroll
      for (int j = 0; j < M; ++j) {
        // scanning in index order, a later equal element is not stronger: strict >
        const bool take = !((kept >> j) & 1u) && static_cast<int>(a[G0 + j]) > best_a;
        best_a = take ? static_cast<int>(a[G0 + j]) : best_a;
        best_j = take ? j : best_j;
      }
      kept |= 1u << best_j;
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
// One thread = 8 contiguous weights (one group of 8, or two groups of 4).
template <int M, int NK>
__global__ void __launch_bounds__(kQmThreads) qm_mask_codes_kernel(const float4* __restrict__ w4, int64_t n8, int n_keep,
                                                                    const float* __restrict__ gamma_ptr,
                                                                    uint8_t* __restrict__ mask_out,
                                                                    uint16_t* __restrict__ codes_out,
                                                                    uint2* __restrict__ w_i8_out) {
  static_assert(M == 4 || M == 8, "groups of 4 or 8");
  const float gamma = *gamma_ptr;
  const bool gamma_ok = isfinite(gamma) && gamma > 0.0f;
  const uint32_t half_gamma_bits = __float_as_uint(0.5f * gamma);   // 0.5 * gamma is exact
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 v0 = __ldcs(w4 + 2 * i);
    const float4 v1 = __ldcs(w4 + 2 * i + 1);
    const uint32_t b[8] = {__float_as_uint(v0.x), __float_as_uint(v0.y), __float_as_uint(v0.z), __float_as_uint(v0.w),
                           __float_as_uint(v1.x), __float_as_uint(v1.y), __float_as_uint(v1.z), __float_as_uint(v1.w)};
    uint32_t a[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) a[j] = b[j] & 0x7fffffffu;   // |w| bits: order-preserving
    uint32_t keep = group_keep<M, NK, 0>(a, n_keep);
    if (M == 4) keep |= group_keep<M, NK, 4>(a, n_keep);
    const uint32_t code_keep = gamma_ok ? keep : 0u;   // range error: all codes 0 (gamma is NaN)

    uint32_t packed = 0, lo = 0, hi = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t nz = ((code_keep >> j) & 1u) & (a[j] > half_gamma_bits ? 1u : 0u);
      const uint32_t neg = b[j] >> 31;
      const uint32_t enc = nz * (1u | (neg << 1));                 // 00 = 0, 01 = +1, 11 = -1
      const uint32_t byte = nz * (neg ? 0xFFu : 0x01u);           // int8 -1 / +1 / 0
      packed |= enc << (2 * j);
      if (j < 4) lo |= byte << (8 * j);
      else hi |= byte << (8 * (j - 4));
    }
    codes_out[i] = static_cast<uint16_t>(packed);
    if (mask_out != nullptr) {
      if (M == 8) mask_out[i] = static_cast<uint8_t>(keep);
      else reinterpret_cast<uint16_t*>(mask_out)[i] = static_cast<uint16_t>((keep & 0xFu) | ((keep >> 4) << 8));
    }
    if (w_i8_out != nullptr) w_i8_out[i] = make_uint2(lo, hi);
  }
}

}  // namespace bl
