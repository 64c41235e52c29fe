// Kernels that read the packed 2-bit ternary codes directly.
//
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 四: four ternary values per
// byte, loaded from HBM and unpacked to {-1, 0, +1} before the product with int8
// activations. Code layout: element k at bits 2*(k mod 4) of byte k/4 of its row,
// 0b00 = 0, 0b01 = +1, 0b11 = -1 (0b10 is never written and reads as 0).
//
//   expand_codes_bf16_kernel: codes -> bf16 {-1, 0, +1} matrix (the exact
//     effective weight up to the scalar gamma) for the input-gradient product.
//   fwd_codes_mma_kernel: grouped forward product for short token batches (decode),
//     streaming the 2-bit codes (details below).
#pragma once

#include "common.cuh"

namespace bl {

__device__ __forceinline__ uint32_t code_to_bf16_bits(uint32_t f) {
  return (f & 1u) ? ((f & 2u) ? 0xBF80u : 0x3F80u) : 0u;
}

// One thread = one 32-bit word of codes = 16 weights -> 32 bytes of bf16.
__global__ void __launch_bounds__(256) expand_codes_bf16_kernel(const uint32_t* __restrict__ codes, int64_t nwords,
                                                                uint4* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords; i += stride) {
    const uint32_t c = __ldg(codes + i);
    uint32_t p[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const uint32_t lo = code_to_bf16_bits((c >> (4 * h)) & 3u);
      const uint32_t hi = code_to_bf16_bits((c >> (4 * h + 2)) & 3u);
      p[h] = lo | (hi << 16);
    }
    out[2 * i] = make_uint4(p[0], p[1], p[2], p[3]);
    out[2 * i + 1] = make_uint4(p[4], p[5], p[6], p[7]);
  }
}

// ---------------------------------------------------------------- grouped decode product
//
// One launch computes y = (xq . masked_codes^T) * absmax/127 * gamma for up to
// kMaxFwdGroup independent problems (e.g. every BitLinear of a layer stack at one
// decode step). Work is split into tasks of 16 weight rows x 32 tokens; persistent
// warps stride over the concatenated task list.
//
// Per task a warp streams its 16 rows' codes once (16-byte loads, L1 bypass) and
// feeds mma.sync.m16n8k32.s8 with the weights decoded straight into A fragments in
// registers: weights never pass through shared memory. Inside each chunk of 256
// weights the reduction order is permuted so that thread (group g, index tig) owns
// logical weights [64*tig, 64*tig + 64): MMA step s, A/B slot 4*tig + i holds weight
// 64*tig + 8*s + i and slot 4*tig + 16 + i holds 64*tig + 8*s + 4 + i. A thread then
// reads 16 contiguous code bytes per row and 64 contiguous int8 activations per
// token; the same permutation on both operands leaves every dot product unchanged.
// Code bytes become int8x4 words through a 256-entry table replicated per lane
// (entry e of lane l at word 32*e + l: conflict-free).
constexpr int kMaxFwdGroup = 256;
constexpr int kDecodeThreads = 256;

struct FwdProblem {
  const uint8_t* codes;    // [n_out, k_in/4]
  const int8_t* xq;        // [t, k_in]
  const float* absmax;     // [t]
  const float* w_scale;    // [1]
  void* y;                 // [t, n_out]
  int32_t* acc;            // [t, n_out] or null
  int t, k_in, n_out;
  int task_begin;          // first task index of this problem
};

struct FwdGroup {
  FwdProblem p[kMaxFwdGroup];
  int count;
  int total_tasks;
  int y_f32;
};

__device__ __forceinline__ void mma_m16n8k32_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t byte_of(const uint4& v, int i) {
  const uint32_t w = i < 4 ? v.x : (i < 8 ? v.y : (i < 12 ? v.z : v.w));
  return (w >> (8 * (i & 3))) & 0xFFu;
}

template <int NG>   // token groups of 8 per task (1, 2 or 4)
__global__ void __launch_bounds__(kDecodeThreads) fwd_codes_mma_kernel(const __grid_constant__ FwdGroup G) {
  __shared__ uint32_t lut[256 * 32];
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const uint32_t e = static_cast<uint32_t>(i) >> 5;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t f = (e >> (2 * j)) & 3u;
      word |= ((f & 1u) ? ((f & 2u) ? 0xFFu : 0x01u) : 0u) << (8 * j);
    }
    lut[i] = word;
  }
  __syncthreads();
  const uint32_t* my_lut = lut + lane;
  const int g = lane >> 2, tig = lane & 3;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int task = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; task < G.total_tasks; task += warps) {
    int lo = 0, hi = G.count - 1;   // last problem with task_begin <= task
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (G.p[mid].task_begin <= task) lo = mid;
      else hi = mid - 1;
    }
    const FwdProblem& P = G.p[lo];
    const int row_blocks = P.n_out >> 4;
    const int local = task - P.task_begin;
    const int n0 = (local % row_blocks) * 16;
    const int t0 = (local / row_blocks) * (8 * NG);
    const int K = P.k_in;
    const int kb = K >> 2;   // code bytes per row
    const uint8_t* crow0 = P.codes + static_cast<int64_t>(n0 + g) * kb + tig * 16;
    const uint8_t* crow1 = crow0 + 8 * static_cast<int64_t>(kb);
    int acc[NG][4];
#pragma unroll
    for (int j = 0; j < NG; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0;
    const int nchunks = (K + 255) >> 8;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    uint4 c0n = (64 * tig < K) ? ld_stream_u4(crow0) : zero;
    uint4 c1n = (64 * tig < K) ? ld_stream_u4(crow1) : zero;
    for (int ch = 0; ch < nchunks; ++ch) {
      const uint4 c0 = c0n, c1 = c1n;
      const bool mine = ch * 256 + 64 * tig < K;   // this thread's 64 weights exist
      if (ch + 1 < nchunks) {
        const bool next = (ch + 1) * 256 + 64 * tig < K;
        c0n = next ? ld_stream_u4(crow0 + (ch + 1) * 64) : zero;
        c1n = next ? ld_stream_u4(crow1 + (ch + 1) * 64) : zero;
      }
      uint4 xv[NG][4];
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const int tok = t0 + 8 * j + g;
        const bool ok = mine && tok < P.t;
        const uint4* xp = reinterpret_cast<const uint4*>(P.xq + static_cast<int64_t>(tok) * K + ch * 256 + tig * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[j][q] = ok ? __ldg(xp + q) : zero;
      }
#pragma unroll
      for (int st = 0; st < 8; ++st) {
        const uint32_t a0 = my_lut[byte_of(c0, 2 * st) << 5];
        const uint32_t a2 = my_lut[byte_of(c0, 2 * st + 1) << 5];
        const uint32_t a1 = my_lut[byte_of(c1, 2 * st) << 5];
        const uint32_t a3 = my_lut[byte_of(c1, 2 * st + 1) << 5];
#pragma unroll
        for (int j = 0; j < NG; ++j) {
          const uint4& xa = xv[j][st >> 1];
          const uint32_t b0 = (st & 1) ? xa.z : xa.x;
          const uint32_t b1 = (st & 1) ? xa.w : xa.y;
          mma_m16n8k32_s8(acc[j], a0, a1, a2, a3, b0, b1);
        }
      }
    }
    // C fragment: acc[j][0..1] = row g, tokens 2*tig, 2*tig+1; acc[j][2..3] = row g+8
    const float gamma = *P.w_scale;
#pragma unroll
    for (int j = 0; j < NG; ++j) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int tok = t0 + 8 * j + 2 * tig + (v & 1);
        const int n = n0 + g + ((v >> 1) << 3);
        if (tok < P.t) {
          const float rs = __fmul_rn(__fdiv_rn(P.absmax[tok], 127.0f), gamma);
          const float y = __fmul_rn(static_cast<float>(acc[j][v]), rs);
          const int64_t off = static_cast<int64_t>(tok) * P.n_out + n;
          if (G.y_f32) static_cast<float*>(P.y)[off] = y;
          else static_cast<__nv_bfloat16*>(P.y)[off] = __float2bfloat16_rn(y);
          if (P.acc != nullptr) P.acc[off] = acc[j][v];
        }
      }
    }
  }
}

}  // namespace bl
