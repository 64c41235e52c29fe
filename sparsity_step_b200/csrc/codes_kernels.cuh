// Kernels that read the packed 2-bit ternary codes directly.
//
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 四: four ternary values per
// byte, loaded from HBM and unpacked to {-1, 0, +1} before the product with int8
// activations. Code layout: element k at bits 2*(k mod 4) of byte k/4 of its row,
// 0b00 = 0, 0b01 = +1, 0b11 = -1 (0b10 is never written and reads as 0).
//
//   expand_codes_bf16_kernel: codes -> bf16 {-1, 0, +1} matrix (the exact
//     effective weight up to the scalar gamma) for the input-gradient product.
//   fwd_codes_kernel: CUDA-core forward product for short token batches (decode):
//     one warp per output row streams that row's codes once per 8 tokens, turns each
//     code byte into four int8 weights with a 256-entry table and accumulates with
//     dp4a against the int8 activations; the warp sum is exact in int32.
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

constexpr int kCodesTokTile = 8;
constexpr int kCodesWarps = 8;

__global__ void __launch_bounds__(kCodesWarps * 32) fwd_codes_kernel(const int8_t* __restrict__ xq, const float* __restrict__ absmax,
                                                                     const uint8_t* __restrict__ codes,
                                                                     const float* __restrict__ w_scale, int t, int k_in,
                                                                     int n_out, int32_t* __restrict__ acc_out,
                                                                     void* __restrict__ y_out, int y_f32) {
  __shared__ uint32_t lut[256];   // code byte -> four int8 weights
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t f = (static_cast<uint32_t>(b) >> (2 * j)) & 3u;
      const uint32_t byte = (f & 1u) ? ((f & 2u) ? 0xFFu : 0x01u) : 0u;
      word |= byte << (8 * j);
    }
    lut[b] = word;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * kCodesWarps + (threadIdx.x >> 5);
  if (n >= n_out) return;
  const float gamma = *w_scale;
  const int kw = k_in / 16;   // 32-bit code words per row (16 weights each)
  const uint32_t* crow = reinterpret_cast<const uint32_t*>(codes + static_cast<int64_t>(n) * (k_in / 4));
  for (int t0 = 0; t0 < t; t0 += kCodesTokTile) {
    int acc[kCodesTokTile];
#pragma unroll
    for (int j = 0; j < kCodesTokTile; ++j) acc[j] = 0;
    for (int w = lane; w < kw; w += 32) {
      const uint32_t c = __ldg(crow + w);
      const int w0 = static_cast<int>(lut[c & 0xFFu]), w1 = static_cast<int>(lut[(c >> 8) & 0xFFu]);
      const int w2 = static_cast<int>(lut[(c >> 16) & 0xFFu]), w3 = static_cast<int>(lut[c >> 24]);
#pragma unroll
      for (int j = 0; j < kCodesTokTile; ++j) {
        if (t0 + j < t) {
          const int4 xv = __ldg(reinterpret_cast<const int4*>(xq + static_cast<int64_t>(t0 + j) * k_in) + w);
          int a = acc[j];
          a = __dp4a(xv.x, w0, a);
          a = __dp4a(xv.y, w1, a);
          a = __dp4a(xv.z, w2, a);
          a = __dp4a(xv.w, w3, a);
          acc[j] = a;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kCodesTokTile; ++j) {
      int a = acc[j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      const int tt = t0 + j;
      if (lane == 0 && tt < t) {
        const float rs = __fmul_rn(__fdiv_rn(absmax[tt], 127.0f), gamma);
        const float y = __fmul_rn(static_cast<float>(a), rs);
        const int64_t off = static_cast<int64_t>(tt) * n_out + n;
        if (y_f32) static_cast<float*>(y_out)[off] = y;
        else static_cast<__nv_bfloat16*>(y_out)[off] = __float2bfloat16_rn(y);
        if (acc_out != nullptr) acc_out[off] = a;
      }
    }
  }
}

}  // namespace bl
