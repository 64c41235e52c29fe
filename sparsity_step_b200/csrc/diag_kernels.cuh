// Kernels outside the forward/backward products:
//
//   threshold_hist_kernel<M>: threshold-decoupling diagnostic. Sparse-BitNet article,
//     section 五: every group of 8 weights gets a threshold that splits kept from
//     dropped weights, and in the 1.58-bit model that threshold stays in the near-zero
//     region. Per group the threshold is the largest dropped |w|; the kernel bins it in
//     units of gamma (bins of 1/8 over [0, 2), then [2, inf)), deciding each bin edge
//     exactly (8|w| against k * gamma in fp64: both products are exact), and counts the
//     dropped weights and those among them with a nonzero ternary code (2|w| > gamma).
//
//   expand_codes_t_i8_kernel: packed codes [n_out, k_in/4] -> the transposed int8
//     matrix C^T [k_in, n_out] (the K-major B operand of the int8-dY input gradient).
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kHistBins = 17;
constexpr int kHistWords = kHistBins + 2;   // bins, dropped, dropped_core

template <int M>
__global__ void __launch_bounds__(256) threshold_hist_kernel(const float* __restrict__ w,
                                                             const uint8_t* __restrict__ mask,
                                                             const float* __restrict__ w_scale, int64_t ngroups,
                                                             unsigned long long* __restrict__ out) {
  static_assert(M == 4 || M == 8, "groups of 4 or 8");
  __shared__ unsigned int bins[kHistBins];
  __shared__ unsigned long long tot[2];
  if (threadIdx.x < kHistBins) bins[threadIdx.x] = 0;
  if (threadIdx.x < 2) tot[threadIdx.x] = 0;
  __syncthreads();
  const float gamma = *w_scale;
  const double g64 = static_cast<double>(gamma);
  const int lane = threadIdx.x & 31;
  unsigned long long dropped = 0, core = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // every lane runs the same number of iterations (warp-collective match below)
  const int64_t first = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31);
  for (int64_t gw = first; gw < ngroups; gw += stride) {
    const int64_t g = gw + lane;
    int b = 31;   // no bin
    if (g < ngroups) {
      float v[M];
      const float4* p = reinterpret_cast<const float4*>(w + g * M);
#pragma unroll
      for (int q = 0; q < M / 4; ++q) {
        const float4 f = __ldg(p + q);
        v[4 * q] = f.x;
        v[4 * q + 1] = f.y;
        v[4 * q + 2] = f.z;
        v[4 * q + 3] = f.w;
      }
      const unsigned keep = mask[g];
      float tmax = 0.0f;
      int nd = 0;
#pragma unroll
      for (int j = 0; j < M; ++j) {
        if (!((keep >> j) & 1u)) {
          const float a = fabsf(v[j]);
          ++nd;
          core += (2.0f * a > gamma) ? 1u : 0u;
          tmax = fmaxf(tmax, a);
        }
      }
      if (nd > 0) {
        dropped += static_cast<unsigned>(nd);
        const double t8 = 8.0 * static_cast<double>(tmax);
        b = 0;
#pragma unroll
        for (int k = 1; k < kHistBins; ++k) b += (t8 >= static_cast<double>(k) * g64) ? 1 : 0;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, b);
    if (b != 31 && lane == __ffs(peers) - 1) atomicAdd(&bins[b], static_cast<unsigned>(__popc(peers)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dropped += __shfl_xor_sync(0xffffffffu, dropped, o);
    core += __shfl_xor_sync(0xffffffffu, core, o);
  }
  if (lane == 0) {
    atomicAdd(&tot[0], dropped);
    atomicAdd(&tot[1], core);
  }
  __syncthreads();
  if (threadIdx.x < kHistBins && bins[threadIdx.x]) atomicAdd(&out[threadIdx.x], bins[threadIdx.x]);
  if (threadIdx.x < 2 && tot[threadIdx.x]) atomicAdd(&out[kHistBins + threadIdx.x], tot[threadIdx.x]);
}

// One CTA per 64 x 64 tile: codes of 64 rows x 64 weights -> C^T rows of 64 bytes.
// Code layout: element k at bits 2*(k mod 4) of byte k/4 (0b01 = +1, 0b11 = -1).
__global__ void __launch_bounds__(256) expand_codes_t_i8_kernel(const uint8_t* __restrict__ codes, int n_out, int k_in,
                                                                int8_t* __restrict__ ct) {
  __shared__ __align__(16) int8_t tile[64][64 + 4];   // [k][n], padded rows
  const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  {
    const int row = threadIdx.x >> 2, word = threadIdx.x & 3;   // 16 codes per thread
    const int n = n0 + row;
    uint32_t c = 0;
    if (n < n_out) c = __ldg(reinterpret_cast<const uint32_t*>(codes + static_cast<int64_t>(n) * (k_in >> 2) + (k0 >> 2)) + word);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t f = (c >> (2 * j)) & 3u;
      tile[16 * word + j][row] = static_cast<int8_t>((f & 1u) ? ((f & 2u) ? -1 : 1) : 0);
    }
  }
  __syncthreads();
  const int k = threadIdx.x >> 2, part = threadIdx.x & 3;   // 16 bytes of row k
  const int n = n0 + 16 * part;
  if (n < n_out) {
    uint32_t v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = *reinterpret_cast<const uint32_t*>(&tile[k][16 * part + 4 * q]);
    *reinterpret_cast<uint4*>(ct + static_cast<int64_t>(k0 + k) * n_out + n) = make_uint4(v[0], v[1], v[2], v[3]);
  }
}

}  // namespace bl
