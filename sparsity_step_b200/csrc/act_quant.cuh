// Step a3: per-token absmax int8 activation quantisation, fused into one read.
//
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 一: activations are quantised
// to 8-bit integers; section 四: W1.58A8 (ternary weights x int8 activations).
//
// Every kernel reads a row once: a row's absmax is a max over |bf16| bit patterns
// (exact, order-free); then q = clamp(rint(x * (127 / a)), -128, 127) with one IEEE
// fp32 division per row, one fp32 multiply per element (no FMA) and one saturating
// round-to-nearest-even conversion, and the int8 rows are written with 8-byte stores.
// HBM traffic: 2 B read + 1 B written per element, + 4 B per row. By row width:
//   act_quant_warp_kernel  k_in <= 4096: one warp per row, row in registers;
//   act_quant_ring_kernel  k_in <= 16384: persistent CTAs streaming their next row into
//                          a shared-memory ring while quantising the current one;
//   act_quant_kernel       k_in <= 32768: one CTA per row, row in registers;
//   act_quant_long_kernel  wider: two reads (max, then quantise).
#pragma once

#include "common.cuh"
#include "cp_async.cuh"

namespace bl {

// Running max of |bf16| bit patterns, both halves at once (16-bit SIMD max; the high
// half is folded in by bf16_absmax_final).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t w, uint32_t m) { return __vmaxu2(m, w & 0x7fff7fffu); }
__device__ __forceinline__ uint32_t bf16_absmax_final(uint32_t m) { return max(m & 0xffffu, m >> 16); }

// q = clamp(rint(x * s), -128, 127): one fp32 multiply, then one conversion that rounds
// to nearest even and saturates to int8 (the low byte of the result).
__device__ __forceinline__ uint32_t quant_one(float xf, float s) {
  uint32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(__fmul_rn(xf, s)));
  return q;
}

// Four bf16 (two words) -> four int8 in one word (element 0 in byte 0).
__device__ __forceinline__ uint32_t quant_pack4(uint32_t w0, uint32_t w1, float s) {
  const uint32_t q0 = quant_one(__uint_as_float(w0 << 16), s), q1 = quant_one(__uint_as_float(w0 & 0xffff0000u), s);
  const uint32_t q2 = quant_one(__uint_as_float(w1 << 16), s), q3 = quant_one(__uint_as_float(w1 & 0xffff0000u), s);
  return __byte_perm(__byte_perm(q0, q1, 0x0040u), __byte_perm(q2, q3, 0x0040u), 0x5410u);
}

__device__ __forceinline__ uint32_t block_max_u32(uint32_t m, uint32_t* s_red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  uint32_t r = 0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) r = max(r, s_red[w]);
  return r;
}

// R rows per CTA, each cached in registers: VPT 16-byte vectors (8 bf16) per thread
// per row. All R rows' loads are in flight before one block reduction of R maxima.
template <int VPT, int R>
__global__ void __launch_bounds__(256) act_quant_kernel(const uint4* __restrict__ x, int64_t t, int k8, int8_t* __restrict__ xq,
                                                        float* __restrict__ absmax_out) {
  __shared__ uint32_t s_red[R][8];
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * R;
  uint4 v[R][VPT];
  uint32_t m[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = 0;
    const bool row_ok = row0 + r < t;
    const uint4* xr = x + (row0 + r) * k8;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * blockDim.x;
      if (row_ok && idx < k8) {
        v[r][i] = __ldcs(xr + idx);
        m[r] = bf16x2_absmax(v[r][i].x, m[r]);
        m[r] = bf16x2_absmax(v[r][i].y, m[r]);
        m[r] = bf16x2_absmax(v[r][i].z, m[r]);
        m[r] = bf16x2_absmax(v[r][i].w, m[r]);
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = bf16_absmax_final(m[r]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m[r] = max(m[r], __shfl_xor_sync(0xffffffffu, m[r], off));
    if (lane == 0) s_red[r][warp] = m[r];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (row0 + r >= t) break;
    uint32_t mm = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) mm = max(mm, s_red[r][w]);
    float a = __uint_as_float(mm << 16);
    if (a == 0.0f) a = 1e-5f;   // an all-zero row quantises to zeros
    const float sc = __fdiv_rn(127.0f, a);
    uint2* out = reinterpret_cast<uint2*>(xq + (row0 + r) * (static_cast<int64_t>(k8) * 8));
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * blockDim.x;
      if (idx < k8) out[idx] = make_uint2(quant_pack4(v[r][i].x, v[r][i].y, sc), quant_pack4(v[r][i].z, v[r][i].w, sc));
    }
    if (threadIdx.x == 0) absmax_out[row0 + r] = a;
  }
}

// Short rows (k8 <= 32 * VPT): one warp per row, the row held in registers (VPT
// 16-byte vectors per lane), warp-shuffle max, no block barrier. Warps stride over the
// rows; the launch gives every row its own warp.
template <int VPT>
__global__ void __launch_bounds__(256) act_quant_warp_kernel(const uint4* __restrict__ x, int64_t t, int k8,
                                                             int8_t* __restrict__ xq, float* __restrict__ absmax_out) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); row < t; row += warps) {
    const uint4* xr = x + row * k8;
    uint4 v[VPT];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = lane + 32 * i;
      if (idx < k8) {
        v[i] = __ldcs(xr + idx);
        m = bf16x2_absmax(v[i].x, m);
        m = bf16x2_absmax(v[i].y, m);
        m = bf16x2_absmax(v[i].z, m);
        m = bf16x2_absmax(v[i].w, m);
      }
    }
    m = bf16_absmax_final(m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    float a = __uint_as_float(m << 16);
    if (a == 0.0f) a = 1e-5f;   // an all-zero row quantises to zeros
    const float sc = __fdiv_rn(127.0f, a);
    uint2* out = reinterpret_cast<uint2*>(xq + row * (static_cast<int64_t>(k8) * 8));
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = lane + 32 * i;
      if (idx < k8) out[idx] = make_uint2(quant_pack4(v[i].x, v[i].y, sc), quant_pack4(v[i].z, v[i].w, sc));
    }
    if (lane == 0) absmax_out[row] = a;
  }
}

// Long rows (k8 > 512) on persistent CTAs: each thread streams its own 16-byte vectors of
// the CTA's next kD - 1 rows into a shared-memory ring with cp.async while it quantises
// the current row from the ring, so the loads of later rows stay in flight through the
// block reduction and the stores of this one. One block barrier per row (the partial
// maxima alternate between two buffers). Ring: kD rows x VPT vectors x 256 threads x 16 B.
template <int VPT, int kD>
__global__ void __launch_bounds__(256) act_quant_ring_kernel(const uint4* __restrict__ x, int64_t t, int k8,
                                                             int8_t* __restrict__ xq, float* __restrict__ absmax_out) {
  extern __shared__ __align__(16) uint8_t aq_ring[];
  __shared__ uint32_t s_red[2][8];
  const uint32_t base = smem_u32(aq_ring) + threadIdx.x * 16u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto slot = [&](int s, int i) { return base + static_cast<uint32_t>((s * VPT + i) * 256) * 16u; };
  auto issue = [&](int s, int64_t row) {   // this thread's vectors of `row` into ring slot s
    if (row < t) {
      const uint4* xr = x + row * k8;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int idx = threadIdx.x + i * 256;
        if (idx < k8) cp_async16(slot(s, i), xr + idx, true);
      }
    }
    cp_async_commit();
  };
  const int64_t step = gridDim.x;
  int64_t row = blockIdx.x;
#pragma unroll
  for (int j = 0; j < kD - 1; ++j) issue(j, row + j * step);
  for (int it = 0; row < t; ++it, row += step) {
    const int s = it % kD;
    issue((it + kD - 1) % kD, row + (kD - 1) * step);
    cp_async_wait<kD - 1>();   // this thread's copies of `row` have landed
    uint4 v[VPT];
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * 256;
      if (idx < k8) {
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                     : "r"(slot(s, i)));
        m = bf16x2_absmax(v[i].x, m);
        m = bf16x2_absmax(v[i].y, m);
        m = bf16x2_absmax(v[i].z, m);
        m = bf16x2_absmax(v[i].w, m);
      }
    }
    m = bf16_absmax_final(m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) s_red[it & 1][warp] = m;
    __syncthreads();
    uint32_t mm = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) mm = max(mm, s_red[it & 1][w]);
    float a = __uint_as_float(mm << 16);
    if (a == 0.0f) a = 1e-5f;   // an all-zero row quantises to zeros
    const float sc = __fdiv_rn(127.0f, a);
    uint2* out = reinterpret_cast<uint2*>(xq + row * (static_cast<int64_t>(k8) * 8));
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * 256;
      if (idx < k8) out[idx] = make_uint2(quant_pack4(v[i].x, v[i].y, sc), quant_pack4(v[i].z, v[i].w, sc));
    }
    if (threadIdx.x == 0) absmax_out[row] = a;
  }
  cp_async_wait<0>();
}

// Rows too long to cache in registers: read the row twice (max, then quantise).
__global__ void __launch_bounds__(256) act_quant_long_kernel(const uint4* __restrict__ x, int k8, int8_t* __restrict__ xq,
                                                             float* __restrict__ absmax_out) {
  __shared__ uint32_t s_red[8];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * k8;
  uint32_t m = 0;
  for (int idx = threadIdx.x; idx < k8; idx += blockDim.x) {
    const uint4 v = xr[idx];
    m = bf16x2_absmax(v.x, m);
    m = bf16x2_absmax(v.y, m);
    m = bf16x2_absmax(v.z, m);
    m = bf16x2_absmax(v.w, m);
  }
  m = block_max_u32(bf16_absmax_final(m), s_red);
  float a = __uint_as_float(m << 16);
  if (a == 0.0f) a = 1e-5f;
  const float s = __fdiv_rn(127.0f, a);
  uint2* out = reinterpret_cast<uint2*>(xq + row * (static_cast<int64_t>(k8) * 8));
  for (int idx = threadIdx.x; idx < k8; idx += blockDim.x) {
    const uint4 v = __ldcs(xr + idx);
    out[idx] = make_uint2(quant_pack4(v.x, v.y, s), quant_pack4(v.z, v.w, s));
  }
  if (threadIdx.x == 0) absmax_out[row] = a;
}

}  // namespace bl

namespace bl {

// Dequantised activations for the optional grad_W reading: x_deq[t, k] = q[t, k] * a_t / 127
// rounded to bf16 (one fp32 division per row, one fp32 multiply per element, then
// round to nearest even). One thread = 16 int8 elements of one row (k_in % 64 == 0,
// so a 16-element chunk never crosses a row): one 16-byte load, two 16-byte stores.
__global__ void __launch_bounds__(256) dequant_x_bf16_kernel(const uint4* __restrict__ xq, const float* __restrict__ absmax,
                                                             int64_t nchunks, int k16, uint4* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunks; i += stride) {
    const float sc = __fdiv_rn(absmax[i / k16], 127.0f);
    const uint4 v = xq[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t b = w[j] >> (16 * h);
        const float f0 = __fmul_rn(static_cast<float>(static_cast<int8_t>(b & 0xffu)), sc);
        const float f1 = __fmul_rn(static_cast<float>(static_cast<int8_t>((b >> 8) & 0xffu)), sc);
        const __nv_bfloat162 p = __floats2bfloat162_rn(f0, f1);
        o[2 * j + h] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
    out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace bl
