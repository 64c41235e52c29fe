// Probes (measurement and self-tests only, not part of the BitLinear ABI).
//
// Tensor-pipe throughput probe:
// every CTA issues back-to-back 128x256 tcgen05.mma instructions on operands that
// stay in shared memory, so the result is the dense MMA rate of one B200 at the
// clock it runs at, with no memory traffic. Built as libblprobe.so; bench.py uses it
// to report the int8 and bf16 tensor peaks its roofline fractions refer to.
#include <cstdint>

#include "common.cuh"

namespace {

constexpr int kProbeThreads = 128;
constexpr int kProbeSmem = 1024 + 16384 + 32768 + 64;

// KIND 0: bf16 (kind::f16), 1: int8 (kind::i8), 2: 2:4-sparse int8 (kind::i8 .sp, logical
// K = 64 per MMA, metadata 0x4 = positions 0 and 1 in every group, in TMEM columns 256-263).
template <int KIND>
__global__ void __launch_bounds__(kProbeThreads, 1) mma_peak_kernel(int iters, unsigned int* status) {
  constexpr bool kI8 = KIND != 0;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = bl::smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  // small finite operand values (int8 1, bf16 1.0 / 0) keep the accumulators finite
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem)[i] = kI8 ? 0x01010101u : 0x00003F80u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 16384 + 32768);
  const uint32_t bar = bl::smem_u32(tmem_slot + 2);
  const int warp = threadIdx.x >> 5;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x == 0) {
    bl::mbar_init(bar, 1);
    bl::fence_mbar_init();
  }
  if (warp == 0) {
    bl::tmem_alloc(bl::smem_u32(tmem_slot), 512);
    bl::tmem_relinquish();
  }
  bl::tc_fence_before_sync();
  __syncthreads();
  bl::tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (KIND == 2) {   // valid metadata for every row (lane = row, 32 lanes per warp)
    const uint32_t m = 0x44444444u;
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(
                     tmem + (static_cast<uint32_t>(32 * warp) << 16) + 256u),
                 "r"(m)
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    bl::tc_fence_before_sync();
    __syncthreads();
    bl::tc_fence_after_sync();
  }
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = KIND == 2   ? (bl::make_idesc(2u, 1u, 1u, 0u, 0u, 256, 128) | (1u << 2))
                               : KIND == 1 ? bl::make_idesc(2u, 1u, 1u, 0u, 0u, 256, 128)
                                           : bl::make_idesc(1u, 1u, 1u, 0u, 0u, 256, 128);
    for (int i = 0; i < iters; ++i) {
      // dense: two 256-column accumulators in turn; sparse: one (columns 256+ hold the metadata)
      const uint32_t d = tmem + static_cast<uint32_t>(KIND == 2 ? 0 : (i & 1) * 256);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = bl::make_sw128_desc(base + kk * 32, 16, 1024);
        const uint32_t acc = (i > 1 || kk > 0) ? 1u : 0u;
        if (KIND == 2) {
          const uint64_t bd = bl::make_sw128_desc(base + 16384 + (kk & 1) * 64, 16, 1024);
          asm volatile(
              "{\n\t.reg .pred p;\n\t"
              "setp.ne.b32 p, %5, 0;\n\t"
              "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d),
              "l"(ad), "l"(bd), "r"(tmem + 256u + 2u * kk), "r"(idesc), "r"(acc)
              : "memory");
        } else {
          const uint64_t bd = bl::make_sw128_desc(base + 16384 + kk * 32, 16, 1024);
          if (kI8) bl::tc_mma_i8(d, ad, bd, idesc, acc);
          else bl::tc_mma_f16(d, ad, bd, idesc, acc);
        }
      }
    }
    bl::tc_commit(bar);
    const uint64_t t0 = bl::global_timer_ns();
    while (!bl::mbar_try_wait(bar, 0)) {
      if (bl::global_timer_ns() - t0 > bl::kWaitTimeoutNs) {
        atomicOr(status, 1u);
        break;
      }
    }
  }
  __syncthreads();
  if (warp == 0) {
    bl::tc_fence_after_sync();
    bl::tmem_dealloc(tmem, 512);
  }
}

// Failure-detection self-test: one thread waits, with the library's bounded wait, on an
// mbarrier that nothing ever arrives on. The wait must give up after kWaitTimeoutNs and
// the kernel must return normally, leaving the context usable; it records the outcome
// and the time waited.
__global__ void wait_timeout_kernel(unsigned int* out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    bl::mbar_init(bl::smem_u32(&bar), 1);
    abort_flag = 0;
    bl::fence_mbar_init();
    const uint64_t t0 = bl::global_timer_ns();
    const bool got = bl::mbar_wait(bl::smem_u32(&bar), 0, &abort_flag);
    const uint64_t dt = bl::global_timer_ns() - t0;
    out[0] = got ? 0u : 1u;
    out[1] = static_cast<unsigned int>(dt / 1000000ull);
  }
}

}  // namespace

// Runs the bounded-wait self-test (about 2 s). out_host[0] = 1 if the wait gave up (the
// expected outcome), out_host[1] = milliseconds waited. Returns 0, or -1 on a CUDA error.
extern "C" int blprobe_wait_timeout(unsigned int* out_host, void* stream) {
  static unsigned int* out = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!out && cudaMalloc(&out, 2 * sizeof(unsigned int)) != cudaSuccess) return -1;
  if (cudaMemsetAsync(out, 0, 2 * sizeof(unsigned int), st) != cudaSuccess) return -1;
  wait_timeout_kernel<<<1, 32, 0, st>>>(out);
  if (cudaGetLastError() != cudaSuccess) return -1;
  if (cudaMemcpyAsync(out_host, out, 2 * sizeof(unsigned int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return -1;
  return cudaStreamSynchronize(st) == cudaSuccess ? 0 : -1;
}

// Runs the probe: `kind` 0 = bf16 (kind::f16), 1 = int8 (kind::i8), 2 = 2:4-sparse int8
// (kind::i8 .sp); `ctas` CTAs of `iters` x 4 MMAs of 128x256x(16|32|64 logical). Returns
// 0, or -1 on a CUDA error, -6 on a timeout. The caller times it (CUDA events on `stream`).
extern "C" int blprobe_mma_peak(int kind, int ctas, int iters, void* stream) {
  static unsigned int* status = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!status && cudaMalloc(&status, sizeof(unsigned int)) != cudaSuccess) return -1;
  cudaMemsetAsync(status, 0, sizeof(unsigned int), st);
  if (kind == 2) {
    cudaFuncSetAttribute(mma_peak_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    mma_peak_kernel<2><<<ctas, kProbeThreads, kProbeSmem, st>>>(iters, status);
  } else if (kind == 1) {
    cudaFuncSetAttribute(mma_peak_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    mma_peak_kernel<1><<<ctas, kProbeThreads, kProbeSmem, st>>>(iters, status);
  } else {
    cudaFuncSetAttribute(mma_peak_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kProbeSmem);
    mma_peak_kernel<0><<<ctas, kProbeThreads, kProbeSmem, st>>>(iters, status);
  }
  if (cudaGetLastError() != cudaSuccess) return -1;
  unsigned int h = 0;
  if (cudaMemcpyAsync(&h, status, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return -1;
  if (cudaStreamSynchronize(st) != cudaSuccess) return -1;
  return h ? -6 : 0;
}
