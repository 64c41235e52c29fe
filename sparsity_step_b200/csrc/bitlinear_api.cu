// C ABI of the BitLinear path (declared in include/bitlinear.h): argument checks,
// workspace layout, TMA descriptor encoding and kernel dispatch. No allocation:
// the caller owns every buffer.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/bitlinear.h"
#include "act_quant.cuh"
#include "codes_kernels.cuh"
#include "codes_tc.cuh"
#include "common.cuh"
#include "diag_kernels.cuh"
#include "gemm_tc.cuh"
#include "gemm_sp2.cuh"
#include "gemm_tc2.cuh"
#include "quant_mask.cuh"

namespace {

thread_local char g_err[512] = "";

bl_status fail(bl_status st, const char* fmt, ...) {
  char msg[sizeof(g_err)];   // formatted apart from g_err: an argument may be g_err itself
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(msg, sizeof(msg), fmt, ap);
  va_end(ap);
  memcpy(g_err, msg, sizeof(g_err));
  return st;
}

bl_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// One-time setup of a kernel on a device: its dynamic shared-memory limit and the
// occupancy figure the launch sizes its grid by. A kernel attribute belongs to the
// context of the device that was current when it was set, so a process that drives
// several devices sets it up once per device. Threads that race on the first call both
// run the setup (idempotent) and store the same value.
constexpr int kMaxSetupDevices = 64;
struct PerDeviceSetup {
  std::atomic<int> v[kMaxSetupDevices];   // value + 1; 0 = not set up on that device
};

template <class F>
bl_status per_device_setup(PerDeviceSetup& c, int* out, F&& setup) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxSetupDevices) return fail(BL_ERR_INVALID_ARG, "device ordinal %d not supported", dev);
  int v = c.v[dev].load(std::memory_order_acquire);
  if (v == 0) {
    int r = 0;
    if (bl_status s = setup(&r)) return s;
    v = r + 1;
    c.v[dev].store(v, std::memory_order_release);
  }
  *out = v - 1;
  return BL_OK;
}

bl_status check_shape(int64_t t, int64_t k_in, int64_t n_out) {
  if (t < 0 || t > (int64_t(1) << 31) - 1) return fail(BL_ERR_UNSUPPORTED_SHAPE, "t=%lld out of range", (long long)t);
  if (k_in < 64 || k_in > 131072 || k_in % 64)
    return fail(BL_ERR_UNSUPPORTED_SHAPE, "k_in=%lld: need 64 <= k_in <= 131072, k_in %% 64 == 0", (long long)k_in);
  if (n_out < 16 || n_out % 16 || n_out > (int64_t(1) << 30))
    return fail(BL_ERR_UNSUPPORTED_SHAPE, "n_out=%lld: need n_out >= 16, n_out %% 16 == 0", (long long)n_out);
  return BL_OK;
}

int device_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  return sms;
}

// ------------------------------------------------------------------ TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner], boxes of [box_outer, box_inner], 128-byte
// swizzled unless `swizzle` is false.
bl_status make_map(CUtensorMap* m, CUtensorMapDataType dt, size_t elem, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_inner, uint32_t box_outer, bool swizzle = true) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(BL_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return BL_OK;
}

// Output tensor map of the TMA-store epilogue: [M, N] row-major, boxes of 32 rows x
// 128 bytes (64 bf16 or 32 fp32 columns), 128-byte swizzle.
bl_status make_out_map(CUtensorMap* m, const void* out, int64_t rows, int64_t cols, bool f32) {
  return make_map(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 ? 4 : 2, out, cols, rows,
                  f32 ? 32 : 64, 32);
}

template <bool kI8, bool kAMN, bool kBMN, int kEpi, bool kTmaStore>
bl_status launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tout, const bl::GemmArgs& g,
                      cudaStream_t st) {
  auto kern = bl::gemm_tc_kernel<kI8, kAMN, kBMN, kEpi, kTmaStore>;
  constexpr size_t smem = bl::gemm_smem_bytes(kTmaStore);
  static PerDeviceSetup setup;   // per instantiation
  int unused = 0;
  if (bl_status s = per_device_setup(setup, &unused, [&](int* r) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm)");
        *r = 1;
        return BL_OK;
      }))
    return s;
  const int tiles = g.num_m_blocks * g.num_n_blocks;
  const int grid = tiles < device_sm_count() ? tiles : device_sm_count();
  kern<<<grid, bl::kGemmThreads, smem, st>>>(ta, tb, tout, g);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return BL_OK;
}

// Two-SM version: clusters of two CTAs, each pair computing 256 x 256 output tiles
// (g.num_m_blocks / g.num_n_blocks count 256-wide blocks). Sets *launched to false and
// launches nothing when no CTA pair fits on the device, so the caller can fall back.
template <bool kI8, bool kAMN, bool kBMN, int kEpi>
bl_status launch_gemm2(const bl::GemmGroup2& G, cudaStream_t st, bool* launched) {
  *launched = false;
  auto kern = bl::gemm_tc2_kernel<kI8, kAMN, kBMN, kEpi>;
  constexpr size_t smem = bl::gemm2_smem_bytes();
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(bl::kGemmThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static PerDeviceSetup setup;   // per instantiation
  int max_clusters = 0;
  if (bl_status s = per_device_setup(setup, &max_clusters, [&](int* r) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemm2)");
        cudaLaunchConfig_t probe = cfg;
        probe.gridDim = dim3(2 * (device_sm_count() / 2));
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &probe);
        if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(gemm2)");
        *r = n > 0 ? n : 0;
        return BL_OK;
      }))
    return s;
  if (max_clusters <= 0) return BL_OK;
  const int tiles = G.total_tiles;
  const int clusters = tiles < max_clusters ? tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, G);
  if (e != cudaSuccess) return cuda_fail(e, "gemm2 launch");
  *launched = true;
  return BL_OK;
}

// A product as a group of one for the pair kernel (g counts 256-wide blocks).
bl::GemmGroup2 one_problem(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tout, const bl::GemmArgs& g) {
  bl::GemmGroup2 G{};
  G.p[0].tmA = ta;
  G.p[0].tmB = tb;
  G.p[0].tmOut = tout;
  G.p[0].g = g;
  G.p[0].tile_begin = 0;
  G.count = 1;
  G.total_tiles = g.num_m_blocks * g.num_n_blocks;
  G.num_k_blocks = g.num_k_blocks;
  return G;
}

// Pairs pay off once the output has at least two 128-row blocks; a single block would
// leave half of each pair's tensor work on rows outside the output.
inline bool use_cta_pair(int64_t m) { return m > bl::kBM; }

// Raster order of one product. By default tiles walk n blocks fastest (every wave
// re-reads all of B). When B is larger than L2 and A is small enough to stay there, m
// blocks go fastest instead, so that A is re-read from L2 and B streams once (grad_W of
// the down projection: X [16384 x 11008] bf16 is 360 MB; measured 1.91 -> 0.64 GB of
// DRAM reads per launch with the serpentine K order of the kernels). Eviction hints on
// the loads were measured and dropped: evict-first on the streamed operand doubled the
// DRAM reads (its lines left L2 before the other tiles of the same wave read them), and
// the hinted TMA form cost ~2 % of forward time.
void set_raster(bl::GemmArgs& g, double a_bytes, double b_bytes) {
  constexpr double kL2Bytes = 96e6;   // usable share of the 126 MB L2
  g.m_fastest = (b_bytes > kL2Bytes && a_bytes < b_bytes && a_bytes <= 0.7 * kL2Bytes) ? 1 : 0;
}

// ------------------------------------------------------------------ grouped codes product

// The warp-MMA decode kernel keeps its lookup table at a fixed shared-window address
// (bl::kDecLutAddr) below which its first ring slot must fit. Where the dynamic shared
// memory starts depends on the device and the driver, so the first launch on each device
// runs one CTA of the kernel in probe mode, reads that address back (synchronously: the
// first call must not be under stream capture) and remembers the result. A device
// where the table does not fit gets BL_ERR_CUDA from every call, before anything is
// enqueued, instead of a launch that would leave y unwritten.
constexpr int kMaxLayoutDevices = 64;
std::mutex g_dec_layout_mu;

template <int NG, int RB>
bl_status check_decode_layout(cudaStream_t st) {
  using C = bl::DecCfg<NG, RB>;
  static int g_dec_layout[kMaxLayoutDevices] = {};   // per kernel: 0 unchecked, 1 fits, -1 does not fit
  static unsigned int g_dec_base_seen[kMaxLayoutDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxLayoutDevices) return fail(BL_ERR_INVALID_ARG, "device ordinal %d not supported", dev);
  std::lock_guard<std::mutex> lock(g_dec_layout_mu);
  if (g_dec_layout[dev] == 0) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    if (cap != cudaStreamCaptureStatusNone)
      return fail(BL_ERR_CUDA, "the first decode-kernel call on a device checks its shared-memory layout "
                               "synchronously: make it before stream capture");
    e = cudaFuncSetAttribute(bl::fwd_codes_mma_kernel<NG, RB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
    static thread_local bl::FwdGroup probe;   // ~16 KB: kept off the stack
    probe.count = 0;
    probe.total_tasks = 0;
    probe.y_f32 = 0;
    probe.layout_probe = 1;
    bl::fwd_codes_mma_kernel<NG, RB><<<1, C::kThreads, C::kSmemBytes, st>>>(probe);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "decode layout probe launch");
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "decode layout probe");
    unsigned int base = 0;
    e = cudaMemcpyFromSymbol(&base, bl::g_dec_smem_base, sizeof(base));
    if (e != cudaSuccess) return cuda_fail(e, "decode layout read");
    g_dec_base_seen[dev] = base;
    g_dec_layout[dev] = (base + C::kSlotBytes <= bl::kDecLutAddr) ? 1 : -1;
  }
  if (g_dec_layout[dev] < 0)
    return fail(BL_ERR_CUDA, "decode kernel: dynamic shared memory starts at 0x%x, where its fixed-address lookup "
                             "table does not fit; use the int8-weight product (w_i8) or batches of 9+ tokens",
                g_dec_base_seen[dev]);
  return BL_OK;
}

template <int NG, int RB>
bl_status launch_fwd_codes_ng(const bl::FwdGroup& grp, cudaStream_t st) {
  using C = bl::DecCfg<NG, RB>;
  if (bl_status s = check_decode_layout<NG, RB>(st)) return s;
  int64_t blocks = (static_cast<int64_t>(grp.total_tasks) + C::kWarps - 1) / C::kWarps;
  const int64_t cap = int64_t(device_sm_count());   // one CTA per SM (persistent)
  if (blocks > cap) blocks = cap;
  bl::fwd_codes_mma_kernel<NG, RB><<<static_cast<unsigned>(blocks), C::kThreads, C::kSmemBytes, st>>>(grp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return BL_OK;
}

// Problems are already validated. Builds the task table in kernel parameters.
// Tensor-core product from codes: up to 128 tokens per task, 128 weight rows.
bl_status launch_fwd_codes_tc(const bl_fwd_problem* problems, int count, bool y_f32, cudaStream_t st) {
  static thread_local bl::FwdGroup grp;
  int64_t tasks = 0;
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const bl_fwd_problem& q = problems[i];
    if (q.t == 0) continue;
    bl::FwdProblem& d = grp.p[n++];
    d.codes = q.codes;
    d.xq = q.xq;
    d.absmax = q.absmax;
    d.w_scale = q.w_scale;
    d.y = q.y_out;
    d.acc = q.acc_out;
    d.t = static_cast<int>(q.t);
    d.k_in = static_cast<int>(q.k_in);
    d.n_out = static_cast<int>(q.n_out);
    d.task_begin = static_cast<int>(tasks);
    const int64_t nt = q.t < bl::kTcMaxN ? (q.t + 15) / 16 * 16 : bl::kTcMaxN;
    d.n_tile = static_cast<int>(nt);
    tasks += ((q.n_out + bl::kTcRows - 1) / bl::kTcRows) * ((q.t + nt - 1) / nt);
    if (tasks > INT32_MAX) return fail(BL_ERR_UNSUPPORTED_SHAPE, "too much work in one call");
  }
  grp.count = n;
  grp.total_tasks = static_cast<int>(tasks);
  grp.y_f32 = y_f32 ? 1 : 0;
  grp.layout_probe = 0;
  static PerDeviceSetup setup;
  int unused = 0;
  if (bl_status s = per_device_setup(setup, &unused, [&](int* r) {
        cudaError_t e = cudaFuncSetAttribute(bl::fwd_codes_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             bl::kTcSmemBytes);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(codes tc)");
        *r = 1;
        return BL_OK;
      }))
    return s;
  const int64_t blocks = tasks < device_sm_count() ? tasks : device_sm_count();
  bl::fwd_codes_tc_kernel<<<static_cast<unsigned>(blocks), bl::kTcThreads, bl::kTcSmemBytes, st>>>(grp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "codes tc launch");
  return BL_OK;
}

// Token batches of more than 8 tokens (the largest in a call) take the tensor-core
// product from codes; up to 8 the warp-MMA kernel (one 8-token MMA column group).
// Measured on the 36-layer decode stack: 12 and 16 tokens on two warp-MMA column groups
// (32-row tasks) 0.377 and 0.391 ms, on the tensor cores 0.374 and 0.377 ms.
constexpr int64_t kCodesTcMinTokens = 9;

// Warp-MMA decode kernel with NG token groups of 8 per task (problems validated).
template <int NG>
bl_status launch_fwd_codes_mma(const bl_fwd_problem* problems, int count, bool y_f32, cudaStream_t st) {
  static thread_local bl::FwdGroup grp;   // ~16 KB: kept off the stack
  // tasks of RB 16-row blocks: the largest RB in {2, 1} that divides every problem's rows
  // (measured on B200, 36-layer 3B decode step: RB = 2 0.180 ms at batch 1, RB = 4 with a
  // quarter of the warps 0.194 ms, RB = 1 0.209 ms)
  int rb = 2;
  for (int i = 0; i < count; ++i)
    while (problems[i].t != 0 && problems[i].n_out % (16 * rb) != 0) rb >>= 1;
  const int rows = 16 * rb;
  int64_t tasks = 0;
  int n = 0;
  for (int i = 0; i < count; ++i) {
    const bl_fwd_problem& q = problems[i];
    if (q.t == 0) continue;
    bl::FwdProblem& d = grp.p[n++];
    d.codes = q.codes;
    d.xq = q.xq;
    d.absmax = q.absmax;
    d.w_scale = q.w_scale;
    d.y = q.y_out;
    d.acc = q.acc_out;
    d.t = static_cast<int>(q.t);
    d.k_in = static_cast<int>(q.k_in);
    d.n_out = static_cast<int>(q.n_out);
    d.task_begin = static_cast<int>(tasks);
    tasks += (q.n_out / rows) * ((q.t + 8 * NG - 1) / (8 * NG));
    if (tasks > INT32_MAX) return fail(BL_ERR_UNSUPPORTED_SHAPE, "too much work in one call");
  }
  grp.count = n;
  grp.total_tasks = static_cast<int>(tasks);
  grp.y_f32 = y_f32 ? 1 : 0;
  grp.layout_probe = 0;
  return rb == 2 ? launch_fwd_codes_ng<NG, 2>(grp, st) : launch_fwd_codes_ng<NG, 1>(grp, st);
}

bl_status launch_fwd_codes(const bl_fwd_problem* problems, int count, bool y_f32, cudaStream_t st) {
  int64_t tmax = 0;
  for (int i = 0; i < count; ++i) tmax = problems[i].t > tmax ? problems[i].t : tmax;
  if (tmax == 0) return BL_OK;
  if (tmax >= kCodesTcMinTokens) return launch_fwd_codes_tc(problems, count, y_f32, st);
  return launch_fwd_codes_mma<1>(problems, count, y_f32, st);
}

// ------------------------------------------------------------------ quant_mask launches

struct QmOutputs {
  uint8_t* mask;
  uint8_t* codes;
  int8_t* w_i8;
  int8_t* sp_values;
  uint8_t* sp_meta;
  int64_t k8, meta_pitch;   // metadata bytes per row and its padded row pitch
};

// The optional latent-weight update fused into pass 1: W <- fp32(W - lr * grad), in place.
struct QmUpdate {
  float* w = nullptr;                // the same tensor as the weights read (updated in place)
  const uint16_t* grad = nullptr;    // bf16 [n_out, k_in]; null: no update
  float lr = 0.0f;
};

// Padded extents of the 2:4 metadata: rows and logical K rounded up to 256, so that the
// sparse product's metadata loads never leave the tensor.
inline int64_t sp_rows(int64_t n_out) { return (n_out + bl::kSpPad - 1) / bl::kSpPad * bl::kSpPad; }
inline int64_t sp_meta_pitch(int64_t k_in) { return (k_in + bl::kSpPad - 1) / bl::kSpPad * bl::kSpPad / 8; }

int qm_blocks(int64_t numel);
int qm_blocks_launch(int64_t numel, int resident);

// Resident 256-thread blocks per SM of a kernel (registers decide it here), looked up
// once per kernel and device; 1 if the query fails.
template <typename K>
int resident_blocks(K kern, PerDeviceSetup& cache) {
  int n = 1;
  per_device_setup(cache, &n, [&](int* r) {
    int m = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, kern, bl::kQmThreads, 0) != cudaSuccess || m <= 0) m = 1;
    *r = m;
    return BL_OK;
  });
  return n > 0 ? n : 1;
}

// Pass 2 for one compile-time N:M and mask source; the 2:4 form exists only for
// 2:4-valid masks (at most two kept per aligned four), so only those instantiate it.
template <int M, int NK, bool kMaskIn>
void launch_codes(const uint4* w4, int64_t n8, int n_keep, float* gamma, const QmOutputs& o, cudaStream_t st) {
  constexpr bool kSpOk = NK <= 2;
  static PerDeviceSetup occ, occ_sp;   // per instantiation
  auto grid = [&](int resident) {
    const int64_t g = (n8 + bl::kQmThreads - 1) / bl::kQmThreads;
    const int64_t cap = int64_t(device_sm_count()) * resident;
    return static_cast<int>(g < cap ? g : cap);
  };
  uint16_t* codes = reinterpret_cast<uint16_t*>(o.codes);
  uint2* w_i8 = reinterpret_cast<uint2*>(o.w_i8);
  if (kSpOk && o.sp_values != nullptr) {
    auto k = bl::qm_codes_kernel<M, NK, kMaskIn, kSpOk>;
    k<<<grid(resident_blocks(k, occ_sp)), bl::kQmThreads, 0, st>>>(w4, n8, n_keep, gamma, o.mask, codes, w_i8,
                                                                     reinterpret_cast<uint32_t*>(o.sp_values),
                                                                     o.sp_meta, o.k8, o.meta_pitch);
  } else {
    auto k = bl::qm_codes_kernel<M, NK, kMaskIn, false>;
    k<<<grid(resident_blocks(k, occ)), bl::kQmThreads, 0, st>>>(w4, n8, n_keep, gamma, o.mask, codes, w_i8, nullptr,
                                                                  nullptr, o.k8, o.meta_pitch);
  }
}

// Pass 1 for one compile-time N:M, mask choice and update choice.
template <int M, int NK, bool kMask, bool kUpdate>
void launch_sum(const uint4* w4, int64_t numel, int n_keep, const QmOutputs& o, const bl::QmScratch& q, float* gamma,
                const QmUpdate& u, cudaStream_t st) {
  static PerDeviceSetup occ;   // per instantiation
  auto k = bl::qm_sum_mask_kernel<M, NK, kMask, kUpdate>;
  const int grid = qm_blocks_launch(numel, device_sm_count() * resident_blocks(k, occ));
  k<<<grid, bl::kQmThreads, 0, st>>>(w4, numel / 8, numel, n_keep, q, gamma, kMask ? o.mask : nullptr,
                                    reinterpret_cast<uint4*>(u.w), reinterpret_cast<const uint4*>(u.grad), u.lr);
}

// Both passes for one compile-time N:M. With a mask output, pass 1 ranks the groups and
// stores the keep bits there, and pass 2 reads them back; without one, pass 2 ranks.
// With an update (u.grad set), pass 1 first applies it to W in place.
// Both grids are one wave of resident blocks (grid-stride loops): a partial second wave
// would leave most SMs idle at the end of each pass.
template <int M, int NK>
void launch_quant_mask(const float* w, int64_t numel, int n_keep, const QmOutputs& o, const bl::QmScratch& q,
                       float* gamma, const QmUpdate& u, cudaStream_t st) {
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  const int64_t n8 = numel / 8;
  const bool upd = u.grad != nullptr;
  if (o.mask != nullptr) {
    if (upd) launch_sum<M, NK, true, true>(w4, numel, n_keep, o, q, gamma, u, st);
    else launch_sum<M, NK, true, false>(w4, numel, n_keep, o, q, gamma, u, st);
    launch_codes<M, NK, true>(w4, n8, n_keep, gamma, o, st);
  } else {
    if (upd) launch_sum<8, 8, false, true>(w4, numel, n_keep, o, q, gamma, u, st);
    else launch_sum<8, 8, false, false>(w4, numel, n_keep, o, q, gamma, u, st);
    launch_codes<M, NK, false>(w4, n8, n_keep, gamma, o, st);
  }
}

// Both passes of steps a1 + a2 on `scratch` (its first 16 bytes are cleared here).
bl_status enqueue_quant_mask(const float* w, int64_t n_out, int64_t k_in, int n_keep, int m_group, const QmOutputs& o,
                             float* gamma, void* scratch, cudaStream_t st, const QmUpdate& u = QmUpdate{}) {
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaError_t e = cudaMemsetAsync(ws, 0, 16, st);   // range flag, status, blocks-done ticket
  if (e != cudaSuccess) return cuda_fail(e, "scratch reset");
  const int64_t numel = n_out * k_in;
  const bl::QmScratch q{reinterpret_cast<unsigned int*>(ws), reinterpret_cast<int*>(ws + 4),
                        reinterpret_cast<unsigned int*>(ws + 8),
                        reinterpret_cast<unsigned long long*>(ws + bl::kQmWsHeader)};
  if (m_group == 8) {
    switch (n_keep) {
      case 8: launch_quant_mask<8, 8>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 7: launch_quant_mask<8, 7>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 6: launch_quant_mask<8, 6>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 5: launch_quant_mask<8, 5>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 4: launch_quant_mask<8, 4>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 3: launch_quant_mask<8, 3>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 2: launch_quant_mask<8, 2>(w, numel, n_keep, o, q, gamma, u, st); break;
      default: launch_quant_mask<8, 1>(w, numel, n_keep, o, q, gamma, u, st); break;
    }
  } else {
    switch (n_keep) {
      case 4: launch_quant_mask<4, 4>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 3: launch_quant_mask<4, 3>(w, numel, n_keep, o, q, gamma, u, st); break;
      case 2: launch_quant_mask<4, 2>(w, numel, n_keep, o, q, gamma, u, st); break;
      default: launch_quant_mask<4, 1>(w, numel, n_keep, o, q, gamma, u, st); break;
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quant_mask launch");
  if (o.sp_meta != nullptr) {   // padding: the valid pattern 0x4 in every group (positions 0, 1)
    if (o.meta_pitch > o.k8) {
      e = cudaMemset2DAsync(o.sp_meta + o.k8, static_cast<size_t>(o.meta_pitch), 0x44,
                            static_cast<size_t>(o.meta_pitch - o.k8), static_cast<size_t>(n_out), st);
      if (e != cudaSuccess) return cuda_fail(e, "metadata column padding");
    }
    const int64_t pad_rows = sp_rows(n_out) - n_out;
    if (pad_rows > 0) {
      e = cudaMemsetAsync(o.sp_meta + n_out * o.meta_pitch, 0x44, static_cast<size_t>(pad_rows * o.meta_pitch), st);
      if (e != cudaSuccess) return cuda_fail(e, "metadata row padding");
    }
  }
  return BL_OK;
}

// ------------------------------------------------------------------ quant_mask sizing

// Upper bound on the blocks of the sum pass (sizes the workspace: one 16-byte partial per
// block): enough to fill 148 SMs with 8 blocks each, and enough that no thread sums more
// than kQmMaxElemsPerThread weights.
constexpr int kQmTargetBlocks = 148 * 8;

int qm_blocks_bounded(int64_t numel, int64_t target) {
  const int64_t n4 = numel / 4;
  int64_t need = (numel + (int64_t(bl::kQmThreads) * bl::kQmMaxElemsPerThread) - 1) /
                 (int64_t(bl::kQmThreads) * bl::kQmMaxElemsPerThread);   // bounds elements per thread
  int64_t fill = (n4 + bl::kQmThreads - 1) / bl::kQmThreads;
  if (fill > target) fill = target;
  int64_t b = need > fill ? need : fill;
  if (b < 1) b = 1;
  return static_cast<int>(b);
}

int qm_blocks(int64_t numel) { return qm_blocks_bounded(numel, kQmTargetBlocks); }

// Blocks actually launched: one wave of `resident` blocks (never more than the
// workspace bound).
int qm_blocks_launch(int64_t numel, int resident) {
  const int b = qm_blocks_bounded(numel, resident < kQmTargetBlocks ? resident : kQmTargetBlocks);
  const int bound = qm_blocks(numel);
  return b < bound ? b : bound;
}

// Rows of 513..2048 vectors: the persistent ring kernel, a two-row ring per CTA and as
// many CTAs as fit on an SM (shared memory decides), one wave. Measured on B200 for
// 16384 x 11008: 99 us with two rows per ring, 101 us with three, 111 us with four
// (fewer CTAs per SM), 132 us for one CTA per row without a ring.
template <int VPT>
bl_status launch_act_quant_ring(const uint4* xv, int64_t t, int k8, int8_t* xq_out, float* absmax_out,
                                cudaStream_t st) {
  constexpr int kD = 2;
  constexpr int smem = kD * VPT * 256 * 16;
  static PerDeviceSetup setup;   // per instantiation
  int occ = 1;
  if (bl_status s = per_device_setup(setup, &occ, [&](int* r) {
        cudaError_t e = cudaFuncSetAttribute(bl::act_quant_ring_kernel<VPT, kD>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(act_quant ring)");
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, bl::act_quant_ring_kernel<VPT, kD>, 256, smem) !=
                cudaSuccess ||
            n <= 0)
          n = 1;
        *r = n;
        return BL_OK;
      }))
    return s;
  int64_t grid = int64_t(device_sm_count()) * occ;
  if (grid > t) grid = t;
  bl::act_quant_ring_kernel<VPT, kD><<<static_cast<unsigned>(grid), 256, smem, st>>>(xv, t, k8, xq_out, absmax_out);
  return BL_OK;
}

// Launch of the act_quant kernels (arguments already checked).
bl_status enqueue_act_quant(const uint16_t* x, int64_t t, int64_t k_in, int8_t* xq_out, float* absmax_out,
                            cudaStream_t st) {
  const int k8 = static_cast<int>(k_in / 8);
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const unsigned g1 = static_cast<unsigned>(t);
  if (k8 <= 512) {   // k_in <= 4096: one warp per row, one row per warp (blocks that finish
                     // make room for new ones, so row loads overlap other rows' stores;
                     // 5 % faster than persistent warps for 16384 x 2048)
    const int64_t blocks = (t + 7) / 8;
    if (blocks > INT32_MAX) return fail(BL_ERR_UNSUPPORTED_SHAPE, "too many rows");
    const unsigned gb = static_cast<unsigned>(blocks);
    if (k8 <= 128) bl::act_quant_warp_kernel<4><<<gb, 256, 0, st>>>(xv, t, k8, xq_out, absmax_out);
    else if (k8 <= 256) bl::act_quant_warp_kernel<8><<<gb, 256, 0, st>>>(xv, t, k8, xq_out, absmax_out);
    else bl::act_quant_warp_kernel<16><<<gb, 256, 0, st>>>(xv, t, k8, xq_out, absmax_out);
  } else {   // up to 16384 wide: persistent ring CTAs; wider: one CTA per row
    const int vpt = (k8 + 255) / 256;
    bl_status s = BL_OK;
    if (vpt <= 4) s = launch_act_quant_ring<4>(xv, t, k8, xq_out, absmax_out, st);
    else if (vpt <= 6) s = launch_act_quant_ring<6>(xv, t, k8, xq_out, absmax_out, st);
    else if (vpt <= 8) s = launch_act_quant_ring<8>(xv, t, k8, xq_out, absmax_out, st);
    else if (vpt <= 12) bl::act_quant_kernel<12, 1><<<g1, 256, 0, st>>>(xv, t, k8, xq_out, absmax_out);
    else if (vpt <= 16) bl::act_quant_kernel<16, 1><<<g1, 256, 0, st>>>(xv, t, k8, xq_out, absmax_out);
    else bl::act_quant_long_kernel<<<g1, 256, 0, st>>>(xv, k8, xq_out, absmax_out);
    if (s != BL_OK) return s;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "act_quant launch");
  return BL_OK;
}

// The int8 tensor-core product y = (xq . w_i8^T) * (absmax / 127 * gamma) with w_i8
// [n_out, k_in] K-major (arguments already checked).
bl_status enqueue_fwd_i8(const int8_t* xq, const float* absmax, const int8_t* w_i8, const float* w_scale, int64_t t,
                         int64_t k_in, int64_t n_out, int32_t* acc_out, void* y_out, bool y_f32, cudaStream_t st) {
  CUtensorMap ta, tb;
  if (bl_status s = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, k_in, t, 128, bl::kBM)) return s;
  if (bl_status s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_i8, k_in, n_out, 128, bl::kBN)) return s;
  bl::GemmArgs g{};
  g.M = static_cast<int>(t);
  g.N = static_cast<int>(n_out);
  g.num_k_blocks = static_cast<int>((k_in + 127) / 128);
  g.num_m_blocks = static_cast<int>((t + bl::kBM - 1) / bl::kBM);
  g.num_n_blocks = static_cast<int>((n_out + bl::kBN - 1) / bl::kBN);
  g.out = y_out;
  g.out_f32 = y_f32 ? 1 : 0;
  g.acc_out = acc_out;
  g.row_absmax = absmax;
  g.w_scale = w_scale;
  set_raster(g, double(t) * double(k_in), double(n_out) * double(k_in));
  if (acc_out) {   // int32 accumulators requested: per-row direct stores of y and acc
    return launch_gemm<true, false, false, bl::EPI_FWD, false>(ta, tb, ta, g, st);
  }
  CUtensorMap to;
  if (bl_status s = make_out_map(&to, y_out, t, n_out, g.out_f32)) return s;
  if (use_cta_pair(t)) {   // each CTA of a pair loads 128 of the tile's 256 weight rows
    CUtensorMap tb2;
    if (bl_status s = make_map(&tb2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w_i8, k_in, n_out, 128, 128)) return s;
    bl::GemmArgs g2 = g;
    g2.num_m_blocks = static_cast<int>((t + 255) / 256);
    bool launched = false;
    if (bl_status s = launch_gemm2<true, false, false, bl::EPI_FWD>(one_problem(ta, tb2, to, g2), st, &launched))
      return s;
    if (launched) return BL_OK;
  }
  return launch_gemm<true, false, false, bl::EPI_FWD, true>(ta, tb, to, g, st);
}

// The 2:4 sparse product on CTA pairs (weights on M, tokens on N; arguments checked,
// k_in % 128 == 0).
bl_status enqueue_fwd_sp(const int8_t* xq, const float* absmax, const int8_t* sp_values, const uint8_t* sp_meta,
                         const float* w_scale, int64_t t, int64_t k_in, int64_t n_out, int32_t* acc_out, void* y_out,
                         bool y_f32, cudaStream_t st) {
  CUtensorMap ta, tb, te;
  if (bl_status s = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sp_values, k_in / 2, n_out, 128, 128)) return s;
  if (bl_status s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, xq, k_in, t, 128, bl::kSpTokHalf)) return s;
  if (bl_status s = make_map(&te, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, sp_meta, sp_meta_pitch(k_in), sp_rows(n_out), 16,
                             128, false))
    return s;
  CUtensorMap ty;
  const bool tma_store = acc_out == nullptr;
  if (tma_store) {
    if (bl_status s = make_map(&ty, y_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                               y_f32 ? 4 : 2, y_out, n_out, t, 32, 16, false))
      return s;
  } else {
    ty = te;   // unused
  }
  bl::SpGemmArgs g{};
  g.tma_store = tma_store ? 1 : 0;
  g.T = static_cast<int>(t);
  g.n_out = static_cast<int>(n_out);
  g.k_in = static_cast<int>(k_in);
  g.num_k_blocks = static_cast<int>((k_in + bl::kSpKStep - 1) / bl::kSpKStep);
  g.num_row_blocks = static_cast<int>((n_out + bl::kSpRowsPair - 1) / bl::kSpRowsPair);
  g.num_tok_blocks = static_cast<int>((t + bl::kSpTok - 1) / bl::kSpTok);
  g.y = y_out;
  g.y_f32 = y_f32 ? 1 : 0;
  g.acc_out = acc_out;
  g.absmax = absmax;
  g.w_scale = w_scale;
  constexpr size_t smem = bl::gemm_sp2_smem_bytes();
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(bl::kSpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static PerDeviceSetup setup;
  int max_clusters = 0;
  if (bl_status s = per_device_setup(setup, &max_clusters, [&](int* r) {
        cudaError_t e =
            cudaFuncSetAttribute(bl::gemm_sp2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(sparse gemm)");
        cudaLaunchConfig_t probe = cfg;
        probe.gridDim = dim3(2 * (device_sm_count() / 2));
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, bl::gemm_sp2_kernel, &probe);
        if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(sparse gemm)");
        *r = n > 0 ? n : 0;
        return BL_OK;
      }))
    return s;
  if (max_clusters <= 0) return fail(BL_ERR_CUDA, "no CTA pair of the sparse product fits on this device");
  const int tiles = g.num_row_blocks * g.num_tok_blocks;
  const int clusters = tiles < max_clusters ? tiles : max_clusters;
  cfg.gridDim = dim3(2 * clusters);
  cudaError_t e = cudaLaunchKernelEx(&cfg, bl::gemm_sp2_kernel, ta, tb, te, ty, g);
  if (e != cudaSuccess) return cuda_fail(e, "sparse gemm launch");
  return BL_OK;
}

// Choice between the 2:4 sparse and the dense int8 product when the caller gives both
// forms, from the measured crossover (forward per shape on B200): the sparse product wins
// on the Qwen2.5-1.5B MLP products at 8192 tokens (225 GOP dense-equivalent each:
// 1.07-1.32x) and loses on the Qwen2.5-0.5B products at 4096 tokens (up to 36 GOP:
// 0.84-0.93x), where the fixed cost per tile (metadata copy, accumulator hand-off,
// transposed epilogue) is not amortised.
constexpr double kSparseMinOps = 100e9;
inline bool use_sparse_product(int64_t t, int64_t k_in, int64_t n_out) {
  return 2.0 * double(t) * double(k_in) * double(n_out) >= kSparseMinOps;
}

inline size_t round256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

extern "C" {

int bitlinear_abi_version(void) { return 2; }

const char* bitlinear_last_error(void) { return g_err; }

size_t bitlinear_quant_mask_workspace_size(int64_t n_out, int64_t k_in) {
  if (n_out <= 0 || k_in <= 0) return bl::kQmWsHeader;
  return bl::kQmWsHeader + 16 * static_cast<size_t>(qm_blocks(n_out * k_in));
}

bl_status bitlinear_quant_mask(const float* w_latent, int64_t n_out, int64_t k_in, int n_keep, int m_group,
                               uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out, int8_t* sp_values_out,
                               uint8_t* sp_meta_out, float* w_scale_out, void* workspace, size_t workspace_bytes,
                               void* stream) {
  g_err[0] = 0;
  if (!w_latent || !codes_out || !w_scale_out) return fail(BL_ERR_INVALID_ARG, "w_latent, codes_out, w_scale_out are required");
  if (bl_status s = check_shape(0, k_in, n_out)) return s;
  if (!(m_group == 4 || m_group == 8) || n_keep < 1 || n_keep > m_group)
    return fail(BL_ERR_INVALID_ARG, "N:M = %d:%d: need M in {4, 8} and 1 <= N <= M", n_keep, m_group);
  if ((sp_values_out == nullptr) != (sp_meta_out == nullptr))
    return fail(BL_ERR_INVALID_ARG, "give both sp_values_out and sp_meta_out, or neither");
  if (sp_values_out && n_keep > 2)
    return fail(BL_ERR_INVALID_ARG, "N:M = %d:%d is not 2:4-valid (at most 2 kept per aligned 4): no 2:4 storage",
                n_keep, m_group);
  if (!workspace) return fail(BL_ERR_WORKSPACE, "workspace is required");
  if (workspace_bytes < bitlinear_quant_mask_workspace_size(n_out, k_in))
    return fail(BL_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes,
                bitlinear_quant_mask_workspace_size(n_out, k_in));
  if (!aligned16(w_latent) || !aligned16(codes_out) || !aligned16(w_scale_out) || !aligned16(workspace) ||
      (mask_out && !aligned16(mask_out)) || (w_i8_out && !aligned16(w_i8_out)) ||
      (sp_values_out && !aligned16(sp_values_out)) || (sp_meta_out && !aligned16(sp_meta_out)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  const QmOutputs o{mask_out, codes_out, w_i8_out, sp_values_out, sp_meta_out, k_in / 8, sp_meta_pitch(k_in)};
  return enqueue_quant_mask(w_latent, n_out, k_in, n_keep, m_group, o, w_scale_out, workspace, as_stream(stream));
}

bl_status bitlinear_sgd_quant_mask(float* w_latent, const uint16_t* grad_w, float lr, int64_t n_out, int64_t k_in,
                                   int n_keep, int m_group, uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out,
                                   int8_t* sp_values_out, uint8_t* sp_meta_out, float* w_scale_out, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  if (!grad_w) return fail(BL_ERR_INVALID_ARG, "grad_w is required");
  if (!std::isfinite(lr)) return fail(BL_ERR_INVALID_ARG, "lr must be finite");
  if (!aligned16(grad_w)) return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  if (!w_latent || !codes_out || !w_scale_out) return fail(BL_ERR_INVALID_ARG, "w_latent, codes_out, w_scale_out are required");
  if (bl_status s = check_shape(0, k_in, n_out)) return s;
  if (!(m_group == 4 || m_group == 8) || n_keep < 1 || n_keep > m_group)
    return fail(BL_ERR_INVALID_ARG, "N:M = %d:%d: need M in {4, 8} and 1 <= N <= M", n_keep, m_group);
  if ((sp_values_out == nullptr) != (sp_meta_out == nullptr))
    return fail(BL_ERR_INVALID_ARG, "give both sp_values_out and sp_meta_out, or neither");
  if (sp_values_out && n_keep > 2)
    return fail(BL_ERR_INVALID_ARG, "N:M = %d:%d is not 2:4-valid (at most 2 kept per aligned 4): no 2:4 storage",
                n_keep, m_group);
  if (!workspace) return fail(BL_ERR_WORKSPACE, "workspace is required");
  if (workspace_bytes < bitlinear_quant_mask_workspace_size(n_out, k_in))
    return fail(BL_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes,
                bitlinear_quant_mask_workspace_size(n_out, k_in));
  if (!aligned16(w_latent) || !aligned16(codes_out) || !aligned16(w_scale_out) || !aligned16(workspace) ||
      (mask_out && !aligned16(mask_out)) || (w_i8_out && !aligned16(w_i8_out)) ||
      (sp_values_out && !aligned16(sp_values_out)) || (sp_meta_out && !aligned16(sp_meta_out)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  const QmOutputs o{mask_out, codes_out, w_i8_out, sp_values_out, sp_meta_out, k_in / 8, sp_meta_pitch(k_in)};
  QmUpdate u;
  u.w = w_latent;
  u.grad = grad_w;
  u.lr = lr;
  return enqueue_quant_mask(w_latent, n_out, k_in, n_keep, m_group, o, w_scale_out, workspace, as_stream(stream), u);
}

bl_status bitlinear_quant_mask_status(const void* workspace, void* stream) {
  g_err[0] = 0;
  if (!workspace) return fail(BL_ERR_WORKSPACE, "workspace is required");
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int status = 0;
  e = cudaMemcpy(&status, static_cast<const uint8_t*>(workspace) + 4, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (status == BL_ERR_RANGE) return fail(BL_ERR_RANGE, "latent weight non-finite or |w| >= 2^16");
  return BL_OK;
}

bl_status bitlinear_act_quant(const uint16_t* x, int64_t t, int64_t k_in, int8_t* xq_out, float* absmax_out, void* stream) {
  g_err[0] = 0;
  if (bl_status s = check_shape(t, k_in, 16)) return s;
  if (t == 0) return BL_OK;   // empty batch: the t-sized arrays may be NULL
  if (!x || !xq_out || !absmax_out) return fail(BL_ERR_INVALID_ARG, "x, xq_out, absmax_out are required");
  if (!aligned16(x) || !aligned16(xq_out) || !aligned16(absmax_out))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  return enqueue_act_quant(x, t, k_in, xq_out, absmax_out, as_stream(stream));
}

bl_status bitlinear_fwd(const int8_t* xq, const float* absmax, const uint8_t* codes, const int8_t* w_i8,
                        const int8_t* sp_values, const uint8_t* sp_meta, const float* w_scale, int64_t t, int64_t k_in,
                        int64_t n_out, int32_t* acc_out, void* y_out, int y_dtype, void* stream) {
  g_err[0] = 0;
  if (!w_scale) return fail(BL_ERR_INVALID_ARG, "w_scale is required");
  if ((sp_values == nullptr) != (sp_meta == nullptr))
    return fail(BL_ERR_INVALID_ARG, "give both sp_values and sp_meta, or neither");
  if (!codes && !w_i8 && !sp_values) return fail(BL_ERR_INVALID_ARG, "give codes, w_i8 or sp_values + sp_meta");
  if (y_dtype != BL_OUT_BF16 && y_dtype != BL_OUT_F32) return fail(BL_ERR_INVALID_ARG, "y_dtype must be BL_OUT_BF16 or BL_OUT_F32");
  if (bl_status s = check_shape(t, k_in, n_out)) return s;
  if (!aligned16(w_scale) || (codes && !aligned16(codes)) || (w_i8 && !aligned16(w_i8)) ||
      (sp_values && !aligned16(sp_values)) || (sp_meta && !aligned16(sp_meta)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  if (t == 0) return BL_OK;   // empty batch: the t-sized arrays may be NULL
  if (!xq || !absmax || !y_out) return fail(BL_ERR_INVALID_ARG, "xq, absmax, y_out are required");
  if (!aligned16(xq) || !aligned16(absmax) || !aligned16(y_out) || (acc_out && !aligned16(acc_out)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  if (sp_values && (!w_i8 || use_sparse_product(t, k_in, n_out)))
    return enqueue_fwd_sp(xq, absmax, sp_values, sp_meta, w_scale, t, k_in, n_out, acc_out, y_out, y_dtype == BL_OUT_F32, st);
  if (w_i8) return enqueue_fwd_i8(xq, absmax, w_i8, w_scale, t, k_in, n_out, acc_out, y_out, y_dtype == BL_OUT_F32, st);
  bl_fwd_problem prob{xq, absmax, codes, w_scale, t, k_in, n_out, acc_out, y_out};
  return launch_fwd_codes(&prob, 1, y_dtype == BL_OUT_F32, st);
}

bl_status bitlinear_fwd_grouped(const bl_fwd_problem* problems, int count, int y_dtype, void* stream) {
  g_err[0] = 0;
  if (!problems || count < 0) return fail(BL_ERR_INVALID_ARG, "problems is required");
  if (count > bl::kMaxFwdGroup) return fail(BL_ERR_UNSUPPORTED_SHAPE, "at most %d problems per call", bl::kMaxFwdGroup);
  if (y_dtype != BL_OUT_BF16 && y_dtype != BL_OUT_F32) return fail(BL_ERR_INVALID_ARG, "y_dtype must be BL_OUT_BF16 or BL_OUT_F32");
  for (int i = 0; i < count; ++i) {
    const bl_fwd_problem& q = problems[i];
    if (bl_status s = check_shape(q.t, q.k_in, q.n_out)) return fail(s, "problem %d: %s", i, g_err);
    if (!q.codes || !q.w_scale) return fail(BL_ERR_INVALID_ARG, "problem %d: codes and w_scale are required", i);
    if (q.t > 0 && (!q.xq || !q.absmax || !q.y_out)) return fail(BL_ERR_INVALID_ARG, "problem %d: xq, absmax, y_out are required", i);
    if (!aligned16(q.codes) || !aligned16(q.w_scale) || (q.xq && !aligned16(q.xq)) || (q.absmax && !aligned16(q.absmax)) ||
        (q.y_out && !aligned16(q.y_out)) || (q.acc_out && !aligned16(q.acc_out)))
      return fail(BL_ERR_ALIGNMENT, "problem %d: every pointer must be 16-byte aligned", i);
  }
  return launch_fwd_codes(problems, count, y_dtype == BL_OUT_F32, as_stream(stream));
}

size_t bitlinear_bwd_workspace_size(int64_t t, int64_t k_in, int64_t n_out, int want_grad_x, int flags) {
  if (k_in <= 0 || n_out <= 0 || t < 0) return 0;
  size_t b = want_grad_x ? round256(static_cast<size_t>(n_out) * static_cast<size_t>(k_in) * 2) : 0;
  if (flags & BL_GRADW_DEQUANT_X) b += static_cast<size_t>(t) * static_cast<size_t>(k_in) * 2;
  return b;
}

bl_status bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const int8_t* xq, const float* absmax,
                        const uint8_t* codes, const float* w_scale, int64_t t, int64_t k_in, int64_t n_out,
                        uint16_t* grad_x, void* grad_w, int grad_w_dtype, int flags, void* workspace,
                        size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  if (!grad_x && !grad_w) return fail(BL_ERR_INVALID_ARG, "request grad_x, grad_w or both");
  if (flags & ~BL_GRADW_DEQUANT_X) return fail(BL_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  const bool deq = grad_w && (flags & BL_GRADW_DEQUANT_X);
  if (!dy && t != 0) return fail(BL_ERR_INVALID_ARG, "dy is required");
  if (grad_x && (!codes || !w_scale)) return fail(BL_ERR_INVALID_ARG, "grad_x needs codes and w_scale");
  if (grad_w && !deq && !x && t != 0) return fail(BL_ERR_INVALID_ARG, "grad_w needs x");
  if (deq && (!xq || !absmax) && t != 0)
    return fail(BL_ERR_INVALID_ARG, "BL_GRADW_DEQUANT_X needs xq and absmax");
  if (grad_w && grad_w_dtype != BL_OUT_BF16 && grad_w_dtype != BL_OUT_F32)
    return fail(BL_ERR_INVALID_ARG, "grad_w_dtype must be BL_OUT_BF16 or BL_OUT_F32");
  if (bl_status s = check_shape(t, k_in, n_out)) return s;
  if ((dy && !aligned16(dy)) || (x && !aligned16(x)) || (xq && !aligned16(xq)) || (absmax && !aligned16(absmax)) ||
      (codes && !aligned16(codes)) || (w_scale && !aligned16(w_scale)) || (grad_x && !aligned16(grad_x)) ||
      (grad_w && !aligned16(grad_w)) || (workspace && !aligned16(workspace)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  const size_t need = bitlinear_bwd_workspace_size(t, k_in, n_out, grad_x != nullptr, deq ? BL_GRADW_DEQUANT_X : 0);
  if (need && (!workspace || workspace_bytes < need))
    return fail(BL_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes, need);
  cudaStream_t st = as_stream(stream);
  if (t == 0) {
    if (grad_w) {
      const size_t bytes = static_cast<size_t>(n_out) * k_in * (grad_w_dtype == BL_OUT_F32 ? 4 : 2);
      cudaError_t e = cudaMemsetAsync(grad_w, 0, bytes, st);
      if (e != cudaSuccess) return cuda_fail(e, "grad_w zero");
    }
    return BL_OK;
  }
  if (grad_x) {
    // effective ternary matrix C [n_out, k_in] in bf16 (exact), gamma applied in the epilogue
    const int64_t nwords = n_out * k_in / 16;
    int64_t grid = (nwords + 255) / 256;
    const int64_t cap = int64_t(device_sm_count()) * 16;
    if (grid > cap) grid = cap;
    bl::expand_codes_bf16_kernel<<<(int)grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(codes), nwords,
                                                           static_cast<uint4*>(workspace));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "expand launch");
    CUtensorMap ta, tb;
    // A = dY [t, n_out], K-major (reduction over n_out); B = C [n_out, k_in], MN-major
    if (bl_status s = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dy, n_out, t, 64, bl::kBM)) return s;
    if (bl_status s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, workspace, k_in, n_out, 64, 64)) return s;
    bl::GemmArgs g{};
    g.M = static_cast<int>(t);
    g.N = static_cast<int>(k_in);
    g.num_k_blocks = static_cast<int>((n_out + 63) / 64);
    g.num_m_blocks = static_cast<int>((t + bl::kBM - 1) / bl::kBM);
    g.num_n_blocks = static_cast<int>((k_in + bl::kBN - 1) / bl::kBN);
    g.out = grad_x;
    g.out_f32 = 0;
    g.w_scale = w_scale;
    set_raster(g, 2.0 * double(t) * double(n_out), 2.0 * double(n_out) * double(k_in));
    CUtensorMap to;
    if (bl_status s = make_out_map(&to, grad_x, t, k_in, false)) return s;
    bool launched = false;
    if (use_cta_pair(t)) {
      bl::GemmArgs g2 = g;
      g2.num_m_blocks = static_cast<int>((t + 255) / 256);
      if (bl_status s = launch_gemm2<false, false, true, bl::EPI_GRADX>(one_problem(ta, tb, to, g2), st, &launched))
        return s;
    }
    if (!launched)
      if (bl_status s = launch_gemm<false, false, true, bl::EPI_GRADX, true>(ta, tb, to, g, st)) return s;
  }
  if (grad_w) {
    const void* xb = x;
    if (deq) {   // X_deq = q * a / 127 in bf16, after the ternary matrix in the workspace
      uint8_t* xd = static_cast<uint8_t*>(workspace) +
                    (grad_x ? round256(static_cast<size_t>(n_out) * static_cast<size_t>(k_in) * 2) : 0);
      const int64_t nchunks = t * k_in / 16;
      int64_t grid = (nchunks + 255) / 256;
      const int64_t cap = int64_t(device_sm_count()) * 16;
      if (grid > cap) grid = cap;
      bl::dequant_x_bf16_kernel<<<(int)grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(xq), absmax, nchunks,
                                                          static_cast<int>(k_in / 16), reinterpret_cast<uint4*>(xd));
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
      xb = xd;
    }
    CUtensorMap ta, tb;
    // A = dY^T: dY [t, n_out] read MN-major (reduction over t); B = X [t, k_in], MN-major
    if (bl_status s = make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dy, n_out, t, 64, 64)) return s;
    if (bl_status s = make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xb, k_in, t, 64, 64)) return s;
    bl::GemmArgs g{};
    g.M = static_cast<int>(n_out);
    g.N = static_cast<int>(k_in);
    g.num_k_blocks = static_cast<int>((t + 63) / 64);
    g.num_m_blocks = static_cast<int>((n_out + bl::kBM - 1) / bl::kBM);
    g.num_n_blocks = static_cast<int>((k_in + bl::kBN - 1) / bl::kBN);
    g.out = grad_w;
    g.out_f32 = grad_w_dtype == BL_OUT_F32;
    set_raster(g, 2.0 * double(n_out) * double(t), 2.0 * double(t) * double(k_in));
    CUtensorMap to;
    if (bl_status s = make_out_map(&to, grad_w, n_out, k_in, g.out_f32)) return s;
    bool launched = false;
    if (use_cta_pair(n_out)) {
      bl::GemmArgs g2 = g;
      g2.num_m_blocks = static_cast<int>((n_out + 255) / 256);
      if (bl_status s = launch_gemm2<false, true, true, bl::EPI_GRADW>(one_problem(ta, tb, to, g2), st, &launched))
        return s;
    }
    if (!launched)
      if (bl_status s = launch_gemm<false, true, true, bl::EPI_GRADW, true>(ta, tb, to, g, st)) return s;
  }
  return BL_OK;
}

bl_status bitlinear_grad_w_grouped(const bl_grad_w_problem* problems, int count, int64_t t, void* stream) {
  g_err[0] = 0;
  if (!problems || count < 1 || count > bl::kMaxGemmGroup)
    return fail(BL_ERR_INVALID_ARG, "need 1 to %d problems", bl::kMaxGemmGroup);
  for (int i = 0; i < count; ++i) {
    const bl_grad_w_problem& q = problems[i];
    if (!q.grad_w) return fail(BL_ERR_INVALID_ARG, "problem %d: grad_w is required", i);
    if ((!q.dy || !q.x) && t != 0) return fail(BL_ERR_INVALID_ARG, "problem %d: dy and x are required", i);
    if (q.grad_w_dtype != BL_OUT_BF16 && q.grad_w_dtype != BL_OUT_F32)
      return fail(BL_ERR_INVALID_ARG, "problem %d: grad_w_dtype must be BL_OUT_BF16 or BL_OUT_F32", i);
    if (bl_status s = check_shape(t, q.k_in, q.n_out)) return s;
    if ((q.dy && !aligned16(q.dy)) || (q.x && !aligned16(q.x)) || !aligned16(q.grad_w))
      return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  }
  cudaStream_t st = as_stream(stream);
  bool pairs = count > 1 && t > 0;
  for (int i = 0; i < count; ++i) pairs = pairs && use_cta_pair(problems[i].n_out);
  if (!pairs) {   // one product at a time (single problem, empty batch or narrow outputs)
    for (int i = 0; i < count; ++i) {
      const bl_grad_w_problem& q = problems[i];
      if (bl_status s = bitlinear_bwd(q.dy, q.x, nullptr, nullptr, nullptr, nullptr, t, q.k_in, q.n_out, nullptr,
                                      q.grad_w, q.grad_w_dtype, 0, nullptr, 0, stream))
        return s;
    }
    return BL_OK;
  }
  bl::GemmGroup2 G{};
  int tiles = 0;
  for (int i = 0; i < count; ++i) {
    const bl_grad_w_problem& q = problems[i];
    bl::GemmProblem2& P = G.p[i];
    // A = dY^T: dY [t, n_out] read MN-major (reduction over t); B = X [t, k_in], MN-major
    if (bl_status s = make_map(&P.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.dy, q.n_out, t, 64, 64)) return s;
    if (bl_status s = make_map(&P.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q.x, q.k_in, t, 64, 64)) return s;
    bl::GemmArgs& g = P.g;
    g.M = static_cast<int>(q.n_out);
    g.N = static_cast<int>(q.k_in);
    g.num_k_blocks = static_cast<int>((t + 63) / 64);
    g.num_m_blocks = static_cast<int>((q.n_out + 255) / 256);
    g.num_n_blocks = static_cast<int>((q.k_in + bl::kBN - 1) / bl::kBN);
    g.out = q.grad_w;
    g.out_f32 = q.grad_w_dtype == BL_OUT_F32;
    set_raster(g, 2.0 * double(q.n_out) * double(t), 2.0 * double(t) * double(q.k_in));
    if (bl_status s = make_out_map(&P.tmOut, q.grad_w, q.n_out, q.k_in, g.out_f32)) return s;
    P.tile_begin = tiles;
    tiles += g.num_m_blocks * g.num_n_blocks;
  }
  G.count = count;
  G.total_tiles = tiles;
  G.num_k_blocks = static_cast<int>((t + 63) / 64);
  bool launched = false;
  if (bl_status s = launch_gemm2<false, true, true, bl::EPI_GRADW>(G, st, &launched)) return s;
  if (launched) return BL_OK;
  for (int i = 0; i < count; ++i) {   // no CTA pair fits on this device: one at a time
    const bl_grad_w_problem& q = problems[i];
    if (bl_status s = bitlinear_bwd(q.dy, q.x, nullptr, nullptr, nullptr, nullptr, t, q.k_in, q.n_out, nullptr,
                                    q.grad_w, q.grad_w_dtype, 0, nullptr, 0, stream))
      return s;
  }
  return BL_OK;
}

size_t bitlinear_grad_x_i8_workspace_size(int64_t t, int64_t k_in, int64_t n_out) {
  if (t <= 0 || k_in <= 0 || n_out <= 0) return 0;
  return round256(static_cast<size_t>(t) * n_out) + round256(static_cast<size_t>(t) * 4) +
         static_cast<size_t>(k_in) * static_cast<size_t>(n_out);
}

bl_status bitlinear_grad_x_i8(const uint16_t* dy, const uint8_t* codes, const float* w_scale, int64_t t, int64_t k_in,
                              int64_t n_out, uint16_t* grad_x, int32_t* acc_out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  if (!codes || !w_scale) return fail(BL_ERR_INVALID_ARG, "codes and w_scale are required");
  if (bl_status s = check_shape(t, k_in, n_out)) return s;
  if (n_out % 64) return fail(BL_ERR_UNSUPPORTED_SHAPE, "n_out=%lld: the int8-dY gradient needs n_out %% 64 == 0", (long long)n_out);
  if (!aligned16(codes) || !aligned16(w_scale)) return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  if (t == 0) return BL_OK;
  if (!dy || !grad_x) return fail(BL_ERR_INVALID_ARG, "dy and grad_x are required");
  if (!aligned16(dy) || !aligned16(grad_x) || (acc_out && !aligned16(acc_out)) || (workspace && !aligned16(workspace)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  const size_t need = bitlinear_grad_x_i8_workspace_size(t, k_in, n_out);
  if (!workspace || workspace_bytes < need) return fail(BL_ERR_WORKSPACE, "workspace too small: %zu < %zu", workspace_bytes, need);
  cudaStream_t st = as_stream(stream);
  int8_t* dyq = static_cast<int8_t*>(workspace);
  float* a = reinterpret_cast<float*>(static_cast<char*>(workspace) + round256(static_cast<size_t>(t) * n_out));
  int8_t* ct = static_cast<int8_t*>(workspace) + round256(static_cast<size_t>(t) * n_out) + round256(static_cast<size_t>(t) * 4);
  if (bl_status s = enqueue_act_quant(dy, t, n_out, dyq, a, st)) return s;
  const dim3 grid(static_cast<unsigned>((n_out + 63) / 64), static_cast<unsigned>(k_in / 64));
  bl::expand_codes_t_i8_kernel<<<grid, 256, 0, st>>>(codes, static_cast<int>(n_out), static_cast<int>(k_in), ct);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "transpose-expand launch");
  // grad_x[t, k] = sum_n dyq[t, n] * C^T[k, n], rescaled by a_t / 127 * gamma
  return enqueue_fwd_i8(dyq, a, ct, w_scale, t, n_out, k_in, acc_out, grad_x, false, st);
}

bl_status bitlinear_mask_threshold_hist(const float* w_latent, const uint8_t* mask, const float* w_scale, int64_t n_out,
                                        int64_t k_in, int m_group, unsigned long long* hist_out, void* stream) {
  g_err[0] = 0;
  if (!w_latent || !mask || !w_scale || !hist_out) return fail(BL_ERR_INVALID_ARG, "w_latent, mask, w_scale, hist_out are required");
  if (m_group != 4 && m_group != 8) return fail(BL_ERR_INVALID_ARG, "m_group must be 4 or 8");
  if (bl_status s = check_shape(0, k_in, n_out)) return s;
  if (!aligned16(w_latent) || !aligned16(w_scale) || !aligned16(hist_out))
    return fail(BL_ERR_ALIGNMENT, "w_latent, w_scale and hist_out must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  cudaError_t e = cudaMemsetAsync(hist_out, 0, bl::kHistWords * sizeof(unsigned long long), st);
  if (e != cudaSuccess) return cuda_fail(e, "histogram clear");
  const int64_t ngroups = n_out * k_in / m_group;
  int64_t blocks = (ngroups + 255) / 256;
  const int64_t cap = int64_t(device_sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (m_group == 8)
    bl::threshold_hist_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, st>>>(w_latent, mask, w_scale, ngroups, hist_out);
  else
    bl::threshold_hist_kernel<4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(w_latent, mask, w_scale, ngroups, hist_out);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "histogram launch");
  return BL_OK;
}

bl_status bitlinear_device_status(unsigned int* bits) {
  g_err[0] = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "device synchronize");
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, bl::g_device_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  e = cudaMemcpyToSymbol(bl::g_device_status, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  if (bits) *bits = v;
  if (v & bl::DEV_ST_SMEM_LAYOUT)
    return fail(BL_ERR_CUDA, "a kernel found its shared memory at an unexpected address and skipped its work (status bits 0x%x)", v);
  if (v) return fail(BL_ERR_TIMEOUT, "a kernel gave up on a bounded wait (status bits 0x%x)", v);
  return BL_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ quant_mask without allocation
//
// Some callers cannot allocate device memory at all: code that runs inside a host
// framework owning every byte of device memory (a fixed arena or a caching pool that
// forbids outside cudaMalloc), and latency-critical paths where cudaMalloc/cudaFree
// (which may synchronise the whole device) are not allowed. For them,
// bitlinear_quant_mask_noalloc keeps its scratch (range flag, status word and the
// per-block partial sums) in the file-scope array below instead of a caller workspace.
//
// The array is a host-side stand-in in host code: its device address is fetched with
// cudaGetSymbolAddress once per device (with that device current) on the first call
// made on that device, and that address is what the kernels receive. Every call on a
// device shares the array: calls that overlap on the GPU (different streams, no
// ordering between them) race on it. Each call clears the header it needs at zero.

namespace {

constexpr size_t kNoAllocScratchBytes = 19200;   // 256-byte header + 16 B x 1184 block partials
static __device__ __align__(256) unsigned char g_qm_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

bl_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BL_ERR_INVALID_ARG, "device ordinal %d not supported", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_qm_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BL_OK;
}

}  // namespace

extern "C" bl_status bitlinear_quant_mask_noalloc(const float* w_latent, int64_t n_out, int64_t k_in, int n_keep,
                                                  int m_group, uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out,
                                                  float* w_scale_out, void* stream) {
  g_err[0] = 0;
  if (!w_latent || !codes_out || !w_scale_out) return fail(BL_ERR_INVALID_ARG, "w_latent, codes_out, w_scale_out are required");
  if (bl_status s = check_shape(0, k_in, n_out)) return s;
  if (!(m_group == 4 || m_group == 8) || n_keep < 1 || n_keep > m_group)
    return fail(BL_ERR_INVALID_ARG, "N:M = %d:%d: need M in {4, 8} and 1 <= N <= M", n_keep, m_group);
  const int64_t numel = n_out * k_in;
  const size_t need = bitlinear_quant_mask_workspace_size(n_out, k_in);
  if (need > kNoAllocScratchBytes)
    return fail(BL_ERR_UNSUPPORTED_SHAPE,
                "tensor of %lld weights needs %zu scratch bytes; the built-in scratch holds %zu "
                "(at most 4966055936 weights): use bitlinear_quant_mask with a workspace",
                (long long)numel, need, kNoAllocScratchBytes);
  if (!aligned16(w_latent) || !aligned16(codes_out) || !aligned16(w_scale_out) || (mask_out && !aligned16(mask_out)) ||
      (w_i8_out && !aligned16(w_i8_out)))
    return fail(BL_ERR_ALIGNMENT, "every pointer must be 16-byte aligned");
  void* scratch = nullptr;
  if (bl_status s = noalloc_scratch(&scratch)) return s;
  const QmOutputs o{mask_out, codes_out, w_i8_out, nullptr, nullptr, k_in / 8, k_in / 8};
  return enqueue_quant_mask(w_latent, n_out, k_in, n_keep, m_group, o, w_scale_out, scratch, as_stream(stream));
}
