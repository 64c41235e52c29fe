// Grouped forward product from the packed 2-bit codes on the 5th-generation tensor
// cores, for token batches of 16 and more (decode at larger batch, short prefill).
//
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 四: ternary weights travel from HBM
// in packed form and are unpacked on chip before the product with 8-bit activations.
// Here the unpacked weights never touch shared memory: they are written into tensor
// memory and the MMA reads its A operand from there.
//
// Per task (one problem, 128 weight rows, up to 128 tokens) the product is computed
// with the weights on M, so Y^T[n, t] = sum_k W[n, k] * Xq[t, k] accumulates in TMEM:
//   warps 0-1   cp.async producers: per stage the task's codes [128 rows x 64 B] (256
//               weights of K) and activations [tokens x 256 B] into a shared-memory
//               ring of 4 stages; completion through cp.async.mbarrier.arrive.
//   warp 2      TMEM allocator and MMA issuer: 8 x tcgen05.mma kind::i8 per stage with
//               A (M = 128, K = 32) from TMEM and B from shared memory (128B swizzle).
//   warps 3-10  decoders and epilogue: thread = one weight row; code bytes become
//               int8x4 words through a per-lane table and are stored into the stage's
//               A columns with tcgen05.st; after a task's last stage they read the
//               accumulator and write y[t, n] = acc * (a_t / 127) * gamma.
// Every wait is bounded (see common.cuh).
#pragma once

#include "codes_kernels.cuh"
#include "common.cuh"

namespace bl {

constexpr int kTcRows = 128;
constexpr int kTcMaxN = 128;                              // tokens per task
constexpr int kTcStages = 4;
constexpr int kTcCodeBytes = kTcRows * 64;                // 8 KB: 256 weights of 128 rows
constexpr int kTcBSub = kTcMaxN * 128;                    // one 128-byte-wide K slice of B
constexpr int kTcStageBytes = kTcCodeBytes + 2 * kTcBSub;  // 40 KB
constexpr int kTcProdWarps = 2;
constexpr int kTcMmaWarp = kTcProdWarps;
constexpr int kTcDecWarps = 8;
constexpr int kTcThreads = 32 * (kTcProdWarps + 1 + kTcDecWarps);
constexpr uint32_t kTcLutBytes = 256 * 128;               // entry e of lane l at 128*e + 4*l
constexpr uint32_t kTcDCols = 128;                        // accumulator columns
constexpr uint32_t kTcACols = 64;                         // A columns per stage (256 int8)
constexpr int kTcBarBytes = 256;
// worst case: 32 KB of padding to align the table, then table, stages, barriers
constexpr int kTcSmemBytes = 32767 + static_cast<int>(kTcLutBytes) + kTcStages * kTcStageBytes + kTcBarBytes;
static_assert(kTcSmemBytes <= 232448, "codes tensor-core kernel exceeds the shared memory of a CTA");

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem]^T, int8 inputs, int32 accumulate.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrive on `bar` once every cp.async issued so far by this thread has landed
// (the barrier's expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Per-lane table lookup of code byte J of w: entry e of lane l at lut + 128*e + 4*l, the
// table 32 KB-aligned so that `lanebase` = lut | 4*lane is OR-ed in.
template <int J>
__device__ __forceinline__ uint32_t lut128_lookup(uint32_t w, uint32_t lanebase) {
  const uint32_t off = ((J == 0 ? (w << 7) : (w >> (8 * J - 7))) & 0x7F80u) | lanebase;
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(off));
  return v;
}

struct TcTask {
  const FwdProblem* P;
  int n0, t0, nch;
};

// Tasks of problem p: ceil(n_out / 128) row blocks x ceil(t / n_tile) token blocks,
// row blocks fastest.
__device__ __forceinline__ TcTask tc_task(const FwdGroup& G, int task) {
  int lo = 0, hi = G.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (G.p[mid].task_begin <= task) lo = mid;
    else hi = mid - 1;
  }
  const FwdProblem& P = G.p[lo];
  const int row_blocks = (P.n_out + kTcRows - 1) / kTcRows;
  const int local = task - P.task_begin;
  TcTask d;
  d.P = &P;
  d.n0 = (local % row_blocks) * kTcRows;
  d.t0 = (local / row_blocks) * P.n_tile;
  d.nch = (P.k_in + 255) >> 8;
  return d;
}

__global__ void __launch_bounds__(kTcThreads, 1) fwd_codes_tc_kernel(const __grid_constant__ FwdGroup G) {
  extern __shared__ __align__(1024) uint8_t dsmem[];
  const uint32_t base = smem_u32(dsmem);
  const uint32_t lut = (base + 0x7FFFu) & ~0x7FFFu;
  const uint32_t stage0 = lut + kTcLutBytes;
  auto st_codes = [&](int s) { return stage0 + static_cast<uint32_t>(s * kTcStageBytes); };
  auto st_b = [&](int s) { return stage0 + static_cast<uint32_t>(s * kTcStageBytes + kTcCodeBytes); };
  const uint32_t bar0 = stage0 + kTcStages * kTcStageBytes;
  const uint32_t full0 = bar0, afull0 = bar0 + 8u * kTcStages, empty0 = bar0 + 16u * kTcStages;
  const uint32_t dfull = bar0 + 24u * kTcStages, dempty = dfull + 8u, done_bar = dfull + 16u;
  uint8_t* bar_gen = dsmem + (bar0 - base);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_gen + 24 * kTcStages + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const uint32_t e = static_cast<uint32_t>(i) >> 5, l = static_cast<uint32_t>(i) & 31u;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t f = (e >> (2 * j)) & 3u;
      word |= ((f & 1u) ? ((f & 2u) ? 0xFFu : 0x01u) : 0u) << (8 * j);
    }
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(lut + 128u * e + 4u * l), "r"(word) : "memory");
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(full0 + 8u * s, 32 * kTcProdWarps);   // every producer lane's cp.async arrive
      mbar_init(afull0 + 8u * s, kTcDecWarps);
      mbar_init(empty0 + 8u * s, 1);           // MMA commit
    }
    mbar_init(dfull, 1);
    mbar_init(dempty, kTcDecWarps);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < kTcProdWarps) {
    // ------------------------------------------------------------- cp.async producers
    // Producer warp pw copies, per stage, code rows (lane >> 2) + 8i and token rows
    // (lane >> 4) + 2i for i = pw, pw + kTcProdWarps, ...; a lane's 16-byte column
    // within a row never changes, so only row offsets advance.
    const int pw = warp;
    const int cc = lane & 3, crow0 = (lane >> 2) + 8 * pw;                 // codes
    const uint32_t cswz = static_cast<uint32_t>((cc ^ ((lane >> 3) & 3)) << 4);
    const int bc16 = lane & 15, brow0 = (lane >> 4) + 2 * pw;              // activations
    const uint32_t bsub = static_cast<uint32_t>((bc16 >> 3) * kTcBSub);
    const int bc = bc16 & 7;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int task = blockIdx.x; task < G.total_tasks && ok; task += gridDim.x) {
      const TcTask d = tc_task(G, task);
      const uint8_t* const codes = d.P->codes;
      const int8_t* const xq = d.P->xq;
      const int K = d.P->k_in, kb = K >> 2;
      const int rows_valid = min(kTcRows, d.P->n_out - d.n0);
      const int toks_valid = min(d.P->n_tile, d.P->t - d.t0);
      const int n_tile = d.P->n_tile;
      const uint8_t* csrc = codes + static_cast<int64_t>(d.n0 + crow0) * kb + cc * 16;
      const int8_t* bsrc = xq + static_cast<int64_t>(d.t0 + brow0) * K + bc16 * 16;
      const int64_t cstep = static_cast<int64_t>(8 * kTcProdWarps) * kb;
      const int64_t bstep = static_cast<int64_t>(2 * kTcProdWarps) * K;
      for (int ch = 0; ch < d.nch; ++ch) {
        const bool got = mbar_wait(empty0 + 8u * s, ph ^ 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const uint32_t cdst = st_codes(s) + cswz;
        const bool ck = ch * 64 + cc * 16 < kb;
        const uint8_t* src = csrc + ch * 64;
#pragma unroll
        for (int row = crow0; row < kTcRows; row += 8 * kTcProdWarps) {
          const bool valid = ck && row < rows_valid;
          cp_async16(cdst + static_cast<uint32_t>(row * 64), valid ? src : codes, valid);
          src += cstep;
        }
        const uint32_t bdst = st_b(s) + bsub;
        const bool bk = ch * 256 + bc16 * 16 < K;
        const int8_t* bs = bsrc + ch * 256;
        for (int row = brow0; row < n_tile; row += 2 * kTcProdWarps) {
          const bool valid = bk && row < toks_valid;
          cp_async16(bdst + static_cast<uint32_t>(row * 128 + ((bc ^ (row & 7)) << 4)), valid ? bs : xq, valid);
          bs += bstep;
        }
        cp_async_arrive_noinc(full0 + 8u * s);
        if (++s == kTcStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(&g_device_status, DEV_ST_TIMEOUT_PRODUCER);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight when the thread exits
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int task = blockIdx.x; task < G.total_tasks && ok; task += gridDim.x, ++local) {
        const TcTask d = tc_task(G, task);
        const uint32_t idesc = make_idesc(2u, 1u, 1u, 0u, 0u, static_cast<uint32_t>(d.P->n_tile), kTcRows);
        if (!mbar_wait(dempty, (static_cast<uint32_t>(local) & 1u) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int ch = 0; ch < d.nch; ++ch) {
          if (!mbar_wait(afull0 + 8u * s, ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          fence_proxy_async_smem();   // activations were written by cp.async (generic proxy)
          const uint32_t a_stage = tmem_base + kTcDCols + static_cast<uint32_t>(s) * kTcACols;
          const uint32_t b_stage = st_b(s);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bd = make_sw128_desc(b_stage + (kk >> 2) * kTcBSub + (kk & 3) * 32, 16, 1024);
            tc_mma_i8_ts(tmem_base, a_stage + static_cast<uint32_t>(kk * 8), bd, idesc, (ch | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty0 + 8u * s);   // frees the shared-memory stage and the A columns
          if (++s == kTcStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(dfull);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_MMA);
      }
      tc_commit(done_bar);
      if (!mbar_wait_plain(done_bar, 0)) atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------- decoders + epilogue
    const int e = warp - (kTcMmaWarp + 1), q = warp & 3, h = e >> 2;
    const int r = 32 * q + lane;                         // weight row in the task = TMEM lane
    const uint32_t lanebase = lut | (static_cast<uint32_t>(lane) << 2);
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    int s = 0;
    uint32_t ph = 0;
    int local = 0;
    bool ok = true;
    for (int task = blockIdx.x; task < G.total_tasks && ok; task += gridDim.x, ++local) {
      const TcTask d = tc_task(G, task);
      const FwdProblem& P = *d.P;
      for (int ch = 0; ch < d.nch; ++ch) {
        const bool got = mbar_wait(full0 + 8u * s, ph, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        uint32_t w[8];
        const uint32_t crow = st_codes(s) + static_cast<uint32_t>(r * 64);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint32_t a = crow + static_cast<uint32_t>(((2 * h + i) ^ ((r >> 1) & 3)) << 4);
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[4 * i]), "=r"(w[4 * i + 1]), "=r"(w[4 * i + 2]), "=r"(w[4 * i + 3])
                       : "r"(a));
        }
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          v[4 * i] = lut128_lookup<0>(w[i], lanebase);
          v[4 * i + 1] = lut128_lookup<1>(w[i], lanebase);
          v[4 * i + 2] = lut128_lookup<2>(w[i], lanebase);
          v[4 * i + 3] = lut128_lookup<3>(w[i], lanebase);
        }
        tmem_st_32x32b_x32(tmem_base + lane_off + kTcDCols + static_cast<uint32_t>(s) * kTcACols + 32u * h, v);
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull0 + 8u * s);
        if (++s == kTcStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      // epilogue: this warp's half of the task's token columns
      const bool got = mbar_wait(dfull, static_cast<uint32_t>(local) & 1u, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const float gamma = *P.w_scale;
      const float* const absmax = P.absmax;
      void* const yout = P.y;
      int32_t* const accout = P.acc;
      const int n_out = P.n_out, n_tile = P.n_tile;
      const int toks_valid = min(n_tile, P.t - d.t0);
      const int n = d.n0 + r;
      const bool row_ok = n < n_out;
      const bool y_f32 = G.y_f32 != 0;
      const int half = n_tile >> 1;
      for (int cb = h * half; cb < (h + 1) * half; cb += 32) {
        // row scales of up to 32 token columns: lane j holds column cb + j
        float rs_l = 0.0f;
        if (cb + lane < (h + 1) * half && cb + lane < toks_valid)
          rs_l = __fmul_rn(__fdiv_rn(absmax[d.t0 + cb + lane], 127.0f), gamma);
        const int cend = min(cb + 32, (h + 1) * half);
        for (int c0 = cb; c0 < cend; c0 += 8) {
          uint32_t a8[8];
          tmem_ld_32x32b_x8(tmem_base + lane_off + static_cast<uint32_t>(c0), a8);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float rs = __shfl_sync(0xffffffffu, rs_l, c0 - cb + j);
            const int col = c0 + j;
            if (col < toks_valid && row_ok) {
              const int acc = static_cast<int>(a8[j]);
              const float y = __fmul_rn(static_cast<float>(acc), rs);
              const int64_t off = static_cast<int64_t>(d.t0 + col) * n_out + n;
              if (y_f32) static_cast<float*>(yout)[off] = y;
              else static_cast<__nv_bfloat16*>(yout)[off] = __float2bfloat16_rn(y);
              if (accout != nullptr) accout[off] = acc;
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(&g_device_status, DEV_ST_TIMEOUT_EPILOGUE);
    }
  }

  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace bl
