// 2:4 structured-sparse forward product on CTA pairs: tcgen05.mma.sp ... kind::i8.
//
// Sparse-BitNet article (m.top168.com), section 七: NVIDIA's sparse tensor cores take
// the 2:4 pattern (at most two nonzero weights in every aligned group of four along
// K); Sparse-BitNet digest (shd-paper.top), abstract: the N:M-sparse ternary layer
// runs on a sparse tensor-core operator. Masks with at most two kept weights per
// aligned four (2:4, 2:8, 1:4, 1:8) are stored as two int8 values plus a 4-bit
// position nibble per group (bitlinear_quant_mask's sp_values / sp_meta outputs), and
// the sparse MMA consumes them directly: half the weight bytes and, on the tensor
// core, half the cycles of the dense product over the same logical K.
//
// Only the A operand of a sparse MMA can be sparse, so the weights take the M side:
//   Y^T[n, t] = sum_k W[n, k] * Xq[t, k]  accumulates in TMEM (lane = weight row),
// and the epilogue writes y[t, n] = acc * (a_t / 127 * gamma) transposed.
//
// A cluster of two CTAs on two SMs computes one tile of 256 weight rows x 224 tokens.
// CTA r loads weight rows [128r, 128r+128) of the tile (compressed values, 128 B per
// row per stage = 256 logical K, one 128B-swizzled TMA box), tokens [112r, 112r+112) of
// the activations (two 128B-swizzled boxes per stage) and its rows' metadata (two boxes
// of 128 rows x 16 B, each landing as the canonical no-swizzle layout: 8-row core
// matrices of 128 B); every load of both CTAs completes on the leader's barrier. The
// leader's single thread then copies the stage's metadata into both CTAs' TMEM with two
// tcgen05.cp.cta_group::2.128x128b (4 columns each: 2 per MMA, column 0 = groups 0-7,
// column 1 = groups 8-15 of its 64 logical K, nibble g % 8 of the word) and issues four
// M = 256 sparse MMAs (logical K = 64 each); copies and MMAs of one thread execute in
// issue order. The metadata tensor is padded to 256 rows and 256 logical K with the
// valid pattern 0x4 (positions 0 and 1), so no metadata load leaves it.
//
// TMEM per CTA (512 columns): two 224-column int32 accumulators (the epilogue of one
// tile overlaps the main loop of the next), then 4 stages x 8 metadata columns. The
// epilogue (8 warps: TMEM lane quarter x half of the tile's tokens) stages y
// transposed in shared memory and writes it with TMA stores (direct stores when the
// int32 accumulators are requested too).
// Every wait is bounded (common.cuh); on a timeout the CTA raises a status bit, lets
// its copies and MMAs retire, frees TMEM and returns. No load uses multicast.
#pragma once

#include "gemm_tc2.cuh"

namespace bl {

constexpr int kSpRowsPair = 256;                 // weight rows per pair tile (M of the MMA)
constexpr int kSpTok = 224;                      // tokens per pair tile (N of the MMA)
constexpr int kSpTokHalf = kSpTok / 2;           // tokens loaded by each CTA
constexpr int kSpStages = 4;
constexpr int kSpKStep = 256;                    // logical K per stage (4 MMAs of 64)
constexpr int kSpABytes = 128 * 128;             // 128 rows x 128 compressed bytes
constexpr int kSpBSlice = kSpTokHalf * 128;      // one 128-byte K slice of this CTA's tokens
constexpr int kSpBBytes = 2 * kSpBSlice;
constexpr int kSpEBytes = 128 * 32;              // 128 rows x 32 metadata bytes: two 2 KB blocks
constexpr int kSpStageBytes = kSpABytes + kSpBBytes + kSpEBytes;   // 48 KB
constexpr int kSpEpiWarps = 8;
constexpr int kSpFirstEpiWarp = 2;
constexpr int kSpThreads = 32 * (kSpFirstEpiWarp + kSpEpiWarps);   // 320
constexpr uint32_t kSpDCols = kSpTok;
constexpr uint32_t kSpECol0 = 2 * kSpDCols;      // 448: metadata columns after the accumulators
constexpr int kSpPad = 256;                      // metadata padding of rows and logical K
constexpr int kSpBarBytes = 256;
// epilogue: per warp two staging buffers of 16 tokens x 32 weight rows (bf16: 64 B per
// token row, fp32: 128 B) for TMA stores of y (all buffers first, each 2 KB-aligned: a
// TMA copy's shared-memory address must be 128-byte aligned), then 16 column scales per warp
constexpr int kSpStgBytes = 16 * 128;
constexpr int kSpEpiBytes = kSpEpiWarps * (2 * kSpStgBytes + 64);
static_assert(kSpBSlice % 1024 == 0 && kSpStageBytes % 1024 == 0, "128B-swizzle atoms need 1 KB alignment");
static_assert(kSpABytes % 1024 == 0 && (kSpABytes + kSpBBytes) % 1024 == 0 && 2048 % 128 == 0,
              "TMA destinations (values, activations, both metadata boxes) 1 KB / 128 B aligned");
static_assert((kSpStages * kSpStageBytes) % 1024 == 0 && kSpStgBytes % 128 == 0, "TMA store sources 128 B aligned");
static_assert(kSpECol0 + kSpStages * 8 <= 512, "accumulators and metadata exceed the TMEM of a CTA");
constexpr size_t gemm_sp2_smem_bytes() {
  return 1024 + static_cast<size_t>(kSpStages) * kSpStageBytes + kSpEpiBytes + kSpBarBytes;
}
static_assert(gemm_sp2_smem_bytes() <= 232448, "sparse GEMM exceeds the shared memory of a CTA");

struct SpGemmArgs {
  int T, n_out, k_in;          // tokens, weight rows, logical K (the metadata is padded)
  int tma_store;               // 1: y through shared memory and TMA stores (no acc_out)
  int num_k_blocks;            // ceil(k_in / 256)
  int num_row_blocks;          // ceil(n_out / 256)
  int num_tok_blocks;          // ceil(T / 224)
  void* y;                     // [T, n_out] bf16 or f32
  int y_f32;
  int32_t* acc_out;            // [T, n_out] or null
  const float* absmax;         // [T]
  const float* w_scale;        // [1]
};

// Instruction descriptor of tcgen05.mma.sp kind::i8: the dense fields plus the
// sparsity flag (bit 2). The sparsity selector (bits 0-1) stays 0: one MMA's
// metadata fills whole TMEM columns for 8-bit kinds.
__host__ __device__ constexpr uint32_t make_idesc_sp_i8(uint32_t n, uint32_t m) {
  return make_idesc(2u, 1u, 1u, 0u, 0u, n, m) | (1u << 2);
}

__device__ __forceinline__ void tc_mma_sp_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                                  uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(idesc), "r"(acc)
      : "memory");
}

// Copy 128 rows x 16 B of shared memory (canonical no-swizzle layout) into 4 TMEM
// columns of lanes 0-127, in each CTA of the pair from its own shared memory.
__device__ __forceinline__ void tc_cp_128x128b_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a K-major block without swizzle: core matrices of 8 rows x
// 16 B (128 B contiguous), SBO between 8-row groups, LBO between 16-byte column groups.
__device__ __forceinline__ uint64_t make_noswz_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;   // layout type 0: no swizzle
}

// Arrive on a barrier of the leader CTA without ordering this thread's memory writes
// (the epilogue's global stores need no ordering with the next tile's MMAs; the TMEM
// reads before it are ordered by tcgen05.wait::ld and the tcgen05 fence).
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__global__ void __launch_bounds__(kSpThreads, 1)
    gemm_sp2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY,
                    const SpGemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  auto st_a = [&](int s) { return base + static_cast<uint32_t>(s * kSpStageBytes); };
  auto st_b = [&](int s) { return base + static_cast<uint32_t>(s * kSpStageBytes + kSpABytes); };
  auto st_e = [&](int s) { return base + static_cast<uint32_t>(s * kSpStageBytes + kSpABytes + kSpBBytes); };
  const uint32_t sEpi = base + static_cast<uint32_t>(kSpStages * kSpStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSpStages * kSpStageBytes + kSpEpiBytes);
  const uint32_t bar0 = smem_u32(bars);
  // full[S] | empty[S] | tfull[2] | tempty[2] | done
  const uint32_t full0 = bar0, empty0 = bar0 + 8u * kSpStages;
  const uint32_t tfull0 = bar0 + 16u * kSpStages, tempty0 = tfull0 + 16u, done_bar = tempty0 + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kSpStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSpStages; ++s) {
      mbar_init(full0 + 8u * s, 1);                  // leader's producer (+ both CTAs' bytes)
      mbar_init(empty0 + 8u * s, 1);                 // one multicast commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8u * b, 1);
      mbar_init(tempty0 + 8u * b, 2 * kSpEpiWarps);  // epilogue warps of both CTAs
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmE);
    if (g.tma_store) tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = map_to_rank(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  const int num_tiles = g.num_row_blocks * g.num_tok_blocks;   // token blocks fastest
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_rank(full0, 0);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters) {
        const int m0 = (tile / g.num_tok_blocks) * kSpRowsPair + 128 * static_cast<int>(rank);
        const int t0 = (tile % g.num_tok_blocks) * kSpTok + kSpTokHalf * static_cast<int>(rank);
        for (int kb = 0; kb < g.num_k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8u * s, ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_leader0 + 8u * s;
          if (leader) mbar_arrive_expect_tx(full0 + 8u * s, 2 * kSpStageBytes);
          tma_load_2d_pair(st_a(s), &tmA, fb, kb * 128, m0);
          tma_load_2d_pair(st_b(s), &tmB, fb, kb * kSpKStep, t0);
          tma_load_2d_pair(st_b(s) + kSpBSlice, &tmB, fb, kb * kSpKStep + 128, t0);
          tma_load_2d_pair(st_e(s), &tmE, fb, kb * 32, m0);
          tma_load_2d_pair(st_e(s) + 2048, &tmE, fb, kb * 32 + 16, m0);
          ++issued;
          if (++s == kSpStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        pair_abort(abort_flag, peer_abort);
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_PRODUCER);
        if (leader) {   // the leader's full barriers count both CTAs' copies: drain them
          const long long first = issued > kSpStages ? issued - kSpStages : 0;
          for (long long i = first; i < issued; ++i)
            if (!mbar_wait_plain(full0 + 8u * static_cast<uint32_t>(i % kSpStages), static_cast<uint32_t>((i / kSpStages) & 1)))
              atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = make_idesc_sp_i8(kSpTok, kSpRowsPair);
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters, ++local) {
        const int buf = local & 1;
        const uint32_t tph = static_cast<uint32_t>(local >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8u * buf, tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * kSpDCols;
        for (int kb = 0; kb < g.num_k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8u * s, ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_base = st_a(s), b_base = st_b(s);
          const uint32_t e_stage = tmem_base + kSpECol0 + static_cast<uint32_t>(s) * 8u;
          // this stage's metadata into both CTAs' TMEM (MMAs 0-1, then 2-3)
          tc_cp_128x128b_pair(e_stage, make_noswz_desc(st_e(s), 2048, 128));
          tc_cp_128x128b_pair(e_stage + 4u, make_noswz_desc(st_e(s) + 2048, 2048, 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // A: 32 compressed bytes (64 logical K) per MMA inside the swizzled row;
            // B: 64 bytes per MMA, two MMAs per 128-byte slice
            const uint64_t ad = make_sw128_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = make_sw128_desc(b_base + (kk >> 1) * kSpBSlice + (kk & 1) * 64, 16, 1024);
            tc_mma_sp_i8_pair(d_tmem, ad, bd, e_stage + 2u * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair(empty0 + 8u * s);   // frees this stage (shared memory and metadata columns) in both CTAs
          if (++s == kSpStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(tfull0 + 8u * buf);
      }
      if (!ok) {
        pair_abort(abort_flag, peer_abort);
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_MMA);
      }
      tc_commit_pair_local(done_bar);
      if (!mbar_wait_plain(done_bar, 0)) atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------- epilogue (8 warps, both CTAs)
    const int e = warp - kSpFirstEpiWarp;
    const int quad = warp & 3;
    const int c_begin = (e >> 2) * kSpTokHalf;   // this warp's half of the tile's token columns
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tempty_leader0 = map_to_rank(tempty0, 0);
    const float gamma = *g.w_scale;
    const uint32_t stg0 = sEpi + static_cast<uint32_t>(e) * (2 * kSpStgBytes);        // two staging buffers
    const uint32_t scales = sEpi + static_cast<uint32_t>(kSpEpiWarps * 2 * kSpStgBytes + e * 64);   // 16 scales
    int cnt = 0;   // TMA stores issued by this warp
    int local = 0;
    bool ok = true;
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
      const int buf = local & 1;
      const uint32_t tph = static_cast<uint32_t>(local >> 1) & 1u;
      const int n = (tile / g.num_tok_blocks) * kSpRowsPair + 128 * static_cast<int>(rank) + quad * 32 + lane;
      const int t0 = (tile % g.num_tok_blocks) * kSpTok + c_begin;
      const bool row_ok = n < g.n_out;
      const bool got = mbar_wait(tfull0 + 8u * buf, tph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t_cols = tmem_base + lane_off + static_cast<uint32_t>(buf) * kSpDCols + static_cast<uint32_t>(c_begin);
      if (g.tma_store) {
        // y through shared memory: the warp's 32 weight rows x 16 tokens, stored
        // transposed ([token][row], one 2- or 4-byte store per element: a warp writes one
        // contiguous token row per instruction), then one TMA store of the block
        const uint32_t esz = g.y_f32 ? 4u : 2u;
        const int n_blk = (tile / g.num_tok_blocks) * kSpRowsPair + 128 * static_cast<int>(rank) + quad * 32;
#pragma unroll 1
        for (int c0 = 0; c0 < kSpTokHalf; c0 += 16, ++cnt) {
          uint32_t a[16];
          tmem_ld_32x32b_x16(t_cols + static_cast<uint32_t>(c0), a);
          if (lane < 16) {   // column scales a_t / 127 * gamma of these 16 tokens
            const int tl = t0 + c0 + lane;
            const float rs = tl < g.T ? __fmul_rn(__fdiv_rn(g.absmax[tl], 127.0f), gamma) : 0.0f;
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(scales + 4u * lane), "f"(rs) : "memory");
          }
          __syncwarp();
          float rs[16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(rs[4 * q]), "=f"(rs[4 * q + 1]), "=f"(rs[4 * q + 2]), "=f"(rs[4 * q + 3])
                         : "r"(scales + 16u * q)
                         : "memory");
          const uint32_t stg = stg0 + static_cast<uint32_t>(cnt & 1) * kSpStgBytes;
          if (cnt >= 2) {   // the store issued from this buffer two chunks ago has read it
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
          }
          tmem_ld_wait();
          const uint32_t row_addr = stg + esz * static_cast<uint32_t>(lane);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float y = __fmul_rn(static_cast<float>(static_cast<int>(a[j])), rs[j]);   // exact int32 -> f32
            if (g.y_f32) {
              asm volatile("st.shared.f32 [%0], %1;" ::"r"(row_addr + 128u * j), "f"(y) : "memory");
            } else {
              const __nv_bfloat16 h = __float2bfloat16_rn(y);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(row_addr + 64u * j), "h"(*reinterpret_cast<const uint16_t*>(&h))
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmY, stg, n_blk, t0 + c0);   // rows past T and columns past n_out are not written
            bulk_commit_group();
          }
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < kSpTokHalf; c0 += 16) {
          uint32_t a[16];
          tmem_ld_32x32b_x16(t_cols + static_cast<uint32_t>(c0), a);
          // column scales a_t / 127 * gamma of these 16 tokens: lane j < 16 holds token j
          const int tl = t0 + c0 + (lane & 15);
          const float rs_l = tl < g.T ? __fmul_rn(__fdiv_rn(g.absmax[tl], 127.0f), gamma) : 0.0f;
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float rs = __shfl_sync(0xffffffffu, rs_l, j);
            const int t = t0 + c0 + j;
            if (row_ok && t < g.T) {
              const int acc = static_cast<int>(a[j]);
              const float y = __fmul_rn(static_cast<float>(acc), rs);   // int32 -> f32 exact (|acc| < 2^24)
              const int64_t off = static_cast<int64_t>(t) * g.n_out + n;
              if (g.y_f32) static_cast<float*>(g.y)[off] = y;
              else static_cast<__nv_bfloat16*>(g.y)[off] = __float2bfloat16_rn(y);
              if (g.acc_out != nullptr) g.acc_out[off] = acc;
            }
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote_relaxed(tempty_leader0 + 8u * buf);
    }
    if (!ok && lane == 0) {
      pair_abort(abort_flag, peer_abort);
      atomicOr(&g_device_status, DEV_ST_TIMEOUT_EPILOGUE);
    }
    if (lane == 0) bulk_wait_group_all();   // stores complete before the CTA exits
  }

  __syncthreads();
  tc_fence_before_sync();
  cluster_sync();   // the peer no longer reads this CTA's shared memory, barriers or TMEM
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace bl
