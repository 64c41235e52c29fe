// Two-SM (cta_group::2) version of the persistent tcgen05 GEMM of gemm_tc.cuh.
//
// A cluster of two CTAs on two SMs computes one 256 x 256 output tile. CTA r of the
// pair loads rows [128r, 128r+128) of the tile's A block and columns [128r, 128r+128)
// of its B block (32 KB per 128-byte K step instead of 48 KB for a 128 x 256 tile on
// one SM), so each SM moves a third less operand data per multiply-accumulate. The
// leader CTA (rank 0) issues every MMA for the pair; each CTA's tensor core produces
// its own 128 rows x 256 columns in its own TMEM, and each CTA runs its own epilogue.
//
// Synchronisation of the pair (all waits bounded, see common.cuh):
//   full[s]  (leader)    : the leader's producer posts the byte count of both CTAs'
//                          loads; both CTAs' TMA loads complete on it (.cta_group::2).
//   empty[s] (each CTA)  : the leader's MMA commit arrives on both (multicast).
//   tfull[b] (each CTA)  : the leader's commit after a tile's last K step (multicast).
//   tempty[b] (leader)   : every epilogue warp of both CTAs arrives (remote arrive).
// A cluster barrier follows barrier initialisation and precedes TMEM release, so no
// CTA touches a peer barrier before it exists or after the peer has exited.
// No load uses multicast; only tcgen05.commit does.
#pragma once

#include "gemm_tc.cuh"

namespace bl {

constexpr int kStages2 = 6;
constexpr int kAHalfBytes = 128 * kBKBytes;   // 16 KB: this CTA's 128 rows of A
constexpr int kBHalfBytes = 128 * kBKBytes;   // 16 KB: this CTA's 128 columns of B
constexpr int kStage2Bytes = kAHalfBytes + kBHalfBytes;
constexpr size_t gemm2_smem_bytes() {
  return 1024 + static_cast<size_t>(kStages2) * kStage2Bytes + kOutStagingBytes + kBarrierBytes;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Raise the abort flag in this CTA and in its peer, so both leave their waits early.
__device__ __forceinline__ void pair_abort(volatile int* abort_flag, uint32_t peer_flag) {
  *abort_flag = 1;
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_flag), "r"(1) : "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive on this CTA's `bar` once every pair MMA issued so far is done. (Every tcgen05
// instruction of a kernel uses the same cta_group, so the pair kernel has its own.)
__device__ __forceinline__ void tc_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// Arrive on `bar` (same offset) in both CTAs of the pair once all prior MMAs are done.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   bar),
               "h"(static_cast<uint16_t>(3))
               : "memory");
}
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

// One launch may run several products of the same kind and the same K (e.g. the grad_W
// of every linear of an MLP over one token batch): their 256 x 256 tiles are numbered
// consecutively (problem i owns tiles [tile_begin, tile_begin + m blocks * n blocks))
// and the pairs stride over the concatenated list, so the last wave of one product no
// longer leaves pairs idle. A single product is a group of one.
constexpr int kMaxGemmGroup = 4;
struct GemmProblem2 {
  CUtensorMap tmA, tmB, tmOut;
  GemmArgs g;
  int tile_begin;
};
struct GemmGroup2 {
  GemmProblem2 p[kMaxGemmGroup];
  int count;
  int total_tiles;
  int num_k_blocks;   // the same for every problem of the group
};
// Problem of a tile in the concatenated list (tile_begin ascending).
__device__ __forceinline__ int group_problem(const GemmGroup2& G, int tile) {
  int i = 0;
#pragma unroll
  for (int j = 1; j < kMaxGemmGroup; ++j) i += (j < G.count && tile >= G.p[j].tile_begin) ? 1 : 0;
  return i;
}

template <bool kI8, bool kAMN, bool kBMN, int kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ GemmGroup2 G) {
  static_assert(!(kI8 && (kAMN || kBMN)), "the int8 product uses K-major operands only");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sA = base;                               // stage s: sA + s * kAHalfBytes
  const uint32_t sB = base + kStages2 * kAHalfBytes;      // stage s: sB + s * kBHalfBytes
  const uint32_t sOut = base + kStages2 * kStage2Bytes;   // epilogue staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages2 * kStage2Bytes + kOutStagingBytes);
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t full0 = bar0, empty0 = bar0 + 8u * kStages2;
  const uint32_t tfull0 = bar0 + 16u * kStages2, tempty0 = tfull0 + 16u, done_bar = tempty0 + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages2 + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(full0 + 8u * s, 1);    // the leader's producer arrival (+ both CTAs' bytes)
      mbar_init(empty0 + 8u * s, 1);   // one multicast commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8u * b, 1);
      mbar_init(tempty0 + 8u * b, 2 * kEpiWarps);   // epilogue warps of both CTAs
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < G.count; ++i) {
      tma_prefetch_desc(&G.p[i].tmA);
      tma_prefetch_desc(&G.p[i].tmB);
      tma_prefetch_desc(&G.p[i].tmOut);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = map_to_rank(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  const int num_tiles = G.total_tiles;   // 256 x 256 tiles of every problem
  const int num_k_blocks = G.num_k_blocks;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to_rank(full0, 0);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      int local = 0;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters, ++local) {
        const GemmProblem2& P = G.p[group_problem(G, tile)];
        int mb, nb;
        tile_coords(P.g, tile - P.tile_begin, mb, nb);
        const int m0 = mb * 256 + 128 * static_cast<int>(rank);
        const int n0 = nb * 256 + 128 * static_cast<int>(rank);
        const CUtensorMap* tmA = &P.tmA;
        const CUtensorMap* tmB = &P.tmB;
        for (int kq = 0; kq < num_k_blocks; ++kq) {
          const int kb = (local & 1) ? num_k_blocks - 1 - kq : kq;   // serpentine K order
          if (!mbar_wait(empty0 + 8u * s, ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = full_leader0 + 8u * s;
          if (leader) mbar_arrive_expect_tx(full0 + 8u * s, 2 * kStage2Bytes);
          const uint32_t a_dst = sA + s * kAHalfBytes, b_dst = sB + s * kBHalfBytes;
          const int kc = kI8 ? kb * 128 : kb * 64;
          if (kAMN) {
            tma_load_2d_pair(a_dst, tmA, fb, m0, kc);
            tma_load_2d_pair(a_dst + 8192, tmA, fb, m0 + 64, kc);
          } else {
            tma_load_2d_pair(a_dst, tmA, fb, kc, m0);
          }
          if (kBMN) {
            tma_load_2d_pair(b_dst, tmB, fb, n0, kc);
            tma_load_2d_pair(b_dst + 8192, tmB, fb, n0 + 64, kc);
          } else {
            tma_load_2d_pair(b_dst, tmB, fb, kc, n0);
          }
          ++issued;
          if (++s == kStages2) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        pair_abort(abort_flag, peer_abort);
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_PRODUCER);
        if (leader) {   // the leader's full barriers count both CTAs' copies: drain them
          const long long first = issued > kStages2 ? issued - kStages2 : 0;
          for (long long i = first; i < issued; ++i)
            if (!mbar_wait_plain(full0 + 8u * static_cast<uint32_t>(i % kStages2), static_cast<uint32_t>((i / kStages2) & 1)))
              atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = kI8 ? make_idesc(2u, 1u, 1u, 0u, 0u, 256, 256)
                                     : make_idesc(1u, 1u, 1u, kAMN ? 1u : 0u, kBMN ? 1u : 0u, 256, 256);
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
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
        for (int kb = 0; kb < num_k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8u * s, ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_base = sA + s * kAHalfBytes, b_base = sB + s * kBHalfBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = kAMN ? make_sw128_desc(a_base + kk * 2048, 8192, 1024) : make_sw128_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = kBMN ? make_sw128_desc(b_base + kk * 2048, 8192, 1024) : make_sw128_desc(b_base + kk * 32, 16, 1024);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (kI8) tc_mma_i8_pair(d_tmem, ad, bd, idesc, accum);
            else tc_mma_f16_pair(d_tmem, ad, bd, idesc, accum);
          }
          tc_commit_pair(empty0 + 8u * s);   // frees this stage in both CTAs
          if (++s == kStages2) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(tfull0 + 8u * buf);   // both CTAs' accumulators complete
      }
      if (!ok) {
        pair_abort(abort_flag, peer_abort);
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_MMA);
      }
      tc_commit_pair_local(done_bar);
      if (!mbar_wait_plain(done_bar, 0)) atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..9, both CTAs)
    const int e = warp - 2;
    const int quad = warp & 3;
    const int col_begin = (e >> 2) * (kBN / 2);
    const int row_in_tile = 128 * static_cast<int>(rank) + quad * 32 + lane;
    const uint32_t stage_buf = sOut + static_cast<uint32_t>(e * kStageOutBytes);
    const uint32_t tempty_leader0 = map_to_rank(tempty0, 0);
    int cnt = 0;
    int local = 0;
    bool ok = true;
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++local) {
      const int buf = local & 1;
      const uint32_t tph = static_cast<uint32_t>(local >> 1) & 1u;
      const GemmProblem2& P = G.p[group_problem(G, tile)];
      int mb, nb;
      tile_coords(P.g, tile - P.tile_begin, mb, nb);
      const int row = mb * 256 + row_in_tile;
      const int n0 = nb * kBN;
      const bool row_ok = row < P.g.M;
      const float gamma = (kEpi == EPI_GRADW) ? 1.0f : *P.g.w_scale;
      float rs = 1.0f;
      if (kEpi == EPI_FWD) {
        if (row_ok) rs = __fmul_rn(__fdiv_rn(P.g.row_absmax[row], 127.0f), gamma);
      } else if (kEpi == EPI_GRADX) {
        rs = gamma;
      }
      const bool got = mbar_wait(tfull0 + 8u * buf, tph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t_row = tmem_base + static_cast<uint32_t>(buf * kBN) + (static_cast<uint32_t>(quad * 32) << 16);
      epilogue_tile_tma<kEpi>(P.g, &P.tmOut, t_row, stage_buf, cnt, row - lane, n0, col_begin, rs, lane);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader0 + 8u * buf);
    }
    if (!ok && lane == 0) {
      pair_abort(abort_flag, peer_abort);
      atomicOr(&g_device_status, DEV_ST_TIMEOUT_EPILOGUE);
    }
    if (lane == 0) bulk_wait_group_all();
  }

  __syncthreads();
  tc_fence_before_sync();
  cluster_sync();   // the peer no longer reads this CTA's shared memory or barriers
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace bl
