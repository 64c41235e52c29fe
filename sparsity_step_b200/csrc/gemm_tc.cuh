// Persistent, warp-specialised tcgen05 GEMM for the BitLinear products (steps a4-a6).
//
//   EPI_FWD  : acc[t,n] = sum_k Xq[t,k] * Wq[n,k]   (kind::i8, int32 in TMEM)
//              y = acc * (a_t / 127 * gamma) -> bf16 | f32, optional int32 acc
//   EPI_GRADX: grad_X[t,k] = gamma * sum_n dY[t,n] * C[n,k]  (kind::f16, f32 in TMEM)
//   EPI_GRADW: grad_W[n,k] = sum_t dY[t,n] * X[t,k]           (kind::f16, f32 in TMEM)
//
// BitNet b1.58 2B4T article (lsdiaocha.cn), section 四: ternary weights are moved
// from HBM to shared memory and multiplied with 8-bit activations. Sparse-BitNet
// article (m.top168.com), sections 三 and 六: the dual straight-through backward
// uses the effective weight for the input gradient and gives every latent weight
// (masked ones included) the dense gradient dY^T X.
//
// Tile 128 x 256, K step 128 bytes (64 bf16 or 128 int8) per pipeline stage, 4
// stages of 48 KB. Warp 0: TMA producer (one thread). Warp 1: TMEM allocator and
// MMA issuer (one thread). Warps 2-9: epilogue (TMEM -> registers -> global), two
// warps on the 32 TMEM lanes (= tile rows) their warp-rank-in-quad may access, each
// converting half of the tile's columns.
// Two 256-column fp32/int32 accumulators in TMEM (all 512 columns) let the
// epilogue of tile i overlap the main loop of tile i+1. Operands are staged with
// 128-byte swizzle: K-major tiles are one TMA box of [rows x 128 B]; MN-major
// tiles are boxes of [64 elements (128 B) x 64 K-rows], one per 64-wide MN atom.
// Every mbarrier wait is bounded (see common.cuh); on a timeout the CTA raises a
// device status bit, lets in-flight copies and MMAs retire, frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKBytes = 128;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBKBytes;   // 16 KB
constexpr int kBBytes = kBN * kBKBytes;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;                       // two per TMEM lane quarter, half the columns each
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr int kBarrierBytes = 256;
// epilogue staging for TMA stores: per epilogue warp one buffer of 32 rows x 128 B
constexpr int kStageOutBytes = 32 * 128;
constexpr int kOutStagingBytes = kEpiWarps * kStageOutBytes;   // 32 KB
constexpr size_t gemm_smem_bytes(bool tma_store) {
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + (tma_store ? kOutStagingBytes : 0) + kBarrierBytes;
}

enum Epi : int { EPI_FWD = 0, EPI_GRADX = 1, EPI_GRADW = 2 };

struct GemmArgs {
  int M, N;                  // output [M, N], row-major, ld = N
  int num_k_blocks;          // ceil(K * elem_bytes / 128)
  int num_m_blocks, num_n_blocks;
  int m_fastest;             // tile order: 1 = m blocks fastest (A re-read from L2), 0 = n blocks fastest
  void* out;                 // bf16 or f32
  int out_f32;
  int32_t* acc_out;          // EPI_FWD only, nullable
  const float* row_absmax;   // EPI_FWD: a_t per output row
  const float* w_scale;      // gamma (EPI_FWD, EPI_GRADX)
};

// Tile index -> (m block, n block) in the launch's raster order: the operand whose
// blocks vary fastest is re-read across the tiles of a wave and should stay in L2.
__device__ __forceinline__ void tile_coords(const GemmArgs& g, int tile, int& mb, int& nb) {
  if (g.m_fastest) {
    mb = tile % g.num_m_blocks;
    nb = tile / g.num_m_blocks;
  } else {
    mb = tile / g.num_n_blocks;
    nb = tile % g.num_n_blocks;
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int kEpi>
__device__ __forceinline__ void epilogue_store32(const GemmArgs& g, const uint32_t (&r)[32], int row, int col0, float rs) {
  float f[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (kEpi == EPI_FWD) {
      f[j] = __fmul_rn(static_cast<float>(static_cast<int32_t>(r[j])), rs);   // int32 -> f32 exact (|acc| < 2^24)
    } else if (kEpi == EPI_GRADX) {
      f[j] = __fmul_rn(__uint_as_float(r[j]), rs);
    } else {
      f[j] = __uint_as_float(r[j]);
    }
  }
  const int64_t off = static_cast<int64_t>(row) * g.N + col0;
  if (g.out_f32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(g.out) + off);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      if (col0 + 4 * v + 4 <= g.N) o[v] = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
  } else {
    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + off);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      if (col0 + 8 * v + 8 <= g.N)
        o[v] = make_uint4(pack_bf16x2(f[8 * v], f[8 * v + 1]), pack_bf16x2(f[8 * v + 2], f[8 * v + 3]),
                          pack_bf16x2(f[8 * v + 4], f[8 * v + 5]), pack_bf16x2(f[8 * v + 6], f[8 * v + 7]));
  }
  if (kEpi == EPI_FWD && g.acc_out != nullptr) {
    int4* o = reinterpret_cast<int4*>(g.acc_out + off);
#pragma unroll
    for (int v = 0; v < 8; ++v)
      if (col0 + 4 * v + 4 <= g.N)
        o[v] = make_int4(static_cast<int>(r[4 * v]), static_cast<int>(r[4 * v + 1]), static_cast<int>(r[4 * v + 2]),
                         static_cast<int>(r[4 * v + 3]));
  }
}

// Epilogue of one tile row-quarter through shared memory and TMA stores: the warp
// converts 32 rows x 128 B (64 bf16 or 32 fp32 columns) at a time into a 128B-swizzled
// staging buffer (row r at r*128, 16-byte chunk j at position j ^ (r & 7): conflict-free
// and the layout the store's tensor map expects), then one lane stores the box.
template <int kEpi>
__device__ __forceinline__ void epilogue_tile_tma(const GemmArgs& g, const CUtensorMap* tmOut, uint32_t t_row,
                                                  uint32_t buf, int& cnt, int row0, int n0, int col_begin, float rs,
                                                  int lane) {
  const int ecols = g.out_f32 ? 32 : 64;
  for (int c = col_begin / ecols; c < (col_begin + kBN / 2) / ecols; ++c, ++cnt) {
    if (cnt >= 1) {
      if (lane == 0) bulk_wait_group_read<0>();   // the previous store has finished reading the buffer
      __syncwarp();
    }
    uint32_t r0[32], r1[32];
    tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * ecols), r0);
    if (!g.out_f32) tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * ecols + 32), r1);
    tmem_ld_wait();
    uint32_t w[32];   // the 128 bytes of this thread's row
    if (g.out_f32) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float f;
        if (kEpi == EPI_FWD) f = __fmul_rn(static_cast<float>(static_cast<int32_t>(r0[j])), rs);
        else if (kEpi == EPI_GRADX) f = __fmul_rn(__uint_as_float(r0[j]), rs);
        else f = __uint_as_float(r0[j]);
        w[j] = __float_as_uint(f);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint32_t a = j < 16 ? r0[2 * j] : r1[2 * j - 32];
        const uint32_t b = j < 16 ? r0[2 * j + 1] : r1[2 * j - 31];
        float fa, fb;
        if (kEpi == EPI_FWD) {
          fa = __fmul_rn(static_cast<float>(static_cast<int32_t>(a)), rs);
          fb = __fmul_rn(static_cast<float>(static_cast<int32_t>(b)), rs);
        } else if (kEpi == EPI_GRADX) {
          fa = __fmul_rn(__uint_as_float(a), rs);
          fb = __fmul_rn(__uint_as_float(b), rs);
        } else {
          fa = __uint_as_float(a);
          fb = __uint_as_float(b);
        }
        w[j] = pack_bf16x2(fa, fb);
      }
    }
    const uint32_t row_addr = buf + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t dst = row_addr + static_cast<uint32_t>((j ^ (lane & 7)) * 16);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w[4 * j]), "r"(w[4 * j + 1]),
                   "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmOut, buf, n0 + c * ecols, row0);
      bulk_commit_group();
    }
  }
}

template <bool kI8, bool kAMN, bool kBMN, int kEpi, bool kTmaStore>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmOut, const GemmArgs g) {
  static_assert(!(kI8 && (kAMN || kBMN)), "the int8 product uses K-major operands only");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // 128B-swizzle atoms need 1024 B alignment
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t sA = base;
  const uint32_t sB = base + kStages * kABytes;
  const uint32_t sOut = base + kStages * kStageBytes;   // epilogue staging (kTmaStore only)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + (kTmaStore ? kOutStagingBytes : 0));
  const uint32_t bar0 = smem_u32(bars);
  // barrier slots: full[kStages] | empty[kStages] | tmem_full[2] | tmem_empty[2] | done
  const uint32_t full0 = bar0, empty0 = bar0 + 8u * kStages;
  const uint32_t tfull0 = bar0 + 16u * kStages, tempty0 = tfull0 + 16u, done_bar = tempty0 + 16u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8u * b, 1);
      mbar_init(tempty0 + 8u * b, kEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kTmaStore) tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = g.num_m_blocks * g.num_n_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        int mb, nb;
        tile_coords(g, tile, mb, nb);
        const int m0 = mb * kBM;
        const int n0 = nb * kBN;
        for (int kq = 0; kq < g.num_k_blocks; ++kq) {
          const int kb = (local & 1) ? g.num_k_blocks - 1 - kq : kq;   // serpentine K order
          if (!mbar_wait(empty0 + 8u * s, ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8u * s;
          mbar_arrive_expect_tx(fb, kStageBytes);
          const uint32_t a_dst = sA + s * kABytes, b_dst = sB + s * kBBytes;
          const int kc = kI8 ? kb * 128 : kb * 64;   // K coordinate in elements (128 B per stage)
          if (kAMN) {
            tma_load_2d(a_dst, &tmA, fb, m0, kc);
            tma_load_2d(a_dst + 8192, &tmA, fb, m0 + 64, kc);
          } else {
            tma_load_2d(a_dst, &tmA, fb, kc, m0);
          }
          if (kBMN) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d(b_dst + 8192 * j, &tmB, fb, n0 + 64 * j, kc);
          } else {
            tma_load_2d(b_dst, &tmB, fb, kc, n0);
          }
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_PRODUCER);
        // let every copy still in flight land before the CTA may exit
        const long long first = issued > kStages ? issued - kStages : 0;
        for (long long i = first; i < issued; ++i) {
          if (!mbar_wait_plain(full0 + 8u * static_cast<uint32_t>(i % kStages), static_cast<uint32_t>((i / kStages) & 1)))
            atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = kI8 ? make_idesc(2u, 1u, 1u, 0u, 0u, kBN, kBM)
                                     : make_idesc(1u, 1u, 1u, kAMN ? 1u : 0u, kBMN ? 1u : 0u, kBN, kBM);
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t tph = static_cast<uint32_t>(local >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8u * buf, tph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kBN);
        for (int kb = 0; kb < g.num_k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8u * s, ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_base = sA + s * kABytes, b_base = sB + s * kBBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // K-major: advance 32 B inside the swizzle atom row; MN-major: 16 K-rows = 2 atoms
            const uint64_t ad = kAMN ? make_sw128_desc(a_base + kk * 2048, 8192, 1024) : make_sw128_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = kBMN ? make_sw128_desc(b_base + kk * 2048, 8192, 1024) : make_sw128_desc(b_base + kk * 32, 16, 1024);
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            if (kI8) tc_mma_i8(d_tmem, ad, bd, idesc, accum);
            else tc_mma_f16(d_tmem, ad, bd, idesc, accum);
          }
          tc_commit(empty0 + 8u * s);   // frees this smem stage once the MMAs read it
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull0 + 8u * buf);   // accumulator complete
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(&g_device_status, DEV_ST_TIMEOUT_MMA);
      }
      tc_commit(done_bar);   // every MMA issued above has retired once this arrives
      if (!mbar_wait_plain(done_bar, 0)) atomicOr(&g_device_status, DEV_ST_TIMEOUT_DRAIN);
    }
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..9)
    // two warps per TMEM lane quarter: warp 2+e owns lanes [32*quad, +32) and the
    // column half e / 4 of each 256-column accumulator
    const int e = warp - 2;
    const int quad = warp & 3;   // TMEM lanes [32*quad, 32*quad+32) belong to this warp
    const int col_begin = (e >> 2) * (kBN / 2);
    const int row_in_tile = quad * 32 + lane;
    const float gamma = (kEpi == EPI_GRADW) ? 1.0f : *g.w_scale;
    const uint32_t stage_buf = sOut + static_cast<uint32_t>(e * kStageOutBytes);
    int cnt = 0;   // stores issued from the staging buffer so far
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t tph = static_cast<uint32_t>(local >> 1) & 1u;
      // the row scale does not depend on the accumulator: fetch it before waiting
      int mb, nb;
      tile_coords(g, tile, mb, nb);
      const int row = mb * kBM + row_in_tile;
      const int n0 = nb * kBN;
      const bool row_ok = row < g.M;
      float rs = 1.0f;
      if (kEpi == EPI_FWD) {
        if (row_ok) rs = __fmul_rn(__fdiv_rn(g.row_absmax[row], 127.0f), gamma);
      } else if (kEpi == EPI_GRADX) {
        rs = gamma;
      }
      // warp-uniform decision: the TMEM loads below are warp-collective
      const bool got = mbar_wait(tfull0 + 8u * buf, tph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t_row = tmem_base + static_cast<uint32_t>(buf * kBN) + (static_cast<uint32_t>(quad * 32) << 16);
      if (kTmaStore) {
        epilogue_tile_tma<kEpi>(g, &tmOut, t_row, stage_buf, cnt, row - lane, n0, col_begin, rs, lane);
      } else {
#pragma unroll 1
        for (int c = col_begin / 32; c < (col_begin + kBN / 2) / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + static_cast<uint32_t>(c * 32), r);
          tmem_ld_wait();
          const int col0 = n0 + c * 32;
          if (row_ok && col0 < g.N) epilogue_store32<kEpi>(g, r, row, col0, rs);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8u * buf);
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      atomicOr(&g_device_status, DEV_ST_TIMEOUT_EPILOGUE);
    }
    if (kTmaStore && lane == 0) bulk_wait_group_all();   // stores complete before the CTA exits
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace bl
