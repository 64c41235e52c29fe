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
#include "cp_async.cuh"

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
// Per task a warp streams its 16 rows' codes once (each thread prefetches its own 32
// bytes per chunk with cp.async, kDecDepth chunks ahead across task boundaries) and
// feeds mma.sync.m16n8k32.s8 with the weights decoded straight into A fragments in
// registers: decoded weights never pass through shared memory. Inside each chunk of 256
// weights the reduction order is permuted so that thread (group g, index tig) owns
// logical weights [64*tig, 64*tig + 64): MMA step s, A/B slot 4*tig + i holds weight
// 64*tig + 8*s + i and slot 4*tig + 16 + i holds 64*tig + 8*s + 4 + i. A thread then
// reads 16 contiguous code bytes per row and 64 contiguous int8 activations per
// token; the same permutation on both operands leaves every dot product unchanged.
// Code bytes become int8x4 words through a 256-entry table replicated per lane
// (entry e of lane l at word 32*e + l: conflict-free).
constexpr int kMaxFwdGroup = 256;

struct FwdProblem {
  const uint8_t* codes;    // [n_out, k_in/4]
  const int8_t* xq;        // [t, k_in]
  const float* absmax;     // [t]
  const float* w_scale;    // [1]
  void* y;                 // [t, n_out]
  int32_t* acc;            // [t, n_out] or null
  int t, k_in, n_out;
  int task_begin;          // first task index of this problem
  int n_tile;              // tokens per task (tensor-core kernel only)
};

struct FwdGroup {
  FwdProblem p[kMaxFwdGroup];
  int count;
  int total_tasks;
  int y_f32;
  int layout_probe;   // fwd_codes_mma_kernel: record where dynamic shared memory starts, do nothing else
};

// Shared-window address of fwd_codes_mma_kernel's dynamic shared memory, written by a
// one-CTA launch with layout_probe set (the host checks it once per device).
__device__ unsigned int g_dec_smem_base;

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

// The byte -> int8x4 table lives at a fixed shared-window address: entry e of lane l is
// the word at kDecLutAddr + 256*e + 4*l (lanes use the first 128 bytes of each 256-byte
// row), so each lane reads its own bank and the address of code byte j of word w is one
// byte permute: byte 0 <- 4*lane, byte 1 <- byte j of w, byte 2 <- 0x01 (kDecLutAddr
// >> 16), byte 3 <- 0. `lanesel` = 0x00010000 | 4*lane supplies bytes 0, 2 and 3.
constexpr uint32_t kDecLutAddr = 0x10000;
constexpr uint32_t kDecLutSpan = 256 * 256;
constexpr uint32_t kDecHighBase = kDecLutAddr + kDecLutSpan;
static_assert(kDecLutAddr == 0x10000, "lut_lookup builds byte 2 of the address from lanesel");

template <int J>
__device__ __forceinline__ uint32_t lut_lookup(uint32_t w, uint32_t lanesel) {
  const uint32_t addr = __byte_perm(w, lanesel, 0x7604u | (J << 4));
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Sixteen codes (code j at bits 2j of w) -> four int8x4 words in natural order with byte
// permutes only (no table): nibble m of (w & 0x33333333) holds code 2m and nibble m of
// ((w >> 2) & 0x33333333) code 2m+1; as permute selectors into the bytes {0x00, 0x01,
// 0x00, 0xFF} they decode the even and the odd codes, and two more permutes interleave
// them. Same result as four table lookups (byte j of w -> o_j), on the ALU pipe instead of
// the shared-memory pipe; the decode kernel uses it for some words to balance the two.
__device__ __forceinline__ void decode16(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2, uint32_t& o3) {
  constexpr uint32_t kTable = 0xFF000100u;
  const uint32_t ev = w & 0x33333333u, od = (w >> 2) & 0x33333333u;
  const uint32_t e_lo = __byte_perm(kTable, 0u, ev), e_hi = __byte_perm(kTable, 0u, ev >> 16);
  const uint32_t o_lo = __byte_perm(kTable, 0u, od), o_hi = __byte_perm(kTable, 0u, od >> 16);
  o0 = __byte_perm(e_lo, o_lo, 0x5140u);   // codes 0..3
  o1 = __byte_perm(e_lo, o_lo, 0x7362u);   // codes 4..7
  o2 = __byte_perm(e_hi, o_hi, 0x5140u);   // codes 8..11
  o3 = __byte_perm(e_hi, o_hi, 0x7362u);   // codes 12..15
}

// Which of a chunk's eight code words (bit 2h + r: word h of row half r) are decoded by
// byte permutes rather than table lookups: two of eight (measured on B200: batch 1
// 0.234 -> 0.224 ms per 36-layer step; all-table decoding is limited by the shared-memory
// instruction queue, half-and-half by the ALU at batch 1).
constexpr unsigned kDecPrmtWords = 0x22;

template <bool kPrmt>
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t lanesel, uint32_t& o0, uint32_t& o1, uint32_t& o2,
                                            uint32_t& o3) {
  if (kPrmt) {
    decode16(w, o0, o1, o2, o3);
  } else {
    o0 = lut_lookup<0>(w, lanesel);
    o1 = lut_lookup<1>(w, lanesel);
    o2 = lut_lookup<2>(w, lanesel);
    o3 = lut_lookup<3>(w, lanesel);
  }
}

// Accumulators per token group, optionally split into independent sets (summed at
// the end) to shorten the MMA dependency chain; one set measured fastest because
// the registers a split costs lower the number of resident warps.
template <int NG>
struct DecAcc {
  static constexpr int kSets = 1;   // more sets did not help (they cost occupancy)
  int v[kSets][NG][4];
};

// Two MMA steps from one 32-bit word of each row's codes (bytes 0..3 = steps 2h, 2h+1).
template <int NG, int H>
__device__ __forceinline__ void decode_mma_word(DecAcc<NG>& acc, uint32_t lanesel, uint32_t w0, uint32_t w1,
                                                const uint4 (&xv)[NG][4]) {
  constexpr int S = DecAcc<NG>::kSets;
  uint32_t r0[4], r1[4];   // decoded words of row g (w0) and row g+8 (w1)
  decode_word<((kDecPrmtWords >> (2 * H)) & 1u) != 0>(w0, lanesel, r0[0], r0[1], r0[2], r0[3]);
  decode_word<((kDecPrmtWords >> (2 * H + 1)) & 1u) != 0>(w1, lanesel, r1[0], r1[1], r1[2], r1[3]);
  // step 2h: bytes 0 (a0) and 1 (a2) of row g's word, of row g+8's word (a1, a3)
#pragma unroll
  for (int j = 0; j < NG; ++j)
    mma_m16n8k32_s8(acc.v[(2 * H) % S][j], r0[0], r1[0], r0[1], r1[1], xv[j][H].x, xv[j][H].y);
  // step 2h+1: bytes 2, 3
#pragma unroll
  for (int j = 0; j < NG; ++j)
    mma_m16n8k32_s8(acc.v[(2 * H + 1) % S][j], r0[2], r1[2], r0[3], r1[3], xv[j][H].z, xv[j][H].w);
}

template <int NG>
__device__ __forceinline__ void decode_chunk(DecAcc<NG>& acc, uint32_t lanesel, const uint4& c0, const uint4& c1,
                                             const uint4 (&xv)[NG][4]) {
  decode_mma_word<NG, 0>(acc, lanesel, c0.x, c1.x, xv);
  decode_mma_word<NG, 1>(acc, lanesel, c0.y, c1.y, xv);
  decode_mma_word<NG, 2>(acc, lanesel, c0.z, c1.z, xv);
  decode_mma_word<NG, 3>(acc, lanesel, c0.w, c1.w, xv);
}

// Per-thread streaming: each thread copies the 32 code bytes it will itself decode
// per chunk (16 bytes of row g, 16 of row g+8) with cp.async into its own slots of a
// shared-memory ring kDecDepth chunks deep, so up to kDecDepth chunks per warp are in
// flight without holding registers, and no thread ever reads another thread's data.
// Slot layout [row half][thread][16 B]: consecutive threads read consecutive 16-byte
// slots (conflict-free). Slot 0 sits at the start of the dynamic shared memory, below
// the table; slots 1.. sit above it, from kDecHighBase.
constexpr int kDecDepth = 4;

// RB = 16-row blocks per task: a task of RB blocks shares each chunk's activations and the
// ring bookkeeping between RB x 8 MMAs (RB = 2 with half the warps keeps the ring's bytes).
template <int NG, int RB = 1>
struct DecCfg {
  static constexpr int kWarps = (NG == 1 ? 32 : 16) / RB;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kDepth = kDecDepth;   // ring slots (chunks in flight + 1)
  static constexpr uint32_t kSlotBytes = 2u * RB * kThreads * 16u;
  // enough for any start address of the dynamic shared memory: the last slot ends at
  // kDecHighBase + (kDepth - 1) * kSlotBytes
  static constexpr int kSmemBytes = static_cast<int>(kDecHighBase + (kDepth - 1) * kSlotBytes);
};
static_assert(DecCfg<1>::kSmemBytes <= 232448, "decode ring and table exceed the shared memory of a CTA");
static_assert(DecCfg<1, 2>::kSmemBytes <= 232448, "decode ring and table exceed the shared memory of a CTA");

struct DecTask {
  const FwdProblem* P;
  int n0, t0, nch;   // first row, first token, chunks of 256 weights
};

__device__ __forceinline__ DecTask dec_task(const FwdGroup& G, int task, int tok_per_task, int rows_per_task) {
  int lo = 0, hi = G.count - 1;   // last problem with task_begin <= task
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (G.p[mid].task_begin <= task) lo = mid;
    else hi = mid - 1;
  }
  const FwdProblem& P = G.p[lo];
  const int row_blocks = P.n_out / rows_per_task;
  const int local = task - P.task_begin;
  DecTask d;
  d.P = &P;
  d.n0 = (local % row_blocks) * rows_per_task;
  d.t0 = (local / row_blocks) * tok_per_task;
  d.nch = (P.k_in + 255) >> 8;
  return d;
}

template <int NG, int RB>   // token groups of 8 and 16-row blocks per task
__global__ void __launch_bounds__(DecCfg<NG, RB>::kThreads, 1) fwd_codes_mma_kernel(const __grid_constant__ FwdGroup G) {
  using C = DecCfg<NG, RB>;
  extern __shared__ __align__(1024) uint8_t dsmem[];
  const uint32_t base = smem_u32(dsmem);
  if (G.layout_probe) {
    if (threadIdx.x == 0 && blockIdx.x == 0) g_dec_smem_base = base;
    return;
  }
  if (base + C::kSlotBytes > kDecLutAddr) {   // slot 0 would overlap the table: do nothing
    if (threadIdx.x == 0) atomicOr(&g_device_status, DEV_ST_SMEM_LAYOUT);
    return;
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) {
    const uint32_t e = static_cast<uint32_t>(i) >> 5, l = static_cast<uint32_t>(i) & 31u;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t f = (e >> (2 * j)) & 3u;
      word |= ((f & 1u) ? ((f & 2u) ? 0xFFu : 0x01u) : 0u) << (8 * j);
    }
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(kDecLutAddr + 256u * e + 4u * l), "r"(word) : "memory");
  }
  __syncthreads();
  // slot layout [segment][thread][16 B]: segment 2b + h holds row 16b + g + 8h of the task
  constexpr uint32_t kHalf = C::kThreads * 16;
  const uint32_t ring_lo = base + static_cast<uint32_t>(threadIdx.x * 16);
  const uint32_t ring_hi = kDecHighBase - C::kSlotBytes + static_cast<uint32_t>(threadIdx.x * 16);
  auto slot_addr = [&](int s) { return s == 0 ? ring_lo : ring_hi + static_cast<uint32_t>(s) * C::kSlotBytes; };

  const uint32_t lanesel = 0x00010000u | (static_cast<uint32_t>(lane) << 2);
  const int g = lane >> 2, tig = lane & 3;
  const int warps = gridDim.x * C::kWarps;
  const int tok_per_task = 8 * NG;
  const uint4 zero = make_uint4(0, 0, 0, 0);

  // Task order: task t runs on CTA t % gridDim.x (one CTA per SM), on its warp
  // (t / gridDim.x) % kWarps, so consecutive tasks -- neighbouring rows of one product,
  // of equal cost -- go to different SMs and every SM gets a near-equal share of each
  // product's work (assigning consecutive tasks to the warps of one CTA left one SM with
  // up to 3.4x the average work for some layer stacks).
  const int task0 = blockIdx.x + gridDim.x * wid;
  // producer cursor: (task, chunk) running kDepth - 1 chunks ahead, across tasks
  int p_task = task0;
  const uint8_t* p_src = nullptr;   // this thread's 16 code bytes of row n0 + g, next chunk
  int64_t p_kb = 0;                 // code bytes per row
  int p_left = 0;                   // chunks left in the producer's task
  bool p_tail_ok = true;            // this thread's part of a partial last chunk is in range
  auto p_start = [&]() {
    if (p_task < G.total_tasks) {
      const DecTask d = dec_task(G, p_task, tok_per_task, 16 * RB);
      p_kb = d.P->k_in >> 2;
      p_src = d.P->codes + static_cast<int64_t>(d.n0 + g) * p_kb + tig * 16;
      p_left = d.nch;
      const int rem = d.P->k_in & 255;
      p_tail_ok = rem == 0 || 64 * tig < rem;
    }
  };
  p_start();
  int issued = 0;
  auto produce_one = [&]() {   // always commits one group (empty past the end)
    if (p_task < G.total_tasks) {
      const bool valid = p_left > 1 || p_tail_ok;
      const uint32_t dst = slot_addr(issued % C::kDepth);
#pragma unroll
      for (int sg = 0; sg < 2 * RB; ++sg)
        cp_async16(dst + sg * kHalf, valid ? p_src + (16 * (sg >> 1) + 8 * (sg & 1)) * p_kb : G.p[0].codes, valid);
      p_src += 64;
      if (--p_left == 0) {
        p_task += warps;
        p_start();
      }
    }
    cp_async_commit();
    ++issued;
  };
#pragma unroll
  for (int i = 0; i < C::kDepth - 1; ++i) produce_one();

  int consumed = 0;
  for (int task = task0; task < G.total_tasks; task += warps) {
    const DecTask d = dec_task(G, task, tok_per_task, 16 * RB);
    const FwdProblem& P = *d.P;
    const int K = P.k_in;
    const int8_t* xrow[NG];
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      const int tok = min(d.t0 + 8 * j + g, P.t - 1);   // past-the-end tokens feed unstored columns
      xrow[j] = P.xq + static_cast<int64_t>(tok) * K + tig * 64;
    }
    DecAcc<NG> accs[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b)
#pragma unroll
      for (int k = 0; k < DecAcc<NG>::kSets; ++k)
#pragma unroll
        for (int j = 0; j < NG; ++j)
          accs[b].v[k][j][0] = accs[b].v[k][j][1] = accs[b].v[k][j][2] = accs[b].v[k][j][3] = 0;
    // one chunk: this thread's code words of every row block, its activations, 8 MMAs per block
    auto chunk = [&](const uint4 (&xv)[NG][4]) {
      produce_one();                      // chunk consumed + kDepth - 1
      cp_async_wait<C::kDepth - 1>();     // chunk `consumed` has landed (own copies only)
      const uint32_t slot = slot_addr(consumed % C::kDepth);
      ++consumed;
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        uint4 c0, c1;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(c0.x), "=r"(c0.y), "=r"(c0.z), "=r"(c0.w) : "r"(slot + 2 * b * kHalf));
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(c1.x), "=r"(c1.y), "=r"(c1.z), "=r"(c1.w) : "r"(slot + (2 * b + 1) * kHalf));
        decode_chunk<NG>(accs[b], lanesel, c0, c1, xv);
      }
    };
    const int nfull = K >> 8;
    // full chunks: every thread's 64 weights are in range. The chunk's activations are
    // loaded at its start (L1/L2 hits; the resident warps hide the latency): a register
    // prefetch of the next chunk's activations measured 5 % slower at batch 1, from the
    // copies it costs and the registers it holds.
    for (int ch = 0; ch < nfull; ++ch) {
      uint4 xv[NG][4];
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const uint4* xp = reinterpret_cast<const uint4*>(xrow[j] + ch * 256);
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[j][q] = __ldg(xp + q);
      }
      chunk(xv);
    }
    if (K & 255) {   // partial last chunk: threads past the end use zero activations
      const bool mine = nfull * 256 + 64 * tig < K;
      uint4 xv[NG][4];
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const uint4* xp = reinterpret_cast<const uint4*>(xrow[j] + nfull * 256);
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[j][q] = mine ? __ldg(xp + q) : zero;
      }
      chunk(xv);
    }
    // C fragment of block b: acc[j][0..1] = row 16b + g, tokens 2*tig, 2*tig+1;
    // acc[j][2..3] = row 16b + g + 8
    const float gamma = *P.w_scale;
#pragma unroll
    for (int b = 0; b < RB; ++b) {
#pragma unroll
      for (int j = 0; j < NG; ++j) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          int accv = 0;
#pragma unroll
          for (int k = 0; k < DecAcc<NG>::kSets; ++k) accv += accs[b].v[k][j][v];
          const int tok = d.t0 + 8 * j + 2 * tig + (v & 1);
          const int n = d.n0 + 16 * b + g + ((v >> 1) << 3);
          if (tok < P.t) {
            const float rs = __fmul_rn(__fdiv_rn(P.absmax[tok], 127.0f), gamma);
            const float y = __fmul_rn(static_cast<float>(accv), rs);
            const int64_t off = static_cast<int64_t>(tok) * P.n_out + n;
            if (G.y_f32) static_cast<float*>(P.y)[off] = y;
            else static_cast<__nv_bfloat16*>(P.y)[off] = __float2bfloat16_rn(y);
            if (P.acc != nullptr) P.acc[off] = accv;
          }
        }
      }
    }
  }
  cp_async_wait<0>();   // no copy in flight when the thread exits
}

}  // namespace bl
