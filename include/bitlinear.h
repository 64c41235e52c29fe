/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) Sparse-BitNet BitLinear path.
 *
 * One BitLinear layer: a dynamic N:M mask over the latent fp32 weights, absmean
 * ternary codes {-1, 0, +1}, per-token int8 activations, the masked ternary x int8
 * product with int32 accumulation, and the dual straight-through backward.
 *
 * Sources (pages named by title and section):
 *   - Sparse-BitNet article (m.top168.com/news/show-814037), section 三: the mask is
 *     recomputed every training step; the dual straight-through estimator passes
 *     gradients through quantiser and mask; masked weights still get gradients.
 *     Section 五: one threshold per group of 8 weights. Section 六: quantise first,
 *     then sparsify; the mask ranks the full-precision latent weights.
 *   - Sparse-BitNet paper digest (shd-paper.top), abstract: 1.58-bit weights with
 *     dynamic N:M sparsity, run on a custom sparse tensor-core operator.
 *   - BitNet b1.58 2B4T article (lsdiaocha.cn/2025/0716/3169029), section 一:
 *     absmean quantisation of the weights to {-1, 0, +1}, 8-bit integer activations,
 *     BitLinear layers without bias. Section 四: four ternary values per byte, moved
 *     HBM -> shared memory and unpacked before the product with int8 activations.
 *
 * Conventions shared by every entry point:
 *   - Memory: every pointer is a DEVICE pointer owned by the caller; the library
 *     allocates no device memory. All arrays are row-major and contiguous. Every
 *     pointer must be 16-byte aligned (BL_ERR_ALIGNMENT otherwise).
 *   - Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Calls only enqueue work and return; results are ready when the
 *     stream reaches them.
 *   - Devices and threads: a call runs on the calling thread's current device (the
 *     stream and every pointer must belong to it; device ordinals 0-63). Each kernel
 *     is set up (shared-memory limit, occupancy) on the first call that uses it on a
 *     device, so one process may drive several devices, from one thread or several.
 *   - Shapes: k_in % 64 == 0, 64 <= k_in <= 131072, n_out % 16 == 0, n_out >= 16,
 *     t >= 0 (t = 0 is a valid empty batch; the arrays sized by t may then be
 *     NULL). Else BL_ERR_UNSUPPORTED_SHAPE.
 *   - bf16 arrays are passed as uint16_t bit patterns.
 *   - Errors: argument, shape and alignment errors return before anything is
 *     enqueued; a failed launch returns BL_ERR_CUDA. bitlinear_last_error() gives a
 *     message for the last non-OK status of the calling thread.
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = -1,       /* null pointer, bad N:M, bad dtype            */
  BL_ERR_UNSUPPORTED_SHAPE = -2, /* shape outside the rules above               */
  BL_ERR_ALIGNMENT = -3,         /* a pointer is not 16-byte aligned            */
  BL_ERR_RANGE = -4,             /* a latent weight is non-finite or |w| >= 2^16 */
  BL_ERR_CUDA = -5,              /* a CUDA call or kernel launch failed          */
  BL_ERR_TIMEOUT = -6,           /* a kernel gave up on a bounded wait          */
  BL_ERR_WORKSPACE = -7          /* workspace missing or too small               */
} bl_status;

typedef enum { BL_OUT_BF16 = 0, BL_OUT_F32 = 1 } bl_dtype;

/* Bytes of workspace bitlinear_quant_mask needs for a [n_out, k_in] tensor. */
size_t bitlinear_quant_mask_workspace_size(int64_t n_out, int64_t k_in);

/*
 * Steps a1 + a2: absmean scale, N:M mask and masked ternary codes of one latent
 * weight tensor W [n_out, k_in] (fp32). Recompute it every training step.
 *
 *   gamma   = mean|W| + 1e-5 over the whole UNMASKED tensor (quantise first, then
 *             sparsify). The mean is exact and order-independent: every |w| is
 *             truncated to a multiple of 2^-32, summed as an integer, and the sum /
 *             (n * 2^32) is rounded once to fp32 (ties to even).
 *   code    = RoundClip(w / gamma, -1, 1) (fp32 division, round half to even).
 *   mask    = per group of m_group contiguous weights along k_in, keep the n_keep
 *             largest |w| of the LATENT weights; equal |w| go to the lower index.
 *   masked code = mask ? code : 0.
 *
 *   w_latent     [n_out, k_in] fp32, in.
 *   n_keep, m_group: 1 <= n_keep <= m_group, m_group in {4, 8} (8:8 = no mask).
 *   mask_out     [n_out, k_in / m_group] uint8, out, nullable. Bit j of byte g is
 *                element j of group g (bits 0..3 only when m_group == 4).
 *   codes_out    [n_out, k_in / 4] uint8, out. Masked codes, 4 per byte: element k
 *                at bits 2*(k % 4) of byte k / 4; 00 = 0, 01 = +1, 11 = -1.
 *   w_i8_out     [n_out, k_in] int8, out, nullable. Masked codes as int8 (the
 *                operand of the tensor-core forward product).
 *   sp_values_out [n_out, k_in / 2] int8, out, nullable, and
 *   sp_meta_out  [n_sp, k_sp / 8] uint8, out, nullable, with n_sp = n_out and k_sp =
 *                k_in each rounded up to a multiple of 256 (both or neither; only for
 *                masks with at most two kept weights in every aligned group of four:
 *                n_keep <= 2, else BL_ERR_INVALID_ARG). The 2:4 structured form of the
 *                masked codes that sparse tensor cores take (Sparse-BitNet article,
 *                section 七: NVIDIA's sparse tensor cores need the 2:4 pattern): per
 *                aligned group of four, two stored values and their positions i0 < i1
 *                (the kept positions, completed with the lowest unused ones, whose
 *                value is 0). Values of group g at bytes 2g, 2g+1 of the row; metadata
 *                nibble i0 | i1 << 2 of group g in bits 4*(g % 2) of byte g / 2 of the
 *                row. The padding rows and columns of sp_meta hold 0x44 (positions 0
 *                and 1), so that the sparse product reads whole tiles of valid metadata.
 *   w_scale_out  [1] fp32, out: gamma. NaN when the range check fails.
 *   workspace    bitlinear_quant_mask_workspace_size() bytes, scratch, in/out.
 *
 * Range errors (non-finite w or |w| >= 2^16) are found on the device: gamma is then
 * NaN, every code 0, and bitlinear_quant_mask_status() reports BL_ERR_RANGE.
 * Calls that share a workspace must not overlap on the GPU.
 */
bl_status bitlinear_quant_mask(const float* w_latent, int64_t n_out, int64_t k_in, int n_keep, int m_group,
                               uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out, int8_t* sp_values_out,
                               uint8_t* sp_meta_out, float* w_scale_out, void* workspace, size_t workspace_bytes,
                               void* stream);

/*
 * The latent-weight update of a training step fused with steps a1 + a2: the mask and
 * codes are recomputed every step from the weights the optimizer has just updated
 * (Sparse-BitNet article, section 三), so the update and the mask recompute share one
 * read of W instead of two. The pages name no optimizer; this is plain SGD:
 *
 *   W <- fp32(W - lr * G)     (G the bf16 gradient; one rounding per weight: a fused
 *                              multiply-add, round to nearest even)
 *
 * then exactly bitlinear_quant_mask of the updated W (same outputs, layouts and rules).
 *
 *   w_latent  [n_out, k_in] fp32, in/out: updated in place.
 *   grad_w    [n_out, k_in] bf16 (bit patterns), in. The gradient of W, e.g. grad_w
 *             of bitlinear_bwd.
 *   lr        finite fp32, else BL_ERR_INVALID_ARG.
 *   other arguments: as bitlinear_quant_mask.
 *
 * A range error of the UPDATED weights is reported as in bitlinear_quant_mask (the
 * update has then been applied). Calls that share a workspace must not overlap on the
 * GPU; w_latent must not overlap any output.
 */
bl_status bitlinear_sgd_quant_mask(float* w_latent, const uint16_t* grad_w, float lr, int64_t n_out, int64_t k_in,
                                   int n_keep, int m_group, uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out,
                                   int8_t* sp_values_out, uint8_t* sp_meta_out, float* w_scale_out, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then returns the range status (BL_OK or BL_ERR_RANGE) that
 * the last bitlinear_quant_mask using `workspace` recorded. */
bl_status bitlinear_quant_mask_status(const void* workspace, void* stream);

/*
 * bitlinear_quant_mask without a workspace and without any allocation. The paper has
 * no counterpart: this is a library convenience. It is for callers that cannot
 * allocate device memory at all -- code running inside a host framework that owns
 * every byte of device memory, or a latency-critical path where cudaMalloc/cudaFree
 * (which may synchronise the device) are not allowed.
 *
 * Same computation, arguments and outputs as bitlinear_quant_mask, minus the
 * workspace and the 2:4 outputs. Its scratch is a fixed array of 19200 bytes inside
 * the library (every GPU that loads the library holds it until exit), which limits
 * the tensor to n_out * k_in <= 4966055936 weights; larger tensors get
 * BL_ERR_UNSUPPORTED_SHAPE. The first call on each device looks up that array's
 * device address (with the device current) and keeps it for the life of the process;
 * make that first call before any stream capture. A reset of the device's primary
 * context (cudaDeviceReset) invalidates the kept address: do not call this entry
 * point on a device after resetting it. All calls on a device share the array, so
 * calls that overlap on the GPU race: order them on one stream. A range error shows
 * as gamma = NaN and all-zero codes (there is no workspace to read a status from).
 */
bl_status bitlinear_quant_mask_noalloc(const float* w_latent, int64_t n_out, int64_t k_in, int n_keep, int m_group,
                                       uint8_t* mask_out, uint8_t* codes_out, int8_t* w_i8_out, float* w_scale_out,
                                       void* stream);

/*
 * Step a3: per-token absmax int8 activation quantisation of X [t, k_in] (bf16).
 *   a_t = max_k |x_tk|   (a zero row uses a_t = 1e-5, giving q = 0)
 *   q   = clamp(rint(x * fp32(127 / a_t)), -128, 127), one fp32 multiply, ties to even.
 *   xq_out [t, k_in] int8, out. absmax_out [t] fp32, out: a_t.
 * Non-finite activations give unspecified (but in-bounds) results.
 */
bl_status bitlinear_act_quant(const uint16_t* x, int64_t t, int64_t k_in, int8_t* xq_out, float* absmax_out,
                              void* stream);

/*
 * Step a4: the masked ternary x int8 forward product.
 *   acc[t, n] = sum_k xq[t, k] * masked_code[n, k]           (exact, int32)
 *   y[t, n]   = acc * (absmax[t] / 127 * gamma)              (fp32, then bf16 or f32)
 *
 *   xq [t, k_in] int8, absmax [t] fp32 (from bitlinear_act_quant).
 *   The masked weights, in one of three forms (give at least one; the first given
 *   in this order is used, except that with both the 2:4 form and w_i8 the library
 *   picks per shape: the sparse product from 100 GOP dense-equivalent (2*t*k_in*n_out)
 *   up, where it measured faster, the dense one below):
 *     sp_values [n_out, k_in / 2] int8 + sp_meta [n_sp, k_sp / 8] uint8 (padded, see
 *       bitlinear_quant_mask): the 2:4 form from bitlinear_quant_mask (masks with at
 *       most two kept per aligned four). Runs on the sparse tensor cores
 *       (tcgen05.mma.sp kind::i8, CTA pairs): Sparse-BitNet article, section 七.
 *     w_i8 [n_out, k_in] int8 masked codes: the dense tcgen05 int8 tensor cores
 *       (TMA-fed, for prefill and training shapes).
 *     codes [n_out, k_in / 4] packed masked codes: streams the 2-bit codes and
 *       decodes them on chip (for decode batches): BitNet b1.58 2B4T article,
 *       section 四.
 *   w_scale [1] fp32 gamma. acc_out [t, n_out] int32, out, nullable.
 *   y_out [t, n_out], out, bf16 (y_dtype = BL_OUT_BF16) or fp32 (BL_OUT_F32).
 * No bias term.
 * The kernel for up to 8 tokens from codes keeps a lookup table at a fixed shared-memory
 * address: its first use on each device runs a one-CTA check of the shared-memory layout
 * and synchronises `stream` (make that first call before any stream capture). Where the
 * table does not fit, every such call returns BL_ERR_CUDA before enqueueing anything.
 */
bl_status bitlinear_fwd(const int8_t* xq, const float* absmax, const uint8_t* codes, const int8_t* w_i8,
                        const int8_t* sp_values, const uint8_t* sp_meta, const float* w_scale, int64_t t, int64_t k_in,
                        int64_t n_out, int32_t* acc_out, void* y_out, int y_dtype, void* stream);

/* One forward problem of bitlinear_fwd_grouped (same meaning as the arguments of
 * bitlinear_fwd, codes operand only). */
typedef struct {
  const int8_t* xq;       /* [t, k_in] int8 activations            */
  const float* absmax;    /* [t] per-token absmax                   */
  const uint8_t* codes;   /* [n_out, k_in / 4] packed masked codes  */
  const float* w_scale;   /* [1] gamma                              */
  int64_t t, k_in, n_out;
  int32_t* acc_out;       /* [t, n_out] int32, nullable             */
  void* y_out;            /* [t, n_out] bf16 or fp32                */
} bl_fwd_problem;

/*
 * Step a4 for up to 256 independent problems in one launch (e.g. every BitLinear of
 * a layer stack at one decode step, or the q/k/v or gate/up linears that share an
 * input). Same result as bitlinear_fwd with the codes operand for each problem; the
 * packed 2-bit codes are streamed once per 128 tokens (once per 8 tokens when the
 * largest problem has at most 8). `problems` is a HOST array (copied into the
 * launch); y_dtype applies to all problems. Problems may have t = 0.
 * The one-time layout check of bitlinear_fwd applies here too (batches of up to 8).
 * More than 256 problems: BL_ERR_UNSUPPORTED_SHAPE.
 */
bl_status bitlinear_fwd_grouped(const bl_fwd_problem* problems, int count, int y_dtype, void* stream);

/* Flags of bitlinear_bwd. */
enum {
  /* grad_w against the activations the forward product consumed, q * a_t / 127
   * (from bitlinear_act_quant), instead of the layer's bf16 input x. */
  BL_GRADW_DEQUANT_X = 1
};

/* Bytes of workspace bitlinear_bwd needs (0 when neither grad_x nor the
 * BL_GRADW_DEQUANT_X option is requested). */
size_t bitlinear_bwd_workspace_size(int64_t t, int64_t k_in, int64_t n_out, int want_grad_x, int flags);

/*
 * Steps a5 + a6: the dual straight-through backward (Sparse-BitNet article, section
 * 三: masked weights still receive gradients; section 六: the estimator passes the
 * gradient through both the quantiser and the mask).
 *   grad_x[t, k] = sum_n dy[t, n] * gamma * masked_code[n, k]   (bf16 out, fp32 accumulate)
 *   grad_w[n, k] = sum_t dy[t, n] * X[t, k]   for EVERY latent weight, masked ones
 *                  included (the mask does not enter; fp32 accumulate).
 *   X is the layer's bf16 input x by default. With flags & BL_GRADW_DEQUANT_X it is
 *   the dequantised int8 input, X[t, k] = bf16(q[t, k] * fp32(a_t / 127)): what the
 *   forward product consumed. The pages say only "straight-through"; both readings
 *   are offered.
 *
 *   dy [t, n_out] bf16. x [t, k_in] bf16 (needed for grad_w without the flag).
 *   xq [t, k_in] int8 and absmax [t] fp32 (needed for grad_w with the flag).
 *   codes [n_out, k_in / 4] packed masked codes, w_scale [1] gamma (needed for grad_x).
 *   grad_x [t, k_in] bf16, out, nullable. grad_w [n_out, k_in], out, nullable, bf16
 *   (grad_w_dtype = BL_OUT_BF16) or fp32 (BL_OUT_F32). With t = 0, grad_w is zeroed.
 *   flags: 0 or BL_GRADW_DEQUANT_X (other bits: BL_ERR_INVALID_ARG).
 *   workspace bitlinear_bwd_workspace_size() bytes: the bf16 ternary matrix
 *   [n_out, k_in] (for grad_x) followed by the bf16 X_deq [t, k_in] (with the flag).
 */
bl_status bitlinear_bwd(const uint16_t* dy, const uint16_t* x, const int8_t* xq, const float* absmax,
                        const uint8_t* codes, const float* w_scale, int64_t t, int64_t k_in, int64_t n_out,
                        uint16_t* grad_x, void* grad_w, int grad_w_dtype, int flags, void* workspace,
                        size_t workspace_bytes, void* stream);

/* One weight gradient of a group (see bitlinear_grad_w_grouped). */
typedef struct {
  const uint16_t* dy;  /* [t, n_out] bf16, in: gradient of this linear's output */
  const uint16_t* x;   /* [t, k_in] bf16, in: this linear's input */
  int64_t k_in, n_out;
  void* grad_w;        /* [n_out, k_in], out: bf16 (BL_OUT_BF16) or fp32 (BL_OUT_F32) */
  int grad_w_dtype;
} bl_grad_w_problem;

/*
 * Step a6 for several linears over the same t tokens (e.g. the gate, up and down
 * projections of an MLP block) in one launch: for each problem, grad_W = dY^T X exactly
 * as bitlinear_bwd computes it with grad_x = NULL and flags = 0 (the layer's bf16 input,
 * every latent weight including the masked ones; Sparse-BitNet article, sections 三 and
 * 六). The products' output tiles are scheduled together, so the partial last wave of
 * one product is filled with tiles of the next.
 *
 *   problems   count entries, 1 <= count <= 4; every pointer 16-byte aligned; shapes
 *              as bitlinear_bwd (k_in, n_out multiples of 64 and 16); outputs must not
 *              overlap each other or any input.
 *   t          tokens, shared by all problems (t = 0 zeroes every grad_w).
 *
 * Problems with n_out <= 128 (outside the two-SM tiles) run one after another instead.
 */
bl_status bitlinear_grad_w_grouped(const bl_grad_w_problem* problems, int count, int64_t t, void* stream);

/* Bytes of workspace bitlinear_grad_x_i8 needs (0 for an empty problem). */
size_t bitlinear_grad_x_i8_workspace_size(int64_t t, int64_t k_in, int64_t n_out);

/*
 * Step a5 with dY quantised to int8: an approximation of the input gradient that runs
 * on the int8 tensor cores. The pages keep the backward in higher precision; this
 * entry point has no counterpart there (it is the library's faster variant, to be
 * used only where its error is acceptable). dY is quantised per token exactly as
 * bitlinear_act_quant quantises activations (BitNet b1.58 2B4T article, section 一),
 * then multiplied with the masked ternary codes in integers (Sparse-BitNet article,
 * section 六: the input gradient goes through the effective weight):
 *   q, a   = act_quant(dy)                              ([t, n_out] int8, [t] fp32)
 *   acc    = sum_n q[t, n] * masked_code[n, k]          (exact, int32)
 *   grad_x = acc * (a_t / 127 * gamma)                  (fp32, then bf16)
 * Each dY element moves by at most half a quantisation step, so
 *   |grad_x - exact| <= sum_n |masked_code[n, k]| * gamma * a_t / 254  (+ rounding).
 *
 *   dy [t, n_out] bf16; codes [n_out, k_in / 4]; w_scale [1] gamma.
 *   grad_x [t, k_in] bf16, out. acc_out [t, k_in] int32, out, nullable.
 *   workspace bitlinear_grad_x_i8_workspace_size() bytes, 16-byte aligned (holds the
 *   int8 dY, its absmax and the transposed int8 codes).
 * Shapes as bitlinear_bwd, plus n_out % 64 == 0 (BL_ERR_UNSUPPORTED_SHAPE otherwise).
 */
bl_status bitlinear_grad_x_i8(const uint16_t* dy, const uint8_t* codes, const float* w_scale, int64_t t, int64_t k_in,
                              int64_t n_out, uint16_t* grad_x, int32_t* acc_out, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Threshold-decoupling diagnostic (Sparse-BitNet article, section 五: the threshold
 * that splits each group's kept from its dropped weights sits, for 1.58-bit weights,
 * in the near-zero region rather than cutting weights that quantise to +-1).
 *   For every group of m_group weights with at least one dropped weight (mask bit
 *   clear), r = max |w| over its dropped weights / gamma:
 *     hist_out[k]  (k = 0..15) counts groups with k/8 <= r < (k+1)/8,
 *     hist_out[16] counts groups with r >= 2,
 *     hist_out[17] = number of dropped weights,
 *     hist_out[18] = dropped weights with a nonzero ternary code (|w| > gamma / 2).
 *   Bin edges are decided exactly (8|w| against k * gamma in fp64).
 *   w_latent [n_out, k_in] fp32, mask [n_out, k_in / m_group] (bit j = element j kept,
 *   as written by bitlinear_quant_mask), w_scale [1] gamma, m_group 4 or 8.
 *   hist_out: 19 uint64 on the device, 16-byte aligned, overwritten.
 */
bl_status bitlinear_mask_threshold_hist(const float* w_latent, const uint8_t* mask, const float* w_scale, int64_t n_out,
                                        int64_t k_in, int m_group, unsigned long long* hist_out, void* stream);

/* Synchronises the current device, then returns BL_OK; BL_ERR_TIMEOUT if a kernel
 * of this library gave up on a bounded wait since the last call (bits 0-3); or
 * BL_ERR_CUDA if the decode kernel found its dynamic shared memory at an address
 * where its fixed-address lookup table does not fit and skipped its work (bit 4).
 * The raw status bits go to *bits when bits != NULL. Clears the status. */
bl_status bitlinear_device_status(unsigned int* bits);

/* Message for the calling thread's last non-OK status ("" if none). */
const char* bitlinear_last_error(void);

/* ABI version of this header: 2. */
int bitlinear_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H */
