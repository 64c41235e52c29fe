"""CPU oracle of the Sparse-BitNet BitLinear path: plain, slow, obviously correct.

TEST INFRASTRUCTURE. Only the tests, the smoke check of ``__graft_entry__`` and the
CPU legs of ``bench.py`` (``cpu_baseline`` and ``--impl reference``) may import this
module. The product path (the
CUDA library and its Python binding) never imports, calls or falls back to it,
and this module imports nothing from the product package.

Sources. Page names used below:

* "Sparse-BitNet article" -- the Chinese write-up of Sparse-BitNet
  (m.top168.com/news/show-814037.html), cited by its numbered sections.
* "Sparse-BitNet digest" -- the paper digest page "Sparse-BitNet: 1.58-bit LLMs are
  Naturally Friendly to Semi-Structured Sparsity" (shd-paper.top), its abstract.
* "BitNet b1.58 2B4T article" -- the write-up of BitNet b1.58 2B4T
  (lsdiaocha.cn/2025/0716/3169029.shtml), cited by its numbered sections.

The pages print no formula. Each function states the plain reading it computes
and which passage it follows; every reading where the pages are silent is named
``reading:`` in the docstring. Floating point is fp64 except where a reading fixes
fp32 (the ternary and int8 quantisers, whose results are integers and must be
decided in one stated precision).

Every function here is pinned by ``tests/test_oracle_pins.py`` against values worked
by hand, closed forms, invariants and brute force. Parity pinned for all of them.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

EPS_W = np.float32(1e-5)        # the absmean epsilon
EPS_ACT = np.float32(1e-5)      # floor of a zero activation row's absmax (reading)
Q_ACT = np.float32(127.0)       # int8 activation scale numerator
FIXED_SHIFT = 32                # |w| is summed as floor(|w| * 2^32) (reading)
W_ABS_LIMIT = np.float32(65536.0)


class OracleRangeError(ValueError):
    """A latent weight is non-finite or |w| >= 2^16 (outside the summed range)."""


# --------------------------------------------------------------------------- helpers

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def rn_f32_from_rational(num: int, den: int) -> np.float32:
    """num/den (integers, num >= 0, den > 0) rounded to the nearest fp32, ties to even.

    Exact rational arithmetic: find e with 2^e <= q < 2^(e+1), scale q to a 24-bit
    integer mantissa, round half to even, renormalise on carry.
    """
    if num == 0:
        return np.float32(0.0)
    q = Fraction(num, den)
    e = num.bit_length() - den.bit_length()
    if q < Fraction(2) ** e:
        e -= 1
    assert Fraction(2) ** e <= q < Fraction(2) ** (e + 1)
    assert e >= -126, "subnormal means are outside the summed range"
    m = q / Fraction(2) ** (e - 23)          # in [2^23, 2^24)
    mi = m.numerator // m.denominator
    rem = m - mi
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and mi % 2 == 1):
        mi += 1
    if mi == 1 << 24:
        mi, e = 1 << 23, e + 1
    value = Fraction(mi) * Fraction(2) ** (e - 23)
    return np.float32(float(value))          # exact: 24-bit mantissa, normal exponent


# --------------------------------------------------------------------------- step a2: gamma

def absmean_gamma(w: np.ndarray) -> tuple[np.float32, np.float32, int]:
    """gamma = mean|W| + 1e-5 over the WHOLE, UNMASKED weight tensor.

    Follows: BitNet b1.58 2B4T article section 一 (absmean quantisation of the
    weights to {-1, 0, +1}); Sparse-BitNet article section 六 (quantise first, then
    sparsify: the scale is taken before any mask is applied).

    reading (the pages fix no precision or summation order): each |w| is truncated
    to a multiple of 2^-32, u = floor(|w| * 2^32) (exact for |w| < 2^16), the u are
    summed exactly as integers, and mean = S / (n * 2^32) is rounded once to the
    nearest fp32 (ties to even). gamma = fp32(mean + fp32(1e-5)). The truncation
    moves the mean by less than 2^-32; summation order cannot change the result.

    Returns (gamma, mean, S).
    """
    a = np.abs(np.asarray(w, dtype=np.float32).ravel())
    if a.size == 0:
        raise ValueError("mean over an empty tensor is undefined")
    if not np.all(np.isfinite(a)) or np.any(a >= W_ABS_LIMIT):
        raise OracleRangeError("latent weight non-finite or |w| >= 2^16")
    # fp32 -> fp64 is exact; * 2^32 is exact; floor is exact; < 2^48 fits uint64
    u = np.floor(a.astype(np.float64) * float(1 << FIXED_SHIFT)).astype(np.uint64)
    total = 0
    for s in range(0, u.size, 1 << 15):          # each chunk sum < 2^63
        total += int(u[s:s + (1 << 15)].sum(dtype=np.uint64))
    mean = rn_f32_from_rational(total, a.size << FIXED_SHIFT)
    gamma = np.float32(mean + EPS_W)             # one fp32 addition
    return gamma, mean, total


# --------------------------------------------------------------------------- step a2: codes

def ternary_codes(w: np.ndarray, gamma: np.float32) -> np.ndarray:
    """code = RoundClip(w / gamma, -1, 1) as int8, before any mask.

    Follows: BitNet b1.58 2B4T article section 一 (weights take only -1, 0, +1 via
    absmean quantisation).
    reading: w / gamma is one IEEE fp32 division; rounding is to nearest, ties to
    even (so |w/gamma| == 0.5 gives 0); the clip is to [-1, 1].
    """
    w32 = np.asarray(w, dtype=np.float32)
    r = np.rint(w32 / np.float32(gamma))         # fp32 / fp32 -> fp32, then RNE
    return np.clip(r, -1, 1).astype(np.int8)


# --------------------------------------------------------------------------- step a1: mask

def nm_keep(w: np.ndarray, n_keep: int, m_group: int) -> np.ndarray:
    """Boolean keep-mask of the N:M pattern, same shape as w [rows, K].

    Follows: Sparse-BitNet article section 三 (the mask is recomputed at every
    training step by ranking the parameters and keeping the best ones), section 五
    (a threshold per group of 8 parameters: keep 6, drop 2) and section 六 (the
    ranking uses the full-precision latent weights, never the ternary codes, because
    ternary values tie too often).

    Groups are M contiguous elements along K (the input dimension). Within a group,
    element j has rank_j = #{i : |w_i| > |w_j|, or |w_i| == |w_j| and i < j}; it is
    kept iff rank_j < N. reading: ties go to the lower index (the pages are silent).
    """
    w32 = np.asarray(w, dtype=np.float32)
    rows, k = w32.shape
    if k % m_group:
        raise ValueError("K must be a multiple of M")
    a = np.abs(w32).reshape(-1, m_group)
    idx = np.arange(m_group)
    lower = idx[:, None] < idx[None, :]                 # [i, j]: i < j
    keep = np.empty(a.shape, dtype=bool)
    for s in range(0, a.shape[0], 1 << 16):
        g = a[s:s + (1 << 16)]
        ai = g[:, :, None]
        aj = g[:, None, :]
        beats = (ai > aj) | ((ai == aj) & lower[None])  # i outranks j
        rank = beats.sum(axis=1)
        keep[s:s + (1 << 16)] = rank < n_keep
    return keep.reshape(rows, k)


def mask_bytes(keep: np.ndarray, m_group: int) -> np.ndarray:
    """Mask storage: one uint8 per group of M, bit j set iff element j is kept."""
    rows, k = keep.shape
    g = keep.reshape(rows, k // m_group, m_group).astype(np.uint32)
    weights = (1 << np.arange(m_group, dtype=np.uint32))
    return (g * weights).sum(axis=2).astype(np.uint8)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Pack ternary codes 4 per byte: element k at bits 2*(k mod 4) of byte k//4,
    with 0 -> 0b00, +1 -> 0b01, -1 -> 0b11 (0b10 unused).

    Follows: BitNet b1.58 2B4T article section 四 (four ternary values are encoded
    into one 8-bit integer for storage). The bit layout is this library's own.
    """
    c = np.asarray(codes, dtype=np.int8)
    rows, k = c.shape
    enc = np.zeros(c.shape, dtype=np.uint32)
    enc[c == 1] = 0b01
    enc[c == -1] = 0b11
    enc = enc.reshape(rows, k // 4, 4)
    shifts = np.array([0, 2, 4, 6], dtype=np.uint32)
    return (enc << shifts).sum(axis=2).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes; raises on the unused 0b10 pattern."""
    p = np.asarray(packed, dtype=np.uint8)
    rows, kb = p.shape
    fields = (p[:, :, None] >> np.array([0, 2, 4, 6], dtype=np.uint8)) & 3
    if np.any(fields == 0b10):
        raise ValueError("invalid code 0b10")
    out = np.zeros(fields.shape, dtype=np.int8)
    out[fields == 0b01] = 1
    out[fields == 0b11] = -1
    return out.reshape(rows, kb * 4)


def quant_mask(w: np.ndarray, n_keep: int, m_group: int) -> dict:
    """Steps a1 + a2 for one weight tensor: gamma, N:M mask and masked ternary codes.

    Follows: Sparse-BitNet article section 六 (quantise first, then sparsify; the
    mask is built from the latent weights): gamma and the codes come from the
    unmasked tensor; the mask then zeroes the dropped codes.
    """
    gamma, mean, total = absmean_gamma(w)
    code = ternary_codes(w, gamma)
    keep = nm_keep(w, n_keep, m_group)
    mcode = (code * keep).astype(np.int8)
    return {
        "gamma": gamma,
        "mean": mean,
        "abs_sum_fixed": total,
        "code": code,
        "keep": keep,
        "mask": mask_bytes(keep, m_group),
        "mcode": mcode,
        "codes_packed": pack_codes(mcode),
    }


# --------------------------------------------------------------------------- optimizer step + a1, a2

def sgd_update(w: np.ndarray, g_bits: np.ndarray, lr: float) -> np.ndarray:
    """W <- fp32(W - lr * G): the latent-weight update that precedes the mask recompute.

    Follows: Sparse-BitNet article section 三 (the mask is recomputed at every training
    step from the latent weights that step has just updated). reading: the pages name
    no optimizer; the fused update is plain SGD, with G the bf16 gradient of W, lr an
    fp32 scalar, and the exact value W - lr * G rounded once to fp32 (nearest, ties to
    even).

    lr * G is exact in fp64 (24-bit times 8-bit significands). W - lr * G is formed as
    an fp64 sum s plus its exact error e (Knuth's two-sum), so s + e is the exact value;
    s rounded to fp32 is the answer unless s lies exactly halfway between two fp32
    values, where the sign of e decides (e = 0: ties to even).
    """
    w64 = np.asarray(w, dtype=np.float32).astype(np.float64)
    p = -(np.float64(np.float32(lr)) * bf16_to_f32(g_bits).astype(np.float64))   # exact
    s = w64 + p
    bv = s - w64
    e = (w64 - (s - bv)) + (p - bv)                    # s + e == w - lr * g exactly
    r = s.astype(np.float32)                            # nearest fp32, ties to even
    r64 = r.astype(np.float64)
    up = np.nextafter(r, np.float32(np.inf)).astype(np.float64)
    dn = np.nextafter(r, np.float32(-np.inf)).astype(np.float64)
    to_up = (s == (r64 + up) / 2) & (e > 0)             # s is the upper midpoint, true value above it
    to_dn = (s == (r64 + dn) / 2) & (e < 0)             # s is the lower midpoint, true value below it
    out = r.copy()
    out[to_up] = up[to_up].astype(np.float32)
    out[to_dn] = dn[to_dn].astype(np.float32)
    return out


def sgd_quant_mask(w: np.ndarray, g_bits: np.ndarray, lr: float, n_keep: int, m_group: int) -> dict:
    """The optimizer step fused with steps a1 + a2: the updated W, then exactly
    ``quant_mask`` of it (Sparse-BitNet article section 三: mask and codes follow
    the latent weights every step)."""
    w_new = sgd_update(w, g_bits, lr)
    out = quant_mask(w_new, n_keep, m_group)
    out["w"] = w_new
    return out


# --------------------------------------------------------------------------- step a3

def act_quant(x_bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-token absmax int8 quantisation of bf16 activations [T, K].

    Follows: BitNet b1.58 2B4T article section 一 (activations are quantised to
    8-bit integers) and section 四 (W1.58A8: ternary weights times int8
    activations).
    reading: a_t = max_k |x_tk| (exact in fp32); a zero row uses a_t = 1e-5;
    s_t = fp32(127 / a_t); q = clip(rint(fp32(x * s_t)), -128, 127), round half to
    even, one fp32 multiply (no fused multiply-add). Returns (q int8, a_t fp32).
    """
    x = bf16_to_f32(x_bits)
    a = np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)
    a = np.where(a == 0, EPS_ACT, a).astype(np.float32)
    s = (Q_ACT / a).astype(np.float32)
    prod = (x * s[:, None]).astype(np.float32)
    q = np.clip(np.rint(prod), -128, 127).astype(np.int8)
    return q, a


# --------------------------------------------------------------------------- step a4

def fwd(q: np.ndarray, absmax: np.ndarray, mcode: np.ndarray, gamma: np.float32,
        rows: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Masked ternary x int8 product: acc[t,n] = sum_k q[t,k] * mcode[n,k] (exact
    integers), y[t,n] = acc * (a_t / 127) * gamma in fp64.

    Follows: BitNet b1.58 2B4T article section 四 (unpacked ternary weights
    multiplied with 8-bit activations); Sparse-BitNet article section 四 (the 6:8
    sparse operator computes this product); no bias (BitNet b1.58 2B4T article
    section 一: all bias terms are removed).

    The integer sum is formed as an fp64 matrix product: every operand is an integer
    of magnitude <= 128 and every partial sum is below 128 * K < 2^53, so fp64
    represents each partial sum exactly and the result is the exact integer in any
    summation order. ``rows`` selects the tokens to compute (all by default).
    """
    qq = q if rows is None else q[rows]
    aa = absmax if rows is None else absmax[rows]
    k = qq.shape[1]
    assert 128 * k < 2 ** 53
    acc = qq.astype(np.float64) @ mcode.astype(np.float64).T
    acc_i = acc.astype(np.int64)
    assert np.all(acc_i == acc) and np.all(np.abs(acc_i) < 2 ** 31)
    y = acc * (aa.astype(np.float64)[:, None] / 127.0) * float(gamma)
    return acc_i.astype(np.int32), y


# --------------------------------------------------------------------------- steps a5, a6

def grad_x(dy_bits: np.ndarray, mcode: np.ndarray, gamma: np.float32,
           rows: np.ndarray | None = None) -> np.ndarray:
    """grad_X = dY . W_eff with W_eff = gamma * (mask . code), fp64.

    Follows: Sparse-BitNet article section 三 and section 六 (dual straight-through
    estimator: the gradient passes through both the quantiser and the mask, so the
    input gradient uses the effective weight of the forward).
    """
    dy = bf16_to_f32(dy_bits if rows is None else dy_bits[rows]).astype(np.float64)
    w_eff = float(gamma) * mcode.astype(np.float64)
    return dy @ w_eff


def grad_w(dy_bits: np.ndarray, x_bits: np.ndarray, rows: np.ndarray | None = None,
           x_deq: np.ndarray | None = None) -> np.ndarray:
    """grad_W = dY^T . X over EVERY latent weight, masked ones included, fp64.

    Follows: Sparse-BitNet article section 三 (a weight masked in this step still
    receives its gradient, so it can return later) and section 六 (dual
    straight-through estimator).
    reading: X is the layer's bf16 input; ``x_deq`` (fp64 [T, K]) replaces it when
    the caller asks for the dequantised activations instead. ``rows`` selects output
    rows n.
    """
    dy = bf16_to_f32(dy_bits).astype(np.float64)
    if rows is not None:
        dy = dy[:, rows]
    x = bf16_to_f32(x_bits).astype(np.float64) if x_deq is None else x_deq
    return dy.T @ x


def dequant_x(q: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """X_deq = q * a_t / 127 (fp64): what the forward product actually consumed."""
    return q.astype(np.float64) * (absmax.astype(np.float64)[:, None] / 127.0)


def dequant_x_bf16(q: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """X_deq as a bf16 operand (fp64 values of the bf16 numbers): s_t = fp32(a_t / 127),
    one fp32 multiply q * s_t, then round to the nearest bf16 (ties to even).

    reading: the dequantised-activation option of grad_W feeds a bf16 product, so its
    operand is X_deq rounded to bf16; ``dequant_x`` is the exact value it rounds.
    """
    s = (np.asarray(absmax, dtype=np.float32) / np.float32(127.0)).astype(np.float32)
    p = (np.asarray(q, dtype=np.float32) * s[:, None]).astype(np.float32)
    u = p.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)).astype(np.uint32)
    return (r << np.uint32(16)).view(np.float32).astype(np.float64)


def grad_x_int8_dy(dy_bits: np.ndarray, mcode: np.ndarray, gamma: np.float32,
                   rows: np.ndarray | None = None) -> tuple[np.ndarray, np.ndarray, np.ndarray, np.ndarray]:
    """grad_X with dY quantised per token to int8, as an exact integer product.

    An approximation this library offers for the input gradient (the pages keep dY in
    higher precision): dY is quantised with the same per-token absmax rule as the
    activations (BitNet b1.58 2B4T article section 一), then multiplied with the
    masked ternary codes exactly in integers (Sparse-BitNet article section 六: the
    input gradient goes through the effective weight), then rescaled:
        acc[t,k] = sum_n q_dy[t,n] * mcode[n,k],  grad_x ~ acc * (a_t / 127) * gamma.
    Returns (acc int32, grad_x fp64, q_dy, a_dy). ``rows`` selects tokens.
    """
    dyr = dy_bits if rows is None else dy_bits[rows]
    q, a = act_quant(dyr)
    acc, y = fwd(q, a, mcode.T, gamma)
    return acc, y, q, a


# --------------------------------------------------------------------------- 2:4 storage

def compress_2_4(mcode: np.ndarray, keep: np.ndarray) -> dict:
    """2:4 structured storage of masked ternary codes (the form sparse tensor cores take).

    Follows: Sparse-BitNet article section 七 (NVIDIA's sparse tensor cores need the 2:4
    pattern: at most two nonzero weights in every aligned group of four along K).
    reading: every aligned group of 4 stores exactly two values and their positions
    i0 < i1 (2 bits each). Kept positions come first in increasing order; a group with
    fewer than two kept positions is completed with the lowest unused positions, whose
    stored value is 0. Metadata byte j of a row holds group 2j in bits 0-3 and group
    2j+1 in bits 4-7, each nibble = i0 | (i1 << 2). Masks with more than two kept
    positions in a group (6:8, 4:8, 3:8) are not 2:4-valid and raise ValueError.
    Returns {"values": int8 [rows, K/2], "idx": uint8 [rows, K/4, 2], "meta": uint8 [rows, K/8]}.
    """
    c = np.asarray(mcode, dtype=np.int8)
    kp = np.asarray(keep, dtype=bool)
    rows, k = c.shape
    assert k % 8 == 0
    values = np.zeros((rows, k // 2), dtype=np.int8)
    idx = np.zeros((rows, k // 4, 2), dtype=np.uint8)
    meta = np.zeros((rows, k // 8), dtype=np.uint8)
    for r in range(rows):
        for g in range(k // 4):
            kept = [j for j in range(4) if kp[r, 4 * g + j]]
            if len(kept) > 2:
                raise ValueError(f"row {r} group {g}: {len(kept)} kept positions, not 2:4-valid")
            pos = list(kept)
            for j in range(4):
                if len(pos) == 2:
                    break
                if j not in pos:
                    pos.append(j)
            pos.sort()
            for s_, j in enumerate(pos):
                values[r, 2 * g + s_] = c[r, 4 * g + j] if kp[r, 4 * g + j] else 0
                idx[r, g, s_] = j
            nib = pos[0] | (pos[1] << 2)
            meta[r, g // 2] |= np.uint8(nib << (4 * (g % 2)))
    return {"values": values, "idx": idx, "meta": meta}


def decompress_2_4(values: np.ndarray, meta: np.ndarray) -> np.ndarray:
    """Inverse of compress_2_4: scatter each group's two values to the positions its
    metadata nibble names. Returns int8 [rows, K]."""
    rows, half = values.shape
    k = 2 * half
    out = np.zeros((rows, k), dtype=np.int8)
    for r in range(rows):
        for g in range(k // 4):
            nib = (int(meta[r, g // 2]) >> (4 * (g % 2))) & 0xF
            i0, i1 = nib & 3, nib >> 2
            out[r, 4 * g + i0] = values[r, 2 * g]
            out[r, 4 * g + i1] = values[r, 2 * g + 1]
    return out


# --------------------------------------------------------------------------- diagnostics

HIST_BINS = 17   # [k/8, (k+1)/8) of gamma for k = 0..15, then [2, inf)


def threshold_hist(w: np.ndarray, keep: np.ndarray, gamma: np.float32, m_group: int) -> dict:
    """Where the N:M threshold falls relative to the ternary levels.

    Follows: Sparse-BitNet article section 五 (threshold decoupling: each group of 8
    gets a threshold that splits kept from dropped weights; in the 1.58-bit model it
    stays in the near-zero "noise" region instead of cutting into weights that
    matter).
    reading: a group's threshold is the largest magnitude among its dropped weights,
    measured in units of gamma; ``hist[k]`` counts the groups whose threshold r has
    k/8 <= r < (k+1)/8 (k = 0..15) and ``hist[16]`` those with r >= 2, the bin decided
    exactly (8|w| against k * gamma in fp64, both products exact). Groups with no
    dropped weight (N = M) are not counted. ``dropped`` counts dropped weights and
    ``dropped_core`` those whose ternary code is nonzero (|w| > gamma / 2, the
    rounding rule of the ternary quantiser), i.e. weights the mask cut from the
    +-1 levels.
    """
    a = np.abs(np.asarray(w, dtype=np.float32)).astype(np.float64)
    rows, k = a.shape
    groups = a.reshape(rows, k // m_group, m_group)
    kept = np.asarray(keep, dtype=bool).reshape(rows, k // m_group, m_group)
    g64 = float(gamma)
    hist = np.zeros(HIST_BINS, dtype=np.int64)
    dropped = 0
    core = 0
    for r in range(rows):
        for gi in range(k // m_group):
            drop_vals = groups[r, gi][~kept[r, gi]]
            if drop_vals.size == 0:
                continue
            dropped += drop_vals.size
            core += int(np.sum(2.0 * drop_vals > g64))
            t = drop_vals.max()
            b = 0
            while b < HIST_BINS - 1 and 8.0 * t >= (b + 1) * g64:
                b += 1
            hist[b] += 1
    return {"hist": hist, "dropped": dropped, "dropped_core": core}


# --------------------------------------------------------------------------- whole layer

def layer_step(w: np.ndarray, x_bits: np.ndarray, dy_bits: np.ndarray,
               n_keep: int, m_group: int) -> dict:
    """One pass of the whole path for one BitLinear layer: mask + ternary codes,
    int8 activations, forward product, both straight-through gradients."""
    qm = quant_mask(w, n_keep, m_group)
    q, a = act_quant(x_bits)
    acc, y = fwd(q, a, qm["mcode"], qm["gamma"])
    gx = grad_x(dy_bits, qm["mcode"], qm["gamma"])
    gw = grad_w(dy_bits, x_bits)
    return {**qm, "q": q, "absmax": a, "acc": acc, "y": y, "grad_x": gx, "grad_w": gw}
