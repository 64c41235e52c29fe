"""Pins of the CPU oracle against things other than itself (CPU only).

Every check here compares the oracle with a value worked by hand, a closed form,
an invariant the method must satisfy, or a brute-force computation written
differently from the oracle (pure-Python loops, subset enumeration, exact
rationals). None of them re-types the oracle's own formula.
"""
import math
import os
from fractions import Fraction
from itertools import combinations

import numpy as np
import pytest

from oracle import bitlinear_oracle as O
from sparsity_step_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_example.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            vals[k.strip()] = v.split()
    return vals


G = _golden()


def _ints(key):
    return [int(t, 0) for t in G[key]]


def _w_example():
    return np.array([float(t) for t in G["w"]], dtype=np.float32).reshape(1, 8)


def _x_example():
    return synth.f32_to_bf16_bits(np.array([float(t) for t in G["x"]], dtype=np.float32)).reshape(1, 8)


# ----------------------------------------------------------------------- hand-worked values

def test_hand_gamma_and_codes():
    qm = O.quant_mask(_w_example(), 8, 8)
    assert abs(float(qm["gamma"]) - float(G["gamma"][0])) < 2e-8
    assert qm["code"].ravel().tolist() == _ints("codes")


@pytest.mark.parametrize("n,m,key", [(8, 8, "keep_8_8"), (6, 8, "keep_6_8"), (4, 8, "keep_4_8"),
                                     (2, 8, "keep_2_8"), (2, 4, "keep_2_4")])
def test_hand_masks(n, m, key):
    keep = O.nm_keep(_w_example(), n, m)
    assert keep.astype(int).ravel().tolist() == _ints(key)


def test_hand_packed_codes():
    qm = O.quant_mask(_w_example(), 6, 8)
    assert qm["codes_packed"].ravel().tolist() == _ints("packed_6_8")
    # masked codes equal the unmasked ones here: both dropped weights quantise to 0
    assert qm["mcode"].ravel().tolist() == _ints("codes")


def test_hand_act_quant_and_acc():
    q, a = O.act_quant(_x_example())
    assert float(a[0]) == float(G["absmax"][0])
    assert q.ravel().tolist() == _ints("q")
    qm = O.quant_mask(_w_example(), 6, 8)
    acc, _ = O.fwd(q, a, qm["mcode"], qm["gamma"])
    assert int(acc[0, 0]) == _ints("acc_6_8")[0]


# ----------------------------------------------------------------------- ties and operation order

def test_hand_dequant_x_bf16():
    q = np.array([[int(t) for t in G["deq_q"]]], dtype=np.int8)
    a = np.array([float(G["deq_a"][0])], dtype=np.float32)
    got = O.dequant_x_bf16(q, a)
    assert got.ravel().tolist() == [float(t) for t in G["deq_x_bf16"]]
    # the bf16 operand is within half a bf16 step of the exact value it rounds
    exact = O.dequant_x(q, a)
    assert np.all(np.abs(got - exact) <= np.abs(exact) * 2.0 ** -8)


def test_hand_ternary_ties_round_to_even():
    """w/gamma exactly +-0.5 gives code 0 (ties to even), one ulp more gives 1, 1.5 clips."""
    g = np.float32(float(G["tie_gamma"][0]))
    half = np.float32(g / np.float32(2))                 # exact in fp32
    assert float(half) * 2 == float(g)
    w = np.array([half, -half, np.nextafter(half, np.float32(1)), np.float32(1.5) * g], dtype=np.float32)
    assert float(w[3] / g) == 1.5                        # the last ratio is exactly 1.5 as well
    assert O.ternary_codes(w, g).tolist() == _ints("tie_codes")


def _bf16_row(key):
    vals = np.array([float(t) for t in G[key]], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    assert np.array_equal(O.bf16_to_f32(bits), vals), "every value of the row is a bf16"
    return bits.reshape(1, -1)


def test_hand_act_quant_ties_round_to_even():
    q, a = O.act_quant(_bf16_row("tie_x"))
    assert float(a[0]) == 127.0
    assert q.ravel().tolist() == _ints("tie_q")


def test_hand_act_quant_scale_then_one_multiply():
    """Row B of the golden file: s = fp32(127/a) first, then one fp32 multiply. The other
    operation orders (x*127 first, or exact arithmetic) give 64 instead of 63."""
    row = _bf16_row("order_x")
    q, a = O.act_quant(row)
    assert float(a[0]) == 1.1875
    assert q.ravel().tolist() == _ints("order_q")
    # the worked intermediate values, exactly as rationals
    s = np.float32(np.float32(127) / np.float32(1.1875))
    assert Fraction(float(s)) == Fraction(14017805, 2 ** 17)
    assert Fraction(float(np.float32(np.float32(0.59375) * s))) == Fraction(16646143, 2 ** 18)
    assert Fraction(0.59375) * 127 / Fraction(1.1875) == Fraction(127, 2)


# ----------------------------------------------------------------------- gamma: exact rationals

def _exact_mean(w):
    tot = Fraction(0)
    for v in np.abs(w.astype(np.float32)).ravel().tolist():
        tot += Fraction(v)          # Fraction(float) is exact
    return tot / w.size


def test_gamma_within_truncation_bound_of_exact_mean():
    w = synth.latent_weight(11, 37, 64)
    g, mean, _ = O.absmean_gamma(w)
    exact = _exact_mean(w)
    ulp = Fraction(np.spacing(np.float32(mean)).item())
    # truncation costs < 2^-32 per element (so < 2^-32 on the mean); rounding < ulp/2
    assert abs(Fraction(float(mean)) - exact) <= Fraction(1, 2 ** 32) + ulp / 2
    assert g == np.float32(np.float32(mean) + np.float32(1e-5))


def test_gamma_exact_on_grid_values():
    # values on the 2^-32 grid are summed without truncation: the mean must then be
    # the correctly rounded exact mean (checked by enumerating neighbours)
    rng = np.random.default_rng(5)
    ints = rng.integers(0, 2 ** 24, size=999)   # 24-bit: exact in fp32
    w = (ints.astype(np.float64) * 2.0 ** -32).astype(np.float32)
    assert np.all(w.astype(np.float64) * 2 ** 32 == ints)
    _, mean, total = O.absmean_gamma(w.reshape(27, 37))
    exact = Fraction(int(ints.sum()), 999 * 2 ** 32)
    assert total == int(ints.sum())
    m = float(mean)
    lo, hi = float(np.nextafter(np.float32(m), np.float32(0))), float(np.nextafter(np.float32(m), np.float32(1)))
    d = abs(Fraction(m) - exact)
    assert d <= abs(Fraction(lo) - exact) and d <= abs(Fraction(hi) - exact)


def test_gamma_constant_tensor():
    w = np.full((4, 8), -0.375, dtype=np.float32)          # |w| exactly on the grid
    g, mean, _ = O.absmean_gamma(w)
    assert mean == np.float32(0.375)


def test_gamma_rejects_out_of_range():
    w = np.zeros((1, 8), np.float32)
    w[0, 3] = np.nan
    with pytest.raises(O.OracleRangeError):
        O.absmean_gamma(w)
    w[0, 3] = 70000.0
    with pytest.raises(O.OracleRangeError):
        O.absmean_gamma(w)


def test_rn_f32_ties_to_even():
    # 1 + 2^-24 is exactly half-way between 1 and 1 + 2^-23: ties go to even (1.0)
    assert O.rn_f32_from_rational(2 ** 24 + 1, 2 ** 24) == np.float32(1.0)
    # 1 + 3 * 2^-24 is half-way between 1+2^-23 and 1+2^-22: even is 1 + 2^-22
    assert O.rn_f32_from_rational(2 ** 24 + 3, 2 ** 24) == np.float32(1 + 2 ** -22)
    assert O.rn_f32_from_rational(1, 3) == np.float32(1.0 / 3.0)


# ----------------------------------------------------------------------- closed form

def test_gaussian_zero_fraction_closed_form():
    # iid N(0, s^2) weights: gamma ~ E|w| = s*sqrt(2/pi); code 0 iff |w| <= gamma/2,
    # so P(code = 0) = erf(0.5*sqrt(2/pi)/sqrt(2)) = erf(1/(2*sqrt(pi))) ~ 0.3101
    w = synth.latent_weight(2001, 896, 4864)
    qm = O.quant_mask(w, 8, 8)
    frac0 = float(np.mean(qm["code"] == 0))
    expect = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    assert abs(expect - 0.3101) < 1e-4
    assert abs(frac0 - expect) < 0.003


# ----------------------------------------------------------------------- mask invariants

def _tied_weights(seed, rows, k):
    # few distinct magnitudes: plenty of ties inside groups
    rng = np.random.default_rng(seed)
    mag = rng.integers(0, 4, size=(rows, k)).astype(np.float32) * np.float32(0.01)
    sign = np.where(rng.random((rows, k)) < 0.5, -1, 1).astype(np.float32)
    return mag * sign


def _brute_force_keep(group_abs, n):
    # among all N-subsets, the largest sum of |w|; among equal sums, the
    # lexicographically smallest index tuple
    best, best_sum = None, None
    for sub in combinations(range(len(group_abs)), n):
        s = sum(Fraction(float(group_abs[i])) for i in sub)
        if best is None or s > best_sum:
            best, best_sum = sub, s
    keep = [0] * len(group_abs)
    for i in best:
        keep[i] = 1
    return keep


@pytest.mark.parametrize("n,m", [(8, 8), (6, 8), (4, 8), (3, 8), (2, 8), (1, 8), (2, 4), (1, 4), (3, 4)])
def test_mask_brute_force_subsets(n, m):
    for seed, w in ((1, _tied_weights(1, 6, 32)), (2, synth.latent_weight(3, 6, 32))):
        keep = O.nm_keep(w, n, m)
        a = np.abs(w).reshape(-1, m)
        want = np.array([_brute_force_keep(g, n) for g in a]).reshape(w.shape)
        assert np.array_equal(keep.astype(int), want)


@pytest.mark.parametrize("n,m", [(6, 8), (4, 8), (2, 8), (2, 4)])
def test_mask_exactly_n_survivors(n, m):
    w = _tied_weights(7, 64, 256)
    keep = O.nm_keep(w, n, m)
    assert np.all(keep.reshape(-1, m).sum(axis=1) == n)


def test_mask_8_8_is_unmasked_bitnet():
    w = synth.latent_weight(9, 32, 128)
    qm = O.quant_mask(w, 8, 8)
    assert qm["keep"].all()
    assert np.array_equal(qm["mcode"], qm["code"])
    assert np.all(qm["mask"] == 0xFF)


def test_mask_nested_and_2_8_is_2_4_valid():
    w = _tied_weights(13, 16, 128)
    prev = None
    for n in range(1, 9):
        keep = O.nm_keep(w, n, 8)
        if prev is not None:
            assert np.all(keep >= prev)       # survivors of N are survivors of N+1
        prev = keep
    k28 = O.nm_keep(w, 2, 8).reshape(-1, 4)
    assert np.all(k28.sum(axis=1) <= 2)


def test_mask_ranks_latent_not_codes():
    # both weights quantise to +1, but the larger latent weight must win
    w = np.array([[0.30, 0.31, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0]], dtype=np.float32)
    qm = O.quant_mask(w, 1, 8)
    assert qm["code"][0, 0] == 1 and qm["code"][0, 1] == 1
    assert qm["keep"][0].tolist() == [False, True] + [False] * 6


def test_gamma_and_codes_independent_of_nm():
    # quantise-then-sparsify: the scale and the unmasked codes never see the mask
    w = synth.latent_weight(21, 16, 256)
    ref = O.quant_mask(w, 8, 8)
    for n, m in [(6, 8), (4, 8), (2, 8), (2, 4)]:
        qm = O.quant_mask(w, n, m)
        assert qm["gamma"] == ref["gamma"]
        assert np.array_equal(qm["code"], ref["code"])
        assert np.array_equal(qm["mcode"], np.where(qm["keep"], ref["code"], 0))


def test_mask_bytes_bit_layout():
    keep = np.zeros((1, 16), bool)
    keep[0, [0, 3, 9, 15]] = True
    assert O.mask_bytes(keep, 8).ravel().tolist() == [0b00001001, 0b10000010]
    assert O.mask_bytes(keep, 4).ravel().tolist() == [0b1001, 0, 0b0010, 0b1000]


def test_pack_unpack_brute_force():
    rng = np.random.default_rng(4)
    c = rng.integers(-1, 2, size=(3, 64)).astype(np.int8)
    p = O.pack_codes(c)
    for r in range(3):
        for k in range(64):
            field = (int(p[r, k // 4]) >> (2 * (k % 4))) & 3
            assert field == {0: 0, 1: 1, -1: 3}[int(c[r, k])]
    assert np.array_equal(O.unpack_codes(p), c)
    with pytest.raises(ValueError):
        O.unpack_codes(np.array([[0b10]], np.uint8))


# ----------------------------------------------------------------------- activation quantiser

def test_act_quant_invariants():
    x = synth.activation_bf16(31, 48, 256)
    q, a = O.act_quant(x)
    xf = O.bf16_to_f32(x).astype(np.float64)
    amax_idx = np.argmax(np.abs(xf), axis=1)
    for t in range(48):
        assert a[t] == np.max(np.abs(xf[t]))
        assert abs(int(q[t, amax_idx[t]])) == 127          # the absmax maps to +-127
    # reconstruction error of a round-to-nearest quantiser: at most half a step
    step = a.astype(np.float64)[:, None] / 127.0
    assert np.all(np.abs(q * step - xf) <= 0.5 * step * (1 + 1e-6))
    assert q.min() >= -127 and q.max() <= 127


def test_act_quant_scale_invariance_and_zero_row():
    x = synth.activation_bf16(32, 8, 64)
    x2 = synth.f32_to_bf16_bits(O.bf16_to_f32(x) * np.float32(2.0))   # exact doubling
    q1, a1 = O.act_quant(x)
    q2, a2 = O.act_quant(x2)
    assert np.array_equal(q1, q2) and np.array_equal(a2, 2 * a1)
    z = np.zeros((2, 64), np.uint16)
    qz, az = O.act_quant(z)
    assert np.all(qz == 0) and np.all(az == np.float32(1e-5))


# ----------------------------------------------------------------------- forward product

def test_fwd_brute_force_integer_matmul():
    for seed in range(4):
        t, k, n = 5 + seed, 64, 24
        x = synth.activation_bf16(100 + seed, t, k)
        w = synth.latent_weight(200 + seed, n, k)
        qm = O.quant_mask(w, 6, 8)
        q, a = O.act_quant(x)
        acc, _ = O.fwd(q, a, qm["mcode"], qm["gamma"])
        for i in range(t):
            for j in range(n):
                s = 0
                for kk in range(k):
                    s += int(q[i, kk]) * int(qm["mcode"][j, kk])
                assert acc[i, j] == s


def test_fwd_exact_on_quantisation_grid():
    # activations that are half-integers with absmax 63.5 quantise exactly (q = 2x),
    # so y must equal the plain product x . (gamma * masked codes)^T
    rng = np.random.default_rng(8)
    t, k, n = 6, 64, 16
    xv = rng.integers(-127, 128, size=(t, k)).astype(np.float32) * np.float32(0.5)
    xv[:, 0] = 63.5
    x = synth.f32_to_bf16_bits(xv)
    assert np.array_equal(O.bf16_to_f32(x), xv)
    w = synth.latent_weight(301, n, k)
    qm = O.quant_mask(w, 4, 8)
    q, a = O.act_quant(x)
    _, y = O.fwd(q, a, qm["mcode"], qm["gamma"])
    plain = xv.astype(np.float64) @ (float(qm["gamma"]) * qm["mcode"].astype(np.float64)).T
    assert np.allclose(y, plain, rtol=1e-13, atol=1e-13)


def test_fwd_8_8_sparse_equals_dense_masked_matrix():
    # the masked path equals a dense product against the masked ternary matrix
    x = synth.activation_bf16(41, 7, 128)
    w = synth.latent_weight(42, 32, 128)
    q, a = O.act_quant(x)
    for n, m in [(8, 8), (6, 8), (2, 4)]:
        qm = O.quant_mask(w, n, m)
        dense = np.where(qm["keep"], qm["code"], 0).astype(np.int64)
        acc, _ = O.fwd(q, a, qm["mcode"], qm["gamma"])
        assert np.array_equal(acc, q.astype(np.int64) @ dense.T)


# ----------------------------------------------------------------------- backward

def _loops_grad_x(dy, w_eff):
    t, n = dy.shape
    k = w_eff.shape[1]
    out = np.zeros((t, k))
    for i in range(t):
        for j in range(k):
            out[i, j] = math.fsum(dy[i, r] * w_eff[r, j] for r in range(n))
    return out


def _loops_grad_w(dy, x):
    t, n = dy.shape
    k = x.shape[1]
    out = np.zeros((n, k))
    for r in range(n):
        for j in range(k):
            out[r, j] = math.fsum(dy[i, r] * x[i, j] for i in range(t))
    return out


def test_grad_x_and_grad_w_brute_force():
    t, k, n = 6, 32, 16
    x = synth.activation_bf16(51, t, k)
    dy = synth.activation_bf16(52, t, n, std=1e-2, outliers=False)
    w = synth.latent_weight(53, n, k)
    qm = O.quant_mask(w, 6, 8)
    gx = O.grad_x(dy, qm["mcode"], qm["gamma"])
    gw = O.grad_w(dy, x)
    dyf = O.bf16_to_f32(dy).astype(np.float64)
    xf = O.bf16_to_f32(x).astype(np.float64)
    w_eff = float(qm["gamma"]) * np.where(qm["keep"], qm["code"], 0).astype(np.float64)
    assert np.allclose(gx, _loops_grad_x(dyf, w_eff), rtol=1e-12, atol=1e-15)
    assert np.allclose(gw, _loops_grad_w(dyf, xf), rtol=1e-12, atol=1e-15)


def test_straight_through_reaches_masked_weights():
    t, k, n = 16, 64, 8
    x = synth.activation_bf16(61, t, k)
    dy = synth.activation_bf16(62, t, n, std=1e-2, outliers=False)
    w = synth.latent_weight(63, n, k)
    qm = O.quant_mask(w, 2, 8)
    gw = O.grad_w(dy, x)
    dropped = ~qm["keep"]
    assert dropped.sum() > 0
    # masked positions carry the dense gradient, which is non-zero
    assert np.count_nonzero(gw[dropped]) == dropped.sum()
    # and grad_W never depends on the N:M choice (same dY, X)
    assert np.array_equal(gw, O.grad_w(dy, x))


def test_grad_x_8_8_equals_dense_bitnet():
    t, k, n = 4, 64, 16
    dy = synth.activation_bf16(71, t, n, std=1e-2, outliers=False)
    w = synth.latent_weight(72, n, k)
    dense = O.quant_mask(w, 8, 8)
    gx = O.grad_x(dy, dense["mcode"], dense["gamma"])
    unmasked = float(dense["gamma"]) * dense["code"].astype(np.float64)
    assert np.allclose(gx, O.bf16_to_f32(dy).astype(np.float64) @ unmasked, rtol=1e-13)


def test_grad_w_dequant_option_matches_forward_input():
    t, k, n = 5, 32, 8
    x = synth.activation_bf16(81, t, k)
    dy = synth.activation_bf16(82, t, n, std=1e-2, outliers=False)
    q, a = O.act_quant(x)
    xd = O.dequant_x(q, a)
    # dequantised activations sit within half a quantisation step of X
    assert np.all(np.abs(xd - O.bf16_to_f32(x)) <= 0.5 * a[:, None] / 127.0 * (1 + 1e-6))
    gw = O.grad_w(dy, x, x_deq=xd)
    assert np.allclose(gw, _loops_grad_w(O.bf16_to_f32(dy).astype(np.float64), xd), rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------------- threshold diagnostic


@pytest.mark.parametrize("n,m,key", [(6, 8, "6_8"), (4, 8, "4_8"), (2, 8, "2_8"), (2, 4, "2_4")])
def test_hand_threshold_hist(n, m, key):
    w = _w_example()
    qm = O.quant_mask(w, n, m)
    h = O.threshold_hist(w, qm["keep"], qm["gamma"], m)
    want = np.zeros(O.HIST_BINS, dtype=np.int64)
    for b in _ints(f"thr_bins_{key}"):
        want[b] += 1
    assert np.array_equal(h["hist"], want)
    assert h["dropped"] == _ints(f"thr_dropped_{key}")[0]
    assert h["dropped_core"] == _ints(f"thr_core_{key}")[0]


@pytest.mark.parametrize("n,m", [(6, 8), (4, 8), (3, 8), (2, 8), (2, 4), (1, 4)])
def test_threshold_is_the_next_largest_magnitude(n, m):
    # With ties, which tied weight is dropped changes nothing: the group threshold is
    # the (n+1)-th largest magnitude, found here by sorting, without the mask.
    w = _tied_weights(11, 6, 64)
    qm = O.quant_mask(w, n, m)
    h = O.threshold_hist(w, qm["keep"], qm["gamma"], m)
    a = np.sort(np.abs(w).astype(np.float64).reshape(-1, m), axis=1)[:, ::-1]
    thr = a[:, n]
    g = float(qm["gamma"])
    bins = np.array([min(16, sum(1 for k in range(1, 17) if 8.0 * t >= k * g)) for t in thr])
    assert np.array_equal(h["hist"], np.bincount(bins, minlength=O.HIST_BINS))
    groups = w.size // m
    assert h["hist"].sum() == groups and h["dropped"] == groups * (m - n)
    # dropped weights with a nonzero ternary code, counted from the codes themselves
    assert h["dropped_core"] == int(np.sum((qm["code"] != 0) & ~qm["keep"].astype(bool)))


def test_threshold_hist_8_8_is_empty():
    w = synth.latent_weight(5, 8, 64)
    qm = O.quant_mask(w, 8, 8)
    h = O.threshold_hist(w, qm["keep"], qm["gamma"], 8)
    assert h["hist"].sum() == 0 and h["dropped"] == 0 and h["dropped_core"] == 0


def test_threshold_hist_bin_edges_inclusive():
    # gamma = 1: a dropped magnitude of exactly k/8 opens bin k; one ulp below stays in k-1
    for k in range(1, 17):
        for val, want in ((np.float32(k / 8), k), (np.nextafter(np.float32(k / 8), np.float32(0)), k - 1)):
            w = np.array([[4.0, 4.0, 4.0, 4.0, 4.0, 4.0, val, 0.0]], dtype=np.float32)
            keep = np.array([[1, 1, 1, 1, 1, 1, 0, 0]], dtype=np.uint8)
            h = O.threshold_hist(w, keep, np.float32(1.0), 8)
            assert h["hist"][want] == 1, (k, float(val))


# ----------------------------------------------------------------------- int8-dY input gradient


def test_grad_x_int8_dy_brute_force():
    rng = np.random.default_rng(21)
    t, n, k = 3, 16, 8
    dy = synth.f32_to_bf16_bits(rng.standard_normal((t, n)).astype(np.float32) * 0.01)
    mcode = rng.integers(-1, 2, size=(n, k)).astype(np.int8)
    gamma = np.float32(0.0375)
    acc, y, q, a = O.grad_x_int8_dy(dy, mcode, gamma)
    for ti in range(t):
        for ki in range(k):
            s = 0
            for ni in range(n):
                s += int(q[ti, ni]) * int(mcode[ni, ki])
            assert acc[ti, ki] == s
            assert y[ti, ki] == pytest.approx(s * float(a[ti]) / 127.0 * float(gamma), rel=1e-15, abs=0)


def test_grad_x_int8_dy_exact_on_quantisation_grid():
    # dY = q * 2^-e with |q| <= 127 and a 127 in each row: quantisation is lossless, so
    # the integer path gives the exact input gradient
    rng = np.random.default_rng(22)
    t, n, k = 4, 64, 32
    q = rng.integers(-127, 128, size=(t, n))
    q[:, 0] = 127
    dy = synth.f32_to_bf16_bits((q * 2.0 ** -9).astype(np.float32))
    mcode = rng.integers(-1, 2, size=(n, k)).astype(np.int8)
    gamma = np.float32(0.02)
    _, y, qq, _ = O.grad_x_int8_dy(dy, mcode, gamma)
    assert np.array_equal(qq, q)
    assert np.allclose(y, O.grad_x(dy, mcode, gamma), rtol=1e-14, atol=0)


def test_grad_x_int8_dy_error_within_quantisation_bound():
    # each dY element moves by at most half a quantisation step a_t / 254 (plus the
    # fp32 product's rounding), so |error| <= sum_n |c[n,k]| * gamma * a_t / 254 * (1 + 1e-6)
    rng = np.random.default_rng(23)
    t, n, k = 8, 256, 64
    dy = synth.activation_bf16(31, t, n, std=1e-2, outliers=False)
    mcode = rng.integers(-1, 2, size=(n, k)).astype(np.int8)
    gamma = np.float32(0.03)
    _, y, _, a = O.grad_x_int8_dy(dy, mcode, gamma)
    exact = O.grad_x(dy, mcode, gamma)
    bound = (np.abs(mcode).sum(axis=0)[None, :] * float(gamma) * a.astype(np.float64)[:, None] / 254.0) * (1 + 1e-6)
    assert np.all(np.abs(y - exact) <= bound)
    assert np.max(np.abs(y - exact)) > 0   # the approximation is not exact in general


# ----------------------------------------------------------------------- 2:4 storage


def test_hand_compress_2_4():
    w = _w_example()
    qm = O.quant_mask(w, 2, 4)
    sp = O.compress_2_4(qm["mcode"], qm["keep"])
    assert sp["values"].ravel().tolist() == _ints("sp24_values")
    assert sp["meta"].ravel().tolist() == _ints("sp24_meta")


@pytest.mark.parametrize("n,m", [(2, 4), (1, 4), (2, 8), (1, 8)])
def test_compress_2_4_round_trip_and_valid_metadata(n, m):
    w = _tied_weights(13, 8, 128)
    qm = O.quant_mask(w, n, m)
    sp = O.compress_2_4(qm["mcode"], qm["keep"])
    assert np.array_equal(O.decompress_2_4(sp["values"], sp["meta"]), qm["mcode"])
    nibbles = np.concatenate([sp["meta"] & 0xF, sp["meta"] >> 4], axis=1).ravel()
    assert set(np.unique(nibbles).tolist()) <= {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}   # i0 < i1
    # the product over the stored form equals the product over the masked codes
    rng = np.random.default_rng(3)
    q = rng.integers(-128, 128, size=(5, 128)).astype(np.int8)
    dense = q.astype(np.int64) @ qm["mcode"].astype(np.int64).T
    k = 128
    g = np.arange(k // 4)
    acc = np.zeros((5, 8), dtype=np.int64)
    for r in range(8):
        for gi in g:
            for s_ in range(2):
                acc[:, r] += q[:, 4 * gi + sp["idx"][r, gi, s_]].astype(np.int64) * int(sp["values"][r, 2 * gi + s_])
    assert np.array_equal(acc, dense)


@pytest.mark.parametrize("n,m", [(6, 8), (4, 8), (3, 8), (3, 4)])
def test_compress_2_4_rejects_denser_masks(n, m):
    w = _tied_weights(14, 4, 64)
    qm = O.quant_mask(w, n, m)
    with pytest.raises(ValueError):
        O.compress_2_4(qm["mcode"], qm["keep"])


# ----------------------------------------------------------------------- optimizer step

def _rn_f32_exact(v: Fraction) -> float:
    """Nearest fp32 to the rational v (ties to the even significand), by comparing v
    with the candidates around fl64(v) in exact arithmetic (independent of the
    oracle's two-sum method)."""
    c = np.float32(float(v))
    cands = {float(c), float(np.nextafter(c, np.float32(np.inf))), float(np.nextafter(c, np.float32(-np.inf)))}
    best = None
    for x in sorted(cands):
        d = abs(Fraction(x) - v)
        even = (int(np.array(x, dtype=np.float32).view(np.uint32)) & 1) == 0
        key = (d, not even)
        if best is None or key < best[0]:
            best = (key, x)
    return best[1]


def test_hand_sgd_update_ties_and_sticky_error():
    """Golden rows sgd_*: plain SGD rounds W - lr*G once; cases 5 and 6 are a quarter
    fp64 ulp above an fp32 halfway point, where rounding an fp64 sum would tie to even."""
    w = np.array([float(t) for t in G["sgd_w"]], dtype=np.float32)
    g = synth.f32_to_bf16_bits(np.array([float(t) for t in G["sgd_g"]], dtype=np.float32))
    want = np.array([float(t) for t in G["sgd_w_new"]], dtype=np.float32)
    for i, lr in enumerate(float(t) for t in G["sgd_lr"]):
        got = O.sgd_update(w[i:i + 1], g[i:i + 1], lr)
        assert got[0] == want[i], (i, float(got[0]), float(want[i]))


def test_sgd_update_brute_force_exact_rationals():
    """Random W (magnitudes 2^-20 .. 2^10), bf16 G and fp32 lr, including exponent gaps
    wider than fp64 holds: the oracle equals the exactly rounded rational W - lr*G."""
    rng = np.random.default_rng(7)
    n = 4000
    w = (rng.standard_normal(n) * np.exp2(rng.integers(-20, 10, n))).astype(np.float32)
    gf = (rng.standard_normal(n) * np.exp2(rng.integers(-12, 6, n))).astype(np.float32)
    g = synth.f32_to_bf16_bits(gf)
    lrs = (np.exp2(rng.integers(-40, 0, n)) * rng.uniform(0.5, 1.0, n)).astype(np.float32)
    gv = O.bf16_to_f32(g)
    for i in range(n):
        got = O.sgd_update(w[i:i + 1], g[i:i + 1], float(lrs[i]))[0]
        exact = Fraction(float(w[i])) - Fraction(float(lrs[i])) * Fraction(float(gv[i]))
        assert float(got) == _rn_f32_exact(exact), (float(w[i]), float(lrs[i]), float(gv[i]))


def test_sgd_quant_mask_zero_step_is_quant_mask():
    """lr = 0 leaves W unchanged, so the fused step reduces to the plain mask/code step."""
    w = synth.latent_weight(3, 16, 64)
    g = synth.activation_bf16(4, 16, 64)
    a = O.sgd_quant_mask(w, g, 0.0, 6, 8)
    b = O.quant_mask(w, 6, 8)
    assert np.array_equal(a["w"], w)
    assert a["gamma"] == b["gamma"] and np.array_equal(a["codes_packed"], b["codes_packed"])
    assert np.array_equal(a["mask"], b["mask"])
