"""Helpers of the GPU parity tests: seeded inputs (via the generator module),
device transfer, and the comparison rules of the path.

Comparison rules:
  * masks, packed codes, int8 weights, int8 activations, absmax, gamma and int32
    accumulators: bit-exact.
  * fp32 outputs: |y - y_ref| <= 1e-5 * |y_ref| element by element (y_ref fp64).
  * bf16 outputs: within one bf16 ulp of the fp64 reference.
  * bf16 gradients: max |g - g_ref| / max |g_ref| <= 2e-2 (fp64 reference), and the
    same bound element by element with a floor of 1e-3 * max |g_ref|.
"""
from __future__ import annotations

import numpy as np
import torch

from sparsity_step_b200 import synth

GRAD_TOL = 2e-2
F32_RTOL = 1e-5


def dev():
    return torch.device("cuda", 0)


def f32_to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def bits_to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).to(dev()).view(torch.bfloat16)


def bf16_dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def layer_inputs(cfg: int, tensor: int, t: int, k_in: int, n_out: int, outliers: bool = True):
    """Latent W ~ N(0, 0.02^2) fp32, X ~ N(0,1) bf16 (+1% x20 outliers), dY ~ N(0, 1e-2^2)."""
    w = synth.latent_weight(synth.config_seed(cfg, 3 * tensor), n_out, k_in)
    x = synth.activation_bf16(synth.config_seed(cfg, 3 * tensor + 1), t, k_in, outliers=outliers)
    dy = synth.activation_bf16(synth.config_seed(cfg, 3 * tensor + 2), t, n_out, std=1e-2, outliers=False)
    return w, x, dy


def assert_exact(got: np.ndarray, want: np.ndarray, what: str):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {tuple(bad[0])}: {got[tuple(bad[0])]} != {want[tuple(bad[0])]}"


def assert_f32_close(got: np.ndarray, ref: np.ndarray, what: str):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    ok = err <= F32_RTOL * np.abs(ref)
    if not ok.all():
        i = tuple(np.argwhere(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} outside 1e-5 rel, first {i}: {got[i]} vs {ref[i]}")


def assert_bf16_within_ulp(got_bits: np.ndarray, ref: np.ndarray, what: str):
    got = bf16_bits_to_f64(got_bits)
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ulp = np.exp2(e - 7)                         # bf16 keeps 8 significant bits
    ok = np.where(a > 0, np.abs(got - ref) <= ulp, got == 0)
    if not ok.all():
        i = tuple(np.argwhere(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} beyond 1 bf16 ulp, first {i}: {got[i]} vs {ref[i]}")


def assert_grad_close(got_bits_or_f32: np.ndarray, ref: np.ndarray, what: str, is_bf16: bool = True):
    got = bf16_bits_to_f64(got_bits_or_f32) if is_bf16 else np.asarray(got_bits_or_f32, np.float64)
    scale = np.max(np.abs(ref))
    if scale == 0:
        assert np.all(got == 0), what
        return
    normwise = np.max(np.abs(got - ref)) / scale
    assert normwise <= GRAD_TOL, f"{what}: max relative error {normwise:.3e} > {GRAD_TOL}"
    elem = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-3 * scale)
    assert np.max(elem) <= GRAD_TOL, f"{what}: element relative error {np.max(elem):.3e} > {GRAD_TOL}"


def sample_rows(n: int, seed: int, count: int = 64) -> np.ndarray:
    """Rows spanning the first two and the last two 128-row tiles plus random ones."""
    rng = np.random.default_rng(seed)
    head = np.arange(min(n, 136))
    tail = np.arange(max(0, n - 136), n)
    mid = rng.integers(0, n, size=min(count, n))
    return np.unique(np.concatenate([head, tail, mid]))
