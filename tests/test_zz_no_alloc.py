"""The no-allocation variant of the mask/ternary-code entry point.

bitlinear_quant_mask_noalloc serves callers that cannot allocate device memory
(a host framework that owns all device memory, or a path where cudaMalloc may not
block the device); it keeps its scratch in an array built into the library. This
file runs last so that a failure here leaves every other test already run.
"""
import numpy as np
import pytest
import torch

import sparsity_step_b200 as B
from oracle import bitlinear_oracle as O
from sparsity_step_b200 import synth

pytestmark = pytest.mark.gpu


def _outputs(n_out, k_in, m_group, dev):
    return {
        "codes": torch.empty((n_out, k_in // 4), dtype=torch.uint8, device=dev),
        "mask": torch.empty((n_out, k_in // m_group), dtype=torch.uint8, device=dev),
        "w_i8": torch.empty((n_out, k_in), dtype=torch.int8, device=dev),
        "w_scale": torch.empty((4,), dtype=torch.float32, device=dev)[:1],
    }


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    dev = torch.device("cuda", 0)
    cases = [(11008, 2048, 6, 8, 401), (896, 896, 2, 4, 402)]
    for n_out, k_in, n, m, seed in cases:   # two calls in a row share the built-in scratch
        w = torch.from_numpy(synth.latent_weight(seed, n_out, k_in)).to(dev)
        ref = B.bitlinear_quant_mask(w, n, m)
        got = B.bitlinear_quant_mask_noalloc(w, n, m, out=_outputs(n_out, k_in, m, dev))
        torch.cuda.synchronize()
        assert B.bitlinear_quant_mask_status(ref["workspace"]) == 0
        # the integer outputs and gamma are bit-exact in both entry points
        for key in ("codes", "mask", "w_i8"):
            assert torch.equal(got[key], ref[key]), key
        assert np.array_equal(got["w_scale"].cpu().numpy().view(np.uint32), ref["w_scale"].cpu().numpy().view(np.uint32))
        # and directly against the oracle
        want = O.quant_mask(w.cpu().numpy(), n, m)
        assert np.array_equal(got["codes"].cpu().numpy(), want["codes_packed"])
        assert np.array_equal(got["mask"].cpu().numpy(), want["mask"])
        assert got["w_scale"].cpu().numpy()[0] == want["gamma"]


def test_noalloc_range_error_then_clean_call():
    """A non-finite weight gives gamma = NaN and all-zero codes; the next call on clean
    weights is bit-exact again (the last block of each call resets the shared flag and
    ticket in the built-in scratch)."""
    dev = torch.device("cuda", 0)
    n_out, k_in = 256, 896
    w_np = synth.latent_weight(403, n_out, k_in)
    bad = w_np.copy()
    bad[7, 100] = np.inf
    out = _outputs(n_out, k_in, 8, dev)
    B.bitlinear_quant_mask_noalloc(torch.from_numpy(bad).to(dev), 6, 8, out=out)
    torch.cuda.synchronize()
    assert np.isnan(out["w_scale"].cpu().numpy()[0])
    assert int(out["codes"].count_nonzero().item()) == 0
    w = torch.from_numpy(w_np).to(dev)
    got = B.bitlinear_quant_mask_noalloc(w, 6, 8, out=_outputs(n_out, k_in, 8, dev))
    ref = B.bitlinear_quant_mask(w, 6, 8)
    torch.cuda.synchronize()
    for key in ("codes", "mask", "w_i8"):
        assert torch.equal(got[key], ref[key]), key
    assert got["w_scale"].cpu().numpy()[0] == O.quant_mask(w_np, 6, 8)["gamma"]


def test_noalloc_rejects_oversize_tensor():
    dev = torch.device("cuda", 0)
    w = torch.empty((16, 64), dtype=torch.float32, device=dev)
    out = _outputs(16, 64, 8, dev)
    lib = B._lib.lib()
    # 2^20 x 8192 weights exceed the built-in scratch: rejected before any launch
    st = lib.bitlinear_quant_mask_noalloc(w.data_ptr(), 1 << 20, 8192, 6, 8, None, out["codes"].data_ptr(), None,
                                          out["w_scale"].data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == -2
    assert "scratch" in lib.bitlinear_last_error().decode()
