"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument validation rejects bad calls before anything is enqueued (CPU only: no
call here reaches a CUDA API)."""
import ctypes

import pytest

from sparsity_step_b200 import _lib
from sparsity_step_b200.build import build

BAD = 0x1001          # a misaligned fake device address (never dereferenced)
GOOD = 0x10000        # an aligned fake device address (never dereferenced)


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def test_exports_every_header_function(L):
    names = _lib.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.SIGNATURES)


def test_abi_version(L):
    assert L.bitlinear_abi_version() == 2


def _err(L):
    return L.bitlinear_last_error().decode()


def test_quant_mask_validation(L):
    ws = L.bitlinear_quant_mask_workspace_size(896, 896)
    assert ws >= 256 + 16
    # null latent weights
    assert L.bitlinear_quant_mask(None, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
    # bad N:M
    for n, m in [(0, 8), (9, 8), (2, 3), (6, 16)]:
        assert L.bitlinear_quant_mask(GOOD, 896, 896, n, m, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
    # unsupported shapes
    assert L.bitlinear_quant_mask(GOOD, 896, 900, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -2
    assert L.bitlinear_quant_mask(GOOD, 8, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -2
    # workspace
    assert L.bitlinear_quant_mask(GOOD, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, None, ws, None) == -7
    assert L.bitlinear_quant_mask(GOOD, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws - 1, None) == -7
    # the 2:4 outputs: both or neither, and only for masks with at most two kept per four
    assert L.bitlinear_quant_mask(GOOD, 896, 896, 2, 4, GOOD, GOOD, GOOD, GOOD, None, GOOD, GOOD, ws, None) == -1
    assert L.bitlinear_quant_mask(GOOD, 896, 896, 6, 8, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, ws, None) == -1
    assert "2:4" in _err(L)
    assert L.bitlinear_quant_mask(GOOD, 896, 896, 2, 8, GOOD, GOOD, GOOD, BAD, GOOD, GOOD, GOOD, ws, None) == -3
    # alignment
    assert L.bitlinear_quant_mask(BAD, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -3
    assert "aligned" in _err(L)


def test_sgd_quant_mask_validation(L):
    ws = L.bitlinear_quant_mask_workspace_size(896, 896)
    call = L.bitlinear_sgd_quant_mask
    # the gradient and a finite learning rate are required
    assert call(GOOD, None, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
    for lr in (float("nan"), float("inf")):
        assert call(GOOD, GOOD, lr, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
        assert "lr" in _err(L)
    assert call(GOOD, BAD, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -3
    # then the checks of bitlinear_quant_mask
    assert call(None, GOOD, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
    assert call(GOOD, GOOD, 1e-3, 896, 896, 9, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -1
    assert call(GOOD, GOOD, 1e-3, 896, 900, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -2
    assert call(GOOD, GOOD, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws - 1, None) == -7
    assert call(GOOD, GOOD, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, ws, None) == -1
    assert call(BAD, GOOD, 1e-3, 896, 896, 6, 8, GOOD, GOOD, GOOD, None, None, GOOD, GOOD, ws, None) == -3


def test_grad_w_grouped_validation(L):
    def arr(*probs):
        a = (_lib.BlGradWProblem * max(1, len(probs)))()
        for i, p in enumerate(probs):
            a[i] = _lib.BlGradWProblem(*p)
        return a
    good = (GOOD, GOOD, 2048, 11008, GOOD, 0)
    call = L.bitlinear_grad_w_grouped
    assert call(None, 1, 4096, None) == -1
    assert call(arr(good), 0, 4096, None) == -1
    assert call(arr(good, good, good, good, good), 5, 4096, None) == -1
    assert call(arr(good, (GOOD, GOOD, 2048, 11008, None, 0)), 2, 4096, None) == -1   # no output
    assert call(arr(good, (None, GOOD, 2048, 11008, GOOD, 0)), 2, 4096, None) == -1   # no dY
    assert call(arr(good, (GOOD, GOOD, 2048, 11008, GOOD, 7)), 2, 4096, None) == -1   # output dtype
    assert call(arr(good, (GOOD, GOOD, 2000, 11008, GOOD, 0)), 2, 4096, None) == -2   # k_in % 64
    assert call(arr(good, (GOOD, BAD, 2048, 11008, GOOD, 0)), 2, 4096, None) == -3    # alignment


def test_quant_mask_noalloc_validation(L):
    assert L.bitlinear_quant_mask_noalloc(None, 896, 896, 6, 8, GOOD, GOOD, GOOD, GOOD, None) == -1
    assert L.bitlinear_quant_mask_noalloc(GOOD, 896, 896, 9, 8, GOOD, GOOD, GOOD, GOOD, None) == -1
    assert L.bitlinear_quant_mask_noalloc(GOOD, 896, 900, 6, 8, GOOD, GOOD, GOOD, GOOD, None) == -2
    # beyond the built-in scratch (1184 block partials): rejected on the host
    assert L.bitlinear_quant_mask_noalloc(GOOD, 1 << 20, 8192, 6, 8, None, GOOD, None, GOOD, None) == -2
    assert "scratch" in _err(L)
    assert L.bitlinear_quant_mask_noalloc(BAD, 896, 896, 6, 8, GOOD, GOOD, GOOD, GOOD, None) == -3


def test_act_quant_validation(L):
    assert L.bitlinear_act_quant(None, 4, 896, GOOD, GOOD, None) == -1
    assert L.bitlinear_act_quant(GOOD, 4, 100, GOOD, GOOD, None) == -2
    assert L.bitlinear_act_quant(GOOD, -1, 896, GOOD, GOOD, None) == -2
    assert L.bitlinear_act_quant(GOOD, 4, 896, BAD, GOOD, None) == -3
    # an empty batch is valid and enqueues nothing
    assert L.bitlinear_act_quant(GOOD, 0, 896, GOOD, GOOD, None) == 0


def test_fwd_validation(L):
    args = dict(xq=GOOD, a=GOOD, codes=GOOD, wi8=GOOD, g=GOOD)
    #                      xq    absmax codes w_i8  spv   spm   w_scale t  k_in n_out acc  y   dtype stream
    assert L.bitlinear_fwd(GOOD, GOOD, None, None, None, None, GOOD, 4, 896, 896, None, GOOD, 0, None) == -1
    assert L.bitlinear_fwd(GOOD, GOOD, GOOD, GOOD, None, None, GOOD, 4, 896, 896, None, GOOD, 7, None) == -1
    assert L.bitlinear_fwd(GOOD, GOOD, GOOD, GOOD, None, None, GOOD, 4, 896, 100, None, GOOD, 0, None) == -2
    assert L.bitlinear_fwd(GOOD, GOOD, GOOD, GOOD, None, None, GOOD, 4, 896, 896, BAD, GOOD, 0, None) == -3
    assert L.bitlinear_fwd(GOOD, GOOD, GOOD, GOOD, None, None, GOOD, 0, 896, 896, None, GOOD, 0, None) == 0
    # the 2:4 operand: both parts or neither, 16-byte aligned
    assert L.bitlinear_fwd(GOOD, GOOD, None, None, GOOD, None, GOOD, 4, 896, 896, None, GOOD, 0, None) == -1
    assert L.bitlinear_fwd(GOOD, GOOD, None, None, GOOD, BAD, GOOD, 4, 896, 896, None, GOOD, 0, None) == -3
    assert L.bitlinear_fwd(GOOD, GOOD, None, None, GOOD, GOOD, GOOD, 0, 896, 896, None, GOOD, 0, None) == 0
    del args


def test_fwd_grouped_validation(L):
    P = _lib.BlFwdProblem
    arr = (P * 2)(P(GOOD, GOOD, GOOD, GOOD, 4, 896, 896, None, GOOD), P(GOOD, GOOD, GOOD, GOOD, 1, 2048, 256, None, GOOD))
    assert L.bitlinear_fwd_grouped(None, 1, 0, None) == -1
    assert L.bitlinear_fwd_grouped(arr, 257, 0, None) == -2
    assert L.bitlinear_fwd_grouped(arr, 2, 5, None) == -1
    arr[1].k_in = 100
    assert L.bitlinear_fwd_grouped(arr, 2, 0, None) == -2
    assert _err(L).startswith("problem 1: k_in=100")   # the shape message kept inside the problem's
    arr[1].k_in = 2048
    arr[1].codes = None
    assert L.bitlinear_fwd_grouped(arr, 2, 0, None) == -1
    arr[1].codes = BAD
    assert L.bitlinear_fwd_grouped(arr, 2, 0, None) == -3
    # empty problems enqueue nothing
    arr[0].t = 0
    arr[1].t = 0
    arr[1].codes = GOOD
    assert L.bitlinear_fwd_grouped(arr, 2, 0, None) == 0
    assert L.bitlinear_fwd_grouped(arr, 0, 0, None) == 0


def test_bwd_validation(L):
    need = L.bitlinear_bwd_workspace_size(16, 896, 896, 1, 0)
    assert need == 896 * 896 * 2
    assert L.bitlinear_bwd_workspace_size(16, 896, 896, 0, 0) == 0
    # the dequantised-X option adds a bf16 [t, k_in] buffer after the ternary matrix
    assert L.bitlinear_bwd_workspace_size(16, 896, 896, 1, 1) == 896 * 896 * 2 + 16 * 896 * 2
    assert L.bitlinear_bwd_workspace_size(16, 896, 896, 0, 1) == 16 * 896 * 2
    #        dy    x     xq    absmax codes w_scale t  k_in n_out gx gw dtype flags ws  bytes stream
    # nothing requested
    assert L.bitlinear_bwd(GOOD, GOOD, None, None, GOOD, GOOD, 16, 896, 896, None, None, 0, 0, GOOD, need, None) == -1
    # grad_x without codes
    assert L.bitlinear_bwd(GOOD, GOOD, None, None, None, GOOD, 16, 896, 896, GOOD, None, 0, 0, GOOD, need, None) == -1
    # workspace too small for grad_x
    assert L.bitlinear_bwd(GOOD, GOOD, None, None, GOOD, GOOD, 16, 896, 896, GOOD, None, 0, 0, GOOD, need - 16,
                           None) == -7
    # grad_w only needs no workspace; bad dtype is rejected
    assert L.bitlinear_bwd(GOOD, GOOD, None, None, None, None, 16, 896, 896, None, GOOD, 3, 0, None, 0, None) == -1
    assert L.bitlinear_bwd(GOOD, BAD, None, None, None, None, 16, 896, 896, None, GOOD, 0, 0, None, 0, None) == -3
    # unknown flag bits
    assert L.bitlinear_bwd(GOOD, GOOD, None, None, None, None, 16, 896, 896, None, GOOD, 0, 2, None, 0, None) == -1
    assert "flags" in _err(L)
    # the dequantised-X option needs xq and absmax (x is not needed) and its workspace
    deq = L.bitlinear_bwd_workspace_size(16, 896, 896, 0, 1)
    assert L.bitlinear_bwd(GOOD, None, None, GOOD, None, None, 16, 896, 896, None, GOOD, 0, 1, GOOD, deq, None) == -1
    assert L.bitlinear_bwd(GOOD, None, GOOD, None, None, None, 16, 896, 896, None, GOOD, 0, 1, GOOD, deq, None) == -1
    assert L.bitlinear_bwd(GOOD, None, GOOD, GOOD, None, None, 16, 896, 896, None, GOOD, 0, 1, GOOD, deq - 16,
                           None) == -7
    assert L.bitlinear_bwd(GOOD, None, BAD, GOOD, None, None, 16, 896, 896, None, GOOD, 0, 1, GOOD, deq, None) == -3


def test_grad_x_i8_validation(L):
    need = L.bitlinear_grad_x_i8_workspace_size(16, 896, 2048)
    assert need == 16 * 2048 + 256 + 896 * 2048
    assert L.bitlinear_grad_x_i8_workspace_size(0, 896, 2048) == 0
    # n_out must be a multiple of 64 on this path
    assert L.bitlinear_grad_x_i8(GOOD, GOOD, GOOD, 16, 896, 144, GOOD, None, GOOD, 1 << 30, None) == -2
    # codes / w_scale required; workspace checked
    assert L.bitlinear_grad_x_i8(GOOD, None, GOOD, 16, 896, 2048, GOOD, None, GOOD, need, None) == -1
    assert L.bitlinear_grad_x_i8(GOOD, GOOD, GOOD, 16, 896, 2048, GOOD, None, GOOD, need - 16, None) == -7
    assert L.bitlinear_grad_x_i8(GOOD, GOOD, GOOD, 16, 896, 2048, BAD, None, GOOD, need, None) == -3
    # empty batch: nothing to do, the t-sized arrays may be NULL
    assert L.bitlinear_grad_x_i8(None, GOOD, GOOD, 0, 896, 2048, None, None, None, 0, None) == 0


def test_mask_threshold_hist_validation(L):
    assert L.bitlinear_mask_threshold_hist(GOOD, GOOD, GOOD, 896, 896, 6, GOOD, None) == -1
    assert L.bitlinear_mask_threshold_hist(None, GOOD, GOOD, 896, 896, 8, GOOD, None) == -1
    assert L.bitlinear_mask_threshold_hist(GOOD, GOOD, GOOD, 896, 100, 8, GOOD, None) == -2
    assert L.bitlinear_mask_threshold_hist(GOOD, GOOD, GOOD, 896, 896, 8, BAD, None) == -3


def test_last_error_is_thread_local_message(L):
    assert L.bitlinear_act_quant(None, 4, 896, GOOD, GOOD, None) == -1
    assert "required" in _err(L)
    assert L.bitlinear_act_quant(GOOD, 0, 896, GOOD, GOOD, None) == 0
    assert _err(L) == ""


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_LIB", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        _lib.lib()


def test_ctypes_signatures_match_header_arity():
    import re
    with open(_lib.HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    for name, (_, args) in _lib.SIGNATURES.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", text)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), name
    assert ctypes.sizeof(ctypes.c_size_t) == 8


def test_binding_calls_on_the_tensors_device(monkeypatch):
    """Every library call runs with the tensors' device current and that device's stream
    as its last argument; a stream of another device is refused before the call."""
    import contextlib

    import torch

    from sparsity_step_b200 import bitlinear as B

    made_current, asked = [], []

    @contextlib.contextmanager
    def fake_device(dev):
        made_current.append(dev)
        yield

    class FakeStream:
        def __init__(self, dev, handle):
            self.device, self.cuda_stream = dev, handle

    def fake_current_stream(dev=None):
        asked.append(dev)
        return FakeStream(dev, 0x5000 + dev.index)

    current = [0]
    monkeypatch.setattr(torch.cuda, "device", fake_device)
    monkeypatch.setattr(torch.cuda, "current_stream", fake_current_stream)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: current[0])
    seen = []
    fn = lambda *a: seen.append(a) or 0   # noqa: E731
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    # tensors on another device than the current one: switched for the call
    assert B._call(fn, d1, None, 7, 8) == 0
    assert made_current == [d1] and asked == [d1] and seen == [(7, 8, 0x5001)]
    assert B._call(fn, d1, FakeStream(d1, 0x77), 9) == 0
    assert seen[-1] == (9, 0x77)
    with pytest.raises(ValueError, match="stream is on"):
        B._call(fn, d1, FakeStream(d0, 0x66), 9)
    assert len(seen) == 2 and made_current == [d1, d1]
    # tensors on the current device: no switch, that device's stream
    assert B._call(fn, d0, None, 5) == 0
    assert seen[-1] == (5, 0x5000) and made_current == [d1, d1] and asked[-1] == d0


def test_binding_checks_buffers_before_the_library():
    """Host tensors, wrong dtypes and missing operands are refused in Python, before any
    pointer reaches the library (no CUDA call is made)."""
    import torch

    from sparsity_step_b200 import bitlinear as B

    w = torch.zeros((16, 64), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.bitlinear_quant_mask(w, 6, 8)
    with pytest.raises(TypeError, match="float32"):
        B.bitlinear_quant_mask(w.double(), 6, 8)
    with pytest.raises(TypeError, match="bfloat16"):
        B.bitlinear_act_quant(torch.zeros((4, 64), dtype=torch.float16))
    xq = torch.zeros((4, 64), dtype=torch.int8)
    a = torch.ones(4)
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.bitlinear_fwd(xq, a, torch.ones(1), w_i8=torch.zeros((16, 64), dtype=torch.int8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        B.bitlinear_fwd(xq, a, torch.ones(1))   # the dtype/device check of xq comes first
    with pytest.raises(ValueError, match="1 to 4"):
        B.bitlinear_grad_w_grouped([])
    assert B.bitlinear_fwd_grouped([]) == []
    with pytest.raises(TypeError, match="torch.Tensor"):
        B._need([1, 2], torch.int8, None, "x")
