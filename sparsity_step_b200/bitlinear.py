"""Python binding of the BitLinear C ABI (include/bitlinear.h).

Argument marshalling only: each function checks dtypes, devices and contiguity,
allocates missing outputs with torch (device memory is PyTorch's job here), and
passes raw pointers plus a CUDA stream of the tensors' device (its current stream
unless one is given) to the library, with that device current. Every step of the
computation runs in the library's CUDA kernels; there is no other code path.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import BL_OUT_BF16, BL_OUT_F32, check, lib


def _call(fn, dev: torch.device, stream, *args) -> int:
    """One library call on the device that holds the tensors: the library works on the
    calling thread's current device, so that device is made current for the call, and
    the stream (last argument) is the given one or that device's current stream."""
    if stream is not None and stream.device != dev:
        raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
    if torch.cuda.current_device() == dev.index:   # the usual case: no device switch
        s = torch.cuda.current_stream(dev) if stream is None else stream
        return int(fn(*args, int(s.cuda_stream)))
    with torch.cuda.device(dev):
        s = torch.cuda.current_stream(dev) if stream is None else stream
        return int(fn(*args, int(s.cuda_stream)))


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _need(t, dtype, shape, name, device=None):
    """Check one caller buffer before its pointer goes to the library (the C ABI
    cannot see buffer sizes, so an undersized or mistyped buffer must stop here)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _need_vec(t, dtype, min_numel, name, device=None):
    """A contiguous buffer of at least ``min_numel`` elements (per-token or scalar data)."""
    _need(t, dtype, None, name, device)
    if t.numel() < min_numel:
        raise ValueError(f"{name}: needs at least {min_numel} elements, got {t.numel()}")
    return t


def _need_bytes(t, nbytes, name, device=None):
    """A contiguous uint8 workspace of at least ``nbytes`` bytes."""
    return _need_vec(t, torch.uint8, nbytes, name, device)


def sp_meta_shape(n_out: int, k_in: int) -> tuple[int, int]:
    """Shape of the padded 2:4 metadata: rows and logical K rounded up to 256."""
    return (n_out + 255) // 256 * 256, (k_in + 255) // 256 * 256 // 8


def _check_qm_outputs(o: dict, n_out: int, k_in: int, m_group: int, dev) -> None:
    _need(o["codes"], torch.uint8, (n_out, k_in // 4), "codes", dev)
    _need_vec(o["w_scale"], torch.float32, 1, "w_scale", dev)
    if o.get("mask") is not None:
        _need(o["mask"], torch.uint8, (n_out, k_in // m_group), "mask", dev)
    if o.get("w_i8") is not None:
        _need(o["w_i8"], torch.int8, (n_out, k_in), "w_i8", dev)
    if o.get("sp_values") is not None or o.get("sp_meta") is not None:
        _need(o["sp_values"], torch.int8, (n_out, k_in // 2), "sp_values", dev)
        _need(o["sp_meta"], torch.uint8, sp_meta_shape(n_out, k_in), "sp_meta", dev)


def bitlinear_quant_mask_workspace_size(n_out: int, k_in: int) -> int:
    return int(lib().bitlinear_quant_mask_workspace_size(n_out, k_in))


def bitlinear_quant_mask(w: torch.Tensor, n_keep: int, m_group: int, *, want_mask: bool = True,
                         want_w_i8: bool = True, want_sp: bool = False, out: dict | None = None,
                         workspace: torch.Tensor | None = None, stream=None) -> dict:
    """Mask, gamma and masked ternary codes of latent weights w [n_out, k_in] (fp32).

    Returns a dict with ``codes`` (uint8 [n_out, k_in/4]), ``w_scale`` (fp32 [1]),
    and optionally ``mask`` (uint8 [n_out, k_in/m]), ``w_i8`` (int8 [n_out, k_in]) and,
    for masks with at most two kept per aligned four (``want_sp``), the 2:4 form
    ``sp_values`` (int8 [n_out, k_in/2]) and ``sp_meta`` (uint8, padded: ``sp_meta_shape``).
    """
    n_out, k_in = w.shape
    _need(w, torch.float32, None, "w")
    dev = w.device
    o = dict(out or {})
    if "codes" not in o:
        o["codes"] = torch.empty((n_out, k_in // 4), dtype=torch.uint8, device=dev)
    if "w_scale" not in o:
        o["w_scale"] = torch.empty((4,), dtype=torch.float32, device=dev)[:1]
    if want_mask and "mask" not in o:
        o["mask"] = torch.empty((n_out, k_in // m_group), dtype=torch.uint8, device=dev)
    if want_w_i8 and "w_i8" not in o:
        o["w_i8"] = torch.empty((n_out, k_in), dtype=torch.int8, device=dev)
    if want_sp and "sp_values" not in o:
        o["sp_values"] = torch.empty((n_out, k_in // 2), dtype=torch.int8, device=dev)
        o["sp_meta"] = torch.empty(sp_meta_shape(n_out, k_in), dtype=torch.uint8, device=dev)
    if m_group not in (4, 8) or k_in % m_group:
        raise ValueError(f"m_group must be 4 or 8 and divide k_in (got {m_group})")
    _check_qm_outputs(o, n_out, k_in, m_group, dev)
    ws_bytes = bitlinear_quant_mask_workspace_size(n_out, k_in)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _need_bytes(workspace, ws_bytes, "workspace", dev)
    st = _call(lib().bitlinear_quant_mask, dev, stream, _ptr(w), n_out, k_in, n_keep, m_group, _ptr(o.get("mask")),
               _ptr(o["codes"]), _ptr(o.get("w_i8")), _ptr(o.get("sp_values")), _ptr(o.get("sp_meta")),
               _ptr(o["w_scale"]), _ptr(workspace), workspace.numel())
    check(st, "bitlinear_quant_mask")
    o["workspace"] = workspace
    return o


def bitlinear_sgd_quant_mask(w: torch.Tensor, grad_w: torch.Tensor, lr: float, n_keep: int, m_group: int, *,
                             want_mask: bool = True, want_w_i8: bool = True, want_sp: bool = False,
                             out: dict | None = None, workspace: torch.Tensor | None = None, stream=None) -> dict:
    """One SGD step on the latent weights fused with the mask/code recompute:
    w <- fp32(w - lr * grad_w) in place (grad_w bf16 [n_out, k_in]), then the outputs of
    ``bitlinear_quant_mask`` for the updated w."""
    n_out, k_in = w.shape
    _need(w, torch.float32, None, "w")
    _need(grad_w, torch.bfloat16, (n_out, k_in), "grad_w", w.device)
    dev = w.device
    o = dict(out or {})
    if "codes" not in o:
        o["codes"] = torch.empty((n_out, k_in // 4), dtype=torch.uint8, device=dev)
    if "w_scale" not in o:
        o["w_scale"] = torch.empty((4,), dtype=torch.float32, device=dev)[:1]
    if want_mask and "mask" not in o:
        o["mask"] = torch.empty((n_out, k_in // m_group), dtype=torch.uint8, device=dev)
    if want_w_i8 and "w_i8" not in o:
        o["w_i8"] = torch.empty((n_out, k_in), dtype=torch.int8, device=dev)
    if want_sp and "sp_values" not in o:
        o["sp_values"] = torch.empty((n_out, k_in // 2), dtype=torch.int8, device=dev)
        o["sp_meta"] = torch.empty(sp_meta_shape(n_out, k_in), dtype=torch.uint8, device=dev)
    if m_group not in (4, 8) or k_in % m_group:
        raise ValueError(f"m_group must be 4 or 8 and divide k_in (got {m_group})")
    _check_qm_outputs(o, n_out, k_in, m_group, dev)
    ws_bytes = bitlinear_quant_mask_workspace_size(n_out, k_in)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _need_bytes(workspace, ws_bytes, "workspace", dev)
    st = _call(lib().bitlinear_sgd_quant_mask, dev, stream, _ptr(w), _ptr(grad_w), float(lr), n_out, k_in, n_keep,
               m_group, _ptr(o.get("mask")), _ptr(o["codes"]), _ptr(o.get("w_i8")), _ptr(o.get("sp_values")),
               _ptr(o.get("sp_meta")), _ptr(o["w_scale"]), _ptr(workspace), workspace.numel())
    check(st, "bitlinear_sgd_quant_mask")
    o["workspace"] = workspace
    return o


def bitlinear_quant_mask_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the range status (0 or BL_ERR_RANGE = -4); no raise."""
    _need(workspace, torch.uint8, None, "workspace")
    return _call(lib().bitlinear_quant_mask_status, workspace.device, stream, _ptr(workspace))


def bitlinear_quant_mask_noalloc(w: torch.Tensor, n_keep: int, m_group: int, *, out: dict, stream=None) -> dict:
    """bitlinear_quant_mask with no workspace and no allocation inside the library.

    For callers that cannot allocate device memory: every output buffer comes in
    ``out`` (``codes``, ``w_scale``, and optionally ``mask`` and ``w_i8``); the
    library's built-in scratch array is used instead of a workspace. Calls that
    overlap on the GPU share that array and race; a range error gives gamma = NaN.
    """
    n_out, k_in = w.shape
    _need(w, torch.float32, None, "w")
    if m_group not in (4, 8) or k_in % m_group:
        raise ValueError(f"m_group must be 4 or 8 and divide k_in (got {m_group})")
    _check_qm_outputs(out, n_out, k_in, m_group, w.device)
    st = _call(lib().bitlinear_quant_mask_noalloc, w.device, stream, _ptr(w), n_out, k_in, n_keep, m_group,
               _ptr(out.get("mask")), _ptr(out["codes"]), _ptr(out.get("w_i8")), _ptr(out["w_scale"]))
    check(st, "bitlinear_quant_mask_noalloc")
    return out


def bitlinear_act_quant(x: torch.Tensor, *, xq: torch.Tensor | None = None, absmax: torch.Tensor | None = None,
                        stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """int8 activations and per-token absmax of x [t, k_in] (bf16)."""
    t, k_in = x.shape
    _need(x, torch.bfloat16, None, "x")
    if xq is None:
        xq = torch.empty((t, k_in), dtype=torch.int8, device=x.device)
    if absmax is None:
        absmax = torch.empty((max(t, 1) + 3) // 4 * 4, dtype=torch.float32, device=x.device)[:t]
    _need(xq, torch.int8, (t, k_in), "xq", x.device)
    _need_vec(absmax, torch.float32, t, "absmax", x.device)
    st = _call(lib().bitlinear_act_quant, x.device, stream, _ptr(x), t, k_in, _ptr(xq), _ptr(absmax))
    check(st, "bitlinear_act_quant")
    return xq, absmax


def bitlinear_fwd(xq: torch.Tensor, absmax: torch.Tensor, w_scale: torch.Tensor, *, codes: torch.Tensor | None = None,
                  w_i8: torch.Tensor | None = None, sp_values: torch.Tensor | None = None,
                  sp_meta: torch.Tensor | None = None, n_out: int | None = None, y_dtype=torch.bfloat16,
                  want_acc: bool = False, y: torch.Tensor | None = None, acc: torch.Tensor | None = None,
                  stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
    """y = (xq . masked_codes^T) * absmax/127 * gamma; returns (y, acc or None).

    Weight operand: the 2:4 form (``sp_values`` + ``sp_meta``, sparse tensor cores),
    else ``w_i8`` (dense tensor cores), else ``codes`` (2-bit codes decoded on chip).
    With both the 2:4 form and ``w_i8`` the library picks per shape."""
    t, k_in = xq.shape
    dev = xq.device
    _need(xq, torch.int8, None, "xq")
    if w_i8 is None and codes is None and sp_values is None:
        raise ValueError("give codes, w_i8 or sp_values + sp_meta")
    if (sp_values is None) != (sp_meta is None):
        raise ValueError("give both sp_values and sp_meta, or neither")
    if n_out is None:
        n_out = (sp_values if sp_values is not None else w_i8 if w_i8 is not None else codes).shape[0]
    if sp_values is not None:
        _need(sp_values, torch.int8, (n_out, k_in // 2), "sp_values", dev)
        _need(sp_meta, torch.uint8, sp_meta_shape(n_out, k_in), "sp_meta", dev)
    if codes is not None:
        _need(codes, torch.uint8, (n_out, k_in // 4), "codes", dev)
    if w_i8 is not None:
        _need(w_i8, torch.int8, (n_out, k_in), "w_i8", dev)
    _need_vec(absmax, torch.float32, t, "absmax", dev)
    _need_vec(w_scale, torch.float32, 1, "w_scale", dev)
    if y is None:
        y = torch.empty((t, n_out), dtype=y_dtype, device=dev)
    if y.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError(f"y: expected bfloat16 or float32, got {y.dtype}")
    _need(y, y.dtype, (t, n_out), "y", dev)
    if want_acc and acc is None:
        acc = torch.empty((t, n_out), dtype=torch.int32, device=dev)
    if acc is not None:
        _need(acc, torch.int32, (t, n_out), "acc", dev)
    ydt = BL_OUT_F32 if y.dtype == torch.float32 else BL_OUT_BF16
    st = _call(lib().bitlinear_fwd, dev, stream, _ptr(xq), _ptr(absmax), _ptr(codes), _ptr(w_i8), _ptr(sp_values),
               _ptr(sp_meta), _ptr(w_scale), t, k_in, n_out, _ptr(acc), _ptr(y), ydt)
    check(st, "bitlinear_fwd")
    return y, acc


def bitlinear_fwd_grouped(problems: list[dict], *, y_dtype=torch.bfloat16, stream=None) -> list[dict]:
    """Forward product of several independent problems in one launch (codes operand).

    Each problem is a dict with ``xq``, ``absmax``, ``codes``, ``w_scale`` and
    optionally ``y``, ``acc`` (outputs allocated here when missing, ``want_acc`` to
    request the int32 accumulators). Returns the dicts with ``y`` (and ``acc``) set.
    """
    if not problems:
        return []
    arr = (_lib.BlFwdProblem * len(problems))()
    out = []
    dev = problems[0]["xq"].device
    for i, p in enumerate(problems):
        xq, codes = p["xq"], p["codes"]
        _need(xq, torch.int8, None, f"problem {i} xq", dev)
        t, k_in = xq.shape
        n_out = codes.shape[0]
        _need(codes, torch.uint8, (n_out, k_in // 4), f"problem {i} codes", dev)
        _need_vec(p["absmax"], torch.float32, t, f"problem {i} absmax", dev)
        _need_vec(p["w_scale"], torch.float32, 1, f"problem {i} w_scale", dev)
        y = p.get("y")
        if y is None:
            y = torch.empty((t, n_out), dtype=y_dtype, device=dev)
        _need(y, y_dtype, (t, n_out), f"problem {i} y", dev)
        acc = p.get("acc")
        if acc is None and p.get("want_acc"):
            acc = torch.empty((t, n_out), dtype=torch.int32, device=dev)
        if acc is not None:
            _need(acc, torch.int32, (t, n_out), f"problem {i} acc", dev)
        arr[i] = _lib.BlFwdProblem(_ptr(xq), _ptr(p["absmax"]), _ptr(codes), _ptr(p["w_scale"]), t, k_in, n_out,
                                   _ptr(acc), _ptr(y))
        out.append({**p, "y": y, "acc": acc})
    ydt = BL_OUT_F32 if y_dtype == torch.float32 else BL_OUT_BF16
    st = _call(lib().bitlinear_fwd_grouped, dev, stream, arr, len(problems), ydt)
    check(st, "bitlinear_fwd_grouped")
    return out


def bitlinear_grad_w_grouped(problems: list[dict], *, grad_w_dtype=torch.bfloat16, stream=None) -> list[torch.Tensor]:
    """grad_W = dY^T X of several linears over the same tokens in one launch.

    Each problem is a dict with ``dy`` (bf16 [t, n_out]), ``x`` (bf16 [t, k_in]) and
    optionally ``grad_w`` (allocated here when missing). Returns the grad_w tensors.
    """
    if not 1 <= len(problems) <= 4:
        raise ValueError("1 to 4 problems")
    arr = (_lib.BlGradWProblem * len(problems))()
    out = []
    t = problems[0]["dy"].shape[0]
    dev = problems[0]["dy"].device
    for i, p in enumerate(problems):
        dy, x = p["dy"], p["x"]
        _need(dy, torch.bfloat16, None, f"problem {i} dy", dev)
        n_out = dy.shape[1]
        if dy.shape[0] != t:
            raise ValueError(f"problem {i}: every problem needs the same token count ({t})")
        _need(x, torch.bfloat16, (t, x.shape[1]), f"problem {i} x", dev)
        k_in = x.shape[1]
        gw = p.get("grad_w")
        if gw is None:
            gw = torch.empty((n_out, k_in), dtype=grad_w_dtype, device=dev)
        _need(gw, grad_w_dtype, (n_out, k_in), f"problem {i} grad_w", dev)
        arr[i] = _lib.BlGradWProblem(_ptr(dy), _ptr(x), k_in, n_out, _ptr(gw),
                                     BL_OUT_F32 if grad_w_dtype == torch.float32 else BL_OUT_BF16)
        out.append(gw)
    st = _call(lib().bitlinear_grad_w_grouped, dev, stream, arr, len(problems), t)
    check(st, "bitlinear_grad_w_grouped")
    return out


BL_GRADW_DEQUANT_X = 1   # grad_W against the dequantised activations q * a / 127


def bitlinear_bwd_workspace_size(t: int, k_in: int, n_out: int, want_grad_x: bool = True, flags: int = 0) -> int:
    return int(lib().bitlinear_bwd_workspace_size(t, k_in, n_out, int(want_grad_x), int(flags)))


def bitlinear_bwd(dy: torch.Tensor, x: torch.Tensor | None, codes: torch.Tensor | None, w_scale: torch.Tensor | None, *,
                  want_grad_x: bool = True, want_grad_w: bool = True, grad_w_dtype=torch.bfloat16,
                  grad_x: torch.Tensor | None = None, grad_w: torch.Tensor | None = None,
                  workspace: torch.Tensor | None = None, k_in: int | None = None,
                  xq: torch.Tensor | None = None, absmax: torch.Tensor | None = None, flags: int = 0,
                  stream=None) -> tuple[torch.Tensor | None, torch.Tensor | None]:
    """Dual straight-through backward; returns (grad_x or None, grad_w or None).

    ``flags = BL_GRADW_DEQUANT_X`` computes grad_w against q * a / 127 (``xq`` and
    ``absmax`` from bitlinear_act_quant) instead of the bf16 input ``x``.
    """
    t, n_out = dy.shape
    _need(dy, torch.bfloat16, None, "dy")
    dev = dy.device
    deq = bool(flags & BL_GRADW_DEQUANT_X)
    if k_in is None:
        k_in = (xq.shape[1] if deq and xq is not None else
                x.shape[1] if x is not None else codes.shape[1] * 4)
    if want_grad_x and grad_x is None:
        grad_x = torch.empty((t, k_in), dtype=torch.bfloat16, device=dev)
    if want_grad_w and grad_w is None:
        grad_w = torch.empty((n_out, k_in), dtype=grad_w_dtype, device=dev)
    if grad_x is not None:
        _need(grad_x, torch.bfloat16, (t, k_in), "grad_x", dev)
        if codes is None or w_scale is None:
            raise ValueError("grad_x needs codes and w_scale")
    if codes is not None:
        _need(codes, torch.uint8, (n_out, k_in // 4), "codes", dev)
    if w_scale is not None:
        _need_vec(w_scale, torch.float32, 1, "w_scale", dev)
    if grad_w is not None:
        if grad_w.dtype not in (torch.bfloat16, torch.float32):
            raise TypeError(f"grad_w: expected bfloat16 or float32, got {grad_w.dtype}")
        _need(grad_w, grad_w.dtype, (n_out, k_in), "grad_w", dev)
        if deq:
            if xq is None or absmax is None:
                raise ValueError("BL_GRADW_DEQUANT_X needs xq and absmax")
            _need(xq, torch.int8, (t, k_in), "xq", dev)
            _need_vec(absmax, torch.float32, t, "absmax", dev)
        elif x is not None:
            _need(x, torch.bfloat16, (t, k_in), "x", dev)
    gwdt = BL_OUT_F32 if (grad_w is not None and grad_w.dtype == torch.float32) else BL_OUT_BF16
    need = bitlinear_bwd_workspace_size(t, k_in, n_out, grad_x is not None, flags if grad_w is not None else 0)
    if need and workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need_bytes(workspace, need, "workspace", dev)
    st = _call(lib().bitlinear_bwd, dev, stream, _ptr(dy), _ptr(x), _ptr(xq), _ptr(absmax), _ptr(codes),
               _ptr(w_scale), t, k_in, n_out, _ptr(grad_x), _ptr(grad_w), gwdt, int(flags), _ptr(workspace),
               0 if workspace is None else workspace.numel())
    check(st, "bitlinear_bwd")
    return grad_x, grad_w


def bitlinear_grad_x_i8_workspace_size(t: int, k_in: int, n_out: int) -> int:
    return int(lib().bitlinear_grad_x_i8_workspace_size(t, k_in, n_out))


def bitlinear_grad_x_i8(dy: torch.Tensor, codes: torch.Tensor, w_scale: torch.Tensor, *, k_in: int | None = None,
                        grad_x: torch.Tensor | None = None, want_acc: bool = False,
                        workspace: torch.Tensor | None = None, stream=None) -> dict:
    """Input gradient with dY quantised per token to int8 (an approximation); returns
    {"grad_x", "acc" (or None)}."""
    t, n_out = dy.shape
    _need(dy, torch.bfloat16, None, "dy")
    dev = dy.device
    if k_in is None:
        k_in = codes.shape[1] * 4
    _need(codes, torch.uint8, (n_out, k_in // 4), "codes", dev)
    if grad_x is None:
        grad_x = torch.empty((t, k_in), dtype=torch.bfloat16, device=dev)
    _need(grad_x, torch.bfloat16, (t, k_in), "grad_x", dev)
    acc = torch.empty((t, k_in), dtype=torch.int32, device=dev) if want_acc else None
    _need_vec(w_scale, torch.float32, 1, "w_scale", dev)
    need = bitlinear_grad_x_i8_workspace_size(t, k_in, n_out)
    if workspace is None and need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need_bytes(workspace, need, "workspace", dev)
    st = _call(lib().bitlinear_grad_x_i8, dev, stream, _ptr(dy), _ptr(codes), _ptr(w_scale), t, k_in, n_out,
               _ptr(grad_x), _ptr(acc), _ptr(workspace), 0 if workspace is None else workspace.numel())
    check(st, "bitlinear_grad_x_i8")
    return {"grad_x": grad_x, "acc": acc}


def bitlinear_mask_threshold_hist(w: torch.Tensor, mask: torch.Tensor, w_scale: torch.Tensor, m_group: int, *,
                                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Threshold-decoupling histogram: int64 [19] = 17 bins of max dropped |w| / gamma
    (width 1/8, last bin >= 2), dropped weights, dropped weights with a nonzero code."""
    n_out, k_in = w.shape
    _need(w, torch.float32, None, "w")
    if m_group not in (4, 8):
        raise ValueError("m_group must be 4 or 8")
    _need(mask, torch.uint8, (n_out, k_in // m_group), "mask", w.device)
    _need_vec(w_scale, torch.float32, 1, "w_scale", w.device)
    if out is None:
        out = torch.empty((19,), dtype=torch.int64, device=w.device)
    _need(out, torch.int64, (19,), "out", w.device)
    st = _call(lib().bitlinear_mask_threshold_hist, w.device, stream, _ptr(w), _ptr(mask), _ptr(w_scale), n_out,
               k_in, m_group, _ptr(out))
    check(st, "bitlinear_mask_threshold_hist")
    return out


def bitlinear_device_status() -> tuple[int, int]:
    """(status, bits): synchronise the current device and read/clear the library's timeout bits."""
    bits = ctypes.c_uint(0)
    st = lib().bitlinear_device_status(ctypes.byref(bits))
    return int(st), int(bits.value)


def bitlinear_abi_version() -> int:
    return int(lib().bitlinear_abi_version())


__all__ = [
    "bitlinear_quant_mask_workspace_size", "bitlinear_quant_mask", "bitlinear_quant_mask_status",
    "bitlinear_quant_mask_noalloc",
    "bitlinear_act_quant", "bitlinear_fwd", "bitlinear_fwd_grouped", "bitlinear_bwd_workspace_size", "bitlinear_bwd",
    "bitlinear_grad_x_i8_workspace_size", "bitlinear_grad_x_i8", "bitlinear_mask_threshold_hist", "sp_meta_shape",
    "bitlinear_device_status", "bitlinear_abi_version", "BL_OUT_BF16", "BL_OUT_F32", "BL_GRADW_DEQUANT_X", "_lib",
]
