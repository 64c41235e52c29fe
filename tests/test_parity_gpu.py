"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on seeded
inputs of every workload shape (full outputs where the oracle is quick, sampled
rows at full launch sizes) and on the edge cases of the method."""
import numpy as np
import pytest
import torch

import sparsity_step_b200 as B
from oracle import bitlinear_oracle as O
from parity_util import (assert_bf16_within_ulp, assert_exact, assert_f32_close, assert_grad_close, bf16_bits_to_f64,
                         bf16_dev_to_bits, bits_to_dev_bf16, f32_to_dev, layer_inputs, sample_rows)
from sparsity_step_b200 import synth

pytestmark = pytest.mark.gpu

# ------------------------------------------------------------------ shared checks


def gpu_quant_mask(w_np, n, m):
    # masks with at most two kept per aligned four also get their 2:4 form
    out = B.bitlinear_quant_mask(f32_to_dev(w_np), n, m, want_sp=n <= 2)
    torch.cuda.synchronize()
    assert B.bitlinear_quant_mask_status(out["workspace"]) == 0
    return out


def check_quant_mask(out, ref, tag, sp_rows=None, has_mask=True):
    g = out["w_scale"].cpu().numpy()[:1]
    assert_exact(g.view(np.uint32), np.array([ref["gamma"]], np.float32).view(np.uint32), f"{tag} gamma")
    if has_mask:
        assert_exact(out["mask"].cpu().numpy(), ref["mask"], f"{tag} mask")
    else:
        assert "mask" not in out, f"{tag}: a mask came back unasked"
    assert_exact(out["codes"].cpu().numpy(), ref["codes_packed"], f"{tag} codes")
    assert_exact(out["w_i8"].cpu().numpy(), ref["mcode"], f"{tag} w_i8")
    if "sp_values" in out:
        # the oracle's 2:4 storage is pure-Python loops: sampled rows on large tensors
        rows = np.arange(ref["mcode"].shape[0]) if sp_rows is None else sp_rows
        want = O.compress_2_4(ref["mcode"][rows], ref["keep"][rows])
        n_out, k_in = ref["mcode"].shape
        meta = out["sp_meta"].cpu().numpy()
        assert meta.shape == B.sp_meta_shape(n_out, k_in)
        assert_exact(out["sp_values"].cpu().numpy()[rows], want["values"], f"{tag} 2:4 values")
        assert_exact(meta[rows, :k_in // 8], want["meta"], f"{tag} 2:4 metadata")
        # padding rows and columns: positions 0 and 1 in every group
        assert np.all(meta[:, k_in // 8:] == 0x44) and np.all(meta[n_out:, :] == 0x44), f"{tag} metadata padding"


def gpu_act_quant(x_bits):
    xq, a = B.bitlinear_act_quant(bits_to_dev_bf16(x_bits))
    torch.cuda.synchronize()
    return xq, a


def check_act_quant(xq, a, ref_q, ref_a, tag):
    assert_exact(xq.cpu().numpy(), ref_q, f"{tag} xq")
    assert_exact(a.cpu().numpy().view(np.uint32), ref_a.astype(np.float32).view(np.uint32), f"{tag} absmax")


def check_fwd(qm_dev, xq, a, ref_qm, ref_q, ref_a, tag, rows=None, paths=("w_i8",), f32=True):
    """Forward on both requested weight operands; compares acc (exact), bf16 and f32 y."""
    acc_ref, y_ref = O.fwd(ref_q, ref_a, ref_qm["mcode"], ref_qm["gamma"], rows=rows)
    for path in paths:
        kw = ({"w_i8": qm_dev["w_i8"]} if path == "w_i8" else
              {"sp_values": qm_dev["sp_values"], "sp_meta": qm_dev["sp_meta"]} if path == "sp" else
              {"codes": qm_dev["codes"]})
        y, acc = B.bitlinear_fwd(xq, a, qm_dev["w_scale"], n_out=ref_qm["mcode"].shape[0], want_acc=True, **kw)
        torch.cuda.synchronize()
        acc_np = acc.cpu().numpy()
        ybits = bf16_dev_to_bits(y)
        if rows is not None:
            acc_np, ybits = acc_np[rows], ybits[rows]
        assert_exact(acc_np, acc_ref, f"{tag} acc [{path}]")
        assert_bf16_within_ulp(ybits, y_ref, f"{tag} y bf16 [{path}]")
        # without the int32 output the tensor-core path stores y through TMA
        y2, _ = B.bitlinear_fwd(xq, a, qm_dev["w_scale"], n_out=ref_qm["mcode"].shape[0], **kw)
        torch.cuda.synchronize()
        y2bits = bf16_dev_to_bits(y2)
        assert_bf16_within_ulp(y2bits if rows is None else y2bits[rows], y_ref, f"{tag} y bf16 no-acc [{path}]")
        if f32:
            y32, _ = B.bitlinear_fwd(xq, a, qm_dev["w_scale"], n_out=ref_qm["mcode"].shape[0], y_dtype=torch.float32, **kw)
            torch.cuda.synchronize()
            y32 = y32.cpu().numpy()
            if rows is not None:
                y32 = y32[rows]
            assert_f32_close(y32, y_ref, f"{tag} y f32 [{path}]")


def check_bwd(dy_bits, x_bits, qm_dev, ref_qm, tag, rows_t=None, rows_n=None, gw_f32=False):
    dy = bits_to_dev_bf16(dy_bits)
    x = bits_to_dev_bf16(x_bits)
    gx, gw = B.bitlinear_bwd(dy, x, qm_dev["codes"], qm_dev["w_scale"],
                             grad_w_dtype=torch.float32 if gw_f32 else torch.bfloat16)
    torch.cuda.synchronize()
    gx_ref = O.grad_x(dy_bits, ref_qm["mcode"], ref_qm["gamma"], rows=rows_t)
    gw_ref = O.grad_w(dy_bits, x_bits, rows=rows_n)
    gxb = bf16_dev_to_bits(gx)
    assert_grad_close(gxb if rows_t is None else gxb[rows_t], gx_ref, f"{tag} grad_x")
    if gw_f32:
        g = gw.cpu().numpy()
        assert_grad_close(g if rows_n is None else g[rows_n], gw_ref, f"{tag} grad_w f32", is_bf16=False)
    else:
        g = bf16_dev_to_bits(gw)
        assert_grad_close(g if rows_n is None else g[rows_n], gw_ref, f"{tag} grad_w")


def full_layer(cfg, tensor, t, k_in, n_out, n, m, *, outliers=True, bwd=True, paths=("w_i8", "codes"), sample=False):
    w, x, dy = layer_inputs(cfg, tensor, t, k_in, n_out, outliers=outliers)
    tag = f"cfg{cfg} t{tensor} [{t}x{k_in}->{n_out}] {n}:{m}"
    ref_qm = O.quant_mask(w, n, m)
    qm = gpu_quant_mask(w, n, m)
    check_quant_mask(qm, ref_qm, tag, sp_rows=sample_rows(n_out, tensor + 3) if sample else None)
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    check_act_quant(xq, a, ref_q, ref_a, tag)
    rows = sample_rows(t, tensor) if sample else None
    check_fwd(qm, xq, a, ref_qm, ref_q, ref_a, tag, rows=rows, paths=paths)
    if bwd:
        check_bwd(dy, x, qm, ref_qm, tag, rows_t=rows, rows_n=sample_rows(n_out, tensor + 7) if sample else None)


# ------------------------------------------------------------------ the five workloads


def test_config1_single_layer_full():
    """X 64x896 bf16 N(0,1) + 1% x20, W 896x896 N(0,0.02), 6:8, seed 0: every output."""
    full_layer(1, 0, 64, 896, 896, 6, 8)


QWEN05 = [("q", 896, 896), ("k", 896, 128), ("v", 896, 128), ("o", 896, 896),
          ("gate", 896, 4864), ("up", 896, 4864), ("down", 4864, 896)]


@pytest.mark.parametrize("idx", range(len(QWEN05)), ids=[s[0] for s in QWEN05])
def test_config2_qwen05_linears(idx):
    _, k_in, n_out = QWEN05[idx]
    full_layer(2, idx, 4096, k_in, n_out, 6, 8, bwd=False, paths=("w_i8",))


QWEN15_MLP = [("gate", 1536, 8960), ("up", 1536, 8960), ("down", 8960, 1536)]


@pytest.mark.parametrize("nm", [(8, 8), (6, 8), (4, 8), (3, 8), (2, 4), (2, 8)], ids=lambda v: f"{v[0]}of{v[1]}")
@pytest.mark.parametrize("idx", range(3), ids=[s[0] for s in QWEN15_MLP])
def test_config3_nm_sweep(idx, nm):
    _, k_in, n_out = QWEN15_MLP[idx]
    # 2:4-valid masks also run on the sparse tensor cores
    paths = ("w_i8", "sp") if nm[0] <= 2 else ("w_i8",)
    full_layer(3, idx, 8192, k_in, n_out, nm[0], nm[1], outliers=False, bwd=False, paths=paths, sample=True)


@pytest.mark.parametrize("nm", [(2, 4), (2, 8)], ids=lambda v: f"{v[0]}of{v[1]}")
@pytest.mark.parametrize("idx", range(len(QWEN05)), ids=[s[0] for s in QWEN05])
def test_config2_qwen05_linears_sparse_24(idx, nm):
    """The Qwen2.5-0.5B linears at 4096 tokens on the sparse tensor cores (k/v: 128
    weight rows, so the second CTA of every pair tile is past the output)."""
    _, k_in, n_out = QWEN05[idx]
    full_layer(2, 20 + idx, 4096, k_in, n_out, nm[0], nm[1], bwd=False, paths=("sp",), sample=True)


@pytest.mark.parametrize("nm", [(2, 4), (2, 8), (1, 4), (1, 8)], ids=lambda v: f"{v[0]}of{v[1]}")
@pytest.mark.parametrize("t,k_in,n_out", [(1, 128, 128), (100, 640, 896), (224, 896, 272), (225, 1536, 256),
                                          (500, 384, 528), (449, 11008, 144)])
def test_sparse_24_ragged(t, k_in, n_out, nm):
    """Ragged tokens (tile of 224), K (stages of 256 logical: 640, 896, 384 end on half
    or quarter stages), and weight rows (pair tiles of 256) on the sparse product."""
    full_layer(1, 60 + t, t, k_in, n_out, nm[0], nm[1], bwd=False, paths=("sp", "w_i8"))


@pytest.mark.parametrize("t,k_in,n_out", [(300, 896, 896), (8192, 1536, 8960)])
def test_sparse_or_dense_picked_per_shape(t, k_in, n_out):
    """With both the 2:4 form and the int8 weights, the library picks the product per
    shape (dense below 100 GOP, sparse above); either way the accumulators are exact."""
    w, x, _ = layer_inputs(3, 90 + n_out % 7, t, k_in, n_out, outliers=False)
    ref_qm = O.quant_mask(w, 2, 4)
    qm = gpu_quant_mask(w, 2, 4)
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    rows = sample_rows(t, 3)
    acc_ref, y_ref = O.fwd(ref_q, ref_a, ref_qm["mcode"], ref_qm["gamma"], rows=rows)
    y, acc = B.bitlinear_fwd(xq, a, qm["w_scale"], w_i8=qm["w_i8"], sp_values=qm["sp_values"], sp_meta=qm["sp_meta"],
                             want_acc=True)
    y2, _ = B.bitlinear_fwd(xq, a, qm["w_scale"], w_i8=qm["w_i8"], sp_values=qm["sp_values"], sp_meta=qm["sp_meta"])
    torch.cuda.synchronize()
    assert_exact(acc.cpu().numpy()[rows], acc_ref, "acc (picked product)")
    assert_bf16_within_ulp(bf16_dev_to_bits(y)[rows], y_ref, "y (picked product)")
    assert_bf16_within_ulp(bf16_dev_to_bits(y2)[rows], y_ref, "y (picked product, TMA-store epilogue)")


def test_sparse_24_storage_matches_oracle_with_ties():
    """2:4 storage of masks built on tied magnitudes and all-zero groups."""
    rng = np.random.default_rng(11)
    mag = rng.integers(0, 3, size=(48, 256)).astype(np.float32) * np.float32(0.01)
    w = (mag * np.where(rng.random((48, 256)) < 0.5, -1, 1)).astype(np.float32)
    w[0, :8] = 0.0
    for n, m in [(2, 4), (2, 8), (1, 4), (1, 8)]:
        check_quant_mask(gpu_quant_mask(w, n, m), O.quant_mask(w, n, m), f"ties {n}:{m}")


QWEN3B_MLP = [("gate", 2048, 11008), ("up", 2048, 11008), ("down", 11008, 2048)]


@pytest.mark.parametrize("idx", range(3), ids=[s[0] for s in QWEN3B_MLP])
def test_config4_training_step(idx):
    _, k_in, n_out = QWEN3B_MLP[idx]
    full_layer(4, idx, 16384, k_in, n_out, 6, 8, bwd=True, paths=("w_i8",), sample=True)


@pytest.mark.parametrize("f32", [False, True], ids=["bf16", "f32"])
@pytest.mark.parametrize("shapes,t", [([(896, 4864), (896, 4864), (4864, 896)], 1000),
                                      ([(640, 400), (576, 272)], 257),
                                      ([(256, 1536), (896, 128), (128, 384)], 300),
                                      ([(512, 768)], 129)],
                         ids=["mlp-0.5b", "ragged", "with-narrow", "single"])
def test_grad_w_grouped(shapes, t, f32):
    """Several grad_W products in one launch (tiles of all products scheduled together;
    a group with an output of <= 128 rows runs one product at a time): each against the
    oracle's dY^T X."""
    probs, refs = [], []
    for i, (k_in, n_out) in enumerate(shapes):
        x = synth.activation_bf16(300 + i, t, k_in)
        dy = synth.activation_bf16(310 + i, t, n_out, std=1e-2, outliers=False)
        probs.append({"dy": bits_to_dev_bf16(dy), "x": bits_to_dev_bf16(x)})
        refs.append(O.grad_w(dy, x))
    gws = B.bitlinear_grad_w_grouped(probs, grad_w_dtype=torch.float32 if f32 else torch.bfloat16)
    torch.cuda.synchronize()
    for i, (gw, ref) in enumerate(zip(gws, refs)):
        if f32:
            assert_grad_close(gw.cpu().numpy(), ref, f"grouped grad_w {i} f32", is_bf16=False)
        else:
            assert_grad_close(bf16_dev_to_bits(gw), ref, f"grouped grad_w {i}")


def test_grad_w_grouped_training_shape():
    """The three grad_W of the 3B MLP over 16384 tokens in one launch (the bench step's
    call), sampled rows against the oracle."""
    t = 16384
    probs, ins = [], []
    for i, (_, k_in, n_out) in enumerate(QWEN3B_MLP):
        x = synth.activation_bf16(320 + i, t, k_in)
        dy = synth.activation_bf16(330 + i, t, n_out, std=1e-2, outliers=False)
        probs.append({"dy": bits_to_dev_bf16(dy), "x": bits_to_dev_bf16(x)})
        ins.append((dy, x, n_out))
    gws = B.bitlinear_grad_w_grouped(probs)
    torch.cuda.synchronize()
    for i, (gw, (dy, x, n_out)) in enumerate(zip(gws, ins)):
        rows = sample_rows(n_out, 40 + i)
        assert_grad_close(bf16_dev_to_bits(gw)[rows], O.grad_w(dy, x, rows=rows), f"grouped grad_w {i}")


QWEN3B_LAYER = [("q", 2048, 2048), ("k", 2048, 256), ("v", 2048, 256), ("o", 2048, 2048),
                ("gate", 2048, 11008), ("up", 2048, 11008), ("down", 11008, 2048)]


@pytest.mark.parametrize("layer", [0, 35])
@pytest.mark.parametrize("idx", range(len(QWEN3B_LAYER)), ids=[s[0] for s in QWEN3B_LAYER])
def test_config5_decode_batches(idx, layer):
    _, k_in, n_out = QWEN3B_LAYER[idx]
    w = synth.latent_weight(synth.config_seed(5, 100 * layer + idx), n_out, k_in)
    ref_qm = O.quant_mask(w, 6, 8)
    qm = gpu_quant_mask(w, 6, 8)
    check_quant_mask(qm, ref_qm, f"cfg5 L{layer} {QWEN3B_LAYER[idx][0]}")
    for b in (1, 8, 32, 128):
        x = synth.activation_bf16(synth.config_seed(5, 5000 + 10 * idx + b), b, k_in, outliers=False)
        ref_q, ref_a = O.act_quant(x)
        xq, a = gpu_act_quant(x)
        check_act_quant(xq, a, ref_q, ref_a, f"cfg5 b{b}")
        check_fwd(qm, xq, a, ref_qm, ref_q, ref_a, f"cfg5 L{layer} {QWEN3B_LAYER[idx][0]} b{b}", paths=("w_i8", "codes"),
                  f32=(b == 8))


@pytest.mark.parametrize("b", [1, 2, 3, 8, 12, 16, 32, 128])
def test_config5_grouped_layer(b):
    """All seven linears of one layer in one grouped launch, mixed shapes."""
    probs, refs = [], []
    for idx, (_, k_in, n_out) in enumerate(QWEN3B_LAYER):
        w = synth.latent_weight(synth.config_seed(5, 300 + idx), n_out, k_in)
        x = synth.activation_bf16(synth.config_seed(5, 400 + idx + b), b, k_in, outliers=False)
        ref_qm = O.quant_mask(w, 6, 8)
        qm = gpu_quant_mask(w, 6, 8)
        ref_q, ref_a = O.act_quant(x)
        xq, a = gpu_act_quant(x)
        probs.append({"xq": xq, "absmax": a, "codes": qm["codes"], "w_scale": qm["w_scale"], "want_acc": True})
        refs.append(O.fwd(ref_q, ref_a, ref_qm["mcode"], ref_qm["gamma"]))
    out = B.bitlinear_fwd_grouped(probs)
    torch.cuda.synchronize()
    for (acc_ref, y_ref), o, (name, _, _) in zip(refs, out, QWEN3B_LAYER):
        assert_exact(o["acc"].cpu().numpy(), acc_ref, f"grouped b{b} {name} acc")
        assert_bf16_within_ulp(bf16_dev_to_bits(o["y"]), y_ref, f"grouped b{b} {name} y")


@pytest.mark.parametrize("idx", [0, 6], ids=["q", "down"])
def test_config5_prefill_8192(idx):
    _, k_in, n_out = QWEN3B_LAYER[idx]
    w = synth.latent_weight(synth.config_seed(5, idx), n_out, k_in)
    x = synth.activation_bf16(synth.config_seed(5, 7000 + idx), 8192, k_in, outliers=False)
    ref_qm = O.quant_mask(w, 6, 8)
    qm = gpu_quant_mask(w, 6, 8)
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    check_act_quant(xq, a, ref_q, ref_a, "cfg5 prefill")
    check_fwd(qm, xq, a, ref_qm, ref_q, ref_a, "cfg5 prefill", rows=sample_rows(8192, idx), paths=("w_i8",), f32=False)


# ------------------------------------------------------------------ edge cases


@pytest.mark.parametrize("t", [1, 5, 12, 127, 129, 300])
def test_ragged_token_counts(t):
    # k_in = 576 ends the int8 K loop on a half-filled 128-byte stage; n_out = 144
    # ends the bf16 reduction of grad_x on a partial 64-row stage and leaves a
    # ragged last tile in every product.
    full_layer(1, 10 + t, t, 576, 144, 6, 8)


@pytest.mark.parametrize("t,n_out", [(128, 128), (129, 128), (128, 144), (257, 400), (520, 272)])
def test_cta_pair_threshold(t, n_out):
    # Products with more than 128 output rows run on CTA pairs (256-row tiles split
    # over two SMs), the others on single CTAs: both sides of the switch, with rows
    # of the last pair tile beyond the output and a ragged K (k_in = 320).
    full_layer(1, 40 + t + n_out, t, 320, n_out, 6, 8)


@pytest.mark.parametrize("nm", [(6, 8), (4, 8), (3, 8), (2, 4), (1, 4), (8, 8)])
def test_mask_ties(nm):
    n, m = nm
    rng = np.random.default_rng(3)
    mag = rng.integers(0, 4, size=(64, 256)).astype(np.float32) * np.float32(0.01)
    w = (mag * np.where(rng.random((64, 256)) < 0.5, -1, 1)).astype(np.float32)
    w[0, :8] = 0.0   # an all-zero group (all ties, gamma still positive)
    ref = O.quant_mask(w, n, m)
    check_quant_mask(gpu_quant_mask(w, n, m), ref, f"ties {n}:{m}")


@pytest.mark.parametrize("nm", [(6, 8), (2, 4), (3, 4), (2, 8)], ids=lambda v: f"{v[0]}of{v[1]}")
def test_quant_mask_without_mask_output(nm):
    """No mask output wanted: pass 2 ranks the groups itself (the keep bits never reach
    memory); codes, int8 codes, gamma and, for 2:4-valid masks, the 2:4 form stay exact."""
    n, m = nm
    w = synth.latent_weight(410, 272, 896)
    w[5, 8:16] = w[5, 8]   # a tied group
    ref = O.quant_mask(w, n, m)
    out = B.bitlinear_quant_mask(f32_to_dev(w), n, m, want_mask=False, want_sp=n <= 2)
    torch.cuda.synchronize()
    assert B.bitlinear_quant_mask_status(out["workspace"]) == 0
    check_quant_mask(out, ref, f"no mask output {n}:{m}", has_mask=False)
    # the same with the SGD step fused into pass 1
    g = synth.activation_bf16(411, 272, 896)
    ref = O.sgd_quant_mask(w, g, 3e-3, n, m)
    w_dev = f32_to_dev(w)
    out = B.bitlinear_sgd_quant_mask(w_dev, bits_to_dev_bf16(g), 3e-3, n, m, want_mask=False, want_sp=n <= 2)
    torch.cuda.synchronize()
    assert B.bitlinear_quant_mask_status(out["workspace"]) == 0
    assert_exact(w_dev.cpu().numpy().view(np.uint32), ref["w"].view(np.uint32), f"sgd {n}:{m} updated W")
    check_quant_mask(out, ref, f"sgd, no mask output {n}:{m}", has_mask=False)


def test_codes_at_rounding_boundary():
    # weights at exactly +-gamma/2 (ties: code 0), one float above (code +-1), and 1.5 gamma
    w = synth.latent_weight(77, 32, 64)
    g, _, _ = O.absmean_gamma(w)
    half = np.float32(0.5) * np.float32(g)
    qm0 = O.quant_mask(w, 8, 8)
    assert qm0["gamma"] == g
    w2 = w.copy()
    w2[0, 0], w2[0, 1] = half, -half
    w2[0, 2] = np.nextafter(half, np.float32(1))
    w2[0, 3] = np.float32(1.5) * np.float32(g)
    ref = O.quant_mask(w2, 8, 8)
    check_quant_mask(gpu_quant_mask(w2, 8, 8), ref, "boundary")


@pytest.mark.parametrize("k_in", [20480, 32768, 65536], ids=["cta-12", "cta-16", "two-pass"])
def test_act_quant_wide_rows(k_in):
    """Rows wider than the ring kernel takes (one CTA per row with 12 or 16 vectors per
    thread; two reads beyond 32768): bit-exact xq and absmax, a zero row included."""
    x = synth.activation_bf16(400, 5, k_in)
    x[2, :] = 0
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    check_act_quant(xq, a, ref_q, ref_a, f"wide rows k={k_in}")


def test_zero_activation_rows_and_empty_batch():
    x = synth.activation_bf16(88, 6, 896)
    x[2, :] = 0
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    check_act_quant(xq, a, ref_q, ref_a, "zero row")
    # empty batch: every entry point accepts t = 0; grad_w of an empty batch is zero
    w = synth.latent_weight(89, 128, 896)
    qm = gpu_quant_mask(w, 6, 8)
    x0 = torch.empty((0, 896), dtype=torch.bfloat16, device="cuda")
    xq0, a0 = B.bitlinear_act_quant(x0)
    y0, _ = B.bitlinear_fwd(xq0, a0, qm["w_scale"], w_i8=qm["w_i8"])
    assert y0.shape == (0, 128)
    dy0 = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    gw = torch.full((128, 896), 7.0, dtype=torch.bfloat16, device="cuda")
    B.bitlinear_bwd(dy0, x0, qm["codes"], qm["w_scale"], grad_w=gw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(gw).item() == 0


def test_grad_w_f32_and_masked_positions():
    w, x, dy = layer_inputs(1, 40, 200, 896, 256)
    ref_qm = O.quant_mask(w, 2, 8)
    qm = gpu_quant_mask(w, 2, 8)
    check_bwd(dy, x, qm, ref_qm, "gw f32", gw_f32=True)
    # the straight-through gradient reaches masked weights: the GPU grad_W is the
    # same for 2:8 and 8:8 masks
    qm8 = gpu_quant_mask(w, 8, 8)
    _, g2 = B.bitlinear_bwd(bits_to_dev_bf16(dy), bits_to_dev_bf16(x), qm["codes"], qm["w_scale"], want_grad_x=False)
    _, g8 = B.bitlinear_bwd(bits_to_dev_bf16(dy), bits_to_dev_bf16(x), qm8["codes"], qm8["w_scale"], want_grad_x=False)
    torch.cuda.synchronize()
    assert torch.equal(g2, g8)


@pytest.mark.parametrize("t,k_in,n_out,with_grad_x", [(200, 896, 256, False), (1000, 2048, 1024, True)])
def test_grad_w_dequantised_x(t, k_in, n_out, with_grad_x):
    """BL_GRADW_DEQUANT_X: grad_W against q * a / 127 (what the forward consumed),
    alone and together with grad_X in one call (both buffers in one workspace)."""
    w, x, dy = layer_inputs(1, 41, t, k_in, n_out)
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    check_act_quant(xq, a, ref_q, ref_a, "dequant-x")
    ref_qm = O.quant_mask(w, 6, 8)
    qm = gpu_quant_mask(w, 6, 8)
    gx, gw = B.bitlinear_bwd(bits_to_dev_bf16(dy), None, qm["codes"] if with_grad_x else None,
                             qm["w_scale"] if with_grad_x else None, want_grad_x=with_grad_x, xq=xq, absmax=a,
                             flags=B.BL_GRADW_DEQUANT_X)
    torch.cuda.synchronize()
    # element by element against the library's stated operand (X_deq rounded to bf16),
    # and normwise against the exact X_deq the pages' reading rounds
    got = bf16_dev_to_bits(gw)
    assert_grad_close(got, O.grad_w(dy, x, x_deq=O.dequant_x_bf16(ref_q, ref_a)), "grad_w (dequantised x, bf16)")
    ref = O.grad_w(dy, x, x_deq=O.dequant_x(ref_q, ref_a))
    assert np.max(np.abs(bf16_bits_to_f64(got) - ref)) / np.max(np.abs(ref)) <= 2e-2
    # the two readings of X really differ here (1% x20 outliers): element by element far
    # beyond the tolerance, so the option is not a no-op
    raw = O.grad_w(dy, x)
    assert np.max(np.abs(ref - raw) / np.maximum(np.abs(raw), 1e-3 * np.max(np.abs(raw)))) > 0.1
    if with_grad_x:
        assert_grad_close(bf16_dev_to_bits(gx), O.grad_x(dy, ref_qm["mcode"], ref_qm["gamma"]), "grad_x (same call)")


def test_grad_w_dequantised_x_training_shape():
    """Qwen2.5-3B gate shape, 16384 tokens, sampled output rows."""
    t, k_in, n_out = 16384, 2048, 11008
    _, x, dy = layer_inputs(4, 0, t, k_in, n_out)
    ref_q, ref_a = O.act_quant(x)
    xq, a = gpu_act_quant(x)
    _, gw = B.bitlinear_bwd(bits_to_dev_bf16(dy), None, None, None, want_grad_x=False, xq=xq, absmax=a,
                            flags=B.BL_GRADW_DEQUANT_X)
    torch.cuda.synchronize()
    rows = sample_rows(n_out, 5)
    got = bf16_dev_to_bits(gw)[rows]
    assert_grad_close(got, O.grad_w(dy, x, rows=rows, x_deq=O.dequant_x_bf16(ref_q, ref_a)),
                      "grad_w (dequantised x, bf16) training shape")
    ref = O.grad_w(dy, x, rows=rows, x_deq=O.dequant_x(ref_q, ref_a))
    assert np.max(np.abs(bf16_bits_to_f64(got) - ref)) / np.max(np.abs(ref)) <= 2e-2


def test_range_error_reported():
    w = synth.latent_weight(90, 64, 128)
    w[3, 5] = np.nan
    out = B.bitlinear_quant_mask(f32_to_dev(w), 6, 8)
    assert B.bitlinear_quant_mask_status(out["workspace"]) == -4
    assert np.isnan(out["w_scale"].cpu().numpy()[0])
    assert int(out["codes"].cpu().numpy().sum()) == 0
    w[3, 5] = 70000.0
    out = B.bitlinear_quant_mask(f32_to_dev(w), 6, 8, workspace=out["workspace"])
    assert B.bitlinear_quant_mask_status(out["workspace"]) == -4
    # the same workspace works again for valid weights
    w[3, 5] = 0.01
    out = B.bitlinear_quant_mask(f32_to_dev(w), 6, 8, workspace=out["workspace"])
    assert B.bitlinear_quant_mask_status(out["workspace"]) == 0
    check_quant_mask(out, O.quant_mask(w, 6, 8), "after range error")


# ------------------------------------------------------------------ optimizer step fused with the mask recompute


def gpu_sgd_quant_mask(w_np, g_bits, lr, n, m):
    wd = f32_to_dev(w_np)
    out = B.bitlinear_sgd_quant_mask(wd, bits_to_dev_bf16(g_bits), lr, n, m, want_sp=n <= 2)
    torch.cuda.synchronize()
    assert B.bitlinear_quant_mask_status(out["workspace"]) == 0
    return wd.cpu().numpy(), out


@pytest.mark.parametrize("nm", [(6, 8), (2, 4), (8, 8)], ids=lambda v: f"{v[0]}of{v[1]}")
@pytest.mark.parametrize("n_out,k_in", [(272, 896), (16, 64)])
def test_sgd_quant_mask_small(n_out, k_in, nm):
    """W <- fp32(W - lr*G) in place (bit-exact), then gamma, mask, codes and int8 codes
    of the updated W (bit-exact)."""
    n, m = nm
    w = synth.latent_weight(120, n_out, k_in)
    g = synth.activation_bf16(121, n_out, k_in)
    lr = 3e-3
    ref = O.sgd_quant_mask(w, g, lr, n, m)
    w_new, out = gpu_sgd_quant_mask(w, g, lr, n, m)
    assert_exact(w_new.view(np.uint32), ref["w"].view(np.uint32), "updated W")
    check_quant_mask(out, ref, f"sgd {n}:{m}")


def test_sgd_update_rounding_cases():
    """The hand-worked SGD cases (halfway points; a quarter fp64 ulp above one) on the
    device: one fused multiply-add rounds like the exact value."""
    cases = [(1.0, 2.0 ** -24, -1.0, 1.0), (1.0, 2.0 ** -24, -1.0078125, 1.0 + 2.0 ** -23),
             (1.0 + 2.0 ** -23, 2.0 ** -24, 1.0, 1.0), (1.0, 16519105 * 2.0 ** -48, -1.015625, 1.0 + 2.0 ** -23),
             (1.0 + 2.0 ** -23, 7110873 * 2.0 ** -47, 1.1796875, 1.0 + 2.0 ** -23)]
    for w0, lr, g0, want in cases:
        w = np.full((16, 64), w0, np.float32)
        g = synth.f32_to_bf16_bits(np.full((16, 64), g0, np.float32))
        w_new, out = gpu_sgd_quant_mask(w, g, lr, 6, 8)
        assert np.all(w_new == np.float32(want)), (w0, lr, g0)
        check_quant_mask(out, O.sgd_quant_mask(w, g, lr, 6, 8), f"sgd case {w0} {lr} {g0}")


def test_sgd_quant_mask_training_shape():
    """The 3B MLP gate projection (11008 x 2048), one step: the whole updated W and gamma
    bit-exact, mask and codes on sampled rows."""
    n_out, k_in = 11008, 2048
    w = synth.latent_weight(122, n_out, k_in)
    g = synth.activation_bf16(123, n_out, k_in, std=1e-2, outliers=False)
    lr = 0.05
    w_ref = O.sgd_update(w, g, lr)
    w_new, out = gpu_sgd_quant_mask(w, g, lr, 6, 8)
    assert_exact(w_new.view(np.uint32), w_ref.view(np.uint32), "updated W")
    gamma, _, _ = O.absmean_gamma(w_ref)
    assert_exact(out["w_scale"].cpu().numpy()[:1].view(np.uint32), np.array([gamma], np.float32).view(np.uint32), "gamma")
    rows = sample_rows(n_out, 5)
    code = O.ternary_codes(w_ref[rows], gamma)
    keep = O.nm_keep(w_ref[rows], 6, 8)
    mcode = (code * keep).astype(np.int8)
    assert_exact(out["mask"].cpu().numpy()[rows], O.mask_bytes(keep, 8), "mask")
    assert_exact(out["codes"].cpu().numpy()[rows], O.pack_codes(mcode), "codes")
    assert_exact(out["w_i8"].cpu().numpy()[rows], mcode, "w_i8")


def test_no_device_timeouts():
    st, bits = B.bitlinear_device_status()
    assert st == 0 and bits == 0


# ------------------------------------------------------------------ diagnostics and the int8-dY gradient


def _hist_by_sorting(w, gamma, n, m):
    """Threshold histogram from sorted magnitudes (the (n+1)-th largest |w| of each
    group), vectorised; equal to the oracle's threshold_hist by the CPU pins."""
    a = np.sort(np.abs(w).astype(np.float64).reshape(-1, m), axis=1)[:, ::-1]
    g = float(gamma)
    if n == m:
        return np.zeros(O.HIST_BINS, np.int64), 0, 0
    thr = a[:, n]
    b = np.zeros(thr.shape, np.int64)
    for k in range(1, O.HIST_BINS):
        b += (8.0 * thr >= k * g)
    core = int(np.sum(2.0 * a[:, n:] > g))
    return np.bincount(b, minlength=O.HIST_BINS), a.shape[0] * (m - n), core


@pytest.mark.parametrize("nm", [(6, 8), (4, 8), (3, 8), (2, 8), (2, 4), (8, 8)])
def test_threshold_hist_oracle(nm):
    n, m = nm
    w = synth.latent_weight(synth.config_seed(3, 60 + 10 * n + m), 192, 1536)
    ref_qm = O.quant_mask(w, n, m)
    ref = O.threshold_hist(w, ref_qm["keep"], ref_qm["gamma"], m)
    qm = gpu_quant_mask(w, n, m)
    h = B.bitlinear_mask_threshold_hist(f32_to_dev(w), qm["mask"], qm["w_scale"], m).cpu().numpy()
    assert_exact(h[:O.HIST_BINS], ref["hist"], f"hist {n}:{m}")
    assert h[O.HIST_BINS] == ref["dropped"] and h[O.HIST_BINS + 1] == ref["dropped_core"]


@pytest.mark.parametrize("nm", [(6, 8), (2, 4)])
def test_threshold_hist_full_size(nm):
    # the training workload's gate weights, 11008 x 2048
    n, m = nm
    w = synth.latent_weight(synth.config_seed(4, 0), 11008, 2048)
    qm = gpu_quant_mask(w, n, m)
    gamma = qm["w_scale"].cpu().numpy()[0]
    h = B.bitlinear_mask_threshold_hist(f32_to_dev(w), qm["mask"], qm["w_scale"], m).cpu().numpy()
    hist, dropped, core = _hist_by_sorting(w, gamma, n, m)
    assert_exact(h[:O.HIST_BINS], hist, f"full-size hist {n}:{m}")
    assert h[O.HIST_BINS] == dropped and h[O.HIST_BINS + 1] == core


@pytest.mark.parametrize("t,k_in,n_out", [(64, 896, 896), (300, 576, 1536), (1, 2048, 256)])
def test_grad_x_int8_dy(t, k_in, n_out):
    w, _, dy = layer_inputs(1, 70 + t, t, k_in, n_out)
    ref_qm = O.quant_mask(w, 6, 8)
    qm = gpu_quant_mask(w, 6, 8)
    acc_ref, y_ref, _, _ = O.grad_x_int8_dy(dy, ref_qm["mcode"], ref_qm["gamma"])
    dyd = bits_to_dev_bf16(dy)
    out = B.bitlinear_grad_x_i8(dyd, qm["codes"], qm["w_scale"], k_in=k_in, want_acc=True)
    torch.cuda.synchronize()
    assert_exact(out["acc"].cpu().numpy(), acc_ref, f"grad_x_i8 acc {t}x{k_in}<-{n_out}")
    assert_bf16_within_ulp(bf16_dev_to_bits(out["grad_x"]), y_ref, f"grad_x_i8 y (acc path)")
    out2 = B.bitlinear_grad_x_i8(dyd, qm["codes"], qm["w_scale"], k_in=k_in)
    torch.cuda.synchronize()
    assert_bf16_within_ulp(bf16_dev_to_bits(out2["grad_x"]), y_ref, f"grad_x_i8 y")
    # the approximation against the exact input gradient
    exact = O.grad_x(dy, ref_qm["mcode"], ref_qm["gamma"])
    assert np.max(np.abs(y_ref - exact)) <= 2e-2 * np.max(np.abs(exact))


def test_grad_x_int8_dy_training_shape():
    # down projection of the training workload (dY [16384, 2048] -> grad_x [16384, 11008]),
    # sampled token rows against the oracle
    t, k_in, n_out = 16384, 11008, 2048
    w, _, dy = layer_inputs(4, 2, t, k_in, n_out)
    ref_qm = O.quant_mask(w, 6, 8)
    qm = gpu_quant_mask(w, 6, 8)
    rows = sample_rows(t, 5)
    acc_ref, y_ref, _, _ = O.grad_x_int8_dy(dy, ref_qm["mcode"], ref_qm["gamma"], rows=rows)
    out = B.bitlinear_grad_x_i8(bits_to_dev_bf16(dy), qm["codes"], qm["w_scale"], k_in=k_in)
    torch.cuda.synchronize()
    assert_bf16_within_ulp(bf16_dev_to_bits(out["grad_x"])[rows], y_ref, "grad_x_i8 training shape")


# ------------------------------------------------------------------ failure detection


def test_bounded_wait_gives_up_and_context_survives():
    # A wait on an mbarrier that nothing arrives on must end by itself (about 2 s), report
    # it, and leave the context usable: no fault, trap or hang.
    import ctypes
    import os
    probe = ctypes.CDLL(os.path.join(os.path.dirname(B.__file__), "libblprobe.so"))
    probe.blprobe_wait_timeout.restype = ctypes.c_int
    probe.blprobe_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    out = (ctypes.c_uint * 2)()
    assert probe.blprobe_wait_timeout(out, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    assert out[0] == 1, "the bounded wait did not give up"
    assert 1500 <= out[1] <= 10000, f"gave up after {out[1]} ms"
    # the context still runs kernels of the library
    xq, a = B.bitlinear_act_quant(torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert int(xq.abs().sum()) == 0
