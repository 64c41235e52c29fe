"""Benchmark of the Sparse-BitNet BitLinear path on B200.

One step = one pass of the whole path over one batch: for each linear of a
Qwen2.5-3B-shaped MLP (gate 2048->11008, up 2048->11008, down 11008->2048) at
16384 tokens and a 6:8 mask: recompute mask + ternary codes from the latent fp32
weights, quantise the activations to int8, run the forward product, and both
straight-through gradients (grad_X and grad_W over every latent weight).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line (rank 0). ``value`` is tokens per second of the whole job
(all ranks; each rank runs its own batch: weak scaling, no collective on the data
path). ``e2e`` is the same metric through the public API with the step's inputs
copied from pinned host memory and its outputs copied back inside the timed region.
``--impl reference`` times the CPU oracle (the slow reference implementation) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "6:8 ternary BitLinear TOPS & tok/s (fwd/bwd), % roofline, speedup vs 8:8 dense"
WORKLOAD = "train-step Qwen2.5-3B MLP BitLinear (gate/up 2048->11008, down 11008->2048), 16384 tokens, 6:8"
TOKENS = 16384
LINEARS = [("gate", 2048, 11008), ("up", 2048, 11008), ("down", 11008, 2048)]
N_KEEP, M_GROUP = 6, 8
CFG_INDEX = 4   # the training-step workload's seed block

# DRAM traffic per launch of the dominant kernel from an ncu capture, keyed by the
# SHA-256 of the kernel's source files at capture time (reported as null once the
# source has changed).
TRAFFIC = {
    # DRAM bytes per launch from `ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum`
    # (1 pass) on the full-size launches of the current GEMM source (see profiles/);
    # reported only while the kernel source hashes to `sha`.
    # grouped grad_W (gate, up, down over 16384 tokens): 2,072,903,680 read + 129,520,640 written
    "bwd_grad_w": {"sha": "dcba4d5a127e6863", "bytes": 2202424320},
    # grad_X GEMM (16384 x 2048 <- 11008; the code expansion is a separate kernel):
    # 585,053,696 read + 61,331,712 written
    "bwd_grad_x": {"sha": "dcba4d5a127e6863", "bytes": 646385408},
}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for f in ("gemm_tc.cuh", "gemm_tc2.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "sparsity_step_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    def __init__(self, gpu: str):
        self.gpu = gpu   # nvidia-smi id: the device UUID (CUDA_VISIBLE_DEVICES does not apply there)
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        finally:
            if self.path and os.path.exists(self.path):
                os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i - 5] for r in rows for i in range(5, 9) if r[i].lower().startswith("active")})
        loaded = [s for s in sm if s >= 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


def gpu_smi_id(local: int) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local)


class RankSync:
    """Barrier and max-over-ranks of the timed regions (the only collectives of the
    benchmark; the data path has none). Works on any torch.distributed backend: on
    NCCL the reduction tensor lives on this rank's GPU, on gloo on the CPU."""

    def __init__(self, world: int, device=None):
        self.world = world
        self.device = device

    def barrier(self) -> None:
        if self.world > 1:
            import torch.distributed as dist
            if self.device is not None and self.device.type == "cuda":
                dist.barrier(device_ids=[self.device.index])
            else:
                dist.barrier()

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device=self.device if self.device is not None else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def choose_bf16_peak(peaks: dict, clocks: dict, ms_total: float) -> tuple[float, bool, str]:
    """The bf16 roofline denominator for kernels timed inside the step: the measured
    burst rate when the median SM clock under load stayed within 5 % of its maximum
    (the clock the burst figure was taken at), else the sustained (power-capped) rate.
    Without a clock record, a timed region under a second counts as a burst.
    Returns (peak TFLOP/s, burst?, the reason in words)."""
    smhz, smax = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    at_max_clock = bool(smhz and smax and smhz >= 0.95 * smax)
    use_burst = at_max_clock if (smhz and smax) else ms_total < 1000.0
    peak = peaks["bf16_tflops"] if use_burst else peaks["bf16_tflops_sustained"]
    why = "timed region %.0f ms, median SM clock %s of max %s MHz" % (ms_total, smhz, smax)
    return peak, use_burst, why


def job_tokens_per_s(ms_per_step: float, world: int) -> float:
    """Whole-job throughput: every rank processes its own TOKENS per step (weak
    scaling); the step time is the max over ranks."""
    return TOKENS * world / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------- our arm

def make_inputs(rank: int):
    import numpy as np
    import torch

    from sparsity_step_b200 import synth

    off = 100000 * rank
    host = {}
    for i, (name, k_in, n_out) in enumerate(LINEARS):
        host[f"w_{name}"] = synth.latent_weight(synth.config_seed(CFG_INDEX, 3 * i) + off, n_out, k_in)
        host[f"dy_{name}"] = synth.activation_bf16(synth.config_seed(CFG_INDEX, 3 * i + 2) + off, TOKENS, n_out,
                                                   std=1e-2, outliers=False)
    host["x_in"] = synth.activation_bf16(synth.config_seed(CFG_INDEX, 1) + off, TOKENS, 2048)
    host["x_down"] = synth.activation_bf16(synth.config_seed(CFG_INDEX, 7) + off, TOKENS, 11008)

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    return {k: pinned(v) for k, v in host.items()}


class Step:
    """Device buffers and the launches of one training step of the three linears.

    Latent weights, codes and intermediates are shared; the step's inputs (X, dY) and
    outputs (y, grad_X) come in ``n_io`` sets so that copies of one step can overlap
    the compute of another."""

    INPUTS = ["x_in", "x_down"] + [f"dy_{n}" for n, _, _ in LINEARS]

    def __init__(self, host, dev, n_keep=N_KEEP, m_group=M_GROUP, n_io=1):
        import torch

        import sparsity_step_b200 as B

        self.B = B
        self.n_keep, self.m_group = n_keep, m_group
        bf = torch.bfloat16
        T = TOKENS
        self.w = {n: host[f"w_{n}"].to(dev) for n, _, _ in LINEARS}
        self.io = []
        for _ in range(n_io):
            d = {k: host[k].to(dev).view(bf) for k in self.INPUTS}
            self.io.append({
                "d": d,
                "y": {n: torch.empty((T, n_out), dtype=bf, device=dev) for n, _, n_out in LINEARS},
                "gx": {n: torch.empty((T, k_in), dtype=bf, device=dev) for n, k_in, _ in LINEARS},
            })
        self.qm = {}
        self.ws_qm = {}
        for name, k_in, n_out in LINEARS:
            self.qm[name] = {
                "codes": torch.empty((n_out, k_in // 4), dtype=torch.uint8, device=dev),
                "mask": torch.empty((n_out, k_in // m_group), dtype=torch.uint8, device=dev),
                "w_i8": torch.empty((n_out, k_in), dtype=torch.int8, device=dev),
                "w_scale": torch.empty((4,), dtype=torch.float32, device=dev)[:1],
            }
            self.ws_qm[name] = torch.empty((B.bitlinear_quant_mask_workspace_size(n_out, k_in),), dtype=torch.uint8,
                                           device=dev)
        self.xq_in = torch.empty((T, 2048), dtype=torch.int8, device=dev)
        self.a_in = torch.empty((T,), dtype=torch.float32, device=dev)
        self.xq_down = torch.empty((T, 11008), dtype=torch.int8, device=dev)
        self.a_down = torch.empty((T,), dtype=torch.float32, device=dev)
        self.gw = {n: torch.empty((n_out, k_in), dtype=bf, device=dev) for n, k_in, n_out in LINEARS}
        wsb = max(B.bitlinear_bwd_workspace_size(T, k, n, True) for _, k, n in LINEARS)
        self.ws_bwd = torch.empty((wsb,), dtype=torch.uint8, device=dev)
        # kernels per step: quant_mask 2 per weight (plus a 16-byte memset, not a kernel),
        # act_quant 1 per input width, fwd 1 per linear, grad_X 2 per linear (expand + GEMM),
        # grad_W 1 for all three linears
        self.launches_per_step = 3 * 2 + 2 + 3 + 3 * 2 + 1

    def run(self, ev=None, io=0):
        """Enqueue one step on the current stream using I/O set ``io``. ``ev`` maps a
        kernel class to a list that receives (start, end) CUDA events around each of
        its launches."""
        import torch

        B = self.B
        d, y, gx = self.io[io]["d"], self.io[io]["y"], self.io[io]["gx"]

        def timed(key, fn):
            if ev is None:
                fn()
                return
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            ev.setdefault(key, []).append((s, e))

        for name, _, _ in LINEARS:
            q = self.qm[name]
            timed("quant_mask", lambda: B.bitlinear_quant_mask(self.w[name], self.n_keep, self.m_group, out=q,
                                                               workspace=self.ws_qm[name]))
        timed("act_quant", lambda: B.bitlinear_act_quant(d["x_in"], xq=self.xq_in, absmax=self.a_in))
        timed("act_quant", lambda: B.bitlinear_act_quant(d["x_down"], xq=self.xq_down, absmax=self.a_down))
        for name, _, _ in LINEARS:
            xq, a = (self.xq_down, self.a_down) if name == "down" else (self.xq_in, self.a_in)
            q = self.qm[name]
            timed("fwd_i8_gemm", lambda: B.bitlinear_fwd(xq, a, q["w_scale"], w_i8=q["w_i8"], y=y[name]))
        for name, k_in, _ in LINEARS:
            q = self.qm[name]
            dy = d[f"dy_{name}"]
            timed("bwd_grad_x", lambda: B.bitlinear_bwd(dy, None, q["codes"], q["w_scale"], want_grad_w=False,
                                                        grad_x=gx[name], workspace=self.ws_bwd, k_in=k_in))
        # the three weight gradients share the token batch: one launch schedules all their tiles
        timed("bwd_grad_w", lambda: B.bitlinear_grad_w_grouped(
            [{"dy": d[f"dy_{name}"], "x": d["x_down"] if name == "down" else d["x_in"], "grad_w": self.gw[name]}
             for name, _, _ in LINEARS]))

    def outputs(self, io=0):
        return [self.io[io]["y"][n] for n, _, _ in LINEARS] + [self.io[io]["gx"][n] for n, _, _ in LINEARS]


def run_e2e(step, host, steps, warmup, barrier):
    """End-to-end steps through the public API: each step copies its inputs from
    pinned host memory, runs, and copies its outputs back to pinned host memory.
    Copies run on their own streams (host->device and device->host use separate copy
    engines) and overlap the compute of the neighbouring steps through two I/O sets.
    Returns (ms per step, h2d bytes per step, d2h bytes per step)."""
    import torch

    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    outs_host = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in step.outputs(0)] for _ in range(2)]
    h2d = sum(host[k].numel() * host[k].element_size() for k in Step.INPUTS)
    d2h = sum(t.numel() * t.element_size() for t in outs_host[0])
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_done + ev_out:
        e.record(comp)

    def one(i):
        s = i % 2
        io = step.io[s]
        s_in.wait_event(ev_done[s])            # compute two steps back is done with this input set
        with torch.cuda.stream(s_in):
            for k in Step.INPUTS:
                io["d"][k].view(torch.int16).copy_(host[k], non_blocking=True)
        ev_in[s].record(s_in)
        comp.wait_event(ev_in[s])
        comp.wait_event(ev_out[s])             # this output set has been copied out
        step.run(io=s)
        ev_done[s].record(comp)
        s_out.wait_event(ev_done[s])
        with torch.cuda.stream(s_out):
            for hdst, dsrc in zip(outs_host[s], step.outputs(s)):
                hdst.copy_(dsrc, non_blocking=True)
        ev_out[s].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    s_in.wait_event(t0)
    for i in range(steps):
        one(warmup + i)
    comp.wait_event(ev_out[(warmup + steps - 1) % 2])
    t1.record(comp)
    torch.cuda.synchronize()
    barrier()
    return t0.elapsed_time(t1) / steps, h2d, d2h


def algorithmic_counts():
    """Per-step operation counts (dense-equivalent) of the step's products."""
    fwd_ops = sum(2 * TOKENS * k * n for _, k, n in LINEARS)
    bwd_flops = 2 * fwd_ops
    return fwd_ops, bwd_flops


def run_ours(args) -> None:
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    host = make_inputs(rank)
    step = Step(host, dev, n_io=2)
    stream = torch.cuda.current_stream()

    sync = RankSync(world, dev)
    barrier = sync.barrier
    max_over_ranks = sync.max

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()

    # ---------------- device-resident timed region (kernel events inside)
    ev = {}
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_smi_id(local)) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step.run(ev)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1))
    ms_step = ms_total / args.steps
    per_kernel_ms = {k: sum(s.elapsed_time(e) for s, e in v) / args.steps for k, v in ev.items()}
    per_launch_ms = {k: sum(s.elapsed_time(e) for s, e in v) / len(v) for k, v in ev.items()}
    clocks = clk.summary()

    # status of the device-side checks (timeouts, weight range)
    st, bits = step.B.bitlinear_device_status()
    for name, _, _ in LINEARS:
        if step.B.bitlinear_quant_mask_status(step.ws_qm[name]) != 0:
            raise RuntimeError(f"weight range error in {name}")
    if st != 0:
        raise RuntimeError(f"device status {bits:#x}")

    # ---------------- 6:8 versus 8:8 (same step, no mask)
    dense = Step(host, dev, n_keep=8, m_group=8)
    for _ in range(args.warmup):
        dense.run()
    barrier()
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(args.steps):
        dense.run()
    d1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_dense = max_over_ranks(d0.elapsed_time(d1)) / args.steps
    del dense

    # ---------------- end to end: pinned host inputs -> device -> step -> host outputs
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    ms_e2e, h2d, d2h = run_e2e(step, host, e2e_steps, min(args.warmup, 3), barrier)
    ms_e2e = max_over_ranks(ms_e2e)

    # ---------------- forward per shape (N:M sweep) and the 36-layer decode stack
    sweep = decode = None
    if not args.no_extra:
        sweep = measure_sweep(steps=20, warmup=3)
        del step.io[1:]
        torch.cuda.empty_cache()
        layers, code_bytes = build_decode_stack(dev, N_KEEP, M_GROUP, distinct=False, want_w_i8=True)
        decode = {"workload": "Qwen2.5-3B-shaped 36-layer BitLinear stack, 6:8, one decode step = 252 products "
                              "from 2-bit codes (layer 0's codes copied into 35 more distinct buffers); prefill = "
                              "8192 tokens through the 252 products on the int8 tensor-core path",
                  "code_bytes_per_step": code_bytes,
                  "batches": measure_decode(dev, layers, code_bytes, (1, 32), steps=200, warmup=5)}
        try:
            decode["prefill"] = measure_prefill(dev, layers, 8192, 10)
        except (RuntimeError, MemoryError) as exc:   # keep the line: report why it is missing
            decode["prefill"] = {"error": str(exc)[:200]}
        del layers
        torch.cuda.empty_cache()

    # ---------------- raw tensor-pipe rates of this GPU (probe: MMAs from shared memory only)
    try:
        probe = {"int8_tops": round(mma_peak("i8"), 1), "bf16_tflops": round(mma_peak("bf16"), 1),
                 "sparse_int8_tops_dense_equiv": round(mma_peak("sp_i8"), 1)}
    except (OSError, RuntimeError) as exc:
        probe = {"error": str(exc)}

    # ---------------- roofline of the dominant kernel (burst or sustained peak by clock)
    peaks = load_peaks()
    bf16_peak, use_burst, why = choose_bf16_peak(peaks, clocks, ms_total)
    fwd_ops, bwd_flops = algorithmic_counts()
    gemm_flops = 2 * TOKENS * 2048 * 11008          # every product here has this size
    # one bwd_grad_w launch computes all three weight gradients; a bwd_grad_x call is one
    # product (its time includes the 2-bit code expansion that feeds it)
    flops_per_launch = {"bwd_grad_w": 3 * gemm_flops, "bwd_grad_x": gemm_flops}

    def gemm_roofline(cls):
        achieved = flops_per_launch[cls] / (per_launch_ms[cls] * 1e-3) / 1e12
        tr = TRAFFIC.get(cls)
        r = {"kernel": cls, "bound": "tensor", "achieved": round(achieved, 1), "peak": bf16_peak,
             "unit": "TFLOP/s", "frac": round(achieved / bf16_peak, 4),
             "peak_kind": f"bf16 {'burst' if use_burst else 'sustained'} ({peaks['source']}; {why})",
             "frac_vs_burst": round(achieved / peaks["bf16_tflops"], 4),
             "frac_vs_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
             "traffic": tr["bytes"] if tr and tr["sha"] == kernel_source_sha() else None,
             "algorithmic_per_launch": flops_per_launch[cls],
             "note": ("one launch = the three weight gradients" if cls == "bwd_grad_w" else
                      "time per call includes the 2-bit code expansion kernel (~14 us); traffic is the GEMM's")}
        if "bf16_tflops" in probe:
            r["frac_vs_tcgen05_probe"] = round(achieved / probe["bf16_tflops"], 4)
        return r

    # The dominant kernel: the grouped grad_W GEMM, the largest single kernel of the step
    # by time (launch list: 38 % of kernel time, the grad_X GEMM 36 %); the grad_X product
    # is reported beside it.
    roof = gemm_roofline("bwd_grad_w")
    roof_gx = gemm_roofline("bwd_grad_x")
    # INT8: no measured peak in the driver's file; derived as 2 x the bf16 rate chosen above (the
    # nominal int8 / bf16 ratio of B200), with this run's tcgen05 probe beside it
    int8_peak = 2 * bf16_peak
    fwd_tops = fwd_ops / (per_kernel_ms["fwd_i8_gemm"] * 1e-3) / 1e12

    tok_s = job_tokens_per_s(ms_step, world)
    out = {
        "metric": METRIC,
        "value": round(tok_s, 1),
        "unit": "tok/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8+bf16",
        "data": "synthetic (seeded N(0,0.02) fp32 latent W; N(0,1) bf16 X with 1% x20 outliers; N(0,1e-2) bf16 dY)",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": TOKENS, "nm": f"{N_KEEP}:{M_GROUP}",
                   "linears": [f"{n} {k}->{o}" for n, k, o in LINEARS], "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (per-step working set ~1.5 GB vs 126 MB L2); no flush"},
        "tops": {"fwd_int8_dense_equiv": round(fwd_tops, 1),
                 "fwd_int8_useful_6of8": round(fwd_tops * N_KEEP / M_GROUP, 1),
                 "bwd_bf16": round(bwd_flops / ((per_kernel_ms["bwd_grad_x"] + per_kernel_ms["bwd_grad_w"]) * 1e-3) / 1e12, 1),
                 "int8_peak_derived": round(int8_peak, 1),
                 "int8_peak_kind": f"2 x measured {'burst' if use_burst else 'sustained'} bf16 (nominal int8/bf16 "
                                   "ratio), not measured",
                 "fwd_frac_of_int8_peak_derived": round(fwd_tops / int8_peak, 4),
                 "fwd_frac_of_int8_probe": (round(fwd_tops / probe["int8_tops"], 4) if "int8_tops" in probe else None),
                 "tensor_pipe_probe": probe},
        "breakdown_ms_per_step": {k: round(v, 4) for k, v in per_kernel_ms.items()},
        "speedup_vs_8_8": round(ms_dense / ms_step, 4),
        "ms_per_step_8_8": round(ms_dense, 4),
        "roofline": roof,
        "roofline_grad_x": roof_gx,
        "e2e": {"value": round(job_tokens_per_s(ms_e2e, world), 1), "unit": "tok/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 3), "steps": e2e_steps,
                "copies": "pinned host <-> device on separate H2D / D2H streams, overlapped with compute (2 I/O sets)"},
        "gpu_launches": step.launches_per_step * args.steps,
        "sweep_fwd_per_shape": sweep,
        "decode": decode,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- oracle (CPU) arm

def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


# The oracle's timed sample: the whole step (mask + ternary codes, act-quant, forward,
# grad_X, grad_W) for all three linears, narrowed to the first SAMPLE_ROWS output rows of
# each weight tensor, over SAMPLE_TOKENS tokens. Nothing is extrapolated: the reported
# throughput is the sample's own tokens per second.
SAMPLE_ROWS = 256
SAMPLE_TOKENS = 64


def oracle_sample_inputs(seed_off: int = 0) -> list:
    """Seeded inputs of the oracle sample: per linear, W [SAMPLE_ROWS, k_in] fp32,
    X [SAMPLE_TOKENS, k_in] bf16 and dY [SAMPLE_TOKENS, SAMPLE_ROWS] bf16."""
    from sparsity_step_b200 import synth

    out = []
    for i, (name, k_in, n_out) in enumerate(LINEARS):
        w = synth.latent_weight(synth.config_seed(CFG_INDEX, 3 * i) + seed_off, SAMPLE_ROWS, k_in)
        x = synth.activation_bf16(synth.config_seed(CFG_INDEX, 3 * i + 1) + seed_off, SAMPLE_TOKENS, k_in)
        dy = synth.activation_bf16(synth.config_seed(CFG_INDEX, 3 * i + 2) + seed_off, SAMPLE_TOKENS, SAMPLE_ROWS,
                                   std=1e-2, outliers=False)
        out.append((w, x, dy))
    return out


def oracle_step(inputs: list) -> float:
    """One oracle step on the sample; returns its wall-clock seconds."""
    from oracle import bitlinear_oracle as O

    s = time.perf_counter()
    for w, x, dy in inputs:
        qm = O.quant_mask(w, N_KEEP, M_GROUP)
        q, a = O.act_quant(x)
        O.fwd(q, a, qm["mcode"], qm["gamma"])
        O.grad_x(dy, qm["mcode"], qm["gamma"])
        O.grad_w(dy, x)
    return time.perf_counter() - s


def sample_text(threads: int) -> str:
    return (f"each step: the whole path (mask + ternary codes, act-quant, forward, grad_X, grad_W) of the three "
            f"linears narrowed to their first {SAMPLE_ROWS} output rows, over {SAMPLE_TOKENS} tokens; value = "
            f"{SAMPLE_TOKENS} tokens / measured step time (not extrapolated); {threads} BLAS thread(s)")


def cpu_baseline(budget_s: float = 12.0) -> dict:
    """The oracle as it stands, timed on this host: repeated sample steps for about
    ``budget_s`` seconds on all BLAS threads, then a few on one thread."""
    inputs = oracle_sample_inputs()
    oracle_step(inputs)                       # warm-up (imports, first-touch)
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        times.append(oracle_step(inputs))
    step_s = statistics.mean(times)
    threads = _blas_threads()
    out = {"value": round(SAMPLE_TOKENS / step_s, 2), "unit": "tok/s", "cores": threads, "kind": "oracle",
           "sample": sample_text(threads), "steps": len(times), "ms_per_step": round(1e3 * step_s, 1)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t1 = [oracle_step(inputs) for _ in range(3)]
        out["single_thread"] = {"value": round(SAMPLE_TOKENS / statistics.mean(t1), 2), "unit": "tok/s",
                                "cores": 1, "ms_per_step": round(1e3 * statistics.mean(t1), 1),
                                "sample": sample_text(1)}
    except ImportError:
        pass
    return out


def run_reference(args) -> None:
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inputs = oracle_sample_inputs()
    for _ in range(args.warmup):
        oracle_step(inputs)
    t0 = time.perf_counter()
    step_s = [oracle_step(inputs) for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    ms = 1e3 * statistics.mean(step_s)
    v = round(SAMPLE_TOKENS / (ms * 1e-3), 3)
    threads = _blas_threads()
    out = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64+f32 (oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": TOKENS, "nm": f"{N_KEEP}:{M_GROUP}",
                   "linears": [f"{n} {k}->{o}" for n, k, o in LINEARS], "parallelism": "single process (CPU)",
                   "oracle_sample": {"rows_per_linear": SAMPLE_ROWS, "tokens": SAMPLE_TOKENS}},
        "cpu_baseline": {"value": v, "unit": "tok/s", "cores": threads, "kind": "oracle", "sample": sample_text(threads)},
        "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "timed_wall_s": round(wall, 2),
    }
    print(json.dumps(out), flush=True)


def mma_peak(kind: str, iters: int = 4000, reps: int = 3) -> float:
    """tcgen05 MMA rate (TOP/s or TFLOP/s; dense-equivalent for the 2:4-sparse kind) of
    this GPU from the probe library: 148 CTAs issuing back-to-back 128x256 MMAs from
    shared memory (no memory traffic)."""
    import ctypes

    import torch

    lib = ctypes.CDLL(os.path.join(ROOT, "sparsity_step_b200", "libblprobe.so"))
    lib.blprobe_mma_peak.restype = ctypes.c_int
    lib.blprobe_mma_peak.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    k = {"bf16": 0, "i8": 1, "sp_i8": 2}[kind]
    ctas = torch.cuda.get_device_properties(0).multi_processor_count
    st = torch.cuda.current_stream()
    if lib.blprobe_mma_peak(k, ctas, 100, st.cuda_stream) != 0:
        raise RuntimeError("mma probe failed")
    best = 0.0
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(st)
        rc = lib.blprobe_mma_peak(k, ctas, iters, st.cuda_stream)
        e.record(st)
        torch.cuda.synchronize()
        if rc != 0:
            raise RuntimeError(f"mma probe failed ({rc})")
        kdim = {"bf16": 16, "i8": 32, "sp_i8": 64}[kind]   # logical K per MMA
        ops = 2.0 * 128 * 256 * kdim * 4 * iters * ctas
        best = max(best, ops / (s.elapsed_time(e) * 1e-3) / 1e12)
    return best


def run_case(args) -> None:
    """One kernel class alone on a chosen shape (for ncu captures and tuning):
    warm-up launches, then ``--steps`` timed launches; prints one JSON line."""
    import numpy as np
    import torch

    import sparsity_step_b200 as B
    from sparsity_step_b200 import synth

    if args.case.startswith("mma_peak"):
        kind = args.case[len("mma_peak_"):]
        print(json.dumps({"case": args.case, "rate": round(mma_peak(kind), 1),
                          "unit": "TOP/s" if kind == "i8" else "TFLOP/s"}), flush=True)
        return
    dev = torch.device("cuda", 0)
    t, k_in, n_out = args.case_t, args.case_k, args.case_n
    w = torch.from_numpy(synth.latent_weight(11, n_out, k_in)).to(dev)

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    x = bf(synth.activation_bf16(12, t, k_in))
    dy = bf(synth.activation_bf16(13, t, n_out, std=1e-2, outliers=False))
    qm = B.bitlinear_quant_mask(w, N_KEEP, M_GROUP)
    qm24 = B.bitlinear_quant_mask(w, 2, 4, want_sp=True) if args.case == "fwd_sp" else None
    xq, a = B.bitlinear_act_quant(x)
    y = torch.empty((t, n_out), dtype=torch.bfloat16, device=dev)
    gx = torch.empty((t, k_in), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((n_out, k_in), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((B.bitlinear_bwd_workspace_size(t, k_in, n_out, True),), dtype=torch.uint8, device=dev)
    ws_i8 = (torch.empty((B.bitlinear_grad_x_i8_workspace_size(t, k_in, n_out),), dtype=torch.uint8, device=dev)
             if args.case == "grad_x_i8" else None)
    hist = torch.empty((19,), dtype=torch.int64, device=dev)
    g_w = (bf(synth.activation_bf16(14, n_out, k_in, std=1e-2, outliers=False)) if args.case == "sgd_quant_mask"
           else None)
    gw_group = ([{"dy": bf(synth.activation_bf16(15 + i, t, n, std=1e-2, outliers=False)),
                  "x": bf(synth.activation_bf16(18 + i, t, k)),
                  "grad_w": torch.empty((n, k), dtype=torch.bfloat16, device=dev)} for i, (_, k, n) in enumerate(LINEARS)]
                if args.case == "grad_w_grouped" else None)
    flops = 2.0 * t * k_in * n_out
    cases = {
        # algorithmic bytes: W read once (4 B/w), int8 codes, packed codes and mask written
        "quant_mask": (lambda: B.bitlinear_quant_mask(w, N_KEEP, M_GROUP, out=qm, workspace=qm["workspace"]),
                       "GB/s", n_out * k_in * (4 + 1 + 0.25 + 1.0 / M_GROUP)),
        # the same plus the fused SGD step: gradient read (2 B/w), W written back (4 B/w)
        "sgd_quant_mask": (lambda: B.bitlinear_sgd_quant_mask(w, g_w, 1e-3, N_KEEP, M_GROUP, out=qm,
                                                              workspace=qm["workspace"]),
                           "GB/s", n_out * k_in * (4 + 2 + 4 + 1 + 0.25 + 1.0 / M_GROUP)),
        "act_quant": (lambda: B.bitlinear_act_quant(x, xq=xq, absmax=a), "GB/s", t * k_in * 3 + 4 * t),
        "fwd": (lambda: B.bitlinear_fwd(xq, a, qm["w_scale"], w_i8=qm["w_i8"], y=y), "TOP/s", flops),
        # 2:4 mask on the sparse tensor cores: dense-equivalent ops
        "fwd_sp": (lambda: B.bitlinear_fwd(xq, a, qm24["w_scale"], sp_values=qm24["sp_values"], sp_meta=qm24["sp_meta"],
                                           y=y), "TOP/s", flops),
        "fwd_codes": (lambda: B.bitlinear_fwd(xq, a, qm["w_scale"], codes=qm["codes"], y=y), "GB/s",
                      n_out * k_in / 4 + t * k_in + 2 * t * n_out),
        "grad_x": (lambda: B.bitlinear_bwd(dy, None, qm["codes"], qm["w_scale"], want_grad_w=False, grad_x=gx,
                                           workspace=ws, k_in=k_in), "TFLOP/s", flops),
        "grad_w": (lambda: B.bitlinear_bwd(dy, x, None, None, want_grad_x=False, grad_w=gw), "TFLOP/s", flops),
        # the three weight gradients of the 3B MLP (gate, up, down) over t tokens, one launch
        "grad_w_grouped": (lambda: B.bitlinear_grad_w_grouped(gw_group), "TFLOP/s",
                           sum(2.0 * t * k * n for _, k, n in LINEARS)),
        # int8-dY input gradient (an approximation; dY quantised per token): dense-equivalent ops
        "grad_x_i8": (lambda: B.bitlinear_grad_x_i8(dy, qm["codes"], qm["w_scale"], k_in=k_in, grad_x=gx,
                                                    workspace=ws_i8), "TOP/s", flops),
        "mask_hist": (lambda: B.bitlinear_mask_threshold_hist(w, qm["mask"], qm["w_scale"], M_GROUP, out=hist),
                      "GB/s", n_out * k_in * (4 + 1.0 / M_GROUP)),
    }
    fn, unit, work = cases[args.case]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(args.steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / args.steps
    rate = work / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
    print(json.dumps({"case": args.case, "t": t, "k_in": k_in, "n_out": n_out, "ms_per_launch": round(ms, 5),
                      "rate": round(rate, 1), "unit": unit}), flush=True)


DECODE_LAYERS = 36
DECODE_SHAPES = [("q", 2048, 2048, "attn_in"), ("k", 2048, 256, "attn_in"), ("v", 2048, 256, "attn_in"),
                 ("o", 2048, 2048, "o_in"), ("gate", 2048, 11008, "mlp_in"), ("up", 2048, 11008, "mlp_in"),
                 ("down", 11008, 2048, "down_in")]
DECODE_INPUTS = {"attn_in": 2048, "o_in": 2048, "mlp_in": 2048, "down_in": 11008}


def build_decode_stack(dev, n_keep: int, m_group: int, distinct: bool, want_w_i8: bool) -> tuple[list, int]:
    """The 36 layers' weights as packed codes (and int8 weights for the prefill).

    distinct=True generates every layer from its own seed (2.78 G latent weights on
    the host: minutes). distinct=False generates layer 0 and copies its codes into 35
    more distinct device buffers: the decode kernels' work and memory traffic do not
    depend on the code values, and every layer still streams from its own HBM buffer."""
    import torch

    import sparsity_step_b200 as B
    from sparsity_step_b200 import synth

    layers = []
    code_bytes = 0
    for layer in range(DECODE_LAYERS):
        qms = {}
        for i, (name, k_in, n_out, _) in enumerate(DECODE_SHAPES):
            if distinct or layer == 0:
                w = torch.from_numpy(synth.latent_weight(synth.config_seed(5, 100 * layer + i), n_out, k_in)).to(dev)
                qms[name] = B.bitlinear_quant_mask(w, n_keep, m_group, want_mask=False, want_w_i8=want_w_i8)
                qms[name].pop("workspace")
                del w
            else:
                qms[name] = {k: v.clone() for k, v in layers[0][name].items()}
            code_bytes += n_out * k_in // 4
        layers.append(qms)
    torch.cuda.synchronize()
    return layers, code_bytes


def measure_decode(dev, layers, code_bytes: int, batches, steps: int, warmup: int) -> dict:
    """Decode steps at the given batches: per step, 4 act-quant launches and grouped
    forward launches (256 products each) over all 252 products, replayed as a CUDA graph."""
    import numpy as np
    import torch

    import sparsity_step_b200 as B
    from sparsity_step_b200 import synth

    peaks = load_peaks()

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    res = {}
    for b in batches:
        inputs = {k: bf(synth.activation_bf16(synth.config_seed(5, 9000 + kk), b, K, outliers=False))
                  for kk, (k, K) in enumerate(DECODE_INPUTS.items())}
        q = {k: B.bitlinear_act_quant(v) for k, v in inputs.items()}
        probs = []
        for qms in layers:
            for name, k_in, n_out, src in DECODE_SHAPES:
                xq, a = q[src]
                probs.append({"xq": xq, "absmax": a, "codes": qms[name]["codes"], "w_scale": qms[name]["w_scale"],
                              "y": torch.empty((b, n_out), dtype=torch.bfloat16, device=dev)})

        def step():
            for k, v in inputs.items():
                B.bitlinear_act_quant(v, xq=q[k][0], absmax=q[k][1])
            for s0 in range(0, len(probs), 256):
                B.bitlinear_fwd_grouped(probs[s0:s0 + 256])

        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        # one decode step is 5 short launches: replay it as a CUDA graph so that host
        # launch overhead does not pace the GPU
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(warmup):
            graph.replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            graph.replay()
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / steps
        del graph
        act_bytes = sum(b * K * 3 + 4 * b for K in DECODE_INPUTS.values())   # bf16 read + int8 write + absmax
        fwd_bytes = code_bytes + sum(b * k * 1 + 2 * b * n for _, k, n, _ in DECODE_SHAPES) * DECODE_LAYERS
        gbs = (fwd_bytes + act_bytes) / (ms * 1e-3) / 1e9
        res[f"b{b}"] = {"ms_per_step": round(ms, 4), "tok_s": round(b / (ms * 1e-3), 1),
                        "gb_s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                        "launches_per_step": len(DECODE_INPUTS) + (len(probs) + 255) // 256, "cuda_graph": True}
    return res


def measure_prefill(dev, layers, t: int, iters: int) -> dict:
    """A t-token prefill through the 252 products of the stack on the int8 tensor-core
    path (one forward launch per linear, eager), after the four act-quant launches."""
    import numpy as np
    import torch

    import sparsity_step_b200 as B
    from sparsity_step_b200 import synth

    def bf(bits):
        return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)

    inputs = {k: bf(synth.activation_bf16(synth.config_seed(5, 9100 + kk), t, K, outliers=False))
              for kk, (k, K) in enumerate(DECODE_INPUTS.items())}
    q = {k: B.bitlinear_act_quant(v) for k, v in inputs.items()}
    ys = {name: torch.empty((t, n_out), dtype=torch.bfloat16, device=dev) for name, _, n_out, _ in DECODE_SHAPES}

    def pstep():
        for k, v in inputs.items():
            B.bitlinear_act_quant(v, xq=q[k][0], absmax=q[k][1])
        for qms in layers:
            for name, k_in, n_out, src in DECODE_SHAPES:
                xq, a = q[src]
                B.bitlinear_fwd(xq, a, qms[name]["w_scale"], w_i8=qms[name]["w_i8"], y=ys[name])

    pstep()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(iters):
        pstep()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / iters
    ops = 2.0 * t * sum(k * n for _, k, n, _ in DECODE_SHAPES) * DECODE_LAYERS
    return {"tokens": t, "ms": round(ms, 3), "tok_s": round(t / (ms * 1e-3), 1),
            "tops_dense_equiv": round(ops / (ms * 1e-3) / 1e12, 1)}


def run_decode(args) -> None:
    """Qwen2.5-3B-shaped 36-layer stack of BitLinear layers (6:8), forward only:
    decode steps at batch 1/8/32/128 (one grouped launch streams every layer's 2-bit
    codes; the four per-shape inputs are reused across layers) and an 8192-token
    prefill (tensor-core product per linear). Prints one JSON line."""
    import torch

    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    n_keep, m_group = (8, 8) if args.dense else (N_KEEP, M_GROUP)
    layers, code_bytes = build_decode_stack(dev, n_keep, m_group, distinct=not args.clone_layers,
                                            want_w_i8=args.prefill > 0)
    res = {"workload": "Qwen2.5-3B-shaped 36-layer BitLinear stack, forward",
           "nm": f"{n_keep}:{m_group}", "code_bytes_per_step": code_bytes,
           "hbm_peak_gbs": peaks["hbm_gbs"],
           "decode": measure_decode(dev, layers, code_bytes, args.batches, args.steps, args.warmup)}

    if args.prefill > 0:
        res["prefill"] = measure_prefill(dev, layers, args.prefill, max(1, args.steps // 10))
    print(json.dumps(res), flush=True)


SWEEP_SHAPES = {
    "qwen2.5-0.5b T=4096": (4096, [("q", 896, 896), ("k", 896, 128), ("v", 896, 128), ("o", 896, 896),
                                   ("gate", 896, 4864), ("up", 896, 4864), ("down", 4864, 896)]),
    "qwen2.5-1.5b-mlp T=8192": (8192, [("gate", 1536, 8960), ("up", 1536, 8960), ("down", 8960, 1536)]),
}
SWEEP_NM = [(8, 8), (6, 8), (4, 8), (3, 8), (2, 4), (2, 8)]


def measure_sweep(steps: int, warmup: int, nms=None) -> dict:
    """Forward product per shape (inference: masks and codes precomputed) for the
    Qwen2.5-0.5B linears at 4096 tokens and the Qwen2.5-1.5B MLP at 8192 tokens,
    for every N:M of the sweep: time, dense-equivalent and useful TOPS, and the
    speedup over 8:8 of the same shape."""
    import numpy as np
    import torch

    import sparsity_step_b200 as B
    from sparsity_step_b200 import synth

    dev = torch.device("cuda", 0)
    out = {}
    for wl, (t, shapes) in SWEEP_SHAPES.items():
        for name, k_in, n_out in shapes:
            x = torch.from_numpy(synth.activation_bf16(synth.config_seed(3, 50 + k_in % 97), t, k_in).view(np.int16)).to(dev)
            x = x.view(torch.bfloat16)
            xq, a = B.bitlinear_act_quant(x)
            w = torch.from_numpy(synth.latent_weight(synth.config_seed(3, 60 + n_out % 89), n_out, k_in)).to(dev)
            y = torch.empty((t, n_out), dtype=torch.bfloat16, device=dev)
            row = {}
            for n, m in (nms or SWEEP_NM):
                # masks with at most two kept per aligned four also run on the sparse
                # tensor cores ("n:m sparse"); every mask runs on the dense int8 path
                sparse_ok = n <= 2 and k_in % 128 == 0
                qm = B.bitlinear_quant_mask(w, n, m, want_sp=sparse_ok)
                variants = [(f"{n}:{m}", {"w_i8": qm["w_i8"]})]
                if sparse_ok:
                    variants.append((f"{n}:{m} sparse", {"sp_values": qm["sp_values"], "sp_meta": qm["sp_meta"]}))
                for key, kw in variants:
                    for _ in range(warmup):
                        B.bitlinear_fwd(xq, a, qm["w_scale"], y=y, **kw)
                    torch.cuda.synchronize()
                    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    s.record()
                    for _ in range(steps):
                        B.bitlinear_fwd(xq, a, qm["w_scale"], y=y, **kw)
                    e.record()
                    torch.cuda.synchronize()
                    ms = s.elapsed_time(e) / steps
                    ops = 2.0 * t * k_in * n_out
                    row[key] = {"us": round(ms * 1e3, 2), "tops_dense_equiv": round(ops / (ms * 1e-3) / 1e12, 1),
                                "tops_useful": round(ops * n / m / (ms * 1e-3) / 1e12, 1)}
            base = row["8:8"]["us"]
            for k in row:
                row[k]["speedup_vs_8_8"] = round(base / row[k]["us"], 4)
            out[f"{wl} {name} {k_in}->{n_out}"] = row
    return out


def run_sweep(args) -> None:
    print(json.dumps({"workload": "forward per shape, N:M sweep", "shapes": measure_sweep(args.steps, args.warmup)}),
          flush=True)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the N:M sweep and decode sub-records")
    ap.add_argument("--case", choices=["quant_mask", "sgd_quant_mask", "act_quant", "fwd", "fwd_sp", "fwd_codes", "grad_x", "grad_w",
                                       "grad_w_grouped",
                                       "grad_x_i8", "mask_hist", "mma_peak_i8", "mma_peak_bf16", "mma_peak_sp_i8"],
                    help="time one kernel class alone on the --case-t/k/n shape")
    ap.add_argument("--case-t", type=int, default=TOKENS)
    ap.add_argument("--case-k", type=int, default=2048)
    ap.add_argument("--case-n", type=int, default=11008)
    ap.add_argument("--workload", choices=["train", "decode", "sweep"], default="train",
                    help="decode: the 36-layer stack at decode batches and prefill (separate JSON line)")
    ap.add_argument("--batches", type=int, nargs="+", default=[1, 8, 32, 128])
    ap.add_argument("--prefill", type=int, default=8192, help="prefill tokens for --workload decode (0 = skip)")
    ap.add_argument("--dense", action="store_true", help="--workload decode with 8:8 (no mask)")
    ap.add_argument("--clone-layers", action="store_true",
                    help="--workload decode: generate layer 0 and copy its codes into the other 35 layers' buffers")
    args = ap.parse_args(argv)
    if args.workload == "decode":
        run_decode(args)
        return
    if args.workload == "sweep":
        run_sweep(args)
        return
    if args.case:
        run_case(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
