#!/usr/bin/env python
"""Benchmark of the GPTQ layer pass on B200: ms per layer and weights quantized per second.

One step = the whole pass over one layer, through the C ABI:
    H = 0; gptq_hessian_accumulate over all calibration tokens (2 X^T X)
    gptq_prepare_hinv (damping + factor U)      | or gptq_il_quantize_layer
    gptq_quantize_layer (sweep, lazy updates)   |    (intrinsic-LoRA workload)
Default workload: the 2048 x 6144 MLP down-projection layer, 262144 bf16 calibration tokens,
3-bit, groups of 128, lambda = 0.01 mean(diag H), B = 128 (synthetic data).

Timing: W untimed warm-up steps, then K steps between a barrier + device synchronize on each
side, timed with CUDA events on the launching stream; the calibration set (3.2 GB) is larger
than L2, so no flush is needed. With --gpus N (torchrun), each rank quantizes its own layer
(independent problems, no data-path collective): weak scaling, max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the same
workload and extrapolates to the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "weights quantized per second (GPTQ layer pass, 1 layer per GPU per step)"
UNIT = "weights/s"
WORKLOAD_SEEDS = {"tiny": 0, "attn": 1, "mlp_down": 2, "deit_fc1": 3, "deit_fc2": 3, "lowrank": 4}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mlp_down", choices=sorted(WORKLOAD_SEEDS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--refine-rounds", type=int, default=2,
                    help="OLrC + Bid-Up rounds timed after the pass (reported apart, 0: none)")
    ap.add_argument("--no-gemm-times", action="store_true",
                    help="skip the extra pass that times the fp32 GEMM launches per stage")
    ap.add_argument("--no-gptq2d", action="store_true",
                    help="skip the two-sided rounding (GPTQ-2D) timing reported under 'gptq2d'")
    ap.add_argument("--only-gptq2d", action="store_true",
                    help="time only the two-sided rounding (one GPU) and print its JSON object")
    ap.add_argument("--tokens", type=int, default=0,
                    help="use only the first TOKENS calibration rows (small profiling cases)")
    ap.add_argument("--no-il", action="store_true",
                    help="skip the intrinsic-LoRA layer pass reported under 'il'")
    ap.add_argument("--no-reduced", action="store_true",
                    help="skip GPTQ with lattice basis reduction reported under 'reduced'")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (tiny, attn, DeiT fc1/fc2) reported under 'configs'")
    return ap.parse_args(argv)


# ------------------------------------------------------------------------------------------
# ranks
# ------------------------------------------------------------------------------------------

def rank_seed(workload: str, rank: int) -> int:
    """Rank 0 quantizes the workload's own seeded layer; rank r > 0 an independent layer of
    the same recipe (weak scaling: one layer per GPU per step)."""
    return WORKLOAD_SEEDS[workload] + 1000 * rank


def reduce_max(value: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = [ln.split(",") for ln in open(self.path).read().strip().splitlines() if ln.strip()]
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) < 9:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# device arm
# ------------------------------------------------------------------------------------------

class LayerPass:
    """Buffers and calls of one layer pass through the C ABI."""

    def __init__(self, g, layer, stream):
        self.g, self.L, self.s = g, layer, stream
        dev = layer.W.device
        m, n, r = layer.m, layer.n, layer.r
        G = n // layer.group_size if layer.group_size else 1
        self.H = torch.empty(n, n, dtype=torch.float32, device=dev)
        self.U = torch.empty(n, n, dtype=torch.float32, device=dev)
        self.codes = torch.empty(m, n * layer.bits // 32, dtype=torch.int32, device=dev)
        self.scales = torch.empty(m, G, dtype=torch.float32, device=dev)
        self.zeros = torch.empty(m, G, dtype=torch.uint8, device=dev)
        self.loss = torch.empty(m, dtype=torch.float64, device=dev)
        self.lam = torch.empty(1, dtype=torch.float32, device=dev)
        if r:
            self.Lr = torch.empty(n, r, dtype=torch.float32, device=dev)
            self.R = torch.empty(r, m, dtype=torch.float32, device=dev)
            self.ws = g.workspace(g.GPTQ_OP_IL_QUANTIZE, m, n, r, layer.block_size, dev)
        else:
            self.ws_f = g.workspace(g.GPTQ_OP_PREPARE_HINV, m, n, 0, layer.block_size, dev)
            self.ws = g.workspace(g.GPTQ_OP_QUANTIZE, m, n, 0, layer.block_size, dev)
        self.ev = self.new_events()

    @staticmethod
    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def hessian(self, X_chunks):
        for X in X_chunks:
            self.g.gptq_hessian_accumulate(self.H, X, stream=self.s)

    def rest(self, W):
        g, L, s = self.g, self.L, self.s
        if L.r:
            g.gptq_il_quantize_layer(W, self.H, L.r, L.bits, L.group_size, L.lambda_rel,
                                     L.block_size, self.codes, self.scales, self.zeros, self.Lr,
                                     self.R, self.lam, self.loss, self.ws, stream=s)
        else:
            g.gptq_prepare_hinv(self.H, L.lambda_rel, self.U, self.lam, self.ws_f, stream=s)
            g.gptq_quantize_layer(W, self.U, L.bits, L.group_size, L.block_size, self.codes,
                                  self.scales, self.zeros, self.loss, self.ws, stream=s)

    def step(self, ev=None):
        """Device-resident step with stage events: [start, H done, factor done, end]."""
        if ev is not None:
            self.ev = ev
        with torch.cuda.stream(self.s):
            self.ev[0].record(self.s)
            self.H.zero_()
            self.hessian([self.L.X])
            self.ev[1].record(self.s)
            if self.L.r:
                self.ev[2].record(self.s)
                self.rest(self.L.W)
            else:
                g, L = self.g, self.L
                g.gptq_prepare_hinv(self.H, L.lambda_rel, self.U, self.lam, self.ws_f, stream=self.s)
                self.ev[2].record(self.s)
                g.gptq_quantize_layer(L.W, self.U, L.bits, L.group_size, L.block_size, self.codes,
                                      self.scales, self.zeros, self.loss, self.ws, stream=self.s)
            self.ev[3].record(self.s)

    def stage_ms(self):
        e = self.ev
        return (e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]))

    def outputs(self):
        outs = [self.codes, self.scales, self.zeros, self.loss]
        if self.L.r:
            outs += [self.Lr, self.R]
        return outs


def hessian_flops(layer) -> float:
    """Algorithmic flops of the Hessian: k n (n + 1) (one symmetric triangle)."""
    return float(layer.k) * layer.n * (layer.n + 1)


def sweep_bytes(layer) -> float:
    """Algorithmic bytes of the sweep stage: W read once (its stored dtype), the upper triangle
    of U read once, the packed codes, and the per-group scales (fp32) and zero-points (u8)."""
    m, n = layer.m, layer.n
    groups = n // layer.group_size if layer.group_size else 1
    w_bytes = layer.W.element_size()
    return float(m * n * w_bytes + 4 * n * (n + 1) // 2 + m * n * layer.bits // 8 + m * groups * 5)


def sweep_roofline(layer, sweep_ms: float, gemm) -> dict:
    """The sweep against HBM: its algorithmic bytes over the timed stage. The stage is bound by
    its n sequential column steps, not by bandwidth, so the fraction is small by design; with
    the GEMM timing pass, the column loops' own share is the stage time minus the event time of
    the sweep's GEMM launches (two passes of the same code)."""
    hbm = hbm_peak_gbs()
    b = sweep_bytes(layer)
    gbs = b / (sweep_ms * 1e-3) / 1e9
    out = {"bound": "latency (n sequential column steps)", "bytes": b, "achieved_gbs": gbs,
           "peak_gbs": hbm, "frac": gbs / hbm, "peak_source": "measured copy (MEASURED_PEAKS.json)"}
    if gemm:
        g_ms = sum(v["ms"] for k, v in gemm.items() if k.startswith("sweep_") and isinstance(v, dict))
        out["gemm_ms"] = g_ms
        out["column_loop_ms"] = max(sweep_ms - g_ms, 0.0)
    return out


def hessian_traffic(layer):
    """DRAM bytes per Hessian launch from the committed one-pass ncu capture
    (profiles/hessian_tc_traffic.json), for the full 2048x6144 / 262144-token workload only, and
    only while the kernel source is the one profiled."""
    import hashlib
    if (layer.n, layer.k) != (6144, 262144):
        return None
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "hessian_tc_traffic.json")))
        src = open(os.path.join(ROOT, rec["kernel_source"]), "rb").read()
        current = hashlib.sha256(src).hexdigest()[:16]
    except (OSError, KeyError, ValueError):
        return None
    return int(rec["traffic_bytes_per_launch"]) if current == rec["kernel_source_sha256_16"] else None


def run_e2e(g, layer, lp, steps, warmup, chunk_tokens=32768):
    """Same pass, inputs from pinned host memory: per step the calibration tokens and W are
    copied host -> device in 32768-token chunks on a copy stream, the Hessian of each chunk
    starts as soon as that chunk has landed, and the packed codes, scales, zeros and loss are
    read back. Consecutive steps overlap the way a run over many layers does: X and H are
    double-buffered, so the copies of step i+1 wait only for the Hessian that last read the
    same X buffer, not for the factor and sweep of step i."""
    dev = layer.W.device
    X_host = layer.X.cpu().pin_memory()
    W_host = layer.W.cpu().pin_memory()
    k, n = layer.X.shape
    X_dev = [torch.empty(k, n, dtype=layer.X.dtype, device=dev) for _ in range(2)]
    H_dev = [lp.H, torch.empty_like(lp.H)]
    W_dev = [torch.empty_like(layer.W) for _ in range(2)]
    outs_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in lp.outputs()]
    cstream = torch.cuda.Stream(device=dev)
    s = lp.s
    bounds = [(t0, min(k, t0 + chunk_tokens)) for t0 in range(0, k, chunk_tokens)]
    landed = [[torch.cuda.Event() for _ in bounds] for _ in range(2)]
    w_landed = [torch.cuda.Event() for _ in range(2)]
    x_free = [torch.cuda.Event() for _ in range(2)]
    h2d = X_host.numel() * X_host.element_size() + W_host.numel() * W_host.element_size()
    d2h = sum(o.numel() * o.element_size() for o in outs_host)
    state = {"i": 0}

    def one():
        b = state["i"] % 2
        if state["i"] >= 2:
            cstream.wait_event(x_free[b])  # the Hessian of step i-2 has read X_dev[b]
        with torch.cuda.stream(cstream):
            for c, (t0, t1) in enumerate(bounds):
                X_dev[b][t0:t1].copy_(X_host[t0:t1], non_blocking=True)
                landed[b][c].record(cstream)
            W_dev[b].copy_(W_host, non_blocking=True)
            w_landed[b].record(cstream)
        with torch.cuda.stream(s):
            H_dev[b].zero_()
            for c, (t0, t1) in enumerate(bounds):
                s.wait_event(landed[b][c])
                g.gptq_hessian_accumulate(H_dev[b], X_dev[b][t0:t1], stream=s)
            x_free[b].record(s)
            s.wait_event(w_landed[b])
            lp.H = H_dev[b]
            lp.rest(W_dev[b])
            for oh, od in zip(outs_host, lp.outputs()):
                oh.copy_(od, non_blocking=True)
        state["i"] += 1

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    cstream.wait_stream(s)  # no copy of the timed steps starts before e0
    for _ in range(steps):
        one()
    e1.record(s)
    torch.cuda.synchronize(dev)
    lp.H = H_dev[0]
    ms = e0.elapsed_time(e1) / steps
    ms = reduce_max(ms, dev)
    barrier()
    return ms, h2d, d2h


def run_refine(g, layer, lp, rounds):
    """OLrC + Bid-Up refinement (gptq_il_refine) of the pass's output, timed apart from the
    pass: `rounds` rounds on the codes the last timed step produced, with the same H."""
    dev = layer.W.device
    m, n, r = layer.m, layer.n, layer.r
    ws = g.workspace(g.GPTQ_OP_IL_REFINE, m, n, r, 0, dev)
    Lr = torch.empty(n, max(r, 1), device=dev)
    Rr = torch.empty(max(r, 1), m, device=dev)
    hist = torch.empty(2 * rounds, dtype=torch.float64, device=dev)
    start = lp.codes.clone()
    codes = start.clone()
    s = lp.s

    def once():
        codes.copy_(start)
        g.gptq_il_refine(layer.W, lp.H, r, layer.bits, layer.group_size, rounds, codes, lp.scales,
                         lp.zeros, Lr if r else None, Rr if r else None, hist, ws, stream=s)

    with torch.cuda.stream(s):
        once()                                   # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        once()
        e1.record(s)
    torch.cuda.synchronize(dev)
    h = hist.cpu().tolist()
    changed = int((codes != start).sum().item())   # packed words that differ
    ms_round = e0.elapsed_time(e1) / rounds
    # product work of one round: g = D H (2 m n^2) and the Bid-Up lazy updates (about
    # 2 m n^2); with r > 0 also E H and (E H) E^T for OLrC (2 m n^2 + 2 m^2 n)
    flops = 4.0 * m * n * n + (2.0 * m * n * n + 2.0 * m * m * n if r else 0.0)
    tf32x3 = tensor_peak_tflops() * TF32_PER_BF16 / 3.0
    achieved = flops / (ms_round * 1e-3) / 1e12
    return {"rounds": rounds, "ms": e0.elapsed_time(e1), "ms_per_round": ms_round,
            "roofline": {"bound": "tensor", "kernel": "refinement round (tf32x3 products)",
                         "achieved": achieved, "peak": tf32x3, "unit": "TFLOP/s",
                         "frac": achieved / tf32x3,
                         "peak_source": "measured bf16 sustained x nominal tf32/bf16 ratio / 3 passes"},
            "loss_after_first_olrc": h[0], "loss_final": h[-1],
            "loss_drop": (h[0] - h[-1]) / h[0] if h[0] else 0.0, "code_words_changed": changed}


SIMT_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x FMA x max SM clock
TF32_PER_BF16 = 1.1 / 2.25                          # nominal dense tf32 : bf16 throughput


def tensor_peak_tflops() -> float:
    """Measured sustained bf16 tensor throughput (MEASURED_PEAKS.json), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["bf16_tflops_sustained"])
    return 1400.0


def hbm_peak_gbs() -> float:
    """Measured copy bandwidth (MEASURED_PEAKS.json), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["hbm_gbs"])
    return 6650.0


def run_gemm_times(g, lp):
    """One more layer pass, outside the timed region, with GPTQ_FLAG_KERNEL_TIMES: the device
    time and algorithmic work of the fp32 GEMM launches per stage (the factor's trailing and
    inverse updates, the sweep's lazy updates) and path (tf32x3 tensor core, SIMT). A launch's
    time runs from its start event to its stop event on its stream, so a factor update that
    waits for SMs held by the chain counts the wait; the roofline time of a class is the larger
    of its flops at the path's peak and its bytes at the measured HBM bandwidth."""
    g.kernel_times()
    g.gptq_set_flags(g.GPTQ_FLAG_KERNEL_TIMES)
    try:
        lp.step()
        torch.cuda.synchronize()
    finally:
        g.gptq_set_flags(0)
    kt = g.kernel_times()
    tf32x3 = tensor_peak_tflops() * TF32_PER_BF16 / 3.0
    hbm = hbm_peak_gbs()
    out = {"peak_tc": tf32x3, "peak_simt": SIMT_FP32_TFLOPS, "hbm_gbs": hbm,
           "peak_source": "tc: measured bf16 sustained x nominal tf32/bf16 ratio / 3 passes; "
                          "simt: derived 148 SMs x 128 lanes x 2 x 1.965 GHz; hbm: measured copy"}
    for (stage, path), v in sorted(kt.items()):
        sec = v["ms"] * 1e-3
        peak = tf32x3 if path == "tc" else SIMT_FP32_TFLOPS
        t_roof = max(v["flops"] / (peak * 1e12), v["bytes"] / (hbm * 1e9))
        out[f"{stage}_{path}"] = {
            "launches": v["launches"], "ms": v["ms"], "gflop": v["flops"] / 1e9,
            "gbytes": v["bytes"] / 1e9, "tflops": v["flops"] / sec / 1e12,
            "frac_of_peak": v["flops"] / sec / 1e12 / peak, "roofline_ms": t_roof * 1e3,
            "frac_of_roofline": t_roof / sec}
    return out


def run_gptq2d(g, dev, steps):
    """Two-sided rounding (gptq_2d_round) of X 2048 x 6144 under G 2048^2, H 6144^2: the whole
    call (both factorizations and the wavefront), and each factorization alone through
    gptq_prepare_hinv. The call factors G beside H, so the wavefront takes at most the call's
    time minus H's factorization (the figure the roofline uses)."""
    import datagen
    P = datagen.two_sided(device=dev)
    torch.cuda.synchronize(dev)           # the inputs come from the current stream
    m, n = P.X.shape
    Z = torch.empty(m, n, dtype=torch.int32, device=dev)
    ws = g.workspace(g.GPTQ_OP_2D_ROUND, m, n, 0, 0, dev)
    s = torch.cuda.Stream(device=dev)
    UG, UH = torch.empty(m, m, device=dev), torch.empty(n, n, device=dev)
    lam = torch.empty(1, device=dev)
    wsf = g.workspace(g.GPTQ_OP_PREPARE_HINV, 0, max(m, n), 0, 0, dev)

    def full():
        g.gptq_2d_round(P.X, P.G, P.H, Z, None, ws, stream=s)

    def factor_h():
        g.gptq_prepare_hinv(P.H, 0.0, UH, lam, wsf, stream=s)

    def factor_g():
        g.gptq_prepare_hinv(P.G, 0.0, UG, lam, wsf, stream=s)

    def timed(fn, reps):
        with torch.cuda.stream(s):
            fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(reps):
                fn()
            e1.record(s)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    reps = max(1, steps)
    l0 = g.gptq_launch_count()
    ms = timed(full, reps)
    launches = (g.gptq_launch_count() - l0) // (reps + 1)
    fh_ms, fg_ms = timed(factor_h, reps), timed(factor_g, reps)
    st, _ = g.gptq_sync_status(s, raise_on_error=False)
    # inside the call the two factorizations overlap: the wavefront takes at most ms - fh_ms
    wave_ms = ms - fh_ms
    flops = 2.0 * m * n * (m + n)         # every entry receives m + n feedback terms (one FMA each)
    achieved = flops / (wave_ms * 1e-3) / 1e12
    return {"workload": P.name + " fp32, G and H spectral Gram matrices", "ms": ms,
            "entries_per_s": m * n / (ms * 1e-3), "factor_h_ms": fh_ms, "factor_g_ms": fg_ms,
            "wavefront_ms": wave_ms,
            "launches_per_call": int(launches), "device_status": int(st),
            "roofline": {"bound": "alu", "kernel": "wavefront (tile sweeps + band flushes), fp32 FMA",
                         "achieved": achieved, "peak": SIMT_FP32_TFLOPS, "unit": "TFLOP/s",
                         "frac": achieved / SIMT_FP32_TFLOPS,
                         "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"}}


def config_dict(layer, world: int = 1) -> dict:
    """The workload as both arms report it."""
    return {"workload": layer.name, "m": layer.m, "n": layer.n, "k_tokens": layer.k,
            "bits": layer.bits, "group_size": layer.group_size, "r": layer.r,
            "block_size": layer.block_size, "lambda_rel": layer.lambda_rel,
            "l2": "inputs larger than L2 (X is %.1f GB)" % (layer.X.numel() * layer.X.element_size() / 1e9)
            if layer.X.numel() * layer.X.element_size() > 126e6 else
            "inputs smaller than L2 (X is %.1f MB)" % (layer.X.numel() * layer.X.element_size() / 1e6),
            "parallelism": f"{world} independent layers (one per GPU)"}


def time_workload(g, layer, steps: int, warmup: int) -> dict:
    """One workload's whole layer pass (H = 0, Hessian over all tokens, factor or
    intrinsic-LoRA step, sweep) timed like the main step: CUDA events on the launching stream,
    `warmup` untimed passes first. Reported apart from the main line."""
    dev = layer.W.device
    torch.cuda.synchronize(dev)
    s = torch.cuda.Stream(device=dev)
    lp = LayerPass(g, layer, s)
    for _ in range(warmup):
        lp.step()
    torch.cuda.synchronize(dev)
    g.gptq_sync_status(s)
    events = [LayerPass.new_events() for _ in range(steps)]
    l0 = g.gptq_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(steps):
        lp.step(events[i])
    e1.record(s)
    torch.cuda.synchronize(dev)
    launches = (g.gptq_launch_count() - l0) // max(1, steps)
    stage = np.zeros(3)
    for ev in events:
        lp.ev = ev
        stage += np.array(lp.stage_ms())
    stage /= steps
    ms = e0.elapsed_time(e1) / steps
    st, info = g.gptq_sync_status(s, raise_on_error=False)
    out = {"config": config_dict(layer), "ms": ms, "weights_per_s": layer.m * layer.n / (ms * 1e-3),
           "steps": steps, "launches_per_step": int(launches), "device_status": int(st)}
    if layer.r:
        out["stages_ms"] = {"hessian": stage[0], "il_quantize": stage[2]}
    else:
        out["stages_ms"] = {"hessian": stage[0], "factor": stage[1], "sweep": stage[2]}
    out["hessian_tflops"] = hessian_flops(layer) / (stage[0] * 1e-3) / 1e12
    del lp
    return out


def run_other_workloads(g, dev, steps: int, warmup: int, rank: int) -> dict:
    """The other seeded workloads, one layer each, generated on the device in turn."""
    import datagen
    out = {}
    for name in ("tiny", "attn", "deit_fc1", "deit_fc2"):
        layer = datagen.WORKLOADS[name](device=dev, seed=rank_seed(name, rank))
        out[name] = time_workload(g, layer, steps, warmup)
        del layer
        torch.cuda.empty_cache()
    return out


def run_reduced(g, dev, steps: int, rank: int) -> dict:
    """GPTQ with lattice basis reduction (gptq_quantize_layer_reduced) on the DeiT fc1 layer
    (2-bit, per channel) and the tiny layer (4-bit, per channel): the whole entry point (LLL, the
    rounding in the reduced basis, codes and loss) timed with CUDA events after one warm-up call,
    with the LLL statistics and the loss against plain GPTQ on the same per-channel grid."""
    import datagen
    out = {}
    for name, bits in (("deit_fc1", 2), ("tiny", 4)):
        layer = datagen.WORKLOADS[name](device=dev, seed=rank_seed(name, rank))
        m, n = layer.m, layer.n
        s = torch.cuda.Stream(device=dev)
        H = torch.zeros(n, n, device=dev)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(s):
            g.gptq_hessian_accumulate(H, layer.X, stream=s)
        res = dict(codes=torch.empty(m, n * bits // 32, dtype=torch.int32, device=dev),
                   scales=torch.empty(m, device=dev),
                   zeros=torch.empty(m, dtype=torch.uint8, device=dev),
                   loss=torch.empty(m, dtype=torch.float64, device=dev),
                   stats=torch.zeros(8, dtype=torch.int64, device=dev))
        ws = g.workspace(g.GPTQ_OP_REDUCED, m, n, 0, 0, dev)

        def call():
            g.gptq_quantize_layer_reduced(layer.W, H, bits, layer.lambda_rel, res["codes"],
                                          res["scales"], res["zeros"], res["loss"], None,
                                          res["stats"], ws, stream=s)

        with torch.cuda.stream(s):
            call()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            for _ in range(max(1, steps)):
                call()
            e1.record(s)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / max(1, steps)
        st, _ = g.gptq_sync_status(s, raise_on_error=False)
        # plain GPTQ on a per-channel grid, same bits and damping
        plain = g.quantize_layer(layer.W, H=H, bits=bits, group_size=0,
                                 lambda_rel=layer.lambda_rel, check_status=False)
        torch.cuda.synchronize(dev)
        stats = res["stats"].cpu().tolist()
        out[name] = {"workload": f"{layer.name.split(',')[0]}, {layer.k} tokens, {bits}-bit per-channel",
                     "ms": ms,
                     "lll_swaps": stats[0], "lll_size_reductions": stats[1],
                     "max_abs_T": stats[3], "codes_clipped": stats[4], "codes": m * n,
                     "loss_vs_plain": float(res["loss"].sum().item() / plain["loss"].sum().item()),
                     "device_status": int(st)}
        del layer, H, res, ws
        torch.cuda.empty_cache()
    return out


def cpu_baseline(layer, budget_s: float):
    """The fp64 oracle as it stands, on a bounded sample of the same layer, on the host cores:
    Hessian over a slice of the tokens, the full n x n factor, the sweep over a few rows;
    extrapolated linearly in tokens and rows to one whole layer."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max(int(i.get("num_threads", 1)) for i in threadpool_info()) if threadpool_info() else os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    k, n = layer.X.shape
    m = layer.m
    k_s = min(k, 4096)
    m_s = min(m, 8)
    X = layer.X[:k_s].double().cpu().numpy()
    W = layer.W[:m_s].double().cpu().numpy()
    t0 = time.perf_counter()
    H = oracle.hessian(X)
    t_h = time.perf_counter() - t0
    t0 = time.perf_counter()
    if layer.r:
        G = H / 2
        V, _ = oracle.top_singular_directions(G, layer.r)
        Ht, _ = oracle.il_hessian(G, V, layer.lambda_rel)
        U = oracle.eig_qr_factor(Ht)[:n]
        Wt = np.hstack([W, np.zeros((m_s, layer.r))])
    else:
        Hd, _ = oracle.damp(H, layer.lambda_rel)
        U = oracle.inverse_cholesky_upper(Hd)
        Wt = W
    t_f = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.sweep(Wt, U, layer.bits, layer.group_size, n_quant=n)
    t_s = time.perf_counter() - t0
    total = t_h * (k / k_s) + t_f + t_s * (m / m_s)
    return {
        "value": m * n / total,
        "unit": UNIT,
        "cores": cores,
        "kind": "oracle",
        "seconds_per_layer": total,
        "sample": (f"fp64 NumPy oracle: Hessian on {k_s} of {k} tokens ({t_h:.2f} s, scaled x{k / k_s:.0f}), "
                   f"full {n}x{n} factor ({t_f:.2f} s), sweep of {m_s} of {m} rows "
                   f"({t_s:.2f} s, scaled x{m / m_s:.0f}); {total:.0f} s per layer"),
    }


def bench_ours(args):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import datagen
    import post_weight_quantization_06_b200 as g

    layer = datagen.WORKLOADS[args.workload](device=dev, seed=rank_seed(args.workload, rank))
    if args.tokens:
        layer.X = layer.X[: args.tokens].clone()
        torch.cuda.empty_cache()
    torch.cuda.synchronize(dev)           # generated on the current stream, used on others
    stream = torch.cuda.Stream(device=dev)
    lp = LayerPass(g, layer, stream)
    for _ in range(args.warmup):
        lp.step()
    torch.cuda.synchronize(dev)
    g.gptq_sync_status(stream)
    barrier()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)
    events = [LayerPass.new_events() for _ in range(args.steps)]
    l0 = g.gptq_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier()
    e0.record(stream)
    for i in range(args.steps):
        lp.step(events[i])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    launches = g.gptq_launch_count() - l0
    stage = np.zeros(3)
    for ev in events:
        lp.ev = ev
        stage += np.array(lp.stage_ms())
    ms = e0.elapsed_time(e1) / args.steps
    ms = reduce_max(ms, dev)
    barrier()
    clk = clocks.stop()
    st, info = g.gptq_sync_status(stream, raise_on_error=False)
    stage /= args.steps

    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else None
    if peaks:
        peak, peak_src = float(peaks["bf16_tflops_sustained"]), "measured (bf16 sustained)"
    else:
        peak, peak_src = 1400.0, "fallback (bf16 sustained)"
    h_tflops = hessian_flops(layer) / (stage[0] * 1e-3) / 1e12

    gemm = run_gemm_times(g, lp) if not args.no_gemm_times else None

    refine = run_refine(g, layer, lp, args.refine_rounds) if args.refine_rounds > 0 else None

    two_d = run_gptq2d(g, dev, args.steps) if not args.no_gptq2d else None

    e2e = None
    if not args.no_e2e:
        e_ms, h2d, d2h = run_e2e(g, layer, lp, max(1, args.steps), 2)
        e2e = {"value": world * layer.m * layer.n / (e_ms * 1e-3), "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # the other workloads, each timed on its own after the main line's measurements
    other = None
    il = None
    reduced = None
    if not args.no_configs or not args.no_il:
        del lp
        torch.cuda.empty_cache()
        import datagen
        if not args.no_il and args.workload != "lowrank":
            il_layer = datagen.lowrank(device=dev, seed=rank_seed("lowrank", rank))
            il = time_workload(g, il_layer, max(1, args.steps), max(1, min(args.warmup, 3)))
            del il_layer
            torch.cuda.empty_cache()
        if not args.no_configs:
            other = run_other_workloads(g, dev, max(1, args.steps), max(1, min(args.warmup, 3)), rank)
    if not args.no_reduced:
        reduced = run_reduced(g, dev, 2, rank)

    if rank == 0:
        out = {
            "metric": METRIC,
            "value": world * layer.m * layer.n / (ms * 1e-3),
            "unit": UNIT,
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16 X / fp32 accumulate; fp32 factor and sweep",
            "data": "synthetic (seeded; shapes and spectra of the named layer)",
            "config": config_dict(layer, world),
            "stages_ms": {"hessian": stage[0], "factor": stage[1], "sweep": stage[2]},
            "roofline": {"bound": "tensor", "kernel": "hessian (2 X^T X)",
                         "achieved": h_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": h_tflops / peak, "peak_source": peak_src,
                         "traffic": hessian_traffic(layer),
                         "traffic_unit": "bytes per launch (DRAM read + write)"},
            "gpu_launches": int(launches),
            "clocks": clk,
            "device_status": int(st),
        }
        if e2e:
            out["e2e"] = e2e
        out["sweep_roofline"] = sweep_roofline(layer, float(stage[2]), gemm)
        if gemm:
            out["gemm"] = gemm
        if refine:
            out["refine"] = refine
        if two_d:
            out["gptq2d"] = two_d
        if il:
            out["il"] = il
        if other:
            out["configs"] = other
        if reduced:
            out["reduced"] = reduced
        if not args.no_cpu_baseline and world == 1:
            out["cpu_baseline"] = cpu_baseline(layer, args.cpu_budget_s)
        print(json.dumps(out))
    if world > 1:
        dist.destroy_process_group()


def bench_reference(args):
    """The oracle on the host cores, each step a bounded sample of the workload. ms_per_step is
    the measured wall time of one such sample; `value` is the metric the sample gives for the
    whole layer (per-layer time extrapolated as cpu_baseline describes, under its own key)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import datagen
    layer = datagen.WORKLOADS[args.workload](device="cuda" if torch.cuda.is_available() else "cpu",
                                              seed=rank_seed(args.workload, 0))
    if args.tokens:
        layer.X = layer.X[: args.tokens].clone()
    for _ in range(args.warmup):
        cpu_baseline(layer, args.cpu_budget_s)
    vals, secs, walls = [], [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        t1 = time.perf_counter()
        cb = cpu_baseline(layer, args.cpu_budget_s)
        walls.append(time.perf_counter() - t1)
        vals.append(cb["value"])
        secs.append(cb["seconds_per_layer"])
    wall = time.perf_counter() - t0
    value = float(np.median(vals))
    print(json.dumps({
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": float(np.mean(walls)) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; same layer as the device arm)",
        "config": config_dict(layer),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
                         "sample": cb["sample"]},
        "extrapolated_ms_per_layer": float(np.median(secs)) * 1e3,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }))


def main(argv=None):
    args = parse_args(argv)
    if args.only_gptq2d:
        import post_weight_quantization_06_b200 as g
        torch.cuda.set_device(0)
        print(json.dumps(run_gptq2d(g, torch.device("cuda", 0), args.steps)))
        return
    if args.impl == "reference":
        bench_reference(args)
    else:
        bench_ours(args)


if __name__ == "__main__":
    main()
