"""Benchmark of the forward MoE layer (Mixture-of-Kittens hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mok|reference]
                    [--config page] [--mode staged|persistent] [--minibatch 0]

One step = one pass of the whole hot path over one batch of synthetic
tokens already resident in HBM: mok_plan (router top-k, gates, histogram,
pull schedule) + the forward layer (gather, gate/up GEMM + SwiGLU, down GEMM
with push to the token slots, fixed-order combine).  The default workload
is the page shape: T = 8192 tokens, hidden 7168, expert intermediate 2048,
384 experts, top-8, R = 8 source shards, bf16 (synthetic Gaussian data;
33.8 GB of expert weights, far larger than L2, so no flush is needed).

Metric: tokens/s of the forward layer (whole job: sum over ranks).  With N
GPUs each rank runs an independent replica of the workload (the layer on
one GPU does not shard; no collective is on the data path) and the time is
the max over ranks.  Rank 0 prints one JSON line.  The default run also
times, on the device, the persistent SM-partitioned kernel on the same
workload and the zipf-routed shape (T 16384, E 256: the tensor-bound
H7168/I2048 GEMM), as sub-records of the same line.

--impl reference times the CPU oracle (test infrastructure, plain C with
fp64 accumulation) on bounded samples of the same workload: each step is
the oracle's FFN on one whole expert's rows plus that expert's share of the
oracle plan.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import signal
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mokgen  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal dense tensor-core peaks of one B200 (TFLOP/s), for context beside the measured ones
NOMINAL_DENSE_TFLOPS = {"bf16": 2250.0, "fp8": 4500.0}
# a timed region shorter than this is a burst: the tensor peak it is compared
# with is the measured burst figure; longer regions use the sustained one
SUSTAINED_REGION_S = 1.0
# kernel sources whose hash identifies the grouped GEMM a DRAM capture was taken of
GEMM_SOURCES = ("gemm_core.cuh", "gemm_sm100.cu", "mok_device.cuh", "mxfp8.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "combine_device_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, mode: str):
    """DRAM bytes (read + write) of the grouped GEMM's launches of one step
    from a committed ncu capture of THIS kernel source (matched by hash) on
    this workload and mode, or (None, reason)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no capture"
    with open(TRAFFIC_FILE) as f:
        entries = json.load(f).get("entries", [])
    sha = gemm_source_hash()
    for e in entries:
        if e.get("workload") == workload and e.get("mode") == mode:
            if e.get("gemm_source_sha") != sha:
                return None, "the kernel changed since its capture"
            return float(e["bytes_per_step"]), e.get("how", "")
    return None, "no capture of this workload"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region.

    The sampler is started first and the timed region begins only after its
    first line has appeared; each line carries the host time it was read at,
    and only lines read between ``mark_start()`` and ``mark_stop()`` count."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 100

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []          # (host time, csv line)
        self.t0 = self.t1 = None
        self.reader = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True,
                bufsize=1)
        except (OSError, FileNotFoundError):
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        deadline = time.time() + 10.0
        while not self.lines and time.time() < deadline and self.proc.poll() is None:
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_stop(self):
        self.t1 = time.time()
        if self.proc is not None:
            # one more period so the last part of the region is sampled
            time.sleep(self.PERIOD_MS / 1e3 * 1.5)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.send_signal(signal.SIGTERM)
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=5)

    def summary(self):
        if self.proc is None or self.t0 is None:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # a line read at time t describes the GPU within one period before t
        lo, hi = self.t0, self.t1 + self.PERIOD_MS / 1e3
        for t, line in self.lines:
            if not (lo <= t <= hi):
                continue
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "period_ms": self.PERIOD_MS}


# ------------------------------------------------------------------ ranks
def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (the job is as slow as its slowest
    rank); the value itself on one process."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_rate(units_per_rank: float, ms: float, world: int) -> float:
    """Whole-job throughput: the units every rank processed over the (max over
    ranks) time, per second."""
    return units_per_rank * world / (ms / 1e3)


# ------------------------------------------------------------------ workload
def algorithmic_work(cfg):
    """Algorithmic bytes / flops of one forward (one step)."""
    ns = cfg.slots
    if cfg.mxfp8:
        # weights, token rows and h: E4M3 bytes plus one E8M0 scale per 32
        # values; slot outputs bf16
        el, slot = 1.0 + 1.0 / 32, 2.0
    else:
        # bf16 weights, rows and h; slot outputs fp16 with one exponent byte per 128 values
        el, slot = 2.0, 2.0 + 1.0 / 128
    w_bytes = cfg.E * 3 * cfg.H * cfg.I * el
    gemm_bytes = w_bytes + ns * cfg.H * el + 2 * ns * cfg.I * el + ns * cfg.H * slot  # weights, rows, h out+in, slots
    gather_bytes = cfg.T * cfg.H * 2 + ns * cfg.H * el
    combine_bytes = ns * cfg.H * slot + ns * 4 + cfg.T * cfg.H * 2
    return {
        "gemm_flops": 6.0 * cfg.H * cfg.I * ns,
        "gemm_bytes": float(gemm_bytes),
        "weight_bytes": float(w_bytes),
        "gather_bytes": float(gather_bytes),
        "combine_bytes": float(combine_bytes),
        # gather + grouped GEMM + combine: what one mok_moe_forward call must move
        "forward_bytes": float(gather_bytes + gemm_bytes + combine_bytes),
        "plan_bytes": float(cfg.T * cfg.E * 4 + ns * 4 * 8),
    }


class Workload:
    """One configuration's inputs on the device (weights generated per expert
    and uploaded; MXFP8 weights quantised once, untimed)."""

    def __init__(self, cfg, device):
        import combine_device_top_b200 as mok

        self.cfg, self.device = cfg, device
        self.x = mokgen.tokens(cfg)
        self.logits = mokgen.router_logits(cfg, self.x)
        self.dx, self.dlogits = self.x.to(device), self.logits.to(device)
        wg, wu, wd = mokgen.upload_expert_weights(cfg, device)
        self.pack = None
        if cfg.mxfp8:
            self.pack = (*mok.quantize_weights_mxfp8(wg), *mok.quantize_weights_mxfp8(wu),
                         *mok.quantize_weights_mxfp8(wd))
            del wg, wu, wd
            self.w = None
            torch.cuda.empty_cache()
        else:
            self.w = (wg, wu, wd)
        self.x_shards = mok.shards(self.dx, cfg.R)
        self.y = torch.empty_like(self.dx)
        self.y_shards = mok.shards(self.y, cfg.R)
        self.plan = mok.plan(self.dlogits, cfg.k, cfg.R)

    def free(self):
        self.w = self.pack = None
        self.dx = self.dlogits = self.y = self.x_shards = self.y_shards = self.plan = None
        torch.cuda.empty_cache()


def _gpu_index():
    if "CUDA_VISIBLE_DEVICES" in os.environ:
        return int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[torch.cuda.current_device()])
    return torch.cuda.current_device()


def time_steps(wl: Workload, mode: str, steps: int, warmup: int, minibatch: int, dispatch_ctas: int = 0,
               world: int = 1, dispatch_warps: int = 0):
    """Time `steps` steps after `warmup` untimed ones; staged mode goes through
    the per-step ABI calls (the same kernels as mok_moe_forward's staged
    mode) so that events on the launching stream time each phase."""
    import combine_device_top_b200 as mok

    cfg, device = wl.cfg, wl.device
    staged = mode == "staged"
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED if staged else mok.MOK_MODE_PERSISTENT,
                        ring_slots=cfg.ring_slots, mxfp8=cfg.mxfp8, dispatch_ctas=dispatch_ctas,
                        dispatch_warps=dispatch_warps)
    p = wl.plan
    bufs = {}
    if staged:
        if cfg.mxfp8:
            bufs["out"] = torch.empty((cfg.slots, cfg.H), dtype=torch.bfloat16, device=device)
            bufs["rows_q"] = torch.empty((cfg.slots, cfg.H), dtype=torch.uint8, device=device)
            bufs["planes"] = torch.zeros((cfg.H // 128, mok.lib().mok_mxfp8_scale_rows(cfg.slots), 4),
                                         dtype=torch.uint8, device=device)
            bufs["ffn_ws"] = torch.empty(mok.lib().mok_expert_ffn_mxfp8_workspace_bytes(cfg.slots, cfg.I, cfg.E),
                                         dtype=torch.uint8, device=device)
        else:
            # slot rows as MOK_SLOTS_F16S: fp16 values plus one exponent per 128 features
            bufs["out"] = torch.empty(mok.lib().mok_slot_bytes(cfg.slots, cfg.H, mok.MOK_SLOTS_F16S),
                                      dtype=torch.uint8, device=device)
            bufs["rows"] = torch.empty((cfg.slots, cfg.H), dtype=torch.bfloat16, device=device)
            bufs["ffn_ws"] = torch.empty(mok.lib().mok_expert_ffn_workspace_bytes(cfg.slots, cfg.I, cfg.E),
                                         dtype=torch.uint8, device=device)
    else:
        bufs["fws"] = torch.empty(mok.forward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, minibatch, opts),
                                  dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    n_ev = 5 if staged else 3

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        mok.plan(wl.dlogits, cfg.k, cfg.R, ws=p.ws)
        if evs:
            evs[1].record(stream)
        if staged:
            if wl.pack is not None:
                mok.gather_mxfp8(wl.x_shards, p, bufs["rows_q"], bufs["planes"])
            else:
                mok.gather(wl.x_shards, p, bufs["rows"])
            if evs:
                evs[2].record(stream)
            if wl.pack is not None:
                mok.expert_ffn_mxfp8(bufs["rows_q"], bufs["planes"], wl.pack, p, out=bufs["out"], ws=bufs["ffn_ws"])
            else:
                mok.expert_ffn(bufs["rows"], *wl.w, p, out=bufs["out"], ws=bufs["ffn_ws"])
            if evs:
                evs[3].record(stream)
            mok.combine(bufs["out"], p, wl.y_shards)
        elif wl.pack is not None:
            mok.moe_forward_mxfp8(wl.x_shards, wl.pack, p, y_shards=wl.y_shards, ws=bufs["fws"],
                                  minibatch=minibatch, opts=opts)
        else:
            mok.moe_forward(wl.x_shards, *wl.w, p, minibatch, opts, y_shards=wl.y_shards, ws=bufs["fws"])
        if evs:
            evs[n_ev - 1].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    # correctness of the timed configuration is covered by tests; here only a sanity check
    if not torch.isfinite(wl.y.float()).all():
        raise RuntimeError("non-finite output")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(_gpu_index()) as clk:
        clk.mark_start()
        start.record(stream)
        for i in range(steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
        clk.mark_stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(start.elapsed_time(stop), device)
    phases = [[evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(steps)] for j in range(n_ev - 1)]
    res = {"total_ms": total_ms, "phases_ms": [sum(ph) / len(ph) for ph in phases], "clocks": clk.summary(),
           # plan: top-k, rank, scan, scatter; staged: gather, chunk list, gate/up, down, combine;
           # persistent: chunk list, one persistent kernel
           "launches_per_step": (4 + 1 + 1 + 2 + 1) if staged else (4 + 2),
           "max_over_mean_load": (lambda c: c.max().item() / c.mean().item())(p.counts().float())}
    if not staged:
        row0, units = mok.minibatch_bounds(p, cfg.H, cfg.I, minibatch, opts,
                                           w_gate=None if wl.pack is None else _mx_ptr(wl.pack))
        res["minibatches"] = len(row0)
        res["min_units_per_minibatch"] = min(units[:-1]) if len(units) > 1 else units[0]
    del bufs
    torch.cuda.empty_cache()
    return res


def _mx_ptr(pack):
    import ctypes

    import combine_device_top_b200 as mok

    qg, sg, qu, su, qd, sd = pack
    _mx_ptr.keep = mok.MxWeights(qg.data_ptr(), sg.data_ptr(), qu.data_ptr(), su.data_ptr(), qd.data_ptr(),
                                 sd.data_ptr())
    return ctypes.cast(ctypes.byref(_mx_ptr.keep), ctypes.c_void_p)


def time_e2e(wl: Workload, mode: str, steps: int, minibatch: int, world: int, dispatch_ctas: int = 0,
             dispatch_warps: int = 0):
    """End to end from pinned host memory through mok_moe_forward_host_batches:
    every step uploads its x and logits and reads its y back; the library
    overlaps step i+1's upload and step i-1's download with step i's compute."""
    import combine_device_top_b200 as mok

    cfg, device = wl.cfg, wl.device
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED if mode == "staged" else mok.MOK_MODE_PERSISTENT,
                        ring_slots=cfg.ring_slots, mxfp8=cfg.mxfp8, dispatch_ctas=dispatch_ctas,
                        dispatch_warps=dispatch_warps)
    hx, hl = wl.x.pin_memory(), wl.logits.pin_memory()
    hy = torch.empty_like(wl.x).pin_memory()
    wts = (wl.pack, None, None) if wl.pack is not None else wl.w
    hws = torch.empty(mok.forward_host_batches_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, minibatch, opts),
                      dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    mok.moe_forward_host_batches([hx] * 2, [hl] * 2, cfg.k, cfg.R, *wts, minibatch, opts, hws, [hy] * 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(1, steps)
    torch.cuda.synchronize()
    e0.record(stream)
    mok.moe_forward_host_batches([hx] * n, [hl] * n, cfg.k, cfg.R, *wts, minibatch, opts, hws, [hy] * n)
    e1.record(stream)
    torch.cuda.synchronize()
    if not torch.isfinite(hy.float()).all():
        raise RuntimeError("non-finite output")
    del hws
    torch.cuda.empty_cache()
    return {"e2e_ms": max_over_ranks(e0.elapsed_time(e1) / n, device), "h2d": cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4,
            "d2h": cfg.T * cfg.H * 2, "e2e_steps": n}


def time_router(wl: Workload, steps: int, warmup: int):
    """mok_plan_router on the workload's tokens: the router projection on the
    tensor cores fused with the top-k, plus the schedule kernels.  Inputs
    (x, the split router weights) resident in HBM; CUDA events on the
    launching stream."""
    import combine_device_top_b200 as mok

    cfg, device = wl.cfg, wl.device
    w = mokgen.router_weight(cfg).to(device)
    prior = mokgen.zipf_log_prior(cfg.E, cfg.zipf_s).to(device) if cfg.zipf_s else None
    hi, lo = mok.router_prepare(w)
    ws = torch.empty(mok.lib().mok_plan_workspace_bytes(cfg.T, cfg.E, cfg.k), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        mok.plan_router(wl.x_shards, hi, lo, cfg.E, cfg.k, prior, ws=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        mok.plan_router(wl.x_shards, hi, lo, cfg.E, cfg.k, prior, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    if mok.get_status(ws) != mok.MOK_OK:
        raise RuntimeError("router status " + mok.last_error())
    ms = e0.elapsed_time(e1) / steps
    flops = 2.0 * cfg.T * cfg.H * cfg.E            # useful: one projection
    return {"workload": f"{cfg.name}: {cfg.describe()}", "ms_per_call": ms, "tokens_per_s": cfg.T / (ms / 1e3),
            "useful_TFLOPs": flops / (ms / 1e3) / 1e12, "mma_TFLOPs": 2 * flops / (ms / 1e3) / 1e12,
            "x_GBps": cfg.T * cfg.H * 2 / (ms / 1e3) / 1e9, "ctas": 2 * ((cfg.T + 127) // 128), "steps": steps,
            "note": "mok_plan_router: x (w_hi + w_lo) on tcgen05 (two bf16 MMAs per product), a CTA pair per "
                    "128 tokens (half of the experts each), top-k and gates in the same kernel, then the schedule "
                    "kernels"}


def backward_work(cfg):
    """Algorithmic bytes / flops of one backward (bf16 path)."""
    ns, H, I, E, T = cfg.slots, cfg.H, cfg.I, cfg.E, cfg.T
    rc = T * H * 2 + ns * H * (2 + 1 / 128) + ns * H * 2 + T * E * 4  # dy, slot rows in; do rows, dlogits out
    dh = E * I * H * 2 + ns * H * 2 + 2 * ns * I * 2 + 2 * ns * I * 2  # Wd, do; a, b in; da, db out
    dx = 2 * E * H * I * 2 + 2 * ns * I * 2 + ns * H * (2 + 1 / 128)  # Wg, Wu, da, db in; dx rows out (fp16 + exps)
    rd = ns * H * (2 + 1 / 128) + T * H * 2                            # dx rows in, dx out
    wg = 3 * E * H * I * 2 + ns * (2 * H + I + 2 * I + H) * 2        # bf16 dW out; x, h, do, da|db rows in
    return {"flops": 12.0 * H * I * ns, "bytes": float(rc + dh + dx + rd + wg), "wgrad_bytes": float(wg)}


def time_backward(wl: Workload, steps: int, warmup: int):
    """mok_moe_backward on the workload after one staged forward that keeps
    the gate/up pre-activations; dy synthetic N(0,1) bf16 resident in HBM;
    CUDA events on the launching stream around the backward calls only."""
    import combine_device_top_b200 as mok

    cfg, device = wl.cfg, wl.device
    opts = mok.fwd_opts(mode=mok.MOK_MODE_STAGED, save_for_backward=True)
    fws = torch.empty(mok.forward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, 0, opts), dtype=torch.uint8,
                      device=device)
    mok.moe_forward(wl.x_shards, *wl.w, wl.plan, 0, opts, y_shards=wl.y_shards, ws=fws)
    dy = mokgen.normal(cfg.seed, 99, (cfg.T, cfg.H), 1.0).to(device)
    dys = mok.shards(dy, cfg.R)
    dx = torch.empty_like(dy)
    dxs = mok.shards(dx, cfg.R)
    dw = (torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16, device=device),
          torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16, device=device),
          torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=device))
    dl = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=device)
    bws = torch.empty(mok.lib().mok_backward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8,
                      device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        mok.moe_backward(dys, *wl.w, wl.plan, fws, dx_shards=dxs, dw=dw, dlogits=dl, ws=bws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        mok.moe_backward(dys, *wl.w, wl.plan, fws, dx_shards=dxs, dw=dw, dlogits=dl, ws=bws)
    e1.record(stream)
    torch.cuda.synchronize()
    if mok.get_status(bws) != mok.MOK_OK or not torch.isfinite(dx.float()).all():
        raise RuntimeError("backward failed: " + mok.last_error())
    ms = e0.elapsed_time(e1) / steps
    work = backward_work(cfg)
    del fws, bws, dw, dl, dx, dy
    torch.cuda.empty_cache()
    return {"workload": f"{cfg.name}: {cfg.describe()}", "ms_per_call": ms, "tokens_per_s": cfg.T / (ms / 1e3),
            "GBps": work["bytes"] / (ms / 1e3) / 1e9, "TFLOPs": work["flops"] / (ms / 1e3) / 1e12,
            "algorithmic_GB": work["bytes"] / 1e9, "steps": steps,
            "note": "mok_moe_backward: reverse combine, dh + SwiGLU backward, dx, reverse dispatch, weight "
                    "gradients (bf16 dW)"}


def time_ep(cfg, device, steps: int, warmup: int, wl: Workload | None = None):
    """The expert-parallel forward (EpGroup: logits all-gather, plan, pull
    dispatch + FFN + push, combine, device barriers) with this process as one
    rank of the torch.distributed group (or a group of one): the layer's T
    tokens and E experts split over the ranks.  Each rank's tokens and its
    experts' weights resident in HBM; CUDA events on the launching stream;
    max over ranks."""
    import combine_device_top_b200 as mok

    dist = torch.distributed
    world = dist.get_world_size() if dist.is_initialized() else 1
    rank = dist.get_rank() if dist.is_initialized() else 0
    grp = mok.EpGroup(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, device=device, mxfp8=cfg.mxfp8)
    S_r = grp.S_r
    if wl is not None and world == 1:
        x, logits_local = wl.dx, wl.dlogits
        w = (wl.pack, None, None) if cfg.mxfp8 else wl.w
    else:
        x_all = mokgen.tokens(cfg)
        logits_all = mokgen.router_logits(cfg, x_all)
        x = x_all[rank * S_r:(rank + 1) * S_r].to(device)
        logits_local = logits_all[rank * S_r:(rank + 1) * S_r].contiguous().to(device)
        w = (torch.empty((grp.e_loc, cfg.H, cfg.I), dtype=torch.bfloat16, device=device),
             torch.empty((grp.e_loc, cfg.H, cfg.I), dtype=torch.bfloat16, device=device),
             torch.empty((grp.e_loc, cfg.I, cfg.H), dtype=torch.bfloat16, device=device))
        for i, e in enumerate(range(grp.e0, grp.e0 + grp.e_loc)):
            for dst, src in zip(w, mokgen.expert_weights(cfg, e)):
                dst[i].copy_(src)
        if cfg.mxfp8:
            if grp.e_loc:
                pack = tuple(t for wt in w for t in mok.quantize_weights_mxfp8(wt))
            else:
                shapes = [(0, cfg.H, cfg.I), (0, cfg.H // 32, cfg.I)] * 2 + [(0, cfg.I, cfg.H), (0, cfg.I // 32, cfg.H)]
                pack = tuple(torch.empty(sh, dtype=torch.uint8, device=device) for sh in shapes)
            w = (pack, None, None)
    grp.x.copy_(x)
    y = torch.empty((S_r, cfg.H), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        grp.forward(logits_local, *w, y=y)
    torch.cuda.synchronize()
    if dist.is_initialized():
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        grp.forward(logits_local, *w, y=y)
    e1.record(stream)
    torch.cuda.synchronize()
    if grp.status() != mok.MOK_OK:
        raise RuntimeError("EP status " + mok.last_error())
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, device)
    if dist.is_initialized():
        dist.barrier()
    grp.close()
    return {"workload": f"{cfg.name}: {cfg.describe()}", "ranks": world, "ms_per_step": ms,
            "dtype": "mxfp8-e4m3" if cfg.mxfp8 else "bf16",
            "tokens_per_s": cfg.T / (ms / 1e3), "steps": steps,
            "note": "EpGroup.forward per step: all-gather of the logits, mok_plan, mok_ep_dispatch_ffn (barrier, "
                    "pull dispatch of this rank's experts' rows from the ranks' x, grouped SwiGLU FFN, push of "
                    "every slot row into its token's rank's slot buffer), mok_ep_combine (barrier, combine); "
                    + ("one rank: the pull and the push stay in this GPU's HBM" if world == 1 else
                       "peer pointers over NVLink")}


# ------------------------------------------------------------------ roofline
def tensor_peaks(peaks, mxfp8: bool, region_s: float):
    """(peak TFLOP/s of the MMA's dtype for a region this long, its kind)."""
    burst = region_s < SUSTAINED_REGION_S
    bf16 = peaks["bf16_tflops"] if burst else peaks["bf16_tflops_sustained"]
    # fp8 runs at twice the bf16 rate (nominal 4.5 / 2.25 PFLOP/s)
    kind = ("burst" if burst else "sustained") + f" (timed region {region_s:.2f} s)"
    return bf16 * (2.0 if mxfp8 else 1.0), bf16, kind


def staged_roofline(cfg, res, peaks, peak_src, mode, steps):
    work = algorithmic_work(cfg)
    t_plan, t_gather, t_gemm, t_comb = res["phases_ms"]
    gemm_s = t_gemm / 1e3
    tflops = work["gemm_flops"] / gemm_s / 1e12
    gbs = work["gemm_bytes"] / gemm_s / 1e9
    region_s = res["total_ms"] / 1e3
    tc_peak, bf16_peak, kind = tensor_peaks(peaks, cfg.mxfp8, region_s)
    t_tc = work["gemm_flops"] / (tc_peak * 1e12)
    t_hbm = work["gemm_bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": tc_peak, "unit": "TFLOP/s", "frac": tflops / tc_peak}
    traffic, how = measured_traffic(cfg.name, mode)
    nominal = NOMINAL_DENSE_TFLOPS["fp8" if cfg.mxfp8 else "bf16"]
    roof.update({
        "traffic": traffic, "traffic_note": how if traffic else how,
        "kernel": "k_grouped_gemm: the gate/up+SwiGLU and down launches of one step (figures per step)",
        "launches_per_step": 2,
        "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
        "tensor_peak_kind": kind,
        "tensor_frac_of_measured_bf16": tflops / bf16_peak,
        "tensor_frac_of_dtype_peak": tflops / tc_peak,
        "tensor_frac_of_nominal_dense": tflops / nominal,
        # both measured bf16 figures, whichever the region length picked: a
        # power-capped run (clocks in `clocks`) is closer to the sustained one
        "tensor_frac_of_bf16_burst": tflops / (peaks["bf16_tflops"] * (2.0 if cfg.mxfp8 else 1.0)),
        "tensor_frac_of_bf16_sustained": tflops / (peaks["bf16_tflops_sustained"] * (2.0 if cfg.mxfp8 else 1.0)),
    })
    rates = {"gather_GBps": work["gather_bytes"] / (t_gather / 1e3) / 1e9,
             "combine_GBps": work["combine_bytes"] / (t_comb / 1e3) / 1e9,
             "gather_frac_of_hbm": work["gather_bytes"] / (t_gather / 1e3) / 1e9 / peaks["hbm_gbs"],
             "combine_frac_of_hbm": work["combine_bytes"] / (t_comb / 1e3) / 1e9 / peaks["hbm_gbs"],
             "gemm_TFLOPs": tflops, "gemm_GBps": gbs, "plan_share": t_plan / (res["total_ms"] / steps)}
    return roof, {"plan": t_plan, "gather": t_gather, "grouped_gemm": t_gemm, "combine": t_comb}, rates


def persistent_roofline(cfg, res, peaks, peak_src, steps):
    work = algorithmic_work(cfg)
    t_plan, t_fwd = res["phases_ms"]
    fwd_s = t_fwd / 1e3
    gbs = work["forward_bytes"] / fwd_s / 1e9
    tflops = work["gemm_flops"] / fwd_s / 1e12
    tc_peak, bf16_peak, kind = tensor_peaks(peaks, cfg.mxfp8, res["total_ms"] / 1e3)
    roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"], "traffic": measured_traffic(cfg.name, "persistent")[0],
            "kernel": "k_moe_persistent (dispatch, grouped GEMM, combine in one launch; figures per step)",
            "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
            "tensor_peak_kind": kind, "tensor_frac_of_dtype_peak": tflops / tc_peak}
    return roof, {"plan": t_plan, "forward": t_fwd}, {"forward_GBps": gbs, "forward_TFLOPs": tflops,
                                                       "plan_share": t_plan / (res["total_ms"] / steps)}


def sub_record(cfg, mode, res, peaks, peak_src, steps):
    ms = res["total_ms"] / steps
    rec = {"workload": f"{cfg.name}: {cfg.describe()}", "mode": mode, "tokens_per_s": cfg.T / (ms / 1e3),
           "ms_per_step": ms, "steps": steps}
    if mode == "staged":
        roof, ph, rates = staged_roofline(cfg, res, peaks, peak_src, mode, steps)
    else:
        roof, ph, rates = persistent_roofline(cfg, res, peaks, peak_src, steps)
        rec["minibatches"] = res["minibatches"]
        rec["min_gate_up_units_per_minibatch"] = res["min_units_per_minibatch"]
    rec.update({"roofline": roof, "phases_ms": ph, "phase_rates": rates, "clocks": res["clocks"],
                "expert_load_max_over_mean": res["max_over_mean_load"]})
    return rec


# ------------------------------------------------------------------ CPU oracle
def oracle_steps(cfg, steps: int, warmup: int, threads: int = 0):
    """The oracle on bounded samples of the workload: step i runs the
    oracle's SwiGLU FFN over every row of one whole expert (experts taken in
    order, warm-up ones first) plus that expert's share of the full oracle
    plan.  Returns the measured rate (tokens/s = rows/s / k) and what ran."""
    import oracle

    cores = threads if threads > 0 else len(os.sched_getaffinity(0))
    oracle.set_num_threads(cores)
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    t0 = time.perf_counter()
    pl = oracle.plan(logits, cfg.k, cfg.R)
    t_plan = time.perf_counter() - t0
    rows_all = oracle.gather(x, cfg.R, pl["src_rank"], pl["src_index"])
    off = pl["offsets"]
    experts = [e for e in range(cfg.E) if off[e + 1] > off[e]]
    spent, rows_done, ran = 0.0, 0, []
    for i in range(warmup + steps):
        e = experts[i % len(experts)]
        a, b = int(off[e]), int(off[e + 1])
        wg, wu, wd = mokgen.expert_weights(cfg, e)
        t0 = time.perf_counter()
        oracle.expert_ffn(rows_all[a:b], wg, wu, wd)
        dt = time.perf_counter() - t0 + t_plan * (b - a) / cfg.slots
        if i >= warmup:
            spent += dt
            rows_done += b - a
            ran.append(e)
    return {"value": (rows_done / cfg.k) / spent, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "steps_run": steps, "warmup_run": warmup, "sampled_seconds": spent,
            "sample_tokens_per_step": rows_done / cfg.k / steps, "extrapolated": True,
            "sample": f"oracle SwiGLU FFN of whole experts {ran[0]}..{ran[-1]} ({rows_done} of {cfg.slots} rows "
                      f"of the {cfg.name} workload, one expert per step) plus their share of the full oracle plan; "
                      f"tokens/s = rows/s / k, extrapolated from the sample to the layer"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mok", choices=["mok", "reference"])
    ap.add_argument("--config", default="page", choices=list(mokgen.CONFIGS))
    ap.add_argument("--mode", default="staged", choices=["staged", "persistent"])
    ap.add_argument("--minibatch", type=int, default=-1,
                    help="persistent mode: least rows per minibatch (0: the two-wave rule alone; "
                         "default: the configuration's)")
    ap.add_argument("--dispatch-ctas", type=int, default=0,
                    help="persistent mode: CTAs on the dispatch side (0: the library default, 6 bf16 / 16 MXFP8)")
    ap.add_argument("--dispatch-warps", type=int, default=0,
                    help="persistent mode: 1 or 2 dispatch warps in every CTA instead of dispatch CTAs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-records", action="store_true", help="time only the main workload")
    ap.add_argument("--backward", action="store_true",
                    help="time only mok_moe_backward on the workload (after one staged forward that keeps a, b)")
    ap.add_argument("--ep", action="store_true",
                    help="time the expert-parallel forward alone, the layer split over the torchrun ranks")
    ap.add_argument("--router", action="store_true",
                    help="time only mok_plan_router (the router projection, top-k and schedule) on the workload's "
                         "tokens; no expert weights are built")
    ap.add_argument("--cpu-steps", type=int, default=64, help="experts the CPU baseline samples")
    ap.add_argument("--scale-experts", type=int, default=0,
                    help="profiling case: E experts and T scaled by the same factor (same rows per expert)")
    args = ap.parse_args()
    cfg = mokgen.CONFIGS[args.config]
    if args.scale_experts:
        n = args.scale_experts
        T = max(cfg.R, round(cfg.T * n / cfg.E / cfg.R) * cfg.R)
        cfg = mokgen.scaled(cfg, E=n, T=T)
    minibatch = cfg.minibatch if args.minibatch < 0 else args.minibatch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    # value is tokens/s; the tensor-core fraction and the gather/combine GB/s
    # of the same metric are in "roofline" and "phase_rates"
    metric = "MoE fwd tokens/s (H7168/I2048); % BF16 TC peak; gather/combine HBM GB/s"
    wdesc = ("MXFP8 E4M3 weights + E8M0 scales per 32 along K (quantised once, untimed)" if cfg.mxfp8
             else "bf16 weights [E,H,I]/[E,I,H]")
    config = {"workload": f"{cfg.name}: {cfg.describe()}, {wdesc}",
              "tokens_per_step_per_gpu": cfg.T, "mode": args.mode,
              **(({"minibatch": minibatch, "dispatch_warps_per_cta": args.dispatch_warps} if args.dispatch_warps
                  else {"minibatch": minibatch, "dispatch_ctas": args.dispatch_ctas or (16 if cfg.mxfp8 else 6)})
                 if args.mode == "persistent" else {}),
              "l2": f"inputs larger than L2 ({algorithmic_work(cfg)['weight_bytes'] / 1e9:.1f} GB of expert "
                    f"weights streamed per step)"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = oracle_steps(cfg, args.steps, args.warmup)
        line = {"metric": metric, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": cb["sampled_seconds"] / args.steps * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": config, "impl": "reference", "extrapolated": True,
                "sample_tokens_per_step": cb["sample_tokens_per_step"], "sampled_seconds": cb["sampled_seconds"],
                "cpu_baseline": dict(cb),
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if args.router:
        if rank == 0:
            import types
            import combine_device_top_b200 as mok

            x = mokgen.tokens(cfg).to(device)
            lite = types.SimpleNamespace(cfg=cfg, device=device, x_shards=mok.shards(x, cfg.R))
            print(json.dumps(time_router(lite, args.steps, args.warmup)), flush=True)
        return 0
    if args.ep:
        r = time_ep(cfg, device, args.steps, args.warmup, Workload(cfg, device) if world == 1 else None)
        if world > 1:
            torch.distributed.destroy_process_group()
        if rank == 0:
            print(json.dumps(r), flush=True)
        return 0
    wl = Workload(cfg, device)
    if args.backward:
        if rank == 0:
            bw = time_backward(wl, args.steps, args.warmup)
            peaks, _ = load_peaks()
            bw["frac_of_hbm"] = bw["GBps"] / peaks["hbm_gbs"]
            print(json.dumps(bw), flush=True)
        return 0
    res = time_steps(wl, args.mode, args.steps, args.warmup, minibatch, args.dispatch_ctas, world,
                     args.dispatch_warps)
    e2e = time_e2e(wl, args.mode, args.steps, minibatch, world, args.dispatch_ctas, args.dispatch_warps)
    subs = {}
    if not args.no_sub_records and not args.scale_experts and world == 1 and args.config == "page":
        peaks, peak_src = load_peaks()
        other = "persistent" if args.mode == "staged" else "staged"
        r2 = time_steps(wl, other, args.steps, args.warmup, minibatch, args.dispatch_ctas, 1, args.dispatch_warps)
        subs[f"{cfg.name}_{other}"] = sub_record(cfg, other, r2, peaks, peak_src, args.steps)
        subs[f"{cfg.name}_router_plan"] = time_router(wl, args.steps, args.warmup)
        bw = time_backward(wl, max(3, args.steps // 4), 2)
        bw["frac_of_hbm"] = bw["GBps"] / peaks["hbm_gbs"]
        subs[f"{cfg.name}_backward"] = bw
        subs[f"{cfg.name}_expert_parallel_1rank"] = time_ep(cfg, device, args.steps, args.warmup, wl)
        wl.free()
        del wl
        zcfg = mokgen.CONFIGS["zipf"]
        zl = Workload(zcfg, device)
        rz = time_steps(zl, "staged", args.steps, args.warmup, zcfg.minibatch)
        subs["zipf_staged"] = sub_record(zcfg, "staged", rz, peaks, peak_src, args.steps)
        zl.free()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    ms = res["total_ms"] / args.steps
    value = job_rate(cfg.T, ms, world)
    line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp8-e4m3" if cfg.mxfp8 else "bf16",
            "data": "synthetic", "config": config}
    if args.mode == "staged":
        roof, ph, rates = staged_roofline(cfg, res, peaks, peak_src, "staged", args.steps)
    else:
        roof, ph, rates = persistent_roofline(cfg, res, peaks, peak_src, args.steps)
        line["minibatches"] = res["minibatches"]
        line["min_gate_up_units_per_minibatch"] = res["min_units_per_minibatch"]
    line["roofline"] = roof
    line["phases_ms"] = ph
    line["phase_rates"] = rates
    line["e2e"] = {"value": job_rate(cfg.T, e2e["e2e_ms"], world), "unit": "tokens/s",
                   "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["e2e_steps"],
                   "api": "mok_moe_forward_host_batches (pinned host buffers; copies overlap the compute)"}
    line["gpu_launches"] = res["launches_per_step"] * args.steps
    if res["clocks"]:
        line["clocks"] = res["clocks"]
    line["expert_load_max_over_mean"] = res["max_over_mean_load"]
    if subs:
        line["sub_records"] = subs
    if not args.no_cpu_baseline and world == 1:
        cb = oracle_steps(cfg, args.cpu_steps, 1)
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample", "extrapolated")}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
