"""Benchmark of the forward MoE layer (Mixture-of-Kittens hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mok|reference]
                    [--config page] [--mode staged|persistent] [--minibatch 2560]

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
the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (test infrastructure, plain C with
fp64 accumulation) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
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


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


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


# ------------------------------------------------------------------ measured DRAM traffic
# dram__bytes_read.sum + dram__bytes_write.sum of the two grouped-GEMM
# launches of one step, from one ncu capture of a small case of the same
# kernel, scaled to the full workload by the experts (and rows) processed;
# the capture, its command and the scaling are in the profiles/ summary
# named beside each entry.  None where no capture of the current kernel
# exists for that workload.
GEMM_TRAFFIC_GB_PER_STEP = {
    "page": (35.6, "profiles/grouped_gemm_bf16_page_e37.md"),
    "page_mxfp8": (18.9, "profiles/grouped_gemm_mxfp8_page_e32.md"),
}


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
    w_bytes = cfg.E * 3 * cfg.H * cfg.I * 2
    gemm_bytes = w_bytes + ns * cfg.H * 2 + 2 * ns * cfg.I * 2 + ns * cfg.H * 2  # weights, rows in, h out+in, fp16 out
    gather_bytes = cfg.T * cfg.H * 2 + ns * cfg.H * 2
    if cfg.mxfp8:
        # weights, token rows and h: E4M3 bytes plus one E8M0 scale per 32 values
        mx = 1.0 + 1.0 / 32
        w_bytes = cfg.E * 3 * cfg.H * cfg.I * mx
        gemm_bytes = w_bytes + ns * cfg.H * mx + 2 * ns * cfg.I * mx + ns * cfg.H * 2
        gather_bytes = cfg.T * cfg.H * 2 + ns * cfg.H * mx
    combine_bytes = ns * cfg.H * 2 + ns * 4 + cfg.T * cfg.H * 2
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


def run_mok(args, cfg, rank, world, device):
    import combine_device_top_b200 as mok

    torch.cuda.set_device(device)
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    dx, dlogits = x.to(device), logits.to(device)
    wg, wu, wd_bf16 = mokgen.upload_expert_weights(cfg, device)
    pack = None
    if cfg.mxfp8:
        # one-time MXFP8 weight quantisation, untimed
        pack = (*mok.quantize_weights_mxfp8(wg), *mok.quantize_weights_mxfp8(wu), *mok.quantize_weights_mxfp8(wd_bf16))
        del wg, wu, wd_bf16
        wg = wu = wd = None
        torch.cuda.empty_cache()
    else:
        wd = mok.prepare_w_down(wd_bf16)      # one-time weight preparation, untimed
        del wd_bf16
    x_shards = mok.shards(dx, cfg.R)
    y = torch.empty_like(dx)
    y_shards = mok.shards(y, cfg.R)
    mode = mok.MOK_MODE_STAGED if args.mode == "staged" else mok.MOK_MODE_PERSISTENT
    opts = mok.fwd_opts(mode=mode, ring_slots=cfg.ring_slots, mxfp8=cfg.mxfp8, dispatch_ctas=args.dispatch_ctas)
    minibatch = args.minibatch or cfg.minibatch
    p = mok.plan(dlogits, cfg.k, cfg.R)
    fws = torch.empty(mok.forward_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, minibatch, opts),
                      dtype=torch.uint8, device=device)
    # staged mode is timed one ABI step at a time (per-phase events)
    staged = mode == mok.MOK_MODE_STAGED
    if staged:
        out = torch.empty((cfg.slots, cfg.H), dtype=torch.float16, device=device)
        if cfg.mxfp8:
            rows_q = torch.empty((cfg.slots, cfg.H), dtype=torch.uint8, device=device)
            planes = torch.zeros((cfg.H // 128, mok.lib().mok_mxfp8_scale_rows(cfg.slots), 4), dtype=torch.uint8,
                                 device=device)
            ffn_ws = torch.empty(mok.lib().mok_expert_ffn_mxfp8_workspace_bytes(cfg.slots, cfg.I, cfg.E),
                                 dtype=torch.uint8, device=device)
        else:
            rows = torch.empty((cfg.slots, cfg.H), dtype=torch.bfloat16, device=device)
            ffn_ws = torch.empty(mok.lib().mok_expert_ffn_workspace_bytes(cfg.slots, cfg.I, cfg.E),
                                 dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    # A step in staged mode goes through the ABI one step at a time so that
    # each phase is bracketed by events; it runs the same kernels as
    # mok_moe_forward's staged mode.
    n_ev = 5 if staged else 3

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        mok.plan(dlogits, cfg.k, cfg.R, ws=p.ws)
        if evs:
            evs[1].record(stream)
        if staged:
            if pack is not None:
                mok.gather_mxfp8(x_shards, p, rows_q, planes)
            else:
                mok.gather(x_shards, p, rows)
            if evs:
                evs[2].record(stream)
            if pack is not None:
                mok.expert_ffn_mxfp8(rows_q, planes, pack, p, out=out, ws=ffn_ws)
            else:
                mok.expert_ffn(rows, wg, wu, wd, p, out=out, ws=ffn_ws)
            if evs:
                evs[3].record(stream)
            mok.combine(out, p, y_shards)
        elif pack is not None:
            mok.moe_forward_mxfp8(x_shards, pack, p, y_shards=y_shards, ws=fws, minibatch=minibatch, opts=opts)
        else:
            mok.moe_forward(x_shards, wg, wu, wd, p, minibatch, opts, y_shards=y_shards, ws=fws)
        if evs:
            evs[n_ev - 1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # correctness of the timed configuration is covered by tests; here only a sanity check
    if not torch.isfinite(y.float()).all():
        raise RuntimeError("non-finite output")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                      else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[torch.cuda.current_device()])) as clk:
        clk.mark_start()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
        clk.mark_stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(stop)
    phases = [[evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)] for j in range(n_ev - 1)]
    total_ms = max_over_ranks(total_ms, device)

    res = {"total_ms": total_ms, "phases_ms": [sum(ph) / len(ph) for ph in phases], "clocks": clk.summary()}

    # end to end from pinned host memory through mok_moe_forward_host
    if rank == 0 or world > 1:
        hx, hl = x.pin_memory(), logits.pin_memory()
        hy = torch.empty_like(x).pin_memory()
        wts = (pack, None, None) if pack is not None else (wg, wu, wd)
        hws = torch.empty(mok.forward_host_workspace_bytes(cfg.T, cfg.H, cfg.I, cfg.E, cfg.k, minibatch, opts),
                          dtype=torch.uint8, device=device)
        for _ in range(2):
            mok.moe_forward_host(hx, hl, cfg.k, cfg.R, *wts, minibatch, opts, hws, hy)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, min(args.steps, 5))
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            mok.moe_forward_host(hx, hl, cfg.k, cfg.R, *wts, minibatch, opts, hws, hy)
        e1.record(stream)
        torch.cuda.synchronize()
        res["e2e_ms"] = max_over_ranks(e0.elapsed_time(e1) / n_e2e, device)
        res["h2d"] = cfg.T * cfg.H * 2 + cfg.T * cfg.E * 4
        res["d2h"] = cfg.T * cfg.H * 2
        del hws
    # plan: top-k, rank, scan, scatter; staged forward: chunk list, gather, gate/up, down, combine;
    # persistent forward: chunk list, one persistent kernel
    res["launches_per_step"] = (4 + 1 + 1 + 2 + 1) if mode == mok.MOK_MODE_STAGED else (4 + 2)
    res["max_over_mean_load"] = (lambda c: c.max().item() / c.mean().item())(p.counts().float())
    return res


# ------------------------------------------------------------------ CPU oracle
def cpu_oracle_sample(cfg, budget_s: float = 12.0, threads: int = 0):
    """Oracle expert FFN on whole experts of the workload, experts 0, 1, ...
    until about budget_s seconds of CPU work, on `threads` host threads (0:
    every core this process may use); returns tokens/s (= rows/s / k)."""
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
    spent, rows_done, experts = 0.0, 0, 0
    for e in range(cfg.E):
        a, b = int(off[e]), int(off[e + 1])
        if b <= a:
            continue
        wg, wu, wd = mokgen.expert_weights(cfg, e)
        t0 = time.perf_counter()
        oracle.expert_ffn(rows_all[a:b], wg, wu, wd)
        spent += time.perf_counter() - t0
        rows_done += b - a
        experts += 1
        if spent >= budget_s:
            break
    # plan time is charged in proportion to the sampled rows
    t = spent + t_plan * rows_done / cfg.slots
    return {"value": (rows_done / cfg.k) / t, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"oracle SwiGLU FFN of experts 0..{experts - 1} ({rows_done} of {cfg.slots} rows) of the "
                      f"{cfg.name} workload plus its share of the full oracle plan; tokens/s = rows/s / k"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mok", choices=["mok", "reference"])
    ap.add_argument("--config", default="page", choices=list(mokgen.CONFIGS))
    ap.add_argument("--mode", default="staged", choices=["staged", "persistent"])
    ap.add_argument("--minibatch", type=int, default=0)
    ap.add_argument("--dispatch-ctas", type=int, default=0,
                    help="persistent mode: CTAs on the dispatch side (0: the library default, 16)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--scale-experts", type=int, default=0,
                    help="profiling case: E experts and T scaled by the same factor (same rows per expert)")
    args = ap.parse_args()
    cfg = mokgen.CONFIGS[args.config]
    if args.scale_experts:
        n = args.scale_experts
        T = max(cfg.R, round(cfg.T * n / cfg.E / cfg.R) * cfg.R)
        cfg = mokgen.scaled(cfg, E=n, T=T)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    # value is tokens/s; the tensor-core fraction and the gather/combine GB/s
    # of the same metric are in "roofline" and "phase_rates"
    metric = "MoE fwd tokens/s (H7168/I2048); % BF16 TC peak; gather/combine HBM GB/s"
    wdesc = ("MXFP8 E4M3 weights + E8M0 scales per 32 along K (quantised once, untimed)" if cfg.mxfp8
             else "bf16 weights [E,H,I]/[E,I,H]")
    config = {"workload": f"{cfg.name}: {cfg.describe()}, {wdesc}",
              "tokens_per_step_per_gpu": cfg.T, "minibatch": args.minibatch or cfg.minibatch,
              "mode": args.mode,
              **({"dispatch_ctas": args.dispatch_ctas or 16} if args.mode == "persistent" else {}),
              "l2": f"inputs larger than L2 ({algorithmic_work(cfg)['weight_bytes'] / 1e9:.1f} GB of expert "
                    f"weights streamed per step)"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = cpu_oracle_sample(cfg, args.cpu_budget)
        t_step_ms = cfg.T / cb["value"] * 1e3
        line = {"metric": metric, "value": cb["value"], "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step_ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "impl": "reference", "cpu_baseline": dict(cb),
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    device = torch.device("cuda", local_rank)
    res = run_mok(args, cfg, rank, world, device)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    work = algorithmic_work(cfg)
    ms = res["total_ms"] / args.steps
    value = job_rate(cfg.T, ms, world)
    ph = res["phases_ms"]
    line = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp8-e4m3 (bf16 MMA)" if cfg.mxfp8 else "bf16",
            "data": "synthetic", "config": config}
    if len(ph) == 4:
        t_plan, t_gather, t_gemm, t_comb = ph
        gemm_s = t_gemm / 1e3
        tflops = work["gemm_flops"] / gemm_s / 1e12
        gbs = work["gemm_bytes"] / gemm_s / 1e9
        # the MMA's own dtype peak: fp8 runs at twice the measured bf16 rate (nominal 4.5 / 2.25 PFLOP/s)
        tc_peak = peaks["bf16_tflops_sustained"] * (2.0 if cfg.mxfp8 else 1.0)
        t_tc = work["gemm_flops"] / (tc_peak * 1e12)
        t_hbm = work["gemm_bytes"] / (peaks["hbm_gbs"] * 1e9)
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / peaks["hbm_gbs"]}
        else:
            roof = {"bound": "tensor", "achieved": tflops, "peak": tc_peak,
                    "unit": "TFLOP/s", "frac": tflops / tc_peak}
        traffic = GEMM_TRAFFIC_GB_PER_STEP.get(cfg.name) if not args.scale_experts else None
        if traffic and args.mode != "staged" and not cfg.mxfp8:
            traffic = None
        roof.update({"traffic": traffic[0] * 1e9 if traffic else None,
                     "traffic_note": (f"bytes per step, both GEMM launches, scaled from {traffic[1]}" if traffic
                                      else "no capture of this workload"),
                     "kernel": "grouped GEMM (gate/up+SwiGLU and down launches)",
                     "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
                     "tensor_frac_of_bf16_peak": tflops / peaks["bf16_tflops_sustained"],
                     "tensor_frac_of_dtype_peak": tflops / tc_peak})
        line["roofline"] = roof
        line["phases_ms"] = {"plan": t_plan, "gather": t_gather, "grouped_gemm": t_gemm, "combine": t_comb}
        line["phase_rates"] = {
            "gather_GBps": work["gather_bytes"] / (t_gather / 1e3) / 1e9,
            "combine_GBps": work["combine_bytes"] / (t_comb / 1e3) / 1e9,
            "gemm_TFLOPs": tflops, "gemm_GBps": gbs,
            "plan_share": t_plan / ms,
        }
    else:
        # one mok_moe_forward call (gather, grouped GEMM and combine together) is the timed kernel work
        t_plan, t_fwd = ph
        fwd_s = t_fwd / 1e3
        gbs = work["forward_bytes"] / fwd_s / 1e9
        tflops = work["gemm_flops"] / fwd_s / 1e12
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                "kernel": "persistent forward kernel (dispatch, grouped GEMM, combine in one launch)",
                "peak_source": f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'})",
                "tensor_frac_of_bf16_peak": tflops / peaks["bf16_tflops_sustained"]}
        line["roofline"] = roof
        line["phases_ms"] = {"plan": t_plan, "forward": t_fwd}
        line["phase_rates"] = {"forward_GBps": gbs, "forward_TFLOPs": tflops, "plan_share": t_plan / ms}
    if "e2e_ms" in res:
        line["e2e"] = {"value": job_rate(cfg.T, res["e2e_ms"], world), "unit": "tokens/s",
                       "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]}
    line["gpu_launches"] = res["launches_per_step"] * args.steps
    if res["clocks"]:
        line["clocks"] = res["clocks"]
    line["expert_load_max_over_mean"] = res["max_over_mean_load"]
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_sample(cfg, args.cpu_budget)
        line["cpu_baseline_1thread"] = cpu_oracle_sample(cfg, args.cpu_budget / 2, threads=1)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
