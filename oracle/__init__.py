"""CPU oracle of the forward MoE layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (``combine_device_top_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``mok_oracle.c`` (forward), ``mxfp8_oracle.c``
(MXFP8 emulation), ``mok_oracle_bwd.c`` (backward) and
``mok_oracle_router.c`` (router projection): plain C, double
precision, compiled with gcc; this file is ctypes marshalling plus small
conveniences.  Each C
function cites the passage of the pages it follows.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against brute force, closed forms, invariants and textbook special cases.
The MXFP8 emulation is pinned by hand-computed bytes in ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from contextlib import contextmanager
from functools import lru_cache

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, f) for f in ("mok_oracle.c", "mxfp8_oracle.c", "mok_oracle_bwd.c",
                                           "mok_oracle_router.c")]
_SO = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` (gcc, OpenMP) next to the sources."""
    srcs = [s for s in _SRCS if os.path.exists(s)]
    newest = max(os.path.getmtime(s) for s in srcs)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < newest:
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", *CFLAGS, *srcs, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def build_from(srcs, out: str) -> str:
    """Compile the given copies of the oracle's C sources into ``out`` with
    the oracle's own flags (the planted-mistake tests build mutated copies)."""
    subprocess.check_call(["gcc", *CFLAGS, *srcs, "-o", out, "-lm"])
    return out


_override = None


def lib():
    """The oracle's C library: this package's build, or the one a
    :func:`library` block selected."""
    return _override if _override is not None else _own_lib()


@contextmanager
def library(path: str):
    """Run every oracle function inside the block on another build of the
    oracle's sources (test use: mutated copies)."""
    global _override
    prev = _override
    _override = _bind(ctypes.CDLL(path))
    try:
        yield
    finally:
        _override = prev


@lru_cache(maxsize=1)
def _own_lib():
    return _bind(ctypes.CDLL(build()))


def _bind(L):
    i32, vp = ctypes.c_int, ctypes.c_void_p
    L.oracle_topk_gates.argtypes = [vp, i32, i32, i32, vp, vp]
    L.oracle_schedule.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.oracle_gather.argtypes = [vp, i32, i32, i32, i32, vp, vp, vp]
    L.oracle_expert_ffn.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
    L.oracle_combine.argtypes = [vp, vp, i32, i32, i32, vp]
    L.oracle_moe_forward.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    L.oracle_num_threads.argtypes = []
    L.oracle_set_num_threads.argtypes = [i32]
    L.oracle_set_num_threads.restype = None
    if hasattr(L, "oracle_mxfp8_quantize"):
        L.oracle_mxfp8_quantize.argtypes = [vp, ctypes.c_int64, vp, vp]
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_mxfp8_expert_ffn.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    if hasattr(L, "oracle_router_logits"):
        L.oracle_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.oracle_router_logits.restype = ctypes.c_int
    if hasattr(L, "oracle_moe_backward"):
        L.oracle_moe_backward.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.oracle_moe_backward.restype = ctypes.c_int
    for name in ("oracle_topk_gates", "oracle_schedule", "oracle_gather", "oracle_expert_ffn",
                 "oracle_combine", "oracle_moe_forward", "oracle_num_threads"):
        getattr(L, name).restype = ctypes.c_int
    if hasattr(L, "oracle_mxfp8_quantize"):
        L.oracle_mxfp8_quantize.restype = ctypes.c_int
        L.oracle_mxfp8_expert_ffn.restype = ctypes.c_int
    return L


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if isinstance(t, torch.Tensor) else t.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _c(t: torch.Tensor, dtype) -> torch.Tensor:
    assert t.device.type == "cpu"
    return t.to(dtype).contiguous()


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def topk_gates(logits: torch.Tensor, k: int):
    """-> (topk_idx [T,k] int32, gates [T,k] fp32)."""
    logits = _c(logits, torch.float32)
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32)
    g = torch.empty((T, k), dtype=torch.float32)
    _check(lib().oracle_topk_gates(_ptr(logits), T, E, k, _ptr(idx), _ptr(g)), "topk_gates")
    return idx, g


def schedule(topk_idx: torch.Tensor, E: int, R: int):
    """-> dict(counts, offsets, src_rank, src_index, row_slot, pos) (int32)."""
    topk_idx = _c(topk_idx, torch.int32)
    T, k = topk_idx.shape
    ns = T * k
    out = dict(counts=torch.empty(E, dtype=torch.int32), offsets=torch.empty(E + 1, dtype=torch.int32),
               src_rank=torch.empty(ns, dtype=torch.int32), src_index=torch.empty(ns, dtype=torch.int32),
               row_slot=torch.empty(ns, dtype=torch.int32), pos=torch.empty(ns, dtype=torch.int32))
    _check(lib().oracle_schedule(_ptr(topk_idx), T, E, k, R, *(_ptr(out[n]) for n in
           ("counts", "offsets", "src_rank", "src_index", "row_slot", "pos"))), "schedule")
    return out


def plan(logits: torch.Tensor, k: int, R: int):
    idx, g = topk_gates(logits, k)
    p = schedule(idx, logits.shape[1], R)
    p["topk_idx"], p["gates"] = idx, g
    return p


def gather(x: torch.Tensor, R: int, src_rank: torch.Tensor, src_index: torch.Tensor) -> torch.Tensor:
    x = _c(x, torch.bfloat16)
    T, H = x.shape
    n = src_rank.numel()
    rows = torch.empty((n, H), dtype=torch.bfloat16)
    _check(lib().oracle_gather(_ptr(x), T, H, R, n, _ptr(_c(src_rank, torch.int32)),
                               _ptr(_c(src_index, torch.int32)), _ptr(rows)), "gather")
    return rows


def expert_ffn(x_rows: torch.Tensor, wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor) -> torch.Tensor:
    """One expert's SwiGLU FFN; bf16 inputs, float64 result [n, H]."""
    x_rows = _c(x_rows, torch.bfloat16)
    n, H = x_rows.shape
    I = wg.shape[1]
    o = torch.empty((n, H), dtype=torch.float64)
    _check(lib().oracle_expert_ffn(_ptr(x_rows), n, H, I, _ptr(_c(wg, torch.bfloat16)),
                                   _ptr(_c(wu, torch.bfloat16)), _ptr(_c(wd, torch.bfloat16)), _ptr(o)),
           "expert_ffn")
    return o


def mxfp8_expert_ffn(x_rows: torch.Tensor, wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor) -> torch.Tensor:
    """One expert's SwiGLU FFN on the MXFP8 path (x, weights and h quantised
    in 32-blocks, exact accumulation); bf16 inputs, float64 result [n, H]."""
    x_rows = _c(x_rows, torch.bfloat16)
    n, H = x_rows.shape
    I = wg.shape[1]
    o = torch.empty((n, H), dtype=torch.float64)
    _check(lib().oracle_mxfp8_expert_ffn(_ptr(x_rows), n, H, I, _ptr(_c(wg, torch.bfloat16)),
                                         _ptr(_c(wu, torch.bfloat16)), _ptr(_c(wd, torch.bfloat16)), _ptr(o),
                                         None, None, None), "mxfp8_expert_ffn")
    return o


def moe_forward_mxfp8(x, logits, wg, wu, wd, k: int, R: int):
    """Whole layer on the MXFP8 path (small inputs) -> y [T,H] float64."""
    T, H = x.shape
    E = wg.shape[0]
    p = plan(logits, k, R)
    rows = gather(x, R, p["src_rank"], p["src_index"])
    o_slot = torch.zeros((T * k, H), dtype=torch.float64)
    off = p["offsets"]
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            o_slot[p["row_slot"][a:b].long()] = mxfp8_expert_ffn(rows[a:b], wg[e], wu[e], wd[e])
    return combine(o_slot.view(T, k, H), p["gates"])


def combine(o_slot: torch.Tensor, gates: torch.Tensor) -> torch.Tensor:
    """o_slot [T,k,H] float64, gates [T,k] -> y [T,H] float64."""
    o_slot = _c(o_slot, torch.float64)
    T, k, H = o_slot.shape
    y = torch.empty((T, H), dtype=torch.float64)
    _check(lib().oracle_combine(_ptr(o_slot), _ptr(_c(gates, torch.float32)), T, k, H, _ptr(y)), "combine")
    return y


def moe_forward(x, logits, wg, wu, wd, k: int, R: int):
    """Whole layer on small inputs -> (y [T,H] float64, topk_idx, gates)."""
    x = _c(x, torch.bfloat16)
    logits = _c(logits, torch.float32)
    T, H = x.shape
    E, _, I = wg.shape
    y = torch.empty((T, H), dtype=torch.float64)
    idx = torch.empty((T, k), dtype=torch.int32)
    g = torch.empty((T, k), dtype=torch.float32)
    _check(lib().oracle_moe_forward(_ptr(x), _ptr(logits), T, H, I, E, k, R,
                                    _ptr(_c(wg, torch.bfloat16)), _ptr(_c(wu, torch.bfloat16)),
                                    _ptr(_c(wd, torch.bfloat16)), _ptr(y), _ptr(idx), _ptr(g)),
           "moe_forward")
    return y, idx, g


def router_logits(x, w_r, prior=None):
    """Router projection (``mok_oracle_router.c``): x bf16 [T,H], W_r fp32
    [H,E], optional fp32 prior [E] -> logits [T,E] float64."""
    x = _c(x, torch.bfloat16)
    w_r = _c(w_r, torch.float32)
    T, H = x.shape
    E = w_r.shape[1]
    out = torch.empty((T, E), dtype=torch.float64)
    pr = _c(prior, torch.float32) if prior is not None else None
    _check(lib().oracle_router_logits(_ptr(x), _ptr(w_r), _ptr(pr) if pr is not None else None, T, H, E,
                                      _ptr(out)), "router_logits")
    return out


def moe_backward(x, logits, wg, wu, wd, dy, k: int, R: int):
    """Backward of the whole layer on small inputs (``mok_oracle_bwd.c``):
    given dy [T,H], returns dict(dx [T,H], dwg, dwu [E,H,I], dwd [E,I,H],
    dlogits [T,E]), all float64."""
    x = _c(x, torch.bfloat16)
    logits = _c(logits, torch.float32)
    T, H = x.shape
    E, _, I = wg.shape
    out = dict(dx=torch.empty((T, H), dtype=torch.float64), dwg=torch.empty((E, H, I), dtype=torch.float64),
               dwu=torch.empty((E, H, I), dtype=torch.float64), dwd=torch.empty((E, I, H), dtype=torch.float64),
               dlogits=torch.empty((T, E), dtype=torch.float64))
    _check(lib().oracle_moe_backward(_ptr(x), _ptr(logits), T, H, I, E, k, R, _ptr(_c(wg, torch.bfloat16)),
                                     _ptr(_c(wu, torch.bfloat16)), _ptr(_c(wd, torch.bfloat16)),
                                     _ptr(_c(dy, torch.float64)), *(_ptr(out[n]) for n in
                                     ("dx", "dwg", "dwu", "dwd", "dlogits"))), "moe_backward")
    return out


def forward_tokens(cfg, x, logits, token_ids, weight_fn, k=None):
    """y rows for a subset of tokens of a large configuration.

    ``weight_fn(e)`` returns (Wg, Wu, Wd) of expert e on the host; only the
    experts these tokens select are materialised.  Routing uses the full-T
    oracle plan restricted to the chosen tokens (a token's selection and
    gates depend on its own logits only).
    """
    k = cfg.k if k is None else k
    token_ids = torch.as_tensor(token_ids, dtype=torch.int64)
    idx, g = topk_gates(logits[token_ids], k)
    n = token_ids.numel()
    o_slot = torch.zeros((n, k, cfg.H), dtype=torch.float64)
    xs = x[token_ids].contiguous()
    need = {}
    for a in range(n):
        for j in range(k):
            need.setdefault(int(idx[a, j]), []).append((a, j))
    for e, uses in sorted(need.items()):
        wg, wu, wd = weight_fn(e)
        rows = torch.stack([xs[a] for a, _ in uses])
        o = expert_ffn(rows, wg, wu, wd)
        for r, (a, j) in enumerate(uses):
            o_slot[a, j] = o[r]
    return combine(o_slot, g), idx, g
