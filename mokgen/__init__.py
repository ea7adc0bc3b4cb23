"""Seeded synthetic inputs for the MoE forward layer.

This module is shared by the tests, ``bench.py`` and ``__graft_entry__``.  It
generates inputs only; it holds none of the layer's arithmetic (no top-k, no
gates, no schedule, no FFN, no combine).  Both the CUDA path and the oracle
receive exactly the arrays produced here.

Distributions.  Gaussian tensors are drawn through a 65536-entry table of
normal quantiles ``std * Phi^-1((i + 0.5) / 65536)`` rounded once to the
payload type (bf16 or fp32), indexed by a counter-based SplitMix64 stream
(``mokgen.c``).  At bf16 resolution this is a Gaussian truncated at about
4.3 sigma.  Every tensor is addressed by ``(seed, stream)`` with the stream id
derived from the config, the tensor name and the expert, so one expert's
weights can be regenerated on demand without materialising the others.

Workload shapes follow the five configurations of the forward-layer study:
a tiny layer, a Mixtral-shaped layer, the page shape (hidden 7168,
intermediate 2048, 384 experts, top-8), an imbalanced Zipf(1.2) routing case
and the MXFP8 variant of the page shape.
"""
from __future__ import annotations

import ctypes
import hashlib
import math
import os
import subprocess
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mokgen.c")
_SO = os.path.join(_HERE, "libmokgen.so")

CFLAGS = ["-O3", "-march=x86-64-v3", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    """Compile ``libmokgen.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp])
        os.replace(tmp, _SO)
    return _SO


@lru_cache(maxsize=1)
def _lib():
    lib = ctypes.CDLL(build())
    u64, vp = ctypes.c_uint64, ctypes.c_void_p
    for name in ("mokgen_fill_u16", "mokgen_fill_u32"):
        f = getattr(lib, name)
        f.argtypes = [u64, u64, u64, u64, vp, vp]
        f.restype = None
    lib.mokgen_fill_idx16.argtypes = [u64, u64, u64, u64, vp]
    lib.mokgen_fill_idx16.restype = None
    return lib


def stream_id(*parts) -> int:
    """Deterministic 64-bit stream id from a tuple of names/numbers."""
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little")


@lru_cache(maxsize=64)
def _normal_table(std: float, dtype: str) -> np.ndarray:
    from scipy.special import ndtri

    q = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0) * float(std)
    t = torch.from_numpy(q.astype(np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().view(np.uint32).copy()


def normal(seed: int, stream: int, shape, std: float = 1.0, dtype=torch.bfloat16,
           first: int = 0, out: torch.Tensor | None = None) -> torch.Tensor:
    """Gaussian tensor (CPU) of ``shape``; element j is stream position first+j."""
    n = int(np.prod(shape))
    if dtype == torch.bfloat16:
        tab = _normal_table(float(std), "bf16")
        if out is None:
            out = torch.empty(shape, dtype=torch.bfloat16)
        assert out.is_contiguous() and out.dtype == torch.bfloat16 and out.numel() == n
        _lib().mokgen_fill_u16(seed, stream, first, n, tab.ctypes.data, out.data_ptr())
        return out
    if dtype == torch.float32:
        tab = _normal_table(float(std), "f32")
        if out is None:
            out = torch.empty(shape, dtype=torch.float32)
        assert out.is_contiguous() and out.dtype == torch.float32 and out.numel() == n
        _lib().mokgen_fill_u32(seed, stream, first, n, tab.ctypes.data, out.data_ptr())
        return out
    raise TypeError(dtype)


def small_ints(seed: int, stream: int, shape, levels: int) -> torch.Tensor:
    """Integer-valued fp32 tensor with values in [0, levels) (tie-heavy logits)."""
    n = int(np.prod(shape))
    raw = np.empty(n, dtype=np.uint16)
    _lib().mokgen_fill_idx16(seed, stream, 0, n, raw.ctypes.data)
    return torch.from_numpy((raw % levels).astype(np.float32).reshape(shape))


# --------------------------------------------------------------------------
# Workload configurations
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens
    H: int          # hidden
    I: int          # expert intermediate
    E: int          # experts
    k: int          # top-k
    R: int          # logical source shards of the token tensor
    seed: int
    zipf_s: float = 0.0          # >0: add log Zipf(s) expert prior to the logits
    mxfp8: bool = False
    ring_slots: int = 0          # 0: library default
    minibatch: int = 2560
    minibatch_sweep: tuple = field(default=())

    @property
    def slots(self) -> int:
        return self.T * self.k

    @property
    def S_r(self) -> int:
        return self.T // self.R

    def describe(self) -> str:
        return (f"T{self.T} H{self.H} I{self.I} E{self.E} k{self.k} R{self.R}"
                + (f" zipf{self.zipf_s}" if self.zipf_s else "") + (" mxfp8" if self.mxfp8 else ""))


CONFIGS = {
    "tiny": MoEConfig("tiny", T=256, H=512, I=256, E=8, k=2, R=2, seed=0, minibatch=256),
    "mixtral": MoEConfig("mixtral", T=4096, H=4096, I=14336, E=8, k=2, R=8, seed=1, minibatch=2048),
    "page": MoEConfig("page", T=8192, H=7168, I=2048, E=384, k=8, R=8, seed=2,
                      ring_slots=2 * 4096, minibatch=2560,
                      minibatch_sweep=(512, 1024, 2048, 2560, 4096)),
    "zipf": MoEConfig("zipf", T=16384, H=7168, I=2048, E=256, k=8, R=16, seed=3, zipf_s=1.2,
                      ring_slots=8192, minibatch=2560),
    "page_mxfp8": MoEConfig("page_mxfp8", T=8192, H=7168, I=2048, E=384, k=8, R=8, seed=4,
                            mxfp8=True, ring_slots=2 * 4096, minibatch=2560),
}
CONFIG_ORDER = ["tiny", "mixtral", "page", "zipf", "page_mxfp8"]


def scaled(cfg: MoEConfig, **kw) -> MoEConfig:
    """A copy of ``cfg`` with some fields replaced (reduced-size test cases)."""
    d = dict(cfg.__dict__)
    d.update(kw)
    return MoEConfig(**d)


# --------------------------------------------------------------------------
# Tensors of one configuration
# --------------------------------------------------------------------------
def tokens(cfg: MoEConfig) -> torch.Tensor:
    """x [T, H] bf16 ~ N(0, 1); shard r is rows [r*S_r, (r+1)*S_r)."""
    return normal(cfg.seed, stream_id(cfg.name, "x"), (cfg.T, cfg.H), 1.0)


def router_weight(cfg: MoEConfig) -> torch.Tensor:
    """W_r [H, E] fp32 ~ N(0, 1/H)."""
    return normal(cfg.seed, stream_id(cfg.name, "w_router"), (cfg.H, cfg.E),
                  1.0 / math.sqrt(cfg.H), dtype=torch.float32)


def zipf_log_prior(E: int, s: float) -> torch.Tensor:
    """log of a Zipf(s) expert prior, rank = e + 1 (normalised)."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return torch.from_numpy(np.log(p).astype(np.float32))


def router_logits(cfg: MoEConfig, x: torch.Tensor | None = None) -> torch.Tensor:
    """fp32 logits [T, E] = float(x) @ W_r (+ log Zipf prior), computed once on the host.

    The router projection is input preparation: the same fp32 array is handed
    to the GPU path and to the oracle, so the selection can be compared bit
    for bit.
    """
    if x is None:
        x = tokens(cfg)
    logits = x.float() @ router_weight(cfg)
    if cfg.zipf_s:
        logits += zipf_log_prior(cfg.E, cfg.zipf_s)[None, :]
    return logits.contiguous()


def expert_weights(cfg: MoEConfig, e: int):
    """(Wg [H,I], Wu [H,I], Wd [I,H]) of expert e, bf16 ~ N(0, 1/fan_in)."""
    wg = normal(cfg.seed, stream_id(cfg.name, "w_gate", e), (cfg.H, cfg.I), 1.0 / math.sqrt(cfg.H))
    wu = normal(cfg.seed, stream_id(cfg.name, "w_up", e), (cfg.H, cfg.I), 1.0 / math.sqrt(cfg.H))
    wd = normal(cfg.seed, stream_id(cfg.name, "w_down", e), (cfg.I, cfg.H), 1.0 / math.sqrt(cfg.I))
    return wg, wu, wd


def all_expert_weights(cfg: MoEConfig):
    """Stacked host weights [E,H,I], [E,H,I], [E,I,H] (small configs only)."""
    wg = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16)
    wu = torch.empty_like(wg)
    wd = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16)
    for e in range(cfg.E):
        a, b, c = expert_weights(cfg, e)
        wg[e], wu[e], wd[e] = a, b, c
    return wg, wu, wd


def upload_expert_weights(cfg: MoEConfig, device, chunk: int = 8):
    """Generate all expert weights on the host, a few experts at a time, and
    copy them into freshly allocated device tensors [E,H,I], [E,H,I], [E,I,H]."""
    wg = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16, device=device)
    wu = torch.empty_like(wg)
    wd = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=device)
    for e0 in range(0, cfg.E, chunk):
        e1 = min(cfg.E, e0 + chunk)
        hg = torch.empty((e1 - e0, cfg.H, cfg.I), dtype=torch.bfloat16).pin_memory()
        hu = torch.empty_like(hg).pin_memory()
        hd = torch.empty((e1 - e0, cfg.I, cfg.H), dtype=torch.bfloat16).pin_memory()
        for e in range(e0, e1):
            a, b, c = expert_weights(cfg, e)
            hg[e - e0], hu[e - e0], hd[e - e0] = a, b, c
        wg[e0:e1].copy_(hg, non_blocking=True)
        wu[e0:e1].copy_(hu, non_blocking=True)
        wd[e0:e1].copy_(hd, non_blocking=True)
        torch.cuda.current_stream(device).synchronize()
    return wg, wu, wd
