"""Shared helpers for the parity tests (inputs from mokgen, expectations from oracle)."""
from __future__ import annotations

import math

import torch

import mokgen
import oracle

# Tolerances for bf16 outputs (forward layer): relative Frobenius error and
# max abs error relative to rms(y).
REL_FRO_BF16 = 5e-3
MAX_ABS_BF16 = 2e-2
GATES_ATOL = 2e-6


def has_gpu() -> bool:
    return torch.cuda.is_available()


def rel_fro(a: torch.Tensor, b: torch.Tensor) -> float:
    a, b = a.double(), b.double()
    return (torch.linalg.norm(a - b) / torch.linalg.norm(b)).item()


def bf16_half_ulp(v: torch.Tensor) -> torch.Tensor:
    """Half the spacing of the bf16 numbers in the binade of each |v|: the
    most that rounding a real number to the nearest bf16 value ``v`` can
    have moved it (round to nearest never lands in a lower binade than its
    input, so the spacing at the rounded value bounds the move).  bf16 keeps
    8 significant bits, so the spacing in [2^e, 2^(e+1)) is 2^(e-7)."""
    a = v.double().abs().clamp_min(2.0 ** -126)     # bf16 subnormals share the spacing of 2^-126
    return torch.exp2(torch.floor(torch.log2(a)) - 8)


def max_abs_over_rms(a: torch.Tensor, b: torch.Tensor) -> float:
    """Literal max |a - b| / rms(b)."""
    a, b = a.double(), b.double()
    rms = torch.sqrt(torch.mean(b * b)).item()
    return ((a - b).abs().max().item()) / rms


def max_abs_beyond_rounding(got: torch.Tensor, want: torch.Tensor) -> float:
    """max over elements of (|got - want| - the rounding of got to its own
    output type)+ / rms(want).  For bf16 ``got`` this is the error the
    computation made before its final rounding to bf16 (at least); for wider
    types nothing is subtracted.

    The max-abs bound for bf16 outputs is read this way because rounding
    the EXACT result to bf16 alone already moves it by up to 2^-8 |y|: an
    element with |y| >= 2^e > 5.12 rms(y) that lies near a rounding midpoint
    is off by more than 2e-2 rms(y) with no computation error at all.  The
    full zipf-shaped layer (T 16384, H 7168, E 256, k 8) has 64 such
    elements (the exact result rounded to bf16 is 2.5e-2 rms(y) off); no
    bf16 output can meet the literal bound there."""
    g, w = got.double(), want.double()
    rms = torch.sqrt(torch.mean(w * w)).item()
    err = (g - w).abs()
    if got.dtype == torch.bfloat16:
        err = (err - bf16_half_ulp(g)).clamp_min(0.0)
    return err.max().item() / rms


def assert_bf16_close(got: torch.Tensor, want: torch.Tensor, what: str = ""):
    """Relative Frobenius error <= 5e-3 and max abs error <= 2e-2 rms(want),
    the max taken beyond the output's own final rounding (see
    :func:`max_abs_beyond_rounding`)."""
    rf, ma = rel_fro(got, want), max_abs_beyond_rounding(got, want)
    lit = max_abs_over_rms(got, want)
    assert rf <= REL_FRO_BF16, f"{what}: relative Frobenius {rf:.3e} > {REL_FRO_BF16}"
    assert ma <= MAX_ABS_BF16, f"{what}: max abs beyond rounding / rms {ma:.3e} > {MAX_ABS_BF16} (literal {lit:.3e})"
    return rf, ma


def decode_slots(buf: torch.Tensor, n: int, H: int) -> torch.Tensor:
    """fp32 values [n, H] of a MOK_SLOTS_F16S slot buffer (uint8): fp16 values
    times 2^s, one int8 exponent s per 128-feature block of a row."""
    import combine_device_top_b200 as mok

    b = buf.cpu()
    off = mok.lib().mok_slot_exp_offset(n, H)
    v = b[: n * H * 2].view(torch.float16).view(n, H).double()
    e = b[off: off + n * (H // 128)].view(torch.int8).view(n, H // 128).double()
    return v * torch.exp2(e).repeat_interleave(128, dim=1)


def encode_slots(x: torch.Tensor) -> torch.Tensor:
    """MOK_SLOTS_F16S buffer (uint8) of x [n, H]: per 128-feature block of a
    row, s = floor(log2 max|x|) - 14 clamped to [-126, 126] (0 for an
    all-zero block), values fp16(x * 2^-s)."""
    import combine_device_top_b200 as mok

    n, H = x.shape
    xb = x.double().view(n, H // 128, 128)
    m = xb.abs().amax(dim=2)
    s = torch.where(m > 0, torch.floor(torch.log2(m.clamp_min(1e-300))) - 14, torch.zeros_like(m)).clamp(-126, 126)
    v = (xb * torch.exp2(-s)[..., None]).view(n, H).to(torch.float16)
    off = mok.lib().mok_slot_exp_offset(n, H)
    buf = torch.zeros(mok.lib().mok_slot_bytes(n, H, mok.MOK_SLOTS_F16S), dtype=torch.uint8)
    buf[: n * H * 2] = v.view(-1).view(torch.uint8)
    buf[off: off + n * (H // 128)] = s.to(torch.int8).view(-1).view(torch.uint8)
    return buf


class Case:
    """Inputs of one configuration, on the host and on the device."""

    def __init__(self, cfg: mokgen.MoEConfig, device="cuda", weights_on_host: bool = True):
        self.cfg = cfg
        self.x = mokgen.tokens(cfg)
        self.logits = mokgen.router_logits(cfg, self.x)
        self.device = device
        if weights_on_host:
            self.wg, self.wu, self.wd = mokgen.all_expert_weights(cfg)
            self.dwg, self.dwu, dwd = (w.to(device) for w in (self.wg, self.wu, self.wd))
        else:
            self.wg = self.wu = self.wd = None
            self.dwg, self.dwu, dwd = mokgen.upload_expert_weights(cfg, device)
        self.dwd = dwd
        self.dx = self.x.to(device)
        self.dlogits = self.logits.to(device)

    def weight_fn(self, e):
        if self.wg is not None:
            return self.wg[e], self.wu[e], self.wd[e]
        return mokgen.expert_weights(self.cfg, e)

    def x_shards(self):
        R = self.cfg.R
        return list(self.dx.view(R, self.cfg.T // R, self.cfg.H).unbind(0))

    def oracle_y(self, token_ids=None):
        """Oracle y (float64) on all tokens (small configs) or a subset."""
        if token_ids is None and self.wg is not None:
            y, _, _ = oracle.moe_forward(self.x, self.logits, self.wg, self.wu, self.wd, self.cfg.k, self.cfg.R)
            return y
        y, _, _ = oracle.forward_tokens(self.cfg, self.x, self.logits, token_ids, self.weight_fn)
        return y


def sample_tokens(T: int, n: int, seed: int = 0) -> list[int]:
    g = torch.Generator().manual_seed(seed)
    ids = torch.randperm(T, generator=g)[:n].tolist()
    return sorted(set(ids + [0, T - 1]))


def topk_within_tolerance(idx: torch.Tensor, exact: torch.Tensor, tol: torch.Tensor):
    """Check a top-k selection made from rounded logits against exact ones.

    idx [T, k] (rank order), exact [T, E] float64, tol [T] float64: the
    largest difference rounding may cause between two logits of a token.
    Where exact logits lie within tol of each other either order is
    correct; everywhere else the selection and its order are fixed.
    Returns (ok [T], strict [T]): ok = the selection is one of the correct
    ones (k distinct experts, none left out that beats a chosen one by more
    than tol, rank order non-increasing up to tol); strict = the token has a
    single correct selection (every gap that decides it exceeds tol), so it
    must equal the exact top-k with the lower-index tie rule.
    """
    T, k = idx.shape
    E = exact.shape[1]
    idx = idx.long()
    sel = torch.gather(exact, 1, idx)                                  # [T, k]
    chosen = torch.zeros(T, E, dtype=torch.bool).scatter_(1, idx, True)
    distinct = chosen.sum(1) == k
    rest_max = torch.where(chosen, torch.full_like(exact, -math.inf), exact).max(1).values
    kth = sel.min(1).values
    order_ok = (sel[:, :-1] >= sel[:, 1:] - tol[:, None]).all(1) if k > 1 else torch.ones(T, dtype=torch.bool)
    ok = distinct & (kth >= rest_max - tol) & order_ok
    gaps_ok = ((sel[:, :-1] - sel[:, 1:]).abs() > tol[:, None]).all(1) if k > 1 else torch.ones(T, dtype=torch.bool)
    strict = ok & (kth > rest_max + tol) & gaps_ok
    return ok, strict
