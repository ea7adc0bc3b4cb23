"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test fixes a part of the oracle through an independent route: brute
force on tiny inputs, a closed form, a textbook special case evaluated with
library routines, invariants the pages fix, or hand-computed bytes stored
under tests/golden/.  A plausible mistake in the oracle (a dropped term, a
wrong index, a transposed operand, a wrong tie rule) fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import mokgen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(T, H, I, E, k, R, seed, std_w=None):
    cfg = mokgen.MoEConfig("pin", T=T, H=H, I=I, E=E, k=k, R=R, seed=seed)
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    wg, wu, wd = mokgen.all_expert_weights(cfg)
    return cfg, x, logits, wg, wu, wd


# ---------------------------------------------------------------- top-k / gates
@pytest.mark.parametrize("E,k,levels", [(8, 2, 3), (8, 3, 2), (384, 8, 3), (256, 8, 5), (16, 16, 2)])
def test_topk_matches_full_sort_with_ties(E, k, levels):
    """Selection = first k of the order (logit desc, index asc); tie-heavy logits."""
    T = 64
    logits = mokgen.small_ints(7, mokgen.stream_id("ties", E, k), (T, E), levels)
    idx, _ = oracle.topk_gates(logits, k)
    for t in range(T):
        l = logits[t].tolist()
        want = sorted(range(E), key=lambda e: (-l[e], e))[:k]
        assert idx[t].tolist() == want


def test_gates_invariants():
    """Gates are a softmax over the selected logits: positive, sum to one,
    non-increasing in rank, and g_a / g_b = exp(l_a - l_b)."""
    cfg, x, logits, *_ = _rand_case(128, 64, 32, 24, 6, 2, seed=11)
    idx, g = oracle.topk_gates(logits, cfg.k)
    assert (g > 0).all()
    assert torch.allclose(g.double().sum(1), torch.ones(cfg.T, dtype=torch.float64), atol=1e-6)
    assert (g[:, :-1] >= g[:, 1:]).all()
    sel = torch.gather(logits, 1, idx.long()).double()
    ratio = g[:, 0:1].double() / g.double()
    assert torch.allclose(ratio, torch.exp(sel[:, 0:1] - sel), rtol=1e-6)


def test_gates_equal_renormalised_full_softmax():
    """Softmax over the k = full softmax restricted to the k and renormalised."""
    cfg, x, logits, *_ = _rand_case(64, 64, 32, 16, 4, 1, seed=12)
    idx, g = oracle.topk_gates(logits, cfg.k)
    full = torch.softmax(logits.double(), dim=1)
    sub = torch.gather(full, 1, idx.long())
    assert torch.allclose(g.double(), sub / sub.sum(1, keepdim=True), atol=1e-7)


# ---------------------------------------------------------------- schedule
@pytest.mark.parametrize("T,E,k,R", [(256, 8, 2, 2), (512, 384, 8, 8), (96, 5, 5, 3), (64, 256, 8, 16)])
def test_schedule_is_stable_counting_sort(T, E, k, R):
    cfg = mokgen.MoEConfig("sched", T=T, H=64, I=64, E=E, k=k, R=R, seed=5)
    logits = mokgen.normal(5, mokgen.stream_id("sched", T, E), (T, E), 1.0, dtype=torch.float32)
    p = oracle.plan(logits, k, R)
    topk = p["topk_idx"].reshape(-1).numpy()
    ns = T * k
    # counts / offsets
    assert p["counts"].sum().item() == ns
    assert np.array_equal(p["counts"].numpy(), np.bincount(topk, minlength=E))
    assert p["offsets"][0] == 0 and p["offsets"][-1] == ns
    assert np.array_equal(np.diff(p["offsets"].numpy()), p["counts"].numpy())
    # row order = library stable sort of the slots (t-major) by expert
    order = np.argsort(topk, kind="stable")
    assert np.array_equal(p["row_slot"].numpy(), order)
    # pos is the inverse permutation; src = divmod(t, S_r)
    assert np.array_equal(p["pos"].numpy()[order], np.arange(ns))
    t = order // k
    assert np.array_equal(p["src_rank"].numpy(), t // (T // R))
    assert np.array_equal(p["src_index"].numpy(), t % (T // R))
    # each token appears k times at k distinct experts
    assert all(len(set(row)) == k for row in p["topk_idx"].tolist())


def test_schedule_segments_ascending_tokens():
    T, E, k, R = 300, 12, 3, 4
    logits = mokgen.small_ints(3, 99, (T, E), 4)
    p = oracle.plan(logits, k, R)
    tok = p["row_slot"].numpy() // k
    off = p["offsets"].numpy()
    for e in range(E):
        seg = tok[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert all(e in p["topk_idx"][tt].tolist() for tt in seg)


def test_gather_is_the_schedule_copy():
    cfg, x, logits, *_ = _rand_case(96, 64, 32, 6, 2, 3, seed=8)
    p = oracle.plan(logits, cfg.k, cfg.R)
    rows = oracle.gather(x, cfg.R, p["src_rank"], p["src_index"])
    t = (p["row_slot"] // cfg.k).long()
    assert torch.equal(rows, x[t])


# ---------------------------------------------------------------- FFN / layer
def _swiglu_ref(xr, wg, wu, wd):
    """Textbook SwiGLU FFN with torch library ops in float64."""
    xr, wg, wu, wd = (a.double() for a in (xr, wg, wu, wd))
    return (torch.nn.functional.silu(xr @ wg) * (xr @ wu)) @ wd


def test_single_expert_is_dense_swiglu():
    """E = 1, k = 1: the gate is 1 and the layer is a dense SwiGLU FFN."""
    cfg, x, logits, wg, wu, wd = _rand_case(48, 96, 64, 1, 1, 2, seed=21)
    y, idx, g = oracle.moe_forward(x, logits, wg, wu, wd, 1, cfg.R)
    assert torch.all(idx == 0) and torch.all(g == 1.0)
    ref = _swiglu_ref(x, wg[0], wu[0], wd[0])
    assert torch.allclose(y, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("E,k", [(8, 2), (6, 3), (4, 4)])
def test_brute_force_four_tokens(E, k):
    """T = 4: evaluate every expert densely on every token, mask by the
    top-k, weight by the renormalised softmax."""
    cfg, x, logits, wg, wu, wd = _rand_case(4, 64, 48, E, k, 2, seed=30 + E)
    y, _, _ = oracle.moe_forward(x, logits, wg, wu, wd, k, cfg.R)
    dense = torch.stack([_swiglu_ref(x, wg[e], wu[e], wd[e]) for e in range(E)], 1)  # [T,E,H]
    l = logits.double()
    want = torch.zeros_like(y)
    for t in range(4):
        sel = sorted(range(E), key=lambda e: (-l[t, e].item(), e))[:k]
        mask = torch.zeros(E, dtype=torch.float64)
        mask[sel] = 1.0
        w = torch.exp(l[t] - l[t].max()) * mask
        w = (w / w.sum()).float().double()      # gates are an fp32 output
        want[t] = (w[:, None] * dense[t]).sum(0)
    assert torch.allclose(y, want, rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("H,I", [(64, 32), (32, 64), (128, 128)])
def test_scaled_identity_closed_form(H, I):
    """Wg = [I_m; 0], Wu = s_e [I_m; 0], Wd = [I_m | 0], s_e = e + 1:
    y[t,c] = (sum_j g[t,j] s_sel(t,j)) * x_c * silu(x_c) for c < m, else 0."""
    T, E, k, R = 40, 5, 2, 4
    m = min(H, I)
    cfg = mokgen.MoEConfig("ident", T=T, H=H, I=I, E=E, k=k, R=R, seed=41)
    x = mokgen.tokens(cfg)
    logits = mokgen.router_logits(cfg, x)
    eye = torch.zeros(H, I)
    eye[:m, :m] = torch.eye(m)
    wg = eye.expand(E, H, I).to(torch.bfloat16).contiguous()
    wu = torch.stack([(e + 1) * eye for e in range(E)]).to(torch.bfloat16)
    wd = eye.t().expand(E, I, H).to(torch.bfloat16).contiguous()
    y, idx, g = oracle.moe_forward(x, logits, wg, wu, wd, k, R)
    scale = (g.double() * (idx.double() + 1)).sum(1)                 # sum_j g s_e
    xd = x.double()
    want = torch.zeros(T, H, dtype=torch.float64)
    xm = xd[:, :m]
    want[:, :m] = scale[:, None] * xm * (xm / (1 + torch.exp(-xm)))
    assert torch.allclose(y, want, rtol=1e-12, atol=1e-14)


def test_combine_is_weighted_sum():
    T, k, H = 7, 3, 16
    o = torch.randn(T, k, H, dtype=torch.float64, generator=torch.Generator().manual_seed(0))
    g = torch.rand(T, k, generator=torch.Generator().manual_seed(1))
    y = oracle.combine(o, g)
    assert torch.allclose(y, torch.einsum("tk,tkh->th", g.double(), o), rtol=1e-14)


def test_forward_tokens_subset_matches_full_layer():
    """The large-config helper (subset of tokens, experts on demand) equals
    the full small layer on the same tokens."""
    cfg, x, logits, wg, wu, wd = _rand_case(64, 64, 64, 8, 2, 2, seed=51)
    y, _, _ = oracle.moe_forward(x, logits, wg, wu, wd, cfg.k, cfg.R)
    ids = [0, 5, 17, 63]
    ys, _, _ = oracle.forward_tokens(cfg, x, logits, ids, lambda e: (wg[e], wu[e], wd[e]))
    assert torch.allclose(ys, y[ids], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- MXFP8
def _quant(v):
    L = oracle.lib()
    v = np.ascontiguousarray(v, dtype=np.float32)
    nb = v.size // 32
    q = np.zeros(v.size, np.uint8)
    s = np.zeros(nb, np.uint8)
    assert L.oracle_mxfp8_quantize(v.ctypes.data, nb, q.ctypes.data, s.ctypes.data) == 0
    return q, s


def test_mxfp8_golden_blocks():
    with open(os.path.join(GOLDEN, "mxfp8_blocks.json")) as f:
        spec = json.load(f)
    for case in spec["cases"]:
        v = np.zeros(32, np.float32)
        for i, val in case["values"].items():
            v[int(i)] = val
        q, s = _quant(v)
        assert s[0] == int(case["scale"], 16), case["name"]
        for i in range(32):
            want = int(case["bytes"].get(str(i), "0x80" if (v[i] == 0 and math.copysign(1, v[i]) < 0) else "0x00"), 16)
            assert q[i] == want, (case["name"], i, hex(q[i]), hex(want))


def test_e4m3_all_codes_round_trip():
    """Every finite E4M3 code decodes and re-encodes to itself (scale 2^0)."""
    L = oracle.lib()
    for b in range(256):
        if (b & 0x7F) == 0x7F:        # NaN codes
            assert math.isnan(L.oracle_e4m3_decode(b))
            continue
        v = np.zeros(32, np.float32)
        v[0] = 448.0                  # pins the block exponent to 0
        v[1] = L.oracle_e4m3_decode(b)
        q, s = _quant(v)
        assert s[0] == 127 and q[1] == b


def test_e4m3_decode_table_values():
    """Spot values of the E4M3 grid from its definition."""
    L = oracle.lib()
    assert L.oracle_e4m3_decode(0x7E) == 448.0
    assert L.oracle_e4m3_decode(0x08) == 2.0 ** -6
    assert L.oracle_e4m3_decode(0x01) == 2.0 ** -9
    assert L.oracle_e4m3_decode(0x38) == 1.0
    assert L.oracle_e4m3_decode(0xB8) == -1.0
    vals = sorted(L.oracle_e4m3_decode(b) for b in range(0x7F))
    assert len(set(vals)) == 127 and vals[-1] == 448.0


def test_e4m3_midpoints_round_to_even():
    """Round half to even, from the grid alone: the midpoint of two adjacent
    positive E4M3 values (scale 2^0) encodes to the neighbour whose code is
    even, and a point just off the midpoint to the nearer neighbour."""
    L = oracle.lib()
    codes = sorted(range(0x7F), key=L.oracle_e4m3_decode)   # 0x00 .. 0x7E ascending
    for lo, hi in zip(codes[:-1], codes[1:]):
        a, b = L.oracle_e4m3_decode(lo), L.oracle_e4m3_decode(hi)
        mid = (a + b) / 2
        eps = (b - a) / 8
        v = np.zeros(32 * 3, np.float32)
        v[0::32] = 448.0                  # every block's exponent is 0
        v[1], v[33], v[65] = mid, mid - eps, mid + eps
        q, s = _quant(v)
        assert (s == 127).all()
        assert q[1] == (lo if lo % 2 == 0 else hi), (hex(lo), hex(hi))
        assert q[33] == lo and q[65] == hi, (hex(lo), hex(hi))


def test_mxfp8_relative_error_bound():
    """Non-saturated elements above the subnormal range are within 2^-4
    relative of the input (3 mantissa bits, round to nearest)."""
    rng = np.random.default_rng(0)
    v = rng.standard_normal(32 * 256).astype(np.float32) * np.repeat(rng.uniform(1e-3, 1e3, 256), 32).astype(np.float32)
    q, s = _quant(v)
    L = oracle.lib()
    dec = np.array([L.oracle_e4m3_decode(int(b)) for b in q]) * np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32)
    scaled = np.abs(v) / np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32)
    ok = (scaled >= 2.0 ** -6) & (scaled <= 448)
    rel = np.abs(dec[ok] - v[ok]) / np.abs(v[ok])
    assert rel.max() <= 2.0 ** -4


def test_mxfp8_ffn_exact_on_representable_inputs():
    """With x and the weights already on the MXFP8 grid (block maxima fix the
    scale, entries are E4M3 values), the quantisation of x and W is the
    identity, so the GEMMs are exact; h is quantised once."""
    n, H, I = 3, 64, 64
    rng = np.random.default_rng(1)
    L = oracle.lib()
    grid = np.array([L.oracle_e4m3_decode(b) for b in range(0x7F)])
    def grid_tensor(shape, scale, along_rows):
        a = rng.choice(grid[grid <= 64], size=shape) * rng.choice([-1, 1], size=shape)
        a = a * scale
        if along_rows:
            a[::32, :] = 448 * scale        # every 32-block along dim 0 has max 448*scale
        else:
            a[:, ::32] = 448 * scale
        return torch.tensor(a, dtype=torch.float32).to(torch.bfloat16)
    x = grid_tensor((n, H), 2.0 ** -8, False)
    wg = grid_tensor((H, I), 2.0 ** -14, True)
    wu = grid_tensor((H, I), 2.0 ** -14, True)
    wd = grid_tensor((I, H), 2.0 ** -14, True)
    assert torch.equal(x.float().to(torch.bfloat16), x)     # bf16 holds the 4-bit values exactly
    o = np.zeros((n, H))
    hq = np.zeros((n, I), np.uint8)
    hs = np.zeros((n, I // 32), np.uint8)
    xb, gb, ub, db = (t.contiguous() for t in (x, wg, wu, wd))
    assert L.oracle_mxfp8_expert_ffn(xb.data_ptr(), n, H, I, gb.data_ptr(), ub.data_ptr(), db.data_ptr(),
                                     o.ctypes.data, hq.ctypes.data, hs.ctypes.data, None) == 0
    a = x.double() @ wg.double()
    b = x.double() @ wu.double()
    h = (torch.nn.functional.silu(a) * b).float().numpy()
    q, s = _quant(h.reshape(-1))
    assert np.array_equal(q.reshape(n, I), hq) and np.array_equal(s.reshape(n, I // 32), hs)
    hdq = np.array([L.oracle_e4m3_decode(int(v)) for v in q]).reshape(n, I) * \
        np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32).reshape(n, I)
    want = hdq @ wd.double().numpy()
    assert np.allclose(o, want, rtol=1e-12, atol=1e-300)


def _dequant_rows(a: np.ndarray) -> np.ndarray:
    """Rows of a 2D array through the pinned quantiser (blocks of 32 along
    each row) and back to exact values."""
    L = oracle.lib()
    q, s = _quant(np.ascontiguousarray(a, dtype=np.float32).reshape(-1))
    dec = np.array([L.oracle_e4m3_decode(int(v)) for v in q])
    return (dec * np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32)).reshape(a.shape)


def test_mxfp8_ffn_is_quantise_then_exact_gemms():
    """On arbitrary (off-grid) inputs the MXFP8 FFN equals its definition
    assembled from the separately pinned quantiser: x quantised along H, Wg
    and Wu along their contraction index H (per output column), Wd along I
    (per output column), exact products, h rounded to fp32 and quantised
    along I, exact down projection."""
    n, H, I = 3, 96, 64
    g = torch.Generator().manual_seed(9)
    x = torch.randn(n, H, generator=g).to(torch.bfloat16)
    wg, wu = ((torch.randn(H, I, generator=g) / H ** 0.5).to(torch.bfloat16) for _ in range(2))
    wd = (torch.randn(I, H, generator=g) / I ** 0.5).to(torch.bfloat16)
    got = oracle.mxfp8_expert_ffn(x, wg, wu, wd).numpy()
    xq = _dequant_rows(x.float().numpy())
    gq = _dequant_rows(wg.float().numpy().T).T            # blocks along H for each column of Wg
    uq = _dequant_rows(wu.float().numpy().T).T
    dq = _dequant_rows(wd.float().numpy().T).T            # blocks along I for each column of Wd
    a, b = xq @ gq, xq @ uq
    h = (a / (1.0 + np.exp(-a)) * b).astype(np.float32)
    want = _dequant_rows(h) @ dq
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
    # and the quantisation is not the identity on these inputs
    assert not np.allclose(xq, x.double().numpy(), rtol=1e-6)


# ---------------------------------------------------------------- pages' worked number
def test_two_wave_minibatch_golden():
    """The pages' one reproducible number: about 2368 tokens for two full waves
    at hidden 7168 / intermediate 2048 (the reading of the tile count is in
    the fixture)."""
    with open(os.path.join(GOLDEN, "two_wave_minibatch.json")) as f:
        g = json.load(f)
    tiles_per_row = (2 * g["I"] / g["tile_cols"]) / g["tile_rows"]
    m = g["waves"] * g["sms"] / tiles_per_row
    assert m == g["minibatch_min"]


# ---------------------------------------------------------------- backward (next row: the oracle first)
def _dense_layer_autograd(x, logits, wg, wu, wd, dy, k):
    """The forward layer's definition in float64 torch ops, differentiated by
    torch.autograd: every expert evaluated densely, the top-k chosen by the
    (logit desc, index asc) order, gates = torch.softmax of the chosen
    logits.  Returns the gradients of sum(y * dy)."""
    T, E = logits.shape
    xd = x.double().requires_grad_()
    ld = logits.double().requires_grad_()
    ws = [w.double().requires_grad_() for w in (wg, wu, wd)]
    sel = torch.tensor([sorted(range(E), key=lambda e: (-logits[t, e].item(), e))[:k] for t in range(T)])
    g = torch.softmax(torch.gather(ld, 1, sel), dim=1)
    y = torch.zeros(T, x.shape[1], dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(sel[t, j])
            o = (torch.nn.functional.silu(xd[t] @ ws[0][e]) * (xd[t] @ ws[1][e])) @ ws[2][e]
            y[t] = y[t] + g[t, j] * o
    (y * dy).sum().backward()
    return dict(dx=xd.grad, dwg=ws[0].grad, dwu=ws[1].grad, dwd=ws[2].grad, dlogits=ld.grad), sel


@pytest.mark.parametrize("T,H,I,E,k,R", [(6, 32, 24, 5, 2, 2), (4, 16, 40, 3, 3, 4), (5, 24, 16, 6, 1, 1)])
def test_backward_matches_autograd_of_dense_layer(T, H, I, E, k, R):
    cfg, x, logits, wg, wu, wd = _rand_case(T, H, I, E, k, R, seed=60 + T + E)
    dy = torch.randn(T, H, dtype=torch.float64, generator=torch.Generator().manual_seed(T * E))
    got = oracle.moe_backward(x, logits, wg, wu, wd, dy, k, R)
    want, _ = _dense_layer_autograd(x, logits, wg, wu, wd, dy, k)
    for name in ("dx", "dwg", "dwu", "dwd", "dlogits"):
        assert torch.allclose(got[name], want[name], rtol=1e-9, atol=1e-12), name


def test_backward_gate_gradient_invariants():
    """Adding one constant to a token's selected logits leaves y unchanged,
    so their gradients sum to zero; unselected logits get no gradient; with
    k = 1 the gate is constant and every logit gradient is zero."""
    cfg, x, logits, wg, wu, wd = _rand_case(32, 32, 16, 7, 3, 2, seed=71)
    dy = torch.randn(32, 32, dtype=torch.float64, generator=torch.Generator().manual_seed(2))
    got = oracle.moe_backward(x, logits, wg, wu, wd, dy, 3, 2)
    idx, _ = oracle.topk_gates(logits, 3)
    mask = torch.zeros(32, 7, dtype=torch.bool)
    mask.scatter_(1, idx.long(), True)
    dl = got["dlogits"]
    assert (dl[~mask] == 0).all()
    assert torch.allclose(dl.sum(1), torch.zeros(32, dtype=torch.float64), atol=1e-12)
    assert (dl[mask] != 0).any()
    got1 = oracle.moe_backward(x, logits, wg, wu, wd, dy, 1, 2)
    assert (got1["dlogits"] == 0).all()


def test_backward_unselected_expert_gets_no_weight_gradient():
    cfg, x, logits, wg, wu, wd = _rand_case(16, 32, 16, 4, 2, 2, seed=72)
    logits = logits.clone()
    logits[:, 2] = -1e4                      # expert 2 is never chosen
    dy = torch.randn(16, 32, dtype=torch.float64, generator=torch.Generator().manual_seed(3))
    got = oracle.moe_backward(x, logits, wg, wu, wd, dy, 2, 2)
    for name in ("dwg", "dwu", "dwd"):
        assert (got[name][2] == 0).all() and (got[name][0] != 0).any(), name


# ---------------------------------------------------------------- router projection (next row)
def test_router_identity_closed_form():
    """W_r = [I_E; 0] picks the first E features: logits = x[:, :E] (+ prior), exactly."""
    T, H, E = 16, 48, 12
    x = mokgen.normal(1, 5, (T, H), 1.0)
    w = torch.zeros(H, E)
    w[:E, :E] = torch.eye(E)
    prior = torch.linspace(-1.0, 1.0, E)
    assert torch.equal(oracle.router_logits(x, w), x[:, :E].double())
    assert torch.equal(oracle.router_logits(x, w, prior), x[:, :E].double() + prior.double())


@pytest.mark.parametrize("name", ["tiny", "page", "zipf"])
def test_router_matches_fp32_host_logits_within_rounding_bound(name):
    """The harness's fp32 logits (its own fp32 product) lie within the
    textbook bound of an fp32 dot product of H terms plus the prior add,
    gamma_{H+1} * (sum_h |x_h w_he| + |prior_e|), of the oracle's values."""
    cfg = mokgen.scaled(mokgen.CONFIGS[name], T=64)
    x = mokgen.tokens(cfg)
    w = mokgen.router_weight(cfg)
    prior = mokgen.zipf_log_prior(cfg.E, cfg.zipf_s) if cfg.zipf_s else None
    exact = oracle.router_logits(x, w, prior)
    host = mokgen.router_logits(cfg, x).double()
    mag = x.double().abs() @ w.double().abs()
    if prior is not None:
        mag = mag + prior.double().abs()
    n, u = cfg.H + 1, 2.0 ** -24
    bound = n * u / (1 - n * u) * mag
    assert ((host - exact).abs() <= bound).all()
