"""Planted mistakes in the oracle, on the CPU.

Each mutant is a copy of the oracle's C sources with ONE plausible error of
the kinds the pins are there to catch: a tie rule turned round, a wrong
sign, a dropped term, a wrong or transposed index, a forgotten shard base,
a result left at the wrong slot, an off-by-one exponent, another rounding
rule, a term of the backward's chain rule.  The copy is compiled with the
oracle's own flags and every pin of test_oracle_pins.py runs on it; at
least one pin must fail.  An unmodified copy, built the same way, must pass
them all (the control), so a failure comes from the planted mistake and not
from the harness.
"""
import os
import shutil

import pytest

import oracle
import test_oracle_pins as pins

ORACLE_DIR = os.path.dirname(os.path.abspath(oracle.__file__))
SOURCES = ("mok_oracle.c", "mxfp8_oracle.c", "mok_oracle_bwd.c", "mok_oracle_router.c")

# name -> (source file, text as written, text with the mistake)
MUTANTS = {
    # step 1: router top-k and gates
    "tie_goes_to_higher_index": (
        "mok_oracle.c", "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;"),
    "softmax_wrong_sign": (
        "mok_oracle.c", "ex[j] = exp((double)l[topk_idx[(size_t)t * k + j]] - m);",
        "ex[j] = exp(m - (double)l[topk_idx[(size_t)t * k + j]]);"),
    "gates_not_normalised": (
        "mok_oracle.c", "gates[(size_t)t * k + j] = (float)(ex[j] / s);", "gates[(size_t)t * k + j] = (float)ex[j];"),
    # step 2: schedule
    "segment_tokens_descending": (
        "mok_oracle.c",
        "        for (int t = 0; t < T; ++t) {\n            for (int j = 0; j < k; ++j) {\n"
        "                if (topk_idx[(size_t)t * k + j] != e) continue;",
        "        for (int t = T - 1; t >= 0; --t) {\n            for (int j = 0; j < k; ++j) {\n"
        "                if (topk_idx[(size_t)t * k + j] != e) continue;"),
    "shards_round_robin": (
        "mok_oracle.c", "if (src_rank) src_rank[row] = t / S_r;", "if (src_rank) src_rank[row] = t % R;"),
    "slot_index_transposed": (
        "mok_oracle.c", "if (row_slot) row_slot[row] = t * k + j;", "if (row_slot) row_slot[row] = j * T + t;"),
    # step 3: gather
    "gather_ignores_shard_base": (
        "mok_oracle.c", "const uint16_t* shard = x + (size_t)r * S_r * H;", "const uint16_t* shard = x;"),
    # step 4: expert FFN
    "silu_dropped": (
        "mok_oracle.c", "a[i] = a[i] / (1.0 + exp(-a[i])) * b[i];", "a[i] = a[i] * b[i];"),
    "sigmoid_wrong_sign": (
        "mok_oracle.c", "a[i] = a[i] / (1.0 + exp(-a[i])) * b[i];", "a[i] = a[i] / (1.0 + exp(a[i])) * b[i];"),
    "gate_and_up_swapped": (
        "mok_oracle.c",
        "a[i] += xv * bf16_to_double(g[i]);\n                        b[i] += xv * bf16_to_double(u[i]);",
        "a[i] += xv * bf16_to_double(u[i]);\n                        b[i] += xv * bf16_to_double(g[i]);"),
    "down_projection_transposed": (
        "mok_oracle.c", "for (int c = 0; c < H; ++c) orow[c] += hv * bf16_to_double(d[c]);",
        "for (int c = 0; c < H; ++c) orow[c] += hv * bf16_to_double(wd[((size_t)c * I + i) % ((size_t)I * H)]);"),
    # step 5: push combine and weighted merge
    "result_left_at_its_row": (
        "mok_oracle.c", "memcpy(o_slot + (size_t)rslot[row] * H, o_row + row * H, sizeof(double) * (size_t)H);",
        "memcpy(o_slot + row * H, o_row + row * H, sizeof(double) * (size_t)H);"),
    "combine_uses_first_gate": (
        "mok_oracle.c", "double g = (double)gates[(size_t)t * k + j];", "double g = (double)gates[(size_t)t * k];"),
    # MXFP8 emulation
    "mx_scale_exponent_off_by_one": ("mxfp8_oracle.c", "int s = (e - 1) - 8;", "int s = e - 8;"),
    "mx_ties_round_up": (
        "mxfp8_oracle.c", "return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;"),
    "mx_saturates_to_nan": ("mxfp8_oracle.c", "if (a >= 448.0) return sgn | 0x7E;", "if (a >= 448.0) return sgn | 0x7F;"),
    "mx_subnormal_exponent": (
        "mxfp8_oracle.c", "if (ex == 0) v = ldexp((double)m, -9);", "if (ex == 0) v = ldexp((double)m, -10);"),
    "mx_zero_block_scale": ("mxfp8_oracle.c", "if (amax == 0.0) return -127;", "if (amax == 0.0) return 0;"),
    "mx_h_not_quantised": (
        "mxfp8_oracle.c", "mx_roundtrip(hv, I, hq);", "memcpy(hq, hv, sizeof(double) * (size_t)I);"),
    "mx_x_not_quantised": (
        "mxfp8_oracle.c", "mx_roundtrip(xr, H, xq);", "memcpy(xq, xr, sizeof(double) * (size_t)H);"),
    "mx_up_weights_not_quantised": (
        "mxfp8_oracle.c", "mx_roundtrip(col, H, qu + (size_t)i * H);",
        "memcpy(qu + (size_t)i * H, col, sizeof(double) * (size_t)H);"),
    "mx_down_weight_read_transposed": (
        "mxfp8_oracle.c", "for (int k = 0; k < I; ++k) col[k] = o_bf16(wd[(size_t)k * H + c]);",
        "for (int k = 0; k < I; ++k) col[k] = o_bf16(wd[((size_t)c * I + k) % ((size_t)I * H)]);"),
    # router projection
    "router_prior_dropped": (
        "mok_oracle_router.c", "for (int e = 0; e < E; ++e) out[e] = prior ? (double)prior[e] : 0.0;",
        "for (int e = 0; e < E; ++e) out[e] = 0.0;"),
    "router_weight_read_transposed": (
        "mok_oracle_router.c", "out[e] += xv * (double)w[e];",
        "out[e] += xv * (double)wr[((size_t)e * H + h) % ((size_t)H * E)];"),
    # backward
    "bwd_silu_derivative_term_dropped": (
        "mok_oracle_bwd.c", "da[i] = dh[i] * b[i] * (s + a[i] * s * (1.0 - s));", "da[i] = dh[i] * b[i] * s;"),
    "bwd_softmax_dot_dropped": (
        "mok_oracle_bwd.c", "g[(size_t)t * k + j] * (dg[(size_t)t * k + j] - dot);",
        "g[(size_t)t * k + j] * dg[(size_t)t * k + j];"),
    "bwd_reverse_combine_without_gate": (
        "mok_oracle_bwd.c", "dout[c] = g[slot] * dyt[c];", "dout[c] = dyt[c];"),
    "bwd_dwd_from_preactivation": (
        "mok_oracle_bwd.c", "dWd[(size_t)i * H + c] += h[i] * dout[c];", "dWd[(size_t)i * H + c] += a[i] * dout[c];"),
    "bwd_dwu_takes_gate_branch": (
        "mok_oracle_bwd.c", "dWu[(size_t)c * I + i] += xr[c] * db[i];", "dWu[(size_t)c * I + i] += xr[c] * da[i];"),
    "bwd_up_gradient_sign": ("mok_oracle_bwd.c", "db[i] = dh[i] * a[i] * s;", "db[i] = -dh[i] * a[i] * s;"),
    "bwd_dx_pushed_to_wrong_token": (
        "mok_oracle_bwd.c", "dx[(size_t)t * H + c] += acc;", "dx[(size_t)((t + 1) % T) * H + c] += acc;"),
}


def _pin_calls():
    """Every pin of test_oracle_pins.py with each of its parameter sets."""
    calls = []
    for name in sorted(n for n in dir(pins) if n.startswith("test_")):
        fn = getattr(pins, name)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, {}))
            continue
        assert len(marks) == 1, name
        argnames = [a.strip() for a in marks[0].args[0].split(",")]
        for vals in marks[0].args[1]:
            vals = vals if isinstance(vals, (tuple, list)) else (vals,)
            calls.append((f"{name}{list(vals)}", fn, dict(zip(argnames, vals))))
    return calls


def _build(tmp_path, edit=None):
    srcs = []
    for f in SOURCES:
        dst = tmp_path / f
        shutil.copyfile(os.path.join(ORACLE_DIR, f), dst)
        srcs.append(str(dst))
    if edit is not None:
        f, before, after = edit
        text = (tmp_path / f).read_text()
        assert text.count(before) == 1, f"the text to mutate must occur once in {f}: {before!r}"
        (tmp_path / f).write_text(text.replace(before, after))
    return oracle.build_from(srcs, str(tmp_path / "liboracle_copy.so"))


def _failing_pins(path, stop_at_first=True):
    failed = []
    with oracle.library(path):
        for name, fn, kw in _pin_calls():
            try:
                fn(**kw)
            except (AssertionError, RuntimeError, ValueError, IndexError):
                failed.append(name)
                if stop_at_first:
                    break
    return failed


def test_unmodified_copy_passes_every_pin(tmp_path):
    assert _failing_pins(_build(tmp_path), stop_at_first=False) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    failed = _failing_pins(_build(tmp_path, MUTANTS[name]))
    assert failed, f"no pin of the oracle catches the planted mistake {name!r}"
