"""The algorithmic work bench.py divides by, pinned to the per-unit figures
of the kernels (bytes and flops per slot, token and weight), so that the
roofline's `achieved` cannot drift from what the kernels must move.  CPU
only."""
import pytest

import bench
import mokgen


def _per_unit(cfg):
    T, H, I, E, k = cfg.T, cfg.H, cfg.I, cfg.E, cfg.k
    ns = T * k
    el = 1.0 + 1.0 / 32 if cfg.mxfp8 else 2.0       # bytes per weight / row / h element
    weights = 3 * E * H * I * el                     # Wg, Wu, Wd streamed once
    gemm = weights + ns * H * el + 2 * ns * I * el + ns * H * 2   # rows in, h out + in, fp16 slots out
    gather = T * H * 2 + ns * H * el                 # each token read once, written to its k rows
    combine = ns * H * 2 + ns * 4 + T * H * 2        # fp16 slots + gates in, bf16 y out
    return dict(gemm_flops=6.0 * H * I * ns, gemm_bytes=gemm, weight_bytes=weights, gather_bytes=gather,
                combine_bytes=combine, forward_bytes=gather + gemm + combine)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "page", "zipf", "page_mxfp8"])
def test_algorithmic_work_matches_per_unit_figures(name):
    cfg = mokgen.CONFIGS[name]
    got = bench.algorithmic_work(cfg)
    for key, want in _per_unit(cfg).items():
        assert got[key] == pytest.approx(want, rel=1e-12), key


def test_page_shape_totals():
    """The page shape's totals quoted beside the measurements: 33.8 GB of
    bf16 weights and 36.2 GB per GEMM step; 17.4 / 19.1 GB on the MXFP8
    path; 5.77 TFLOP per step."""
    w = bench.algorithmic_work(mokgen.CONFIGS["page"])
    assert w["weight_bytes"] / 1e9 == pytest.approx(33.8, abs=0.05)
    assert w["gemm_bytes"] / 1e9 == pytest.approx(36.2, abs=0.05)
    assert w["gemm_flops"] / 1e12 == pytest.approx(5.77, abs=0.005)
    m = bench.algorithmic_work(mokgen.CONFIGS["page_mxfp8"])
    assert m["weight_bytes"] / 1e9 == pytest.approx(17.4, abs=0.05)
    assert m["gemm_bytes"] / 1e9 == pytest.approx(19.1, abs=0.05)


def test_traffic_entries_cite_existing_profiles():
    import os

    root = os.path.dirname(os.path.abspath(bench.__file__))
    for name, (gb, path) in bench.GEMM_TRAFFIC_GB_PER_STEP.items():
        assert name in mokgen.CONFIGS
        assert os.path.exists(os.path.join(root, path)), path
        # DRAM traffic of a kernel that re-reads nothing is close to its algorithmic bytes
        alg = bench.algorithmic_work(mokgen.CONFIGS[name])["gemm_bytes"] / 1e9
        assert 0.9 * alg <= gb <= 1.1 * alg, (name, gb, alg)
