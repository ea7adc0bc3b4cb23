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
    slot = 2.0 if cfg.mxfp8 else 2.0 + 1.0 / 128     # slot outputs: bf16 (MXFP8 path) or fp16 + block exponents
    weights = 3 * E * H * I * el                     # Wg, Wu, Wd streamed once
    gemm = weights + ns * H * el + 2 * ns * I * el + ns * H * slot   # rows in, h out + in, slots out
    gather = T * H * 2 + ns * H * el                 # each token read once, written to its k rows
    combine = ns * H * slot + ns * 4 + T * H * 2     # slots + gates in, bf16 y out
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
    bf16 weights and 36.2 GB per GEMM step (fp16 slot rows); 17.4 /
    19.1 GB on the MXFP8 path (bf16 slot outputs); 5.77 TFLOP per step."""
    w = bench.algorithmic_work(mokgen.CONFIGS["page"])
    assert w["weight_bytes"] / 1e9 == pytest.approx(33.8, abs=0.05)
    assert w["gemm_bytes"] / 1e9 == pytest.approx(36.25, abs=0.05)
    assert w["gemm_flops"] / 1e12 == pytest.approx(5.77, abs=0.005)
    m = bench.algorithmic_work(mokgen.CONFIGS["page_mxfp8"])
    assert m["weight_bytes"] / 1e9 == pytest.approx(17.4, abs=0.05)
    assert m["gemm_bytes"] / 1e9 == pytest.approx(19.1, abs=0.05)


def test_traffic_only_for_the_captured_kernel_source(tmp_path, monkeypatch):
    """A DRAM capture is reported only for the workload and mode it was taken
    on, and only while the GEMM sources hash to what they were then."""
    import json

    f = tmp_path / "t.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic("page", "staged") == (None, "no capture")
    sha = bench.gemm_source_hash()
    f.write_text(json.dumps({"entries": [
        {"workload": "page", "mode": "staged", "gemm_source_sha": sha, "bytes_per_step": 3.7e10, "how": "x"},
        {"workload": "zipf", "mode": "staged", "gemm_source_sha": "0" * 16, "bytes_per_step": 2.5e10}]}))
    assert bench.measured_traffic("page", "staged") == (3.7e10, "x")
    assert bench.measured_traffic("zipf", "staged")[0] is None
    assert bench.measured_traffic("page", "persistent")[0] is None


def test_committed_traffic_entries_are_plausible():
    """Every committed capture names a known workload and lies near its
    algorithmic bytes (a kernel that re-reads nothing moves about what it
    must)."""
    import json
    import os

    if not os.path.exists(bench.TRAFFIC_FILE):
        pytest.skip("no committed capture")
    with open(bench.TRAFFIC_FILE) as f:
        entries = json.load(f)["entries"]
    for e in entries:
        cfg = mokgen.CONFIGS[e["workload"]]
        alg = bench.algorithmic_work(cfg)["gemm_bytes"]
        assert 0.85 * alg <= e["bytes_per_step"] <= 1.15 * alg, e


def test_tensor_peak_follows_the_timed_region():
    peaks = {"bf16_tflops": 1646.9, "bf16_tflops_sustained": 1385.0, "hbm_gbs": 6547.8}
    assert bench.tensor_peaks(peaks, False, 0.15)[0] == 1646.9
    assert bench.tensor_peaks(peaks, False, 5.0)[0] == 1385.0
    assert bench.tensor_peaks(peaks, True, 0.15)[0] == 2 * 1646.9
