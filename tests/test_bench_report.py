"""The benchmark's per-stage roofline report, computed from given stage times (CPU only)."""
import importlib.util
import os
import sys

import pytest

from block_sparse_long_tcgen05_b200 import accounting, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        spec.loader.exec_module(m)
    finally:
        sys.argv = argv
    return m


def test_stage_rates_match_the_work_counts():
    bench = _bench()
    cfg = synth.CONFIGS["prefill-128k"]
    peaks = {"bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    stages = {"index_topk": {"ms_per_step": 14.0}, "kvouter": {"ms_per_step": 12.0},
              "merge": {"ms_per_step": 6.0}, "csr_scatter": {"ms_per_step": 0.3},
              "csr_count": {"ms_per_step": 0.2}}
    r = bench.stage_rates(stages, cfg, peaks)
    nb = cfg.N // cfg.Bk
    assert r["index_topk"]["tflops"] == pytest.approx(accounting.index_kernel_flops(0, nb, cfg.G, cfg.d_idx) / 14e-3 / 1e12)
    assert r["index_topk"]["frac_bf16_sustained"] == pytest.approx(r["index_topk"]["tflops"] / 1400.0)
    mb = accounting.main_branch_bytes(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.Bk, cfg.k)
    assert r["merge"]["gbs"] == pytest.approx(mb["merge"] / 6e-3 / 1e9)
    assert r["kvouter"]["gbs"] == pytest.approx(mb["kvouter"] / 12e-3 / 1e9)
    assert "tflops" in r["kvouter"]
    assert r["csr (all passes)"]["gbs"] == pytest.approx(12.0 * cfg.N * cfg.G * cfg.k / 0.5e-3 / 1e9)
    assert "csr_scatter" not in r
