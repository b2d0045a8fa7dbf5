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
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    stages = {"index_topk": {"ms_per_step": 14.0}, "kvouter": {"ms_per_step": 12.0},
              "merge": {"ms_per_step": 6.0}, "csr_scatter": {"ms_per_step": 0.3},
              "csr_count": {"ms_per_step": 0.2}}
    r = bench.stage_rates(stages, cfg, peaks)
    nb = cfg.N // cfg.Bk
    assert r["index_topk"]["tflops"] == pytest.approx(accounting.index_kernel_flops(0, nb, cfg.G, cfg.d_idx) / 14e-3 / 1e12)
    assert r["index_topk"]["frac_bf16_burst"] == pytest.approx(r["index_topk"]["tflops"] / 1650.0)
    mb = accounting.main_branch_bytes(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.Bk, cfg.k)
    assert r["merge"]["gbs"] == pytest.approx(mb["merge"] / 6e-3 / 1e9)
    assert r["kvouter"]["gbs"] == pytest.approx(mb["kvouter"] / 12e-3 / 1e9)
    assert "tflops" in r["kvouter"]
    assert r["csr (all passes)"]["gbs"] == pytest.approx(12.0 * cfg.N * cfg.G * cfg.k / 0.5e-3 / 1e9)
    assert "csr_scatter" not in r


def test_roofline_uses_the_burst_peak_and_the_dominant_kernel():
    """The dominant kernel's line divides its algorithmic work per launch by its average launch
    time and by the measured burst peak; the sustained figure is a labelled extra."""
    bench = _bench()
    cfg = synth.CONFIGS["prefill-128k"]
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0, "sustained_sm_mhz": 1350.0}
    steps = 4
    stats = {"index_topk": (steps, 4 * 14.0), "kvouter": (8 * steps, 4 * 12.0), "merge": (8 * steps, 4 * 6.0)}
    r = bench.roofline(stats, steps, cfg, peaks, "measured", {}, 1900.0)
    nb = cfg.N // cfg.Bk
    work = accounting.index_kernel_flops(0, nb, cfg.G, cfg.d_idx)
    assert r["kernel"] == "index_topk" and r["bound"] == "tensor"
    assert r["work_per_launch"] == pytest.approx(work)
    assert r["achieved"] == pytest.approx(work / 14e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1650.0)
    assert r["sustained_extra"]["frac"] == pytest.approx(r["achieved"] / 1400.0)
    assert r["sustained_extra"]["peak_sm_mhz"] == 1350.0
    assert r["achieved_per_sm_ghz"] == pytest.approx(r["achieved"] / 1.9)
    # an HBM-bound dominant kernel (per launch: 8 launches per step)
    r = bench.roofline({"merge": (8 * steps, 4 * 6.0)}, steps, cfg, peaks, "measured", {"merge": 123}, None)
    mb = accounting.main_branch_bytes(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.Bk, cfg.k)["merge"]
    assert r["bound"] == "hbm" and r["traffic"] == 123
    assert r["achieved"] == pytest.approx(mb / 8 / (6e-3 / 8) / 1e9)


def test_memory_bound_rates_name_the_fused_topk():
    bench = _bench()
    cfg = synth.CONFIGS["prefill-128k"]
    peaks = {"bf16_tflops": 1650.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    st = {"index_topk": {"ms_per_step": 14.0}, "merge": {"ms_per_step": 6.0}, "csr_count": {"ms_per_step": 0.2}}
    r = bench.memory_bound_rates(st, cfg, peaks)
    assert set(r) == {"merge", "csr", "topk"} and isinstance(r["topk"], str)
    st = {"index_blockmax": {"ms_per_step": 14.0}, "topk_prefill": {"ms_per_step": 1.0}}
    r = bench.memory_bound_rates(st, cfg, peaks)
    nb = cfg.N // cfg.Bk
    assert r["topk"]["gbs"] == pytest.approx((4.0 * cfg.G * cfg.Bk * nb * (nb - 1) / 2 + 4.0 * cfg.N * cfg.G * cfg.k)
                                             / 1e-3 / 1e9)
