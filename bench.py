"""Benchmark of the MSA hot path on B200: prefill tokens/s and TFLOP/s at 128K, decode tokens/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one msa_forward prefill over the 131072-token sequence (Index Branch: scores +
block max + Top-k; Main Branch: CSR build + KV-outer attention + LSE merge), inputs
resident in HBM. Under torchrun every rank runs its own independent sequence (weak
scaling), or with --shard groups its range of GQA groups of one shared sequence (strong
scaling); no data-path collective either way, the time is the max over ranks. Rank 0
prints one JSON line. `--impl reference` times the fp64 CPU oracle on a bounded sample of query
rows of the same workload instead (rank 0 only).

At N = 1 the same line also reports every synthetic configuration (the 2K tiny prefill, 32K,
128K, decode B = 64 x 128K and 1M) under "configs": tokens/s, useful TFLOP/s and its fraction
of the measured bf16 peak, the HBM rate of the memory-bound kernels, and the oracle's
per-query rate on the host cores beside it (--headline-only skips them).
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_tcgen05_b200 import accounting, synth  # noqa: E402
from block_sparse_long_tcgen05_b200 import dist as mdist  # noqa: E402

METRIC = "prefill tokens/s & TFLOP/s (frac of bf16 peak) at 128K; decode tokens/s"
SPEC_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# Device sources each kernel is built from: DRAM counters taken on a kernel describe it only
# while these files are unchanged.
KERNEL_SOURCES = {
    "index_topk": ["index_topk.cuh", "index_blockmax.cuh", "topk.cuh", "ptx.cuh", "common.cuh"],
    "index_blockmax": ["index_blockmax.cuh", "ptx.cuh", "common.cuh"],
    "topk_prefill": ["topk.cuh", "ptx.cuh", "common.cuh"],
    "kvouter": ["kvouter.cuh", "ptx.cuh", "common.cuh"],
    "merge": ["merge.cuh", "ptx.cuh", "common.cuh"],
}


def kernel_sha256(kernel: str, csrc: str | None = None) -> str | None:
    import hashlib
    files = KERNEL_SOURCES.get(kernel)
    if files is None:
        return None
    csrc = csrc or os.path.join(ROOT, "block_sparse_long_tcgen05_b200", "csrc")
    h = hashlib.sha256()
    for f in files:
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()


def load_peaks():
    """Roofline denominators: the measured HBM copy bandwidth, the measured cuBLAS bf16 burst
    rate (the peak for kernels of a step of tens of milliseconds) and, as a labelled extra,
    the seconds-long sustained rate with the SM clock it ran at."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        out = {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}
        out["sustained_sm_mhz"] = (d.get("clocks_under_load") or {}).get("sm_mhz_median")
        return out, "measured"
    return dict(FALLBACK, sustained_sm_mhz=None), "fallback"


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling (200 ms) of one GPU during a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.proc = subprocess.Popen(["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------------------ dist
def dist_setup():
    return mdist.init("nccl", timeout_s=300)


def max_over_ranks(x: float, world: int) -> float:
    return mdist.max_over_ranks(x, device="cuda") if world > 1 else x


def barrier(world: int):
    mdist.barrier()


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(inp: dict, cfg, rows: int, seed: int):
    """Time the oracle (as it stands) on `rows` seeded query rows; returns (rows/s, seconds)."""
    from oracle import msa_oracle as orc  # test / baseline infrastructure only
    rng = np.random.default_rng(seed)
    sel = sorted(rng.choice(cfg.N, size=rows, replace=False).tolist())
    host = {n: t.detach().cpu() for n, t in inp.items()}
    t0 = time.perf_counter()
    orc.prefill_rows(host, sel, cfg.Bk, cfg.k)
    dt = time.perf_counter() - t0
    return rows / dt, dt


def oracle_rows_rate(inp: dict, cfg, rows: int, seed: int):
    """The oracle on `rows` seeded query rows of a prefill, reading the (device) inputs row by
    row as the long-sequence parity tests do (no host copy of the whole sequence); returns
    (query rows/s, seconds)."""
    from oracle import msa_oracle as orc  # test / baseline infrastructure only
    rng = np.random.default_rng(seed)
    sel = sorted(rng.choice(cfg.N, size=min(rows, cfg.N), replace=False).tolist())
    t0 = time.perf_counter()
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], sel, cfg.Bk, cfg.k)
    orc.attend_rows(inp["q"], inp["k"], inp["v"], ids, sel, cfg.Bk)
    dt = time.perf_counter() - t0
    return len(sel) / dt, dt


def oracle_decode_rate(dinp: dict, dcfg, seqs: int):
    """The oracle on the first `seqs` decode sequences; returns (new tokens/s, seconds)."""
    from oracle import msa_oracle as orc  # test / baseline infrastructure only
    t0 = time.perf_counter()
    orc.decode_rows(dinp, range(seqs), dcfg.Bk, dcfg.k)
    dt = time.perf_counter() - t0
    return seqs / dt, dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def workload_config(cfg, extra=None) -> dict:
    c = {"workload": cfg.name, "N": cfg.N, "Hq": cfg.Hq, "G": cfg.G, "d": cfg.d, "d_idx": cfg.d_idx,
         "Bk": cfg.Bk, "k": cfg.k, "hot_frac": cfg.hot_frac, "seed": cfg.seed,
         "l2": "inputs larger than L2 (q alone is 2.1 GB), no flush needed",
         "parallelism": "one independent sequence per GPU, no collective"}
    if extra:
        c.update(extra)
    return c


def run_reference(args, world, rank):
    if rank != 0:
        return
    cfg = synth.CONFIGS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.prefill_inputs(cfg, device=dev)
    rows = args.ref_rows
    for w in range(args.warmup):
        oracle_sample(inp, cfg, rows, seed=100 + w)
    times = []
    for s in range(args.steps):
        _, dt = oracle_sample(inp, cfg, rows, seed=200 + s)
        times.append(dt)
    tot = sum(times)
    value = rows * args.steps / tot
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} seeded query rows of the {cfg.name} workload per step "
                                       f"(both branches, fp64)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ ours
def timed(fn, steps: int, stream) -> float:
    """ms per call of fn over `steps` calls, CUDA events on the launching stream."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def graph_of(fn) -> "torch.cuda.CUDAGraph":
    """fn captured once as a CUDA graph (after one call outside the capture, which sets the
    kernels' attributes); every step of the library is a launch on the caller's stream, so
    replays run the same kernels on the captured buffers' current contents."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def stage_rates(stages: dict, cfg, peaks: dict) -> dict:
    """Every prefill kernel's achieved rate against its own roofline, from the per-step stage
    times: TFLOP/s of the score and attention products (fraction of the measured bf16 burst
    peak), GB/s of compulsory bytes for the HBM-bound passes (fraction of the measured copy
    bandwidth). The CSR passes together move the block ids twice and write one entry per
    (query, group, slot)."""
    N, Hq, G, d, d_idx, Bk, k = cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.Bk, cfg.k
    nb = (N + Bk - 1) // Bk
    flops = {"index_topk": accounting.index_kernel_flops(0, nb, G, d_idx, Bk),
             "index_blockmax": accounting.index_kernel_flops(0, nb, G, d_idx, Bk),
             "kvouter": accounting.kvouter_flops(N, Hq, d, Bk, k)}
    byts = dict(accounting.main_branch_bytes(N, Hq, G, d, Bk, k))
    byts["topk_prefill"] = 4.0 * G * Bk * nb * (nb - 1) / 2 + 4.0 * N * G * k
    out = {}
    for name, v in stages.items():
        sec = v["ms_per_step"] * 1e-3
        if sec <= 0:
            continue
        r = {}
        if name in flops:
            r["tflops"] = flops[name] / sec / 1e12
            r["frac_bf16_burst"] = r["tflops"] / peaks["bf16_tflops"]
        if name in byts:
            r["gbs"] = byts[name] / sec / 1e9
            r["frac_hbm"] = r["gbs"] / peaks["hbm_gbs"]
        if r:
            out[name] = r
    csr_sec = sum(v["ms_per_step"] for n, v in stages.items() if n.startswith("csr")) * 1e-3
    if csr_sec > 0:
        gbs = 3.0 * 4 * N * G * k / csr_sec / 1e9
        out["csr (all passes)"] = {"gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]}
    return out


def stage_table(stats: dict, steps: int) -> dict:
    total = sum(v[1] for v in stats.values())
    return {name: {"launches_per_step": launches / steps, "ms_per_step": tot / steps,
                   "share": tot / total if total else None}
            for name, (launches, tot) in sorted(stats.items(), key=lambda kv: -kv[1][1])}


def roofline(stats: dict, steps: int, rcfg, peaks: dict, peak_src: str, traffic: dict, sm_mhz) -> dict:
    """The dominant kernel's achieved rate: algorithmic work per launch over its average
    launch time (CUDA events on the launching stream), against the measured burst peak of its
    bound; the sustained bf16 figure and a clock-normalised rate are labelled extras."""
    N = rcfg.N
    nb = (N + rcfg.Bk - 1) // rcfg.Bk
    dom = max(stats.items(), key=lambda kv: kv[1][1])[0]
    dom_launches, dom_ms = stats[dom]
    per_launch_s = dom_ms / dom_launches * 1e-3
    launches_per_step = dom_launches / steps
    traffic_b = traffic.get(dom) if traffic else None
    if dom in ("index_blockmax", "index_topk", "kvouter"):
        if dom == "kvouter":
            work = accounting.kvouter_flops(N, rcfg.Hq, rcfg.d, rcfg.Bk, rcfg.k) / launches_per_step
        else:
            work = accounting.index_kernel_flops(0, nb, rcfg.G, rcfg.d_idx, rcfg.Bk) / launches_per_step
        ach = work / per_launch_s / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"], "traffic": traffic_b,
                "peak_source": f"{peak_src} bf16 burst (cuBLAS 8192^3, best of 10); of {peak_src}",
                "work_per_launch": work,
                "sustained_extra": {"peak": peaks["bf16_tflops_sustained"],
                                    "frac": ach / peaks["bf16_tflops_sustained"],
                                    "peak_sm_mhz": peaks.get("sustained_sm_mhz"),
                                    "note": "seconds-long GEMM loop under the power cap, at a lower SM clock "
                                            "than this step's"}}
    else:
        byts = accounting.main_branch_bytes(N, rcfg.Hq, rcfg.G, rcfg.d, rcfg.Bk, rcfg.k).get(dom, float("nan"))
        work = byts / launches_per_step
        ach = work / per_launch_s / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic_b,
                "peak_source": f"{peak_src} HBM copy; of {peak_src}", "work_per_launch": work}
    if sm_mhz:
        roof["achieved_per_sm_ghz"] = ach / (sm_mhz / 1000.0)
        roof["sm_mhz_median"] = sm_mhz
    return roof


def prefill_rates(rcfg, ms: float, peaks: dict, world: int) -> dict:
    idx_f, main_f = accounting.prefill_useful_flops(rcfg.N, rcfg.Hq, rcfg.G, rcfg.d, rcfg.d_idx, rcfg.Bk, rcfg.k)
    tf = (idx_f + main_f) / (ms * 1e-3) / 1e12
    return {"useful_tflops": tf * world, "useful_tflops_per_gpu": tf,
            "frac_measured_bf16_burst": tf / peaks["bf16_tflops"],
            "frac_spec_bf16_2250": tf / SPEC_BF16_TFLOPS,
            "frac_measured_bf16_sustained_extra": tf / peaks["bf16_tflops_sustained"],
            "useful_tflop_per_step": (idx_f + main_f) / 1e12}


def memory_bound_rates(stages: dict, rcfg, peaks: dict) -> dict:
    """HBM rate of the memory-bound stages of a prefill: the merge, the CSR build and the
    Top-k (a separate pass only on the two-kernel Index Branch; the one-kernel path keeps it in
    the score epilogue, with no block maxima in HBM)."""
    sr = stage_rates(stages, rcfg, peaks)
    out = {}
    for name, key in (("merge", "merge"), ("csr", "csr (all passes)"), ("topk", "topk_prefill")):
        if key in sr:
            out[name] = {"gbs": sr[key]["gbs"], "frac_hbm": sr[key]["frac_hbm"]}
    if "topk_prefill" not in stages and "index_topk" in stages:
        out["topk"] = "fused into index_topk (no block maxima in HBM)"
    return out


def make_prefill(cfg, dev, seed, query_chunk, shard_groups: bool, world: int, rank: int):
    """Inputs, parameters and buffers of one prefill configuration on this rank."""
    from block_sparse_long_tcgen05_b200 import msa
    if shard_groups:
        full = synth.prefill_inputs(cfg, device=dev, seed=cfg.seed)
        inp = mdist.shard_inputs_by_group(full, cfg.G, world, rank)
        del full
        torch.cuda.empty_cache()
        groups, _, _ = mdist.group_slice(cfg.G, cfg.R, world, rank)
        rcfg = dataclasses.replace(cfg, Hq=len(groups) * cfg.R, G=len(groups))
    else:
        inp = synth.prefill_inputs(cfg, device=dev, seed=seed)
        rcfg = cfg
    p = msa.prefill_params(cfg.N, rcfg.Hq, rcfg.G, rcfg.d, rcfg.d_idx, rcfg.k, bk=rcfg.Bk, query_chunk=query_chunk)
    bufs = {"ws": torch.empty(msa.msa_forward_workspace(p), dtype=torch.uint8, device=dev),
            "o": torch.empty_like(inp["q"]),
            "ids": torch.empty(cfg.N, rcfg.G, rcfg.k, dtype=torch.int32, device=dev)}
    return inp, rcfg, p, bufs


def time_prefill(inp, p, bufs, steps: int, warmup: int, stream, dev, world: int, clocks: bool):
    """W untimed steps, then K timed steps between barriers; returns (ms per step as the max
    over ranks, per-kernel stats of this rank, clock record or None)."""
    from block_sparse_long_tcgen05_b200 import msa

    def step():
        msa.msa_forward(p, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], o=bufs["o"],
                        block_ids=bufs["ids"], workspace=bufs["ws"])

    for _ in range(warmup):
        step()
    msa.check_device_error(dev)
    barrier(world)
    sampler = ClockSampler(dev.index) if clocks else None
    msa.msa_profile_start()
    ms = timed(step, steps, stream)
    stats = msa.msa_profile_stop()
    clk = sampler.stop() if sampler else None
    msa.check_device_error(dev)
    ms = max_over_ranks(ms, world)
    barrier(world)
    return ms, stats, clk


def run_decode(args, dev, stream, world, rank, peaks, cpu_baseline: bool) -> dict:
    from block_sparse_long_tcgen05_b200 import msa
    dcfg = synth.DEC128K
    dinp = synth.decode_inputs(dcfg, device=dev, seed=mdist.rank_seed(dcfg.seed, rank))
    dp = msa.decode_params(dcfg.B, dinp["k_cache"].shape[1], dinp["seqlens"], dcfg.Hq, dcfg.G, dcfg.d,
                           dcfg.d_idx, dcfg.k)
    dws = torch.empty(msa.msa_forward_workspace(dp), dtype=torch.uint8, device=dev)
    do = torch.empty_like(dinp["q"])

    def dstep():
        msa.msa_forward(dp, dinp["q"], dinp["k_cache"], dinp["v_cache"], dinp["q_idx"],
                        dinp["k_idx_cache"], o=do, workspace=dws)

    for _ in range(max(3, args.warmup)):
        dstep()
    msa.check_device_error(dev)
    barrier(world)
    msa.msa_profile_start()
    dms = timed(dstep, args.steps, stream)
    dstats = msa.msa_profile_stop()
    msa.check_device_error(dev)
    dms = max_over_ranks(dms, world)
    barrier(world)
    scan_ms = dstats.get("decode_scan", (1, float("nan")))[1] / args.steps
    scan_bytes = accounting.decode_scan_bytes([dcfg.L] * dcfg.B, dcfg.G, dcfg.d_idx)
    d_idx_f, d_main_f = accounting.decode_useful_flops([dcfg.L] * dcfg.B, dcfg.Hq, dcfg.G, dcfg.d,
                                                       dcfg.d_idx, dcfg.Bk, dcfg.k)
    tok_s = world * dcfg.B / (dms * 1e-3)
    scan_gbs = scan_bytes / (scan_ms * 1e-3) / 1e9
    out = {"workload": dcfg.name, "tokens_per_s": tok_s, "ms_per_step": dms,
           "useful_tflops_per_gpu": (d_idx_f + d_main_f) / (dms * 1e-3) / 1e12,
           "frac_measured_bf16_burst": (d_idx_f + d_main_f) / (dms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "scan_hbm_gbs": scan_gbs, "scan_frac_hbm": scan_gbs / peaks["hbm_gbs"],
           "roofline": {"kernel": "decode_scan", "bound": "hbm", "achieved": scan_gbs, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": scan_gbs / peaks["hbm_gbs"],
                        "work_per_launch": scan_bytes,
                        "note": "a read-only stream against a read+write copy peak can read a little above 1"},
           "stages": {k: {"ms_per_step": v[1] / args.steps} for k, v in dstats.items()}}
    # the same step captured once and replayed as a CUDA graph, as a serving loop would run it
    g = graph_of(dstep)
    barrier(world)
    gms = max_over_ranks(timed(g.replay, args.steps, stream), world)
    msa.check_device_error(dev)
    del g
    out["graph"] = {"ms_per_step": gms, "tokens_per_s": world * dcfg.B / (gms * 1e-3),
                    "how": "one CUDA graph of the decode step, replayed; CUDA events on the stream"}
    if cpu_baseline:
        seqs = 2
        rate, dt = oracle_decode_rate(dinp, dcfg, seqs)
        out["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "us_per_query": 1e6 / rate,
                               "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{seqs} decode sequences of {dcfg.L} tokens (both branches, fp64), "
                                         f"{dt:.1f} s"}
        out["gpu_over_oracle"] = tok_s / rate
    del dinp, dws, do
    torch.cuda.empty_cache()
    return out


# oracle rows per configuration for the per-query rate (a few seconds of host time each)
ORACLE_ROWS = {"prefill-2k-tiny": 256, "prefill-32k": 16, "prefill-128k": 16, "prefill-1m": 2}


def config_report(cfg, dev, stream, args, peaks, rank) -> dict:
    """One more prefill configuration at N = 1: tokens/s, useful TFLOP/s, fractions of the
    measured bf16 burst peak, HBM rates of the memory-bound stages and the oracle's per-query
    rate on the host cores."""
    inp, rcfg, p, bufs = make_prefill(cfg, dev, cfg.seed, 0, False, 1, rank)
    steps = args.steps if cfg.N <= 131072 else max(2, min(args.steps, 3))
    ms, stats, _ = time_prefill(inp, p, bufs, steps, max(3, args.warmup), stream, dev, 1, False)
    st = stage_table(stats, steps)
    out = {"tokens_per_s": cfg.N / (ms * 1e-3), "ms_per_step": ms, "steps": steps,
           **prefill_rates(rcfg, ms, peaks, 1), "memory_bound": memory_bound_rates(st, rcfg, peaks),
           "stages": {k: round(v["ms_per_step"], 4) for k, v in st.items()}}
    if cfg.N <= 4096:
        # launch-bound: the forward captured once as a CUDA graph and replayed
        from block_sparse_long_tcgen05_b200 import msa
        g = graph_of(lambda: msa.msa_forward(p, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"],
                                             o=bufs["o"], block_ids=bufs["ids"], workspace=bufs["ws"]))
        gms = timed(g.replay, steps, stream)
        msa.check_device_error(dev)
        del g
        out["graph"] = {"ms_per_step": gms, "tokens_per_s": cfg.N / (gms * 1e-3)}
    if not args.no_cpu_baseline:
        rate, dt = oracle_rows_rate(inp, cfg, ORACLE_ROWS.get(cfg.name, 4), seed=11)
        out["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "us_per_query": 1e6 / rate,
                               "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{ORACLE_ROWS.get(cfg.name, 4)} seeded query rows of {cfg.name} "
                                         f"(both branches, fp64, inputs read from the device row by row), "
                                         f"{dt:.1f} s"}
        out["gpu_over_oracle"] = out["tokens_per_s"] / rate
    del inp, bufs
    torch.cuda.empty_cache()
    return out


def kl_report(cfg, dev, stream, args, peaks) -> dict:
    """The index-branch KL loss forward (msa_index_kl) on one configuration: per step one KL
    pass over every (query, group), given the forward's block ids and log-sum-exp. Useful work:
    per (query, head, selected token) 2 d FLOPs of logits, per (query, group, selected token)
    2 d_idx FLOPs of index scores; the kernel's tensor work also counts the index product on
    all R rows of a query (it repeats the index row per head) and whole blocks."""
    from block_sparse_long_tcgen05_b200 import msa
    inp, rcfg, p, bufs = make_prefill(cfg, dev, cfg.seed, 0, False, 1, 0)
    lse = torch.empty(cfg.N, cfg.Hq, dtype=torch.float32, device=dev)
    msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cfg.k, bk=cfg.Bk, block_ids=bufs["ids"],
                lse=lse, o=bufs["o"], workspace=bufs["ws"])
    kl = torch.empty(cfg.N, cfg.G, dtype=torch.float32, device=dev)
    kp = msa.prefill_params(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.k, bk=cfg.Bk)
    kws = torch.empty(max(256, msa.load_library().msa_index_kl_workspace(ctypes.byref(kp))), dtype=torch.uint8,
                      device=dev)

    def step():
        msa.index_kl(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], bufs["ids"], lse, bk=cfg.Bk, kl=kl,
                     workspace=kws)

    for _ in range(max(3, args.warmup)):
        step()
    msa.check_device_error(dev)
    msa.msa_profile_start()
    steps = max(3, min(args.steps, 10))
    ms = timed(step, steps, stream)
    stats = msa.msa_profile_stop()
    msa.check_device_error(dev)
    i = np.arange(cfg.N, dtype=np.int64)
    sel = accounting._selected_tokens(i, cfg.Bk, cfg.k).sum()
    useful = 2.0 * cfg.d * cfg.Hq * sel + 2.0 * cfg.d_idx * cfg.G * sel
    nsel_blocks = float(np.minimum(i // cfg.Bk + 1, cfg.k).sum())
    tensor = 2.0 * cfg.Bk * nsel_blocks * cfg.Hq * (cfg.d + cfg.d_idx)
    kl_ms = stats.get("kl", (1, ms))[1] / steps
    out = {"workload": cfg.name, "ms_per_step": ms, "steps": steps,
           "useful_tflops": useful / (ms * 1e-3) / 1e12,
           "kl_kernel": {"ms_per_step": kl_ms, "tensor_tflops": tensor / (kl_ms * 1e-3) / 1e12,
                         "frac_bf16_burst": tensor / (kl_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]},
           "stages": {k: round(v[1] / steps, 4) for k, v in stats.items()},
           "mean_kl_nats": float(kl.mean().item())}
    del inp, bufs, lse, kl, kws
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    from block_sparse_long_tcgen05_b200 import msa
    msa.load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    cfg = synth.CONFIGS[args.workload]
    shard_groups = args.shard == "groups"
    inp, rcfg, p, bufs = make_prefill(cfg, dev, mdist.rank_seed(cfg.seed, rank), args.query_chunk, shard_groups,
                                      world, rank)
    seqs_per_job = 1 if shard_groups else world
    parallelism = (f"GQA groups sharded over {world} GPU(s), one sequence, no collective" if shard_groups
                   else "one independent sequence per GPU, no collective")
    N = cfg.N
    warmup = max(3, args.warmup)
    ms, stats, clk = time_prefill(inp, p, bufs, args.steps, warmup, stream, dev, world, rank == 0)
    value = seqs_per_job * N / (ms * 1e-3)   # tokens of the whole job over the slowest rank's time
    stages = stage_table(stats, args.steps)
    gpu_launches = sum(v[0] for v in stats.values())
    rates = prefill_rates(rcfg, ms, peaks, world)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if shard_groups else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based generator)",
            "config": workload_config(cfg, {"parallelism": parallelism}),
            "prefill": {"tokens_per_s": value, **rates},
            "stages": stages,
            "roofline": roofline(stats, args.steps, rcfg, peaks, peak_src, args.traffic,
                                 clk.get("sm_mhz") if clk else None),
            "gpu_launches": gpu_launches, "clocks": clk}
    if clk and clk.get("sm_mhz"):
        line["prefill"]["useful_tflops_per_sm_ghz"] = rates["useful_tflops_per_gpu"] / (clk["sm_mhz"] / 1000.0)
    try:   # reporting only: a failure here must not cost the measurement
        line["stage_rates"] = stage_rates(stages, rcfg, peaks)
        line["prefill"]["memory_bound"] = memory_bound_rates(stages, rcfg, peaks)
    except Exception as e:  # noqa: BLE001
        line["stage_rates"] = {"error": repr(e)}

    # ------------------------------------------------ decode (query-stationary), same ranks
    if not args.no_decode:
        line["decode"] = run_decode(args, dev, stream, world, rank, peaks,
                                    cpu_baseline=(world == 1 and not args.no_cpu_baseline))

    # ------------------------------------------------ end to end from pinned host memory
    if not args.no_e2e:
        # msa_forward_host: page-locked host inputs in, host output back; the library pipelines
        # the copies with the kernels chunk by chunk (all copies inside the timed region)
        host = {n: t.cpu().pin_memory() for n, t in inp.items()}
        o_h = torch.empty(bufs["o"].shape, dtype=bufs["o"].dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = o_h.numel() * o_h.element_size()
        dbuf = torch.empty(msa.msa_forward_host_device_bytes(p), dtype=torch.uint8, device=dev)

        def estep():
            msa.forward_host(p, host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"], o_h,
                             device_buf=dbuf, device=dev)

        estep()
        torch.cuda.synchronize(dev)
        msa.check_device_error(dev)
        same = bool(torch.equal(o_h, bufs["o"].cpu()))   # the same kernels on the same inputs: identical
        barrier(world)
        esteps = max(2, min(args.steps, 10))
        ems = max_over_ranks(timed(estep, esteps, stream), world)
        line["e2e"] = {"value": seqs_per_job * N / (ems * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": esteps,
                       "api": "msa_forward_host", "output_equals_device_path": same}
        del dbuf, host, o_h
        torch.cuda.empty_cache()

    # ------------------------------------------------ CPU oracle baseline (rank 0, N = 1)
    if world == 1 and not args.no_cpu_baseline:
        rate, dt = oracle_sample(inp, cfg, args.ref_rows * 2, seed=7)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{args.ref_rows * 2} seeded query rows of {cfg.name} "
                                          f"(both branches, fp64), {dt:.1f} s"}

    # ------------------------------------------------ the other synthetic configurations (N = 1)
    if world == 1 and not args.headline_only:
        headline = {"tokens_per_s": value, "ms_per_step": ms, "steps": args.steps, **rates,
                    "memory_bound": line["prefill"].get("memory_bound"),
                    "stages": {k: round(v["ms_per_step"], 4) for k, v in stages.items()}}
        if "cpu_baseline" in line:
            headline["cpu_baseline"] = dict(line["cpu_baseline"], us_per_query=1e6 / line["cpu_baseline"]["value"])
            headline["gpu_over_oracle"] = value / line["cpu_baseline"]["value"]
        del inp, bufs
        torch.cuda.empty_cache()
        configs = {}
        for name in ("prefill-2k-tiny", "prefill-32k", "prefill-128k", "decode-b64-128k", "prefill-1m"):
            try:
                if name == cfg.name:
                    configs[name] = headline
                elif name == "decode-b64-128k":
                    configs[name] = line.get("decode") or run_decode(args, dev, stream, 1, rank, peaks,
                                                                     not args.no_cpu_baseline)
                else:
                    configs[name] = config_report(synth.CONFIGS[name], dev, stream, args, peaks, rank)
            except Exception as e:  # noqa: BLE001  (reporting only)
                configs[name] = {"error": repr(e)}
        line["configs"] = configs
        # the block-size ablation's efficiency side (Bk = 64, 32 at the 128K shapes) and the KL loss
        for bk in (64, 32):
            c = dataclasses.replace(synth.P128K, name=f"prefill-128k-bk{bk}", Bk=bk)
            try:
                line.setdefault("block_sizes", {})[c.name] = config_report(c, dev, stream, args, peaks, rank)
            except Exception as e:  # noqa: BLE001
                line.setdefault("block_sizes", {})[c.name] = {"error": repr(e)}
        try:
            line["index_kl"] = kl_report(synth.P128K, dev, stream, args, peaks)
        except Exception as e:  # noqa: BLE001
            line["index_kl"] = {"error": repr(e)}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill-128k", choices=[c for c in synth.CONFIGS if "prefill" in c])
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the report of the other synthetic configurations (N = 1)")
    ap.add_argument("--only-kl", action="store_true",
                    help="measure only the index-branch KL loss forward on --workload (for profiling)")
    ap.add_argument("--shard", choices=["sequences", "groups"], default="sequences",
                    help="N > 1: one independent sequence per GPU (weak scaling) or the GQA groups of one "
                         "sequence split over the GPUs (strong scaling); no collective either way")
    ap.add_argument("--query-chunk", type=int, default=0,
                    help="queries per KV-outer chunk (multiple of 128; 0: the library default, 16384)")
    ap.add_argument("--traffic-json", default=os.path.join(ROOT, "profiles", "traffic.json"),
                    help="per-kernel DRAM bytes per launch from an ncu capture (null when absent)")
    args = ap.parse_args()
    args.traffic = {}
    if args.traffic_json and os.path.exists(args.traffic_json):
        tj = json.load(open(args.traffic_json))
        # counters only describe the kernels they were taken on: drop a kernel's figure once
        # its device source changed
        for kern, ent in tj.get(args.workload, {}).items():
            if isinstance(ent, dict) and ent.get("source_sha256") == kernel_sha256(kern):
                args.traffic[kern] = ent["bytes"]
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.only_kl:
            from block_sparse_long_tcgen05_b200 import msa
            msa.load_library()
            dev = torch.device("cuda", local)
            torch.cuda.set_device(dev)
            peaks, _ = load_peaks()
            out = kl_report(synth.CONFIGS[args.workload], dev, torch.cuda.current_stream(dev), args, peaks)
            if rank == 0:
                print(json.dumps({"index_kl": out}), flush=True)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
