"""The forward as a CUDA graph.

Every step of a forward is a kernel launch on the caller's stream: the library neither
synchronises nor allocates, and its grids depend only on the shapes in msa_params (and, for
decode, on Lmax), never on device data. A forward can therefore be captured once and
replayed on new contents of the captured buffers, which is how a decode step is served
without per-step launch overhead. The pass has no atomics, so a replay gives the eager
result bit for bit.
"""
import pytest
import torch

from block_sparse_long_tcgen05_b200 import msa, synth

pytestmark = pytest.mark.gpu


def _capture(fn) -> torch.cuda.CUDAGraph:
    # first use (kernel attributes, tensor maps) outside the capture
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_prefill_graph_replays_the_eager_forward(cuda_ok):
    cfg = synth.TINY
    inp = synth.prefill_inputs(cfg, device="cuda")
    p = msa.prefill_params(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.k, bk=cfg.Bk)
    ws = torch.empty(msa.msa_forward_workspace(p), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(inp["q"])
    ids = torch.empty(cfg.N, cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    g = _capture(lambda: msa.msa_forward(p, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], o=o,
                                         block_ids=ids, workspace=ws))
    for seed in (cfg.seed, cfg.seed + 1):
        new = synth.prefill_inputs(cfg, device="cuda", seed=seed)
        for name, t in new.items():
            inp[name].copy_(t)
        o.zero_()
        ids.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        msa.check_device_error()
        ids_ref = torch.empty_like(ids)
        o_ref = msa.msa_forward(p, new["q"], new["k"], new["v"], new["q_idx"], new["k_idx"], block_ids=ids_ref)
        msa.check_device_error()
        assert torch.equal(ids, ids_ref)
        assert torch.equal(o, o_ref)


def test_decode_graph_follows_new_lengths(cuda_ok):
    """One decode graph captured at Lmax serves steps whose sequences grow: the lengths are
    read on the device."""
    cfg = synth.DecodeConfig("t", B=5, L=0, Hq=16, G=2, d=128, d_idx=64, k=8, hot_frac=0.05, seed=31)
    Lmax = 3000
    inp = synth.decode_inputs(cfg, device="cuda", lengths=[1, 127, 700, 2048, 2999], Lmax=Lmax)
    o = torch.empty_like(inp["q"])
    ids = torch.empty(cfg.B, cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    p = msa.decode_params(cfg.B, Lmax, inp["seqlens"], cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.k, cfg.Bk)
    ws = torch.empty(msa.msa_forward_workspace(p), dtype=torch.uint8, device="cuda")
    g = _capture(lambda: msa.msa_forward(p, inp["q"], inp["k_cache"], inp["v_cache"], inp["q_idx"],
                                         inp["k_idx_cache"], o=o, block_ids=ids, workspace=ws))
    for lengths in ([1, 127, 700, 2048, 2999], [2, 128, 701, 2049, 3000], [129, 129, 1500, 2500, 3000]):
        new = synth.decode_inputs(cfg, device="cuda", lengths=lengths, Lmax=Lmax)
        for name, t in new.items():
            inp[name].copy_(t)
        o.zero_()
        g.replay()
        torch.cuda.synchronize()
        msa.check_device_error()
        ids_ref = torch.empty_like(ids)
        o_ref = msa.decode(new["q"], new["k_cache"], new["v_cache"], new["q_idx"], new["k_idx_cache"],
                           new["seqlens"], cfg.k, bk=cfg.Bk, block_ids=ids_ref)
        msa.check_device_error()
        assert torch.equal(ids, ids_ref)
        assert torch.equal(o, o_ref)
