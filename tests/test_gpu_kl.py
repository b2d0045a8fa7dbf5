"""GPU parity of the index-branch KL loss forward (msa_index_kl) and of the forward's
log-sum-exp output, against the fp64 CPU oracle.

hyper.ai "MiniMax Sparse Attention", Method (fourth paragraph) and zhichai.net section 5.1:
KL(P_main || P_idx) over the selected tokens, P_main the group-averaged Main Branch
distribution. Tolerances, derived from the arithmetic: the logits come from bf16 inputs with
fp32 accumulation and the exponentials from the hardware ex2 (relative error near 2^-22), so
each probability carries a relative error of a few 1e-6; summed over up to 4096 tokens and
combined as A - c B + C LSE_y (terms of tens of nats) that stays well below
|kl - kl_ref| <= 1e-3 + 1e-3 |kl_ref|. The log-sum-exp: |lse - lse_ref| <= 1e-3 + 1e-4 |lse_ref|.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_tcgen05_b200 import msa, synth
from oracle import msa_oracle as orc

pytestmark = pytest.mark.gpu


def _close(a, ref, atol, rtol, what):
    a = np.asarray(a, dtype=np.float64)
    err = np.abs(a - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} out of tolerance, max err {err.max():.3e}"


@pytest.mark.parametrize("N,Hq,G,d,d_idx,k,Bk,rows", [
    (2048, 8, 2, 64, 32, 4, 128, None),            # the tiny configuration's shapes, every row
    (2500 + 77, 16, 4, 128, 64, 8, 64, None),
    (1800, 8, 2, 64, 128, 16, 32, None),
    (4200, 64, 8, 128, 128, 16, 128, 160),         # the workload dims (R = 8), sampled rows
    (1500, 2, 2, 64, 64, 8, 128, None),            # one head per group (R = 1)
    (1300 + 5, 4, 2, 128, 32, 4, 64, None),        # R = 2
])
def test_index_kl_matches_oracle(cuda_ok, N, Hq, G, d, d_idx, k, Bk, rows):
    cfg = synth.PrefillConfig("t", N=N, Hq=Hq, G=G, d=d, d_idx=d_idx, k=k, idx_range=3 if d_idx == 32 else 4,
                              hot_frac=0.05, seed=90 + k, Bk=Bk)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids = torch.empty(N, G, k, dtype=torch.int32, device="cuda")
    lse = torch.empty(N, Hq, dtype=torch.float32, device="cuda")
    msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], k, bk=Bk, block_ids=ids, lse=lse,
                query_chunk=1024)
    kl = msa.index_kl(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, lse, bk=Bk, query_chunk=1024)
    msa.check_device_error()
    if rows is None:
        sel = list(range(N))
    else:
        rng = np.random.default_rng(3)
        sel = sorted(set([0, 1, Bk - 1, Bk, k * Bk, N - 1] + rng.choice(N, size=rows, replace=False).tolist()))
    host = {n: t.cpu().double().numpy() for n, t in inp.items()}
    ids_ref, _ = orc.index_select_rows(host["q_idx"], host["k_idx"], sel, Bk, k)
    np.testing.assert_array_equal(ids.cpu().numpy()[sel], ids_ref)
    lse_ref = orc.lse_rows(host["q"], host["k"], ids_ref, sel, Bk)
    _close(lse.cpu().numpy()[sel], lse_ref, 1e-3, 1e-4, "lse")
    kl_ref = orc.index_kl_rows(host["q"], host["k"], host["q_idx"], host["k_idx"], ids_ref, sel, Bk)
    _close(kl.cpu().numpy()[sel], kl_ref, 1e-3, 1e-3, "kl")


def test_index_kl_is_deterministic_and_chunk_independent(cuda_ok):
    """The same call twice gives the same bits, and so does another query chunk (slots are
    merged in a fixed order; no atomics)."""
    cfg = synth.PrefillConfig("t", N=3000, Hq=16, G=2, d=128, d_idx=128, k=8, hot_frac=0.05, seed=7)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids = torch.empty(cfg.N, cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    lse = torch.empty(cfg.N, cfg.Hq, dtype=torch.float32, device="cuda")
    msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cfg.k, block_ids=ids, lse=lse)
    a = msa.index_kl(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, lse)
    b = msa.index_kl(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, lse)
    c = msa.index_kl(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, lse, query_chunk=512)
    msa.check_device_error()
    assert torch.equal(a, b) and torch.equal(a, c)
