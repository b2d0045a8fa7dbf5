"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bars: block selections bit-exact; outputs within |o - o_ref| <= 2e-2 + 2e-2 |o_ref|
elementwise (bf16 inputs, fp32 accumulation). Small cases check every row (several
tiles and a ragged tail); the full-size workloads check seeded sampled rows that
always include the edge rows {0, Bk-1, Bk, k*Bk-1, k*Bk, N-1}.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_tcgen05_b200 import msa, synth
from oracle import msa_oracle as orc

pytestmark = pytest.mark.gpu

ATOL = 2e-2
RTOL = 2e-2


def assert_close(o_gpu, o_ref, what=""):
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    bound = ATOL + RTOL * np.abs(o_ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                           f"max err {err.max():.3e}, worst excess {(err - bound).max():.3e}")


def host_f64(inp: dict) -> dict:
    """fp64 numpy copies of the inputs (exact): the oracle then indexes plain arrays, which
    is much faster than converting torch slices row by row."""
    return {n: t.detach().cpu().double().numpy() if t.is_floating_point() else t.detach().cpu().numpy()
            for n, t in inp.items()}


def oracle_prefill(inp: dict, rows, Bk: int, k: int):
    h = host_f64(inp)
    ids, _ = orc.index_select_rows(h["q_idx"], h["k_idx"], rows, Bk, k)
    return ids, orc.attend_rows(h["q"], h["k"], h["v"], ids, rows, Bk)


def sample_rows(N, k, Bk=128, n=64, seed=0):
    must = [0, Bk - 1, Bk, k * Bk - 1, k * Bk, N - 1]
    rng = np.random.default_rng(seed)
    extra = rng.choice(N, size=min(n, N), replace=False).tolist()
    return sorted(set(x for x in must + extra if 0 <= x < N))


def cfg_of(N, Hq, G, d, d_idx, k, hot=0.0, seed=77, idx_range=4, Bk=128):
    return synth.PrefillConfig("t", N=N, Hq=Hq, G=G, d=d, d_idx=d_idx, k=k, idx_range=idx_range,
                               hot_frac=hot, seed=seed, Bk=Bk)


def check_prefill(cfg, rows=None, query_chunk=0, check_all_ids=True):
    dev = torch.device("cuda")
    inp = synth.prefill_inputs(cfg, device=dev)
    ids_gpu = torch.empty(cfg.N, cfg.G, cfg.k, dtype=torch.int32, device=dev)
    o = msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cfg.k, bk=cfg.Bk, block_ids=ids_gpu,
                    query_chunk=query_chunk)
    msa.check_device_error()
    if rows is None:
        rows = list(range(cfg.N))
    if cfg.N * cfg.Hq * cfg.d > (1 << 31):
        # long sequences: the oracle reads the device tensors row by row (one group's index
        # keys at a time) instead of taking a host copy of every input
        ids_ref, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, cfg.Bk, cfg.k)
        o_ref = orc.attend_rows(inp["q"], inp["k"], inp["v"], ids_ref, rows, cfg.Bk)
    else:
        ids_ref, o_ref = oracle_prefill(inp, rows, cfg.Bk, cfg.k)
    ids_g = ids_gpu.cpu().numpy()
    np.testing.assert_array_equal(ids_g[rows], ids_ref)
    if check_all_ids:
        structural_ids_check(ids_g, cfg.Bk, cfg.k)
    rt = torch.as_tensor(rows, device=o.device)
    assert_close(o[rt].float().cpu().numpy(), o_ref, "prefill o")
    return inp, ids_gpu, o


def structural_ids_check(ids_g, Bk, k):
    """Rules every row must satisfy: min(k, bl + 1) valid ids, ascending, -1 padded, the
    local block last."""
    N = ids_g.shape[0]
    bl = np.arange(N) // Bk
    valid = ids_g >= 0
    nval = valid.sum(-1)
    assert np.array_equal(nval, np.broadcast_to(np.minimum(k, bl + 1)[:, None], nval.shape))
    assert not np.any(valid[..., 1:] & ~valid[..., :-1])          # -1 padding only at the end
    both = valid[..., 1:] & valid[..., :-1]
    assert np.all(np.diff(ids_g, axis=-1)[both] > 0)                  # strictly ascending
    last = np.take_along_axis(ids_g, (nval[..., None] - 1), axis=-1)[..., 0]
    assert np.array_equal(last, np.broadcast_to(bl[:, None], last.shape))


# ---------------------------------------------------------------- Index Branch alone

@pytest.mark.parametrize("N,G,d_idx,k", [(2048, 2, 32, 4), (2048 + 77, 3, 64, 8), (1500, 1, 128, 16),
                                         (640, 2, 128, 1), (5000, 2, 128, 32)])
def test_index_select_all_rows_bit_exact(cuda_ok, N, G, d_idx, k):
    cfg = cfg_of(N, G, G, 64, d_idx, k, hot=0.05, idx_range=3)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids = msa.msa_index_select(inp["q_idx"], inp["k_idx"], k)
    msa.check_device_error()
    h = host_f64(inp)
    ref, _ = orc.index_select_rows(h["q_idx"], h["k_idx"], range(N), 128, k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref)


@pytest.mark.parametrize("N,G,d_idx,k,Bk", [(2048 + 77, 2, 128, 16, 64), (3000, 3, 32, 8, 32),
                                             (5000, 2, 64, 32, 32), (4000, 8, 128, 4, 64), (700, 1, 32, 16, 32)])
def test_index_select_block_sizes_bit_exact(cuda_ok, N, G, d_idx, k, Bk):
    """Block sizes 64 and 32 of the block-size ablation (hyper.ai page, Experiment): each
    128-key tile holds several blocks, and rows see the earlier blocks of their own tile."""
    cfg = cfg_of(N, G, G, 64, d_idx, k, hot=0.05, idx_range=3, Bk=Bk)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids = msa.msa_index_select(inp["q_idx"], inp["k_idx"], k, bk=Bk)
    msa.check_device_error()
    h = host_f64(inp)
    ref, _ = orc.index_select_rows(h["q_idx"], h["k_idx"], range(N), Bk, k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref)


def test_index_select_all_equal_scores_tie_rule(cuda_ok):
    """Every block score equal: the lowest block indices win (plus the local block)."""
    N, G, k = 3000, 2, 5
    q_idx = torch.ones(N, G, 32, dtype=torch.bfloat16, device="cuda")
    k_idx = torch.ones(N, G, 32, dtype=torch.bfloat16, device="cuda")
    ids = msa.msa_index_select(q_idx, k_idx, k).cpu().numpy()
    for i in (0, 127, 128, 600, 2999):
        bl = i // 128
        want = list(range(bl + 1))[:k] if bl + 1 <= k else [0, 1, 2, 3, bl]
        want = want + [-1] * (k - len(want))
        assert list(ids[i, 0]) == want and list(ids[i, 1]) == want


def test_index_select_negative_zero_ties(cuda_ok):
    """Scores of exactly zero from opposite-signed terms tie with plain zeros."""
    N, G, k = 1024, 1, 3
    q_idx = torch.zeros(N, G, 32, dtype=torch.bfloat16, device="cuda")
    q_idx[:, :, 0] = 1
    q_idx[:, :, 1] = 1
    k_idx = torch.zeros(N, G, 32, dtype=torch.bfloat16, device="cuda")
    k_idx[256:384, :, 0] = -1      # block 2: scores -1 + 1 = 0 (exact)
    k_idx[256:384, :, 1] = 1
    ids = msa.msa_index_select(q_idx, k_idx, k).cpu().numpy()
    ref, _ = orc.index_select_rows(q_idx.cpu(), k_idx.cpu(), range(N), 128, k)
    np.testing.assert_array_equal(ids, ref)


# ---------------------------------------------------------------- Main Branch alone

@pytest.mark.parametrize("N,Hq,G,d", [(2048, 8, 2, 64), (1000, 16, 2, 128), (777, 4, 4, 64),
                                      (900, 32, 2, 128), (640, 4, 2, 128)])
def test_sparse_attn_all_rows(cuda_ok, N, Hq, G, d):
    cfg = cfg_of(N, Hq, G, d, 32, 4, seed=5)
    inp = synth.prefill_inputs(cfg, device="cuda")
    h = host_f64(inp)
    ref_ids, _ = orc.index_select_rows(h["q_idx"], h["k_idx"], range(N), 128, 4)
    ids = torch.from_numpy(ref_ids).cuda()
    o = msa.msa_sparse_attn(inp["q"], inp["k"], inp["v"], ids)
    msa.check_device_error()
    o_ref = orc.attend_rows(h["q"], h["k"], h["v"], ref_ids, range(N), 128)
    assert_close(o.float().cpu().numpy(), o_ref, "sparse_attn")


def test_sparse_attn_rejects_bad_ids_on_device(cuda_ok):
    """Ids above the query's own block are reported as MSA_ERR_DEVICE_BOUNDS (no fault)."""
    cfg = cfg_of(512, 8, 2, 64, 32, 4)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids = torch.full((512, 2, 4), -1, dtype=torch.int32, device="cuda")
    ids[:, :, 0] = torch.div(torch.arange(512, device="cuda"), 128, rounding_mode="floor")[:, None].int()
    ids[5, 1, 0] = 3                     # row 5 lives in block 0
    msa.msa_sparse_attn(inp["q"], inp["k"], inp["v"], ids)
    assert msa.msa_get_device_error() == 6
    assert msa.msa_get_device_error() == 0   # cleared


# ---------------------------------------------------------------- both branches

def test_forward_tiny_config_all_rows(cuda_ok):
    """The 2K tiny configuration (Hq=8, G=2, d=64, d_idx=32, k=4): every row."""
    check_prefill(synth.TINY)


def test_forward_dense_reduction(cuda_ok):
    """k * Bk covering the context: MSA equals dense causal GQA (oracle, fp64)."""
    cfg = cfg_of(1024 + 50, 8, 2, 64, 32, 9)
    check_prefill(cfg)


@pytest.mark.parametrize("query_chunk", [128, 256, 384])
def test_forward_query_chunks(cuda_ok, query_chunk):
    cfg = cfg_of(1300, 16, 2, 128, 64, 4, hot=0.1)
    check_prefill(cfg, query_chunk=query_chunk)


@pytest.mark.parametrize("N,Hq,G,d,d_idx,k,rows", [(4000, 16, 2, 128, 128, 17, None), (5000, 16, 2, 128, 128, 32, None),
                                                    (4600 + 33, 16, 4, 64, 64, 32, None),
                                                    (5000, 64, 8, 128, 128, 32, 400)])
def test_forward_large_k(cuda_ok, N, Hq, G, d, d_idx, k, rows):
    """k above 16: slot ids 16..31 in the inverted index, the merge's combination of more than
    16 slots, and (k = 32) the one-kernel Index Branch's longest running list; k = 17 takes
    the two-kernel Index Branch. R = 8 heads per group with hot blocks; every row (or, at
    the workload's 64 heads, seeded rows plus the edge rows); the sequences are long enough
    (more than k blocks) that the later rows make a real selection."""
    cfg = cfg_of(N, Hq, G, d, d_idx, k, hot=0.05, seed=40 + k)
    check_prefill(cfg, rows=None if rows is None else sample_rows(N, k, n=rows, seed=k))


@pytest.mark.parametrize("N,Hq,G,d,d_idx,k,Bk", [(3000, 16, 2, 128, 128, 16, 64), (2500, 8, 2, 64, 32, 8, 32),
                                                 (2000 + 33, 64, 8, 128, 128, 32, 32), (1500, 4, 4, 64, 64, 4, 64)])
def test_forward_block_sizes_all_rows(cuda_ok, N, Hq, G, d, d_idx, k, Bk):
    """Both branches at block sizes 64 and 32: K/V blocks of Bk keys in the KV-outer pass, the
    causal mask inside Bk-token local blocks, Bk-block buckets in the inverted index."""
    check_prefill(cfg_of(N, Hq, G, d, d_idx, k, hot=0.05, seed=60 + Bk + k, Bk=Bk), query_chunk=1024)


def test_forward_32k_sampled(cuda_ok):
    check_prefill(synth.P32K, rows=sample_rows(32768, 16, n=96, seed=1))


@pytest.mark.slow
def test_forward_128k_sampled(cuda_ok):
    """The headline 128K configuration, in the launch configuration the bench times."""
    check_prefill(synth.P128K, rows=sample_rows(131072, 16, n=48, seed=2), check_all_ids=True)


@pytest.mark.slow
def test_forward_1m_sampled(cuda_ok):
    """The 1M-token configuration: the two-kernel Index Branch (block maxima in chunks of at
    most 4 GiB) and 64 query chunks of the Main Branch; sampled rows against the oracle,
    structural rules on every row."""
    check_prefill(synth.P1M, rows=sample_rows(1 << 20, 16, n=10, seed=3), check_all_ids=True)


def test_forward_host_matches_device_path(cuda_ok):
    """msa_forward_host (host tensors in and out, copies pipelined with the chunks) gives the
    device path's output and block ids bit for bit; several query chunks and a ragged tail."""
    cfg = cfg_of(5000, 16, 2, 128, 64, 8, hot=0.1, seed=21)
    inp = synth.prefill_inputs(cfg, device="cuda")
    p = msa.prefill_params(cfg.N, cfg.Hq, cfg.G, cfg.d, cfg.d_idx, cfg.k, query_chunk=1024)
    ids_d = torch.empty(cfg.N, cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    o_d = msa.msa_forward(p, inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], block_ids=ids_d)
    host = {n: t.cpu().pin_memory() for n, t in inp.items()}
    o_h = torch.empty(o_d.shape, dtype=o_d.dtype, pin_memory=True)
    ids_h = torch.empty(ids_d.shape, dtype=torch.int32, pin_memory=True)
    for _ in range(2):   # the device buffer is reused by the second call
        o_h.zero_()
        msa.forward_host(p, host["q"], host["k"], host["v"], host["q_idx"], host["k_idx"], o_h, block_ids=ids_h)
        torch.cuda.synchronize()
        msa.check_device_error()
        assert torch.equal(ids_h, ids_d.cpu())
        assert torch.equal(o_h, o_d.cpu())
    rows = sample_rows(cfg.N, cfg.k, n=24, seed=5)
    ids_ref, o_ref = oracle_prefill(inp, rows, cfg.Bk, cfg.k)
    np.testing.assert_array_equal(ids_h.numpy()[rows], ids_ref)
    assert_close(o_h.float().numpy()[rows], o_ref, "forward_host o")


def test_group_shard_equals_slice_of_full_forward(cuda_ok):
    """Group sharding (bench.py --shard groups): the forward on one rank's groups gives, bit for
    bit, those groups' heads and block ids of the full forward (two ranks emulated on one GPU,
    one after the other; no rank waits on another)."""
    from block_sparse_long_tcgen05_b200 import dist as mdist
    cfg = cfg_of(3000, 16, 4, 128, 64, 6, hot=0.1, seed=31)
    inp = synth.prefill_inputs(cfg, device="cuda")
    ids_full = torch.empty(cfg.N, cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    o_full = msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cfg.k, block_ids=ids_full)
    world = 2
    for r in range(world):
        part = mdist.shard_inputs_by_group(inp, cfg.G, world, r)
        groups, hs, gs = mdist.group_slice(cfg.G, cfg.R, world, r)
        ids_p = torch.empty(cfg.N, len(groups), cfg.k, dtype=torch.int32, device="cuda")
        o_p = msa.prefill(part["q"], part["k"], part["v"], part["q_idx"], part["k_idx"], cfg.k, block_ids=ids_p)
        msa.check_device_error()
        assert torch.equal(ids_p, ids_full[:, gs])
        assert torch.equal(o_p, o_full[:, hs])
        # and against the oracle on the rank's own inputs: its groups of the full problem
        rows = sample_rows(cfg.N, cfg.k, n=24, seed=40 + r)
        ids_ref, o_ref = oracle_prefill(inp, rows, cfg.Bk, cfg.k)
        np.testing.assert_array_equal(ids_p.cpu().numpy()[rows], ids_ref[:, gs])
        assert_close(o_p.float().cpu().numpy()[rows], o_ref[:, hs], f"group shard {r}")


# ---------------------------------------------------------------- decode

def check_decode(cfg, lengths, seqs=None, Lmax=None):
    inp = synth.decode_inputs(cfg, device="cuda", lengths=lengths, Lmax=Lmax)
    ids = torch.empty(len(lengths), cfg.G, cfg.k, dtype=torch.int32, device="cuda")
    o = msa.decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["q_idx"], inp["k_idx_cache"], inp["seqlens"],
                   cfg.k, bk=cfg.Bk, block_ids=ids)
    msa.check_device_error()
    seqs = list(range(len(lengths))) if seqs is None else seqs
    ids_ref, o_ref = orc.decode_rows(inp, seqs, cfg.Bk, cfg.k)
    np.testing.assert_array_equal(ids.cpu().numpy()[seqs], ids_ref)
    assert_close(o.float().cpu().numpy()[seqs], o_ref, "decode o")


def test_decode_varied_lengths(cuda_ok):
    cfg = synth.DecodeConfig("t", B=9, L=0, Hq=64, G=8, d=128, d_idx=128, k=16, hot_frac=0.05, seed=9)
    check_decode(cfg, [1, 2, 127, 128, 129, 2048, 2049, 5000, 9000], Lmax=9001)


@pytest.mark.parametrize("k", [17, 32])
def test_decode_large_k(cuda_ok, k):
    """k above 16 on the decode path (its merge combines the slots past the first 16 one by
    one); lengths on both sides of k blocks and with every kind of partial last block."""
    cfg = synth.DecodeConfig("t", B=6, L=0, Hq=64, G=8, d=128, d_idx=128, k=k, hot_frac=0.05, seed=11 + k)
    check_decode(cfg, [k * 128 - 1, k * 128, k * 128 + 1, 5000, 9000, 300], Lmax=9001)


@pytest.mark.parametrize("Bk,k", [(64, 16), (32, 8)])
def test_decode_block_sizes(cuda_ok, Bk, k):
    """Decode at block sizes 64 and 32: a scan CTA covers several blocks of 128 tokens, the
    local block is the last partial Bk-block."""
    cfg = synth.DecodeConfig("t", B=7, L=0, Hq=64, G=8, d=128, d_idx=128, k=k, Bk=Bk, hot_frac=0.05, seed=13 + Bk)
    check_decode(cfg, [1, Bk - 1, Bk, Bk + 1, k * Bk + 3, 3000, 5001], Lmax=5001)


def test_decode_small_dims(cuda_ok):
    cfg = synth.DecodeConfig("t", B=5, L=0, Hq=8, G=2, d=64, d_idx=32, k=4, hot_frac=0.0, seed=10, idx_range=3)
    check_decode(cfg, [300, 700, 128, 1, 4096])


@pytest.mark.slow
def test_decode_full_size_sampled(cuda_ok):
    """Batch 64 x 131073 tokens (the decode configuration); the oracle checks 6 sequences."""
    check_decode(synth.DEC128K, [131073] * 64, seqs=[0, 1, 17, 31, 48, 63])


# ---------------------------------------------------------------- failure detection

def test_wait_timeout_is_reported_and_the_device_stays_usable(cuda_ok):
    """A gating-wait limit of 1 ns makes every pipelined kernel give up at its first wait that
    is not already satisfied: the call reports MSA_ERR_TIMEOUT through the error word (no hang,
    no fault: work already in flight is drained with the normal limit). With the default limit
    restored, the same device computes the tiny configuration exactly as before."""
    cfg = synth.TINY
    inp = synth.prefill_inputs(cfg, device="cuda")
    torch.cuda.synchronize()
    msa.set_wait_limit_ns(1)
    try:
        msa.prefill(inp["q"], inp["k"], inp["v"], inp["q_idx"], inp["k_idx"], cfg.k)
        st = msa.msa_get_device_error()
    finally:
        torch.cuda.synchronize()
        msa.set_wait_limit_ns(0)
    assert st == 5, msa.STATUS.get(st)
    assert msa.msa_get_device_error() == 0   # cleared
    check_prefill(cfg)
