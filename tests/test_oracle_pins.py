"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types the oracle's own code. Each compares it with something else:
a hand-worked example, a set characterisation of Top-k checked exhaustively, a library
attention routine (dense causal GQA), closed forms, or a metamorphic invariant. A
plausible slip in the oracle (a causal off-by-one, a mean instead of a max pool, the
wrong tie direction, a transposed head-to-group map, a wrong softmax scale) fails at
least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import msa_oracle as orc
from block_sparse_long_tcgen05_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------
# Index Branch
# ------------------------------------------------------------------------------------

def test_golden_index_branch_hand_worked():
    """hyper.ai 'MiniMax Sparse Attention', Method (score, Block Max Pooling, Top-k
    with the local block forced): the hand-worked cases in golden/index_branch_hand.json."""
    fx = json.load(open(os.path.join(GOLDEN, "index_branch_hand.json")))
    Bk = fx["Bk"]
    k_idx = np.asarray(fx["k_idx"], dtype=np.float64)[:, None, :]      # [N, G=1, d_idx]
    for case in fx["cases"]:
        i = case["i"]
        q_idx = np.zeros_like(k_idx)
        q_idx[i, 0] = case["q"]
        ids, scores = orc.index_select_rows(q_idx, k_idx, [i], Bk, case["k"])
        assert list(scores[0][0]) == case["block_scores"], case["derivation"]
        assert list(ids[0, 0]) == case["block_ids"], case["derivation"]


def _topk_is_correct(S, k, ids):
    """Set characterisation of the selection (not a sort): size, local block, order,
    padding, and dominance of every chosen non-local block over every unchosen one."""
    bl = len(S) - 1
    n = min(k, bl + 1)
    valid = [int(b) for b in ids if b >= 0]
    if len(valid) != n or any(b >= 0 for b in ids[n:]) or any(b < 0 for b in ids[:n]):
        return False
    if valid != sorted(set(valid)) or bl not in valid or max(valid) > bl:
        return False
    chosen = set(valid) - {bl}
    for b in chosen:
        for c in range(bl):
            if c in chosen:
                continue
            if not (S[b] > S[c] or (S[b] == S[c] and b < c)):
                return False
    return True


def test_topk_exhaustive_small_alphabet():
    """Top-k against its set characterisation on every score vector over {0,1,2}^L,
    L = 1..7, all k = 1..8 (many ties: the lower-index rule is exercised everywhere)."""
    count = 0
    for L in range(1, 8):
        for vec in itertools.product((0.0, 1.0, 2.0), repeat=L):
            S = np.asarray(vec)
            for k in range(1, 9):
                ids = orc.select_blocks(S, k)
                assert len(ids) == k
                assert _topk_is_correct(S, k, ids), (vec, k, ids)
                count += 1
    assert count == 8 * sum(3 ** L for L in range(1, 8))


def test_topk_characterisation_rejects_wrong_answers():
    """The characterisation is strict: wrong tie direction or a dropped local block fail."""
    S = np.asarray([1.0, 1.0, 0.0, 5.0])     # bl = 3
    assert _topk_is_correct(S, 2, np.asarray([0, 3]))
    assert not _topk_is_correct(S, 2, np.asarray([1, 3]))      # tie went to higher index
    assert not _topk_is_correct(S, 2, np.asarray([0, 1]))      # local block dropped
    assert not _topk_is_correct(S, 2, np.asarray([3, 0]))      # not ascending


def test_block_max_pool_brute_force_loops():
    """Block Max Pooling against explicit loops over (row, block, token) on a tiny case."""
    rng = np.random.default_rng(7)
    Bk, L = 4, 23
    scores = rng.integers(-9, 10, size=(L, L)).astype(np.float64)
    rows = np.arange(L)
    pooled = orc.block_max_pool(scores, rows, Bk)
    for i in range(L):
        bl = i // Bk
        assert len(pooled[i]) == bl + 1
        for b in range(bl + 1):
            best = None
            for j in range(b * Bk, (b + 1) * Bk):
                if j <= i and (best is None or scores[i, j] > best):
                    best = scores[i, j]
            assert pooled[i][b] == best


def test_token_scores_exact_for_integer_inputs():
    """Scores of integer index vectors equal the exact integer dot product (int64)."""
    rng = np.random.default_rng(3)
    q = rng.integers(-4, 5, size=(5, 128))
    kk = rng.integers(-6, 7, size=(300, 128))
    s = orc.token_scores(q.astype(np.float64), kk.astype(np.float64))
    exact = q.astype(np.int64) @ kk.astype(np.int64).T
    assert np.array_equal(s, exact.astype(np.float64))


def _tiny_inputs(N=1024, seed=11, **kw):
    cfg = synth.PrefillConfig("t", N=N, Hq=kw.get("Hq", 8), G=kw.get("G", 2),
                              d=kw.get("d", 64), d_idx=kw.get("d_idx", 32),
                              k=kw.get("k", 4), idx_range=3, hot_frac=kw.get("hot", 0.0),
                              seed=seed)
    return cfg, synth.prefill_inputs(cfg)


def test_metamorphic_scaling_index_query_keeps_selection():
    """Exp-free Top-k (zhichai.net section 4.1): selection depends on order only, so a
    positive scale of the index query (x2, exact for these integers) changes nothing."""
    cfg, inp = _tiny_inputs(N=1024, seed=21)
    rows = list(range(0, 1024, 37)) + [1023]
    a, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, cfg.Bk, cfg.k)
    b, _ = orc.index_select_rows(inp["q_idx"] * 2, inp["k_idx"], rows, cfg.Bk, cfg.k)
    assert np.array_equal(a, b)


def test_metamorphic_permuting_inside_blocks_keeps_selection():
    """A block's max does not depend on the order of its tokens: permuting the index
    keys inside every complete block before the queries' own blocks keeps the selection."""
    cfg, inp = _tiny_inputs(N=1024, seed=22)
    Bk = cfg.Bk
    rows = [1023, 1000, 900, 897]                  # all in blocks 7 and 8..; permute blocks 0..6
    perm = torch.arange(1024)
    g = torch.Generator().manual_seed(5)
    for b in range(7):
        perm[b * Bk:(b + 1) * Bk] = b * Bk + torch.randperm(Bk, generator=g)
    a, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, Bk, cfg.k)
    b_, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"][perm], rows, Bk, cfg.k)
    assert np.array_equal(a, b_)


def test_local_block_always_selected():
    """Local block forced (hyper.ai page, Method; zhichai.net section 2), every row."""
    cfg, inp = _tiny_inputs(N=2048, seed=23)
    rows = list(range(0, 2048, 3))
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, cfg.Bk, cfg.k)
    for t, i in enumerate(rows):
        for g in range(cfg.G):
            assert i // cfg.Bk in ids[t, g]
            valid = ids[t, g][ids[t, g] >= 0]
            assert len(valid) == min(cfg.k, i // cfg.Bk + 1)
            assert np.all(np.diff(valid) > 0)


def test_selection_equals_topk_of_all_blocks_with_local_replacement():
    """The reading 'local block is one of the k' agrees with the alternative phrasing:
    take the k best of all visible blocks; if the local one is missing, it replaces the
    k-th. (Both describe the same set whenever the local block is forced.)"""
    rng = np.random.default_rng(9)
    for _ in range(2000):
        bl = int(rng.integers(0, 20))
        k = int(rng.integers(1, 8))
        S = rng.integers(0, 4, size=bl + 1).astype(np.float64)
        ids = orc.select_blocks(S, k)
        order = sorted(range(bl + 1), key=lambda b: (-S[b], b))
        top = order[:k]
        if bl not in top:
            top = top[:k - 1] + [bl]
        top = sorted(top)
        want = np.full(k, -1)
        want[:len(top)] = top
        assert np.array_equal(ids, want), (S, k, ids, want)


# ------------------------------------------------------------------------------------
# Main Branch
# ------------------------------------------------------------------------------------

def _dense_causal_gqa_torch(q, k, v):
    """Dense causal GQA with the library routine, fp64: heads h use kv head h // R."""
    qt = q.double().permute(1, 0, 2)[None]            # [1, Hq, N, d]
    kt = k.double().permute(1, 0, 2)[None]            # [1, G, N, d]
    vt = v.double().permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                         enable_gqa=True)
    return o[0].permute(1, 0, 2).numpy()              # [N, Hq, d]


@pytest.mark.parametrize("N,Hq,G,d,Bk", [(512, 8, 2, 64, 128), (300, 6, 3, 32, 128), (300, 8, 2, 32, 64),
                                          (200, 4, 2, 32, 32)])
def test_dense_reduction_equals_causal_gqa(N, Hq, G, d, Bk):
    """Pin (a): with k * Bk covering the causal context every visible block is selected,
    and the Main Branch ('standard scaled dot-product attention' over the selected
    tokens, hyper.ai page, Method) is dense causal GQA (torch SDPA, fp64). Also at the
    smaller block sizes of the block-size ablation (hyper.ai page, Experiment: 32, 64, 128)."""
    nb = -(-N // Bk)
    cfg, inp = _tiny_inputs(N=N, seed=31, Hq=Hq, G=G, d=d, k=nb)
    rows = list(range(N))
    ids, o = orc.prefill_rows(inp, rows, Bk, nb)
    ref = _dense_causal_gqa_torch(inp["q"], inp["k"], inp["v"])
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    # and the selection really is every visible block
    for i in rows:
        want = list(range(i // Bk + 1)) + [-1] * (nb - i // Bk - 1)
        assert list(ids[i, 0]) == want


def test_first_row_returns_first_value_exactly():
    """Closed form: query 0 sees only token 0, so o[0, h] = v[0, h // R]."""
    cfg, inp = _tiny_inputs(N=256, seed=41)
    ids, o = orc.prefill_rows(inp, [0], cfg.Bk, cfg.k)
    R = cfg.Hq // cfg.G
    for h in range(cfg.Hq):
        assert np.array_equal(o[0, h], inp["v"][0, h // R].double().numpy())


def test_zero_query_gives_mean_of_selected_values():
    """Closed form: q = 0 makes every logit 0, so o is the plain mean of v over the
    selected tokens j <= i (and only those)."""
    cfg, inp = _tiny_inputs(N=1024, seed=42)
    i = 1000
    inp = dict(inp)
    inp["q"] = inp["q"].clone()
    inp["q"][i] = 0
    ids, o = orc.prefill_rows(inp, [i], cfg.Bk, cfg.k)
    R = cfg.Hq // cfg.G
    for g in range(cfg.G):
        toks = [j for b in ids[0, g] if b >= 0 for j in range(b * 128, b * 128 + 128) if j <= i]
        mean = inp["v"][toks, g].double().mean(0).numpy()
        for r in range(R):
            np.testing.assert_allclose(o[0, g * R + r], mean, rtol=1e-12, atol=1e-14)


def test_two_token_softmax_closed_form():
    """Closed form: query 1 sees tokens 0 and 1 only, so
    o = sigmoid(a0 - a1) v0 + sigmoid(a1 - a0) v1 with a_j = q . k_j / sqrt(d)."""
    cfg, inp = _tiny_inputs(N=128, seed=43)
    ids, o = orc.prefill_rows(inp, [1], cfg.Bk, cfg.k)
    R = cfg.Hq // cfg.G
    d = cfg.d
    for h in range(cfg.Hq):
        g = h // R
        q = inp["q"][1, h].double()
        a0 = float(q @ inp["k"][0, g].double()) / math.sqrt(d)
        a1 = float(q @ inp["k"][1, g].double()) / math.sqrt(d)
        w0 = 1.0 / (1.0 + math.exp(a1 - a0))
        want = w0 * inp["v"][0, g].double() + (1 - w0) * inp["v"][1, g].double()
        np.testing.assert_allclose(o[0, h], want.numpy(), rtol=1e-12, atol=1e-14)


def test_unselected_blocks_do_not_influence_output():
    """Main Branch restricted to the selected tokens: changing k/v of a block that no
    row of a group selected leaves that group's outputs unchanged."""
    cfg, inp = _tiny_inputs(N=1024, seed=44)
    i = 1023
    ids, o = orc.prefill_rows(inp, [i], cfg.Bk, cfg.k)
    g = 0
    unselected = [b for b in range(8) if b not in ids[0, g]]
    assert unselected
    inp2 = dict(inp)
    inp2["k"] = inp["k"].clone()
    inp2["v"] = inp["v"].clone()
    b = unselected[0]
    inp2["k"][b * 128:(b + 1) * 128, g] += 3.0
    inp2["v"][b * 128:(b + 1) * 128, g] -= 2.0
    ids2, o2 = orc.prefill_rows(inp2, [i], cfg.Bk, cfg.k)
    assert np.array_equal(ids, ids2)
    R = cfg.Hq // cfg.G
    assert np.array_equal(o[0, :R], o2[0, :R])


def test_decode_query_equals_prefill_row():
    """Decode applies the same definition to the one new query at position L-1: with a
    cache holding a prefill sequence, decode equals that sequence's last prefill row."""
    cfg, inp = _tiny_inputs(N=700, seed=45)
    L = 700
    dec = dict(q=inp["q"][L - 1:L].clone(), q_idx=inp["q_idx"][L - 1:L].clone(),
               k_cache=inp["k"][None].clone(), v_cache=inp["v"][None].clone(),
               k_idx_cache=inp["k_idx"][None].clone(),
               seqlens=torch.tensor([L], dtype=torch.int32))
    ids_d, o_d = orc.decode_rows(dec, [0], cfg.Bk, cfg.k)
    ids_p, o_p = orc.prefill_rows(inp, [L - 1], cfg.Bk, cfg.k)
    assert np.array_equal(ids_d, ids_p)
    np.testing.assert_allclose(o_d, o_p, rtol=1e-13, atol=1e-15)


def test_lse_merge_identity():
    """Identity behind the merge of per-block partials (used by the GPU design and
    checked here in fp64): softmax over the union of blocks equals the log-sum-exp
    weighted combination of per-block normalised outputs."""
    rng = np.random.default_rng(5)
    d, T = 16, 5 * 7
    q = rng.standard_normal(d)
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    full = orc.sdpa(q[None], K, V, 0.25)[0]
    parts, lses = [], []
    for s in range(5):
        sl = slice(7 * s, 7 * s + 7)
        a = (K[sl] @ q) * 0.25
        m = a.max()
        l_ = np.exp(a - m).sum()
        parts.append(np.exp(a - m) @ V[sl] / l_)
        lses.append(m + math.log(l_))
    Lt = max(lses) + math.log(sum(math.exp(x - max(lses)) for x in lses))
    merged = sum(math.exp(x - Lt) * p for x, p in zip(lses, parts))
    np.testing.assert_allclose(merged, full, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("Bk", [32, 64])
def test_block_size_refines_the_selection_consistently(Bk):
    """Block sizes of the ablation (hyper.ai page, Experiment: 32, 64, 128). At Bk the pooled
    score of a block equals the max of the pooled scores of its halves at Bk / 2 (a max over a
    union), for every row and every non-local block; the local block of row i is i // Bk at
    every size; and with k = 1 only the local block is kept."""
    cfg, inp = _tiny_inputs(N=700, seed=53, Hq=4, G=2, d=32, k=4)
    rows = [0, Bk - 1, Bk, 3 * Bk + 5, 699]
    ids_a, sc_a = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, Bk, 4)
    ids_h, sc_h = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, Bk // 2, 4)
    for t, i in enumerate(rows):
        for g in range(2):
            A, H = sc_a[t][g], sc_h[t][g]
            assert len(A) == i // Bk + 1 and len(H) == i // (Bk // 2) + 1
            for b in range(len(A) - 1):
                assert A[b] == max(H[2 * b], H[2 * b + 1])
            assert i // Bk in ids_a[t, g]
    ids1, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, Bk, 1)
    assert [int(x) for x in ids1[:, 0, 0]] == [i // Bk for i in rows]


# ------------------------------------------------------------------------------------
# Index-branch KL loss (hyper.ai page, Method, fourth paragraph; zhichai.net section 五.1)
# ------------------------------------------------------------------------------------

def _kl_inputs(N=300, Hq=4, G=2, d=32, d_idx=32, seed=71, k=3):
    cfg = synth.PrefillConfig("t", N=N, Hq=Hq, G=G, d=d, d_idx=d_idx, k=k, idx_range=3, seed=seed)
    inp = synth.prefill_inputs(cfg)
    return cfg, inp


def test_kl_is_zero_when_the_index_head_mirrors_the_main_head():
    """One head per group (R = 1), index query/key equal to the head's query/key and the same
    scale: the two distributions coincide, so the KL is 0 on every row."""
    cfg, inp = _kl_inputs(Hq=2, G=2)
    rows = list(range(0, cfg.N, 7))
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    kl = orc.index_kl_rows(inp["q"], inp["k"], inp["q"], inp["k"], ids, rows, 128,
                           scale=0.3, idx_scale=0.3)
    assert np.abs(kl).max() < 1e-12


def test_kl_two_token_closed_form():
    """Query 1 sees tokens {0, 1}: with a = mean over the group's heads of sigma(l_h0 - l_h1)
    and b = sigma(c (y_0 - y_1)), KL = a ln(a / b) + (1 - a) ln((1 - a) / (1 - b)). With two
    heads per group this also fixes the order of averaging (mean of the distributions, not of
    per-head KLs) and the direction (Main Branch as the target)."""
    cfg, inp = _kl_inputs(Hq=4, G=2, d=16, d_idx=8, seed=5)
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], [1], 128, cfg.k)
    kl = orc.index_kl_rows(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, [1], 128)
    q = inp["q"].double().numpy()
    k = inp["k"].double().numpy()
    qi = inp["q_idx"].double().numpy()
    ki = inp["k_idx"].double().numpy()
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    for g in range(2):
        a = 0.0
        for h in (2 * g, 2 * g + 1):
            l0 = float(q[1, h] @ k[0, g]) / math.sqrt(16)
            l1 = float(q[1, h] @ k[1, g]) / math.sqrt(16)
            a += sig(l0 - l1) / 2
        b = sig((float(qi[1, g] @ ki[0, g]) - float(qi[1, g] @ ki[1, g])) / math.sqrt(8))
        want = a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b))
        assert kl[0, g] == pytest.approx(want, rel=1e-12, abs=1e-14)
        # the other direction differs on this input, so the test fixes it
        other = b * math.log(b / a) + (1 - b) * math.log((1 - b) / (1 - a))
        assert abs(other - want) > 1e-6


def test_kl_uniform_main_branch_closed_form():
    """Zero queries make every head's softmax uniform over the T selected tokens, so
    KL = -ln T - (1/T) sum_j log P_idx(j), with log P_idx from scipy's logsumexp."""
    from scipy.special import logsumexp
    cfg, inp = _kl_inputs(N=400, Hq=4, G=2, d=32, d_idx=32, seed=9, k=2)
    inp["q"] = torch.zeros_like(inp["q"])
    rows = [0, 5, 130, 255, 399]
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    kl = orc.index_kl_rows(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, rows, 128, idx_scale=0.25)
    qi = inp["q_idx"].double().numpy()
    ki = inp["k_idx"].double().numpy()
    for t, i in enumerate(rows):
        for g in range(2):
            toks = [j for b in ids[t, g] if b >= 0 for j in range(b * 128, min(b * 128 + 128, i + 1))]
            y = 0.25 * (ki[toks, g] @ qi[i, g])
            logp = y - logsumexp(y)
            want = -math.log(len(toks)) - float(np.mean(logp))
            assert kl[t, g] == pytest.approx(want, rel=1e-10, abs=1e-12)


def test_kl_nonnegative_and_zero_on_the_first_row():
    """Gibbs' inequality on every row; query 0 sees one token, both distributions are the
    same point mass."""
    cfg, inp = _kl_inputs(N=600, Hq=8, G=2, d=32, d_idx=16, seed=13, k=2)
    rows = list(range(0, 600, 11)) + [0]
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    kl = orc.index_kl_rows(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], ids, rows, 128)
    assert kl.min() > -1e-12
    assert np.abs(kl[-1]).max() < 1e-15


def test_lse_rows_closed_forms():
    """The Main Branch's log-sum-exp: row 0 sees one token, so lse = scale q0.k0; and exp(lse)
    is the softmax normaliser: sum_j exp(l_j - lse) = 1 over the selected tokens (checked
    with torch.logsumexp on the same logits)."""
    cfg, inp = _kl_inputs(N=400, Hq=4, G=2, d=32, d_idx=16, seed=17, k=2)
    rows = [0, 77, 260, 399]
    ids, _ = orc.index_select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    lse = orc.lse_rows(inp["q"], inp["k"], ids, rows, 128)
    q = inp["q"].double()
    k = inp["k"].double()
    for h in range(4):
        assert lse[0, h] == pytest.approx(float(q[0, h] @ k[0, h // 2]) / math.sqrt(32), rel=1e-13)
    for t, i in enumerate(rows):
        for h in range(4):
            g = h // 2
            toks = [j for b in ids[t, g] if b >= 0 for j in range(b * 128, min(b * 128 + 128, i + 1))]
            want = torch.logsumexp(k[toks, g] @ q[i, h] / math.sqrt(32), dim=0).item()
            assert lse[t, h] == pytest.approx(want, rel=1e-12)
