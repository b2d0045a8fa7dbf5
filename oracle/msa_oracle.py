"""CPU oracle for MiniMax Sparse Attention (MSA): plain, slow, fp64.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only the
tests, the package's smoke check and the benchmark's CPU-baseline leg do. It shares
no code with the CUDA library (no kernels, headers, tables or helpers); the only
common module is the seeded input generator, which holds none of the method's
arithmetic.

What it computes, step by step, in the order the method's description gives:

  Index Branch (hyper.ai "MiniMax Sparse Attention", Method, second paragraph;
  zhichai.net article, section 二 "Index Branch"):
    1. For each GQA group g, one index query head and one shared index key head:
       token score s_g(i, j) = q_idx[i, g] . k_idx[j, g] for every causally visible
       key token j <= i.
    2. Block Max Pooling: S_g(i, b) = max of s_g(i, j) over the tokens j <= i of
       block b (blocks of Bk = 128 consecutive tokens).
    3. Top-k over blocks per (query, group), with the block that holds the query
       (its local block) always included.
  Main Branch (hyper.ai page, Method, third paragraph; zhichai.net section 二
  "Main Branch"):
    4. For every query head h of group g: standard scaled dot-product softmax
       attention over the tokens of the selected blocks (j <= i), scale 1/sqrt(d).
       All heads of a group share the group's block set.

Readings where the pages are silent (each also listed in the design notes):
  * the local block is one of the k (budget k * Bk tokens per query, zhichai.net
    section 二 "关键参数");
  * ties between equal block scores go to the lower block index;
  * with fewer than k visible blocks every visible block is selected, and the row
    is padded with -1;
  * block_ids of a row are listed in ascending block order;
  * query head h belongs to group h // (Hq // G) (contiguous grouping);
  * decode: the new token sits at position L-1 of its sequence, and the same
    definition is applied to that one query.

Index-branch KL loss (hyper.ai page, Method, fourth paragraph; zhichai.net section 五.1):
    5. For every (query i, group g), over the tokens T of the selected blocks (j <= i):
       the Main Branch's group-averaged distribution P_main(j) = mean over the group's
       heads of softmax_T(q[i,h] . k[j,g] * scale), the Index Branch's distribution
       P_idx(j) = softmax_T(s_g(i, j) * idx_scale), and KL(P_main || P_idx) =
       sum_j P_main(j) (log P_main(j) - log P_idx(j)) in natural log units. The pages leave
       the index distribution's normalisation open; the readings taken here (softmax over
       the selected tokens, idx_scale = 1 / sqrt(d_idx) by default, the Main Branch as the
       target) are listed in the design notes.

Precision. Scores are computed with an fp64 matrix product. When every index input
is an integer (all the synthetic workloads), every partial sum is an integer below
2**53, so the scores are exact and the selection is the exact one. The main branch
runs in fp64 with a max-subtracted exp.
"""
from __future__ import annotations

import numpy as np
import torch

NEG_INF = -np.inf


def to_f64(x) -> np.ndarray:
    """Exact upcast of a (bf16) torch tensor or array to a float64 numpy array."""
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------------------
# Index Branch
# --------------------------------------------------------------------------------------

def token_scores(q_idx_rows: np.ndarray, k_idx_g: np.ndarray) -> np.ndarray:
    """Step 1: s(i, j) = q_idx[i] . k_idx[j] for one group (all j; causality is step 2).

    q_idx_rows: [r, d_idx] fp64; k_idx_g: [L, d_idx] fp64 -> [r, L] fp64.
    """
    return q_idx_rows @ k_idx_g.T


def block_max_pool(scores: np.ndarray, positions: np.ndarray, Bk: int) -> list:
    """Step 2: per row, S(b) = max over tokens j <= i of block b, for b = 0..bl(i).

    scores: [r, L] token scores (L >= max position + 1); positions: [r] query
    positions i. Tokens after the query are masked to -inf (causality), the token
    axis is cut into blocks of Bk and each block is reduced with max. Returns a list
    of length-r arrays, row t holding bl(i_t) + 1 block scores; the last one is the
    local block's, which only counts the tokens j <= i.
    """
    r, L = scores.shape
    nbk = -(-L // Bk)
    padded = np.full((r, nbk * Bk), NEG_INF, dtype=np.float64)
    padded[:, :L] = scores
    j = np.arange(nbk * Bk)
    padded[j[None, :] > positions[:, None]] = NEG_INF        # causal: j <= i
    pooled = padded.reshape(r, nbk, Bk).max(axis=2)
    return [pooled[t, :int(i) // Bk + 1].copy() for t, i in enumerate(positions)]


def select_blocks(S_row: np.ndarray, k: int) -> np.ndarray:
    """Step 3: Top-k blocks of one (query, group) row, local block forced.

    S_row holds the block scores of blocks 0..bl, bl being the query's local block.
    Returns k int32 ids: ascending, padded with -1.

    Order of preference among non-local blocks: higher score first, lower block
    index first among equal scores (a full stable sort, so there is no partial
    selection to get wrong). The local block takes one of the k places.
    """
    bl = len(S_row) - 1
    ids = np.full(k, -1, dtype=np.int32)
    if bl + 1 <= k:
        ids[:bl + 1] = np.arange(bl + 1, dtype=np.int32)
        return ids
    # a stable sort on descending score keeps ascending block order within ties
    order = np.argsort(-S_row[:bl], kind="stable")
    chosen = np.sort(np.append(order[:k - 1], bl))
    ids[:] = chosen.astype(np.int32)
    return ids


def index_select_rows(q_idx, k_idx, rows, Bk: int, k: int, row_chunk: int = 256):
    """Index Branch for the given query rows of one sequence.

    q_idx, k_idx: [N, G, d_idx] (torch bf16 or numpy). rows: iterable of query
    positions. Returns (block_ids [r, G, k] int32, block_scores: list over rows of
    [G] lists of score arrays).
    """
    rows = np.asarray(list(rows), dtype=np.int64)
    N, G, _ = k_idx.shape
    out = np.full((len(rows), G, k), -1, dtype=np.int32)
    all_scores = [[None] * G for _ in range(len(rows))]
    for g in range(G):
        kg = to_f64(k_idx[:, g, :])
        for c0 in range(0, len(rows), row_chunk):
            rr = rows[c0:c0 + row_chunk]
            qg = to_f64(q_idx[torch.as_tensor(rr), g, :]) if isinstance(q_idx, torch.Tensor) \
                else to_f64(q_idx[rr, g, :])
            hi = int(rr.max()) + 1
            s = token_scores(qg, kg[:hi])
            pooled = block_max_pool(s, rr, Bk)
            for t, S_row in enumerate(pooled):
                out[c0 + t, g] = select_blocks(S_row, k)
                all_scores[c0 + t][g] = S_row
    return out, all_scores


# --------------------------------------------------------------------------------------
# Main Branch
# --------------------------------------------------------------------------------------

def selected_tokens(ids: np.ndarray, i: int, Bk: int) -> np.ndarray:
    """Token positions of the selected blocks that query i may see (j <= i)."""
    toks = []
    for b in ids:
        if b < 0:
            continue
        lo = int(b) * Bk
        hi = min((int(b) + 1) * Bk, i + 1)
        toks.append(np.arange(lo, hi, dtype=np.int64))
    return np.concatenate(toks) if toks else np.empty(0, dtype=np.int64)


def sdpa(q_heads: np.ndarray, keys: np.ndarray, vals: np.ndarray, scale: float) -> np.ndarray:
    """Standard softmax(q k^T * scale) v in fp64. q_heads [R, d], keys/vals [T, d]."""
    logits = (q_heads @ keys.T) * scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ vals) / p.sum(axis=1, keepdims=True)


def attend_rows(q, k, v, block_ids: np.ndarray, rows, Bk: int, scale: float | None = None):
    """Main Branch for the given query rows.

    q [N, Hq, d], k/v [N, G, d] (torch bf16 or numpy), block_ids [r, G, k] for the
    rows. Returns o [r, Hq, d] fp64.
    """
    rows = np.asarray(list(rows), dtype=np.int64)
    N, Hq, d = q.shape
    G = k.shape[1]
    R = Hq // G
    scale = (1.0 / np.sqrt(d)) if not scale else scale
    out = np.zeros((len(rows), Hq, d), dtype=np.float64)
    for t, i in enumerate(rows):
        i = int(i)
        qi = to_f64(q[i])
        for g in range(G):
            toks = selected_tokens(block_ids[t, g], i, Bk)
            tk = torch.as_tensor(toks) if isinstance(k, torch.Tensor) else toks
            keys = to_f64(k[tk, g, :])
            vals = to_f64(v[tk, g, :])
            out[t, g * R:(g + 1) * R] = sdpa(qi[g * R:(g + 1) * R], keys, vals, scale)
    return out


def lse_rows(q, k, block_ids: np.ndarray, rows, Bk: int, scale: float | None = None) -> np.ndarray:
    """Natural-log log-sum-exp of each (row, head)'s scaled logits over the tokens of its
    group's selected blocks (j <= i): the normaliser of step 4's softmax. [r, Hq] fp64."""
    rows = np.asarray(list(rows), dtype=np.int64)
    N, Hq, d = q.shape
    G = k.shape[1]
    R = Hq // G
    scale = (1.0 / np.sqrt(d)) if not scale else scale
    out = np.zeros((len(rows), Hq), dtype=np.float64)
    for t, i in enumerate(rows):
        i = int(i)
        qi = to_f64(q[i])
        for g in range(G):
            toks = selected_tokens(block_ids[t, g], i, Bk)
            tk = torch.as_tensor(toks) if isinstance(k, torch.Tensor) else toks
            logits = (to_f64(k[tk, g, :]) @ qi[g * R:(g + 1) * R].T).T * scale    # [R, T]
            m = logits.max(axis=1)
            out[t, g * R:(g + 1) * R] = m + np.log(np.exp(logits - m[:, None]).sum(axis=1))
    return out


def prefill_rows(inp: dict, rows, Bk: int, k: int, scale: float | None = None):
    """Both branches for sampled query rows of one prefill sequence.

    inp: dict with q, k, v, q_idx, k_idx (torch, any device; copied to host here).
    Returns (block_ids [r, G, k] int32, o [r, Hq, d] fp64).
    """
    host = {n: t.detach().cpu() for n, t in inp.items()}
    ids, _ = index_select_rows(host["q_idx"], host["k_idx"], rows, Bk, k)
    o = attend_rows(host["q"], host["k"], host["v"], ids, rows, Bk, scale)
    return ids, o


def decode_rows(inp: dict, seqs, Bk: int, k: int, scale: float | None = None):
    """Decode: for each listed sequence b, the one new query at position L_b - 1.

    inp: q [B,Hq,d], q_idx [B,G,d_idx], k_cache/v_cache [B,Lmax,G,d],
    k_idx_cache [B,Lmax,G,d_idx], seqlens [B]. Returns (block_ids [s, G, k],
    o [s, Hq, d] fp64) for the listed sequences.
    """
    seqs = list(seqs)
    G = inp["q_idx"].shape[1]
    Hq, d = inp["q"].shape[1], inp["q"].shape[2]
    ids_out = np.full((len(seqs), G, k), -1, dtype=np.int32)
    o_out = np.zeros((len(seqs), Hq, d), dtype=np.float64)
    lens = inp["seqlens"].detach().cpu().numpy()
    for t, b in enumerate(seqs):
        L = int(lens[b])
        p = L - 1
        kic = inp["k_idx_cache"][b, :L].detach().cpu()
        qi = inp["q_idx"][b].detach().cpu()
        # place the single query at position p of a length-L sequence
        for g in range(G):
            s = token_scores(to_f64(qi[g:g + 1]), to_f64(kic[:, g, :]))
            S_row = block_max_pool(s, np.array([p]), Bk)[0]
            ids_out[t, g] = select_blocks(S_row, k)
        kc = inp["k_cache"][b, :L].detach().cpu()
        vc = inp["v_cache"][b, :L].detach().cpu()
        qf = inp["q"][b].detach().cpu()
        R = Hq // G
        sc = (1.0 / np.sqrt(d)) if not scale else scale
        qh = to_f64(qf)
        for g in range(G):
            toks = torch.as_tensor(selected_tokens(ids_out[t, g], p, Bk))
            o_out[t, g * R:(g + 1) * R] = sdpa(qh[g * R:(g + 1) * R], to_f64(kc[toks, g, :]),
                                               to_f64(vc[toks, g, :]), sc)
    return ids_out, o_out


# --------------------------------------------------------------------------------------
# Index-branch KL loss (forward)
# --------------------------------------------------------------------------------------

def log_softmax(x: np.ndarray) -> np.ndarray:
    """log softmax of a 1-D fp64 array (max-subtracted)."""
    m = x.max()
    return x - m - np.log(np.exp(x - m).sum())


def index_kl_rows(q, k, q_idx, k_idx, block_ids: np.ndarray, rows, Bk: int, scale: float | None = None,
                  idx_scale: float | None = None) -> np.ndarray:
    """Step 5 for the given query rows: KL(P_main || P_idx) per (row, group), fp64.

    q [N, Hq, d], k [N, G, d], q_idx / k_idx [N, G, d_idx] (torch or numpy), block_ids
    [r, G, k] for the rows. The tokens are those the Main Branch attends (selected blocks,
    j <= i); P_main averages the softmax of the group's heads, P_idx is the softmax of the
    index scores over the same tokens.
    """
    rows = np.asarray(list(rows), dtype=np.int64)
    N, Hq, d = q.shape
    G, d_idx = k_idx.shape[1], k_idx.shape[2]
    R = Hq // G
    scale = (1.0 / np.sqrt(d)) if not scale else scale
    idx_scale = (1.0 / np.sqrt(d_idx)) if not idx_scale else idx_scale
    out = np.zeros((len(rows), G), dtype=np.float64)
    for t, i in enumerate(rows):
        i = int(i)
        qi = to_f64(q[i])
        qii = to_f64(q_idx[i])
        for g in range(G):
            toks = selected_tokens(block_ids[t, g], i, Bk)
            tk = torch.as_tensor(toks) if isinstance(k, torch.Tensor) else toks
            keys = to_f64(k[tk, g, :])
            ikeys = to_f64(k_idx[tk, g, :])
            p_main = np.zeros(len(toks), dtype=np.float64)
            for h in range(g * R, (g + 1) * R):
                p_main += np.exp(log_softmax((keys @ qi[h]) * scale))
            p_main /= R
            log_p_idx = log_softmax((ikeys @ qii[g]) * idx_scale)
            nz = p_main > 0
            out[t, g] = float(np.sum(p_main[nz] * (np.log(p_main[nz]) - log_p_idx[nz])))
    return out
