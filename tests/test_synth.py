"""The seeded input generator (CPU): reproducible, counter-based, and with the value ranges
and distributions the workload recipe states."""
import torch

from block_sparse_long_tcgen05_b200 import synth


def _cfg(**kw):
    base = dict(N=1500, Hq=8, G=2, d=64, d_idx=32, k=4, idx_range=3, hot_frac=0.0, seed=11)
    base.update(kw)
    return synth.PrefillConfig("t", **base)


def test_reproducible_and_seed_sensitive():
    a = synth.prefill_inputs(_cfg())
    b = synth.prefill_inputs(_cfg())
    c = synth.prefill_inputs(_cfg(), seed=12)
    for n in a:
        assert torch.equal(a[n], b[n])
        assert not torch.equal(a[n], c[n])


def test_counter_based_prefix():
    """A value depends only on (seed, tensor, position): a shorter sequence is a prefix."""
    full = synth.prefill_inputs(_cfg(N=1500))
    part = synth.prefill_inputs(_cfg(N=700))
    for n in full:
        assert torch.equal(full[n][:700], part[n])


def test_normals_and_integer_ranges():
    z = synth.normal_bf16(5, 1, (1 << 20,)).double()
    assert abs(z.mean().item()) < 0.01 and abs(z.std().item() - 1.0) < 0.01
    assert 0.68 < (z.abs() < 1).double().mean().item() < 0.69          # one-sigma mass
    u = synth.uniform_int(5, 2, (1 << 16,), 4).double()
    assert u.min().item() == -4 and u.max().item() == 4
    assert torch.equal(u, u.round())
    counts = torch.bincount((u + 4).long(), minlength=9).double()
    assert (counts / counts.mean() - 1).abs().max().item() < 0.05    # uniform over the 9 values


def test_hot_blocks_keep_index_keys_exact_integers():
    cfg = _cfg(N=128 * 40, idx_range=4, hot_frac=0.1)
    inp = synth.prefill_inputs(cfg)
    k = inp["k_idx"].double()
    assert torch.equal(k, k.round()) and k.abs().max().item() <= 6
    plain = synth.prefill_inputs(_cfg(N=128 * 40, idx_range=4, hot_frac=0.0))
    moved = (inp["k_idx"] != plain["k_idx"]).any(dim=-1).any(dim=-1)   # tokens whose keys changed
    blocks = moved.view(40, 128).any(dim=1)
    assert 1 <= int(blocks.sum()) <= 4                                 # floor(0.1 * 40) hot blocks
    assert torch.equal(inp["q_idx"], plain["q_idx"]) and torch.equal(inp["q"], plain["q"])


def test_decode_cache_layout():
    cfg = synth.DecodeConfig("t", B=3, L=0, Hq=8, G=2, d=64, d_idx=32, k=4, hot_frac=0.0, seed=9, idx_range=3)
    inp = synth.decode_inputs(cfg, lengths=[5, 300, 1], Lmax=320)
    assert inp["k_cache"].shape == (3, 320, 2, 64) and inp["k_idx_cache"].shape == (3, 320, 2, 32)
    assert inp["seqlens"].tolist() == [5, 300, 1]
    for b, L in enumerate([5, 300, 1]):
        assert torch.count_nonzero(inp["k_cache"][b, L:]) == 0                # rows past the sequence
        assert torch.count_nonzero(inp["v_cache"][b, :L]) > 0
