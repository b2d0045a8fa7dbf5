"""The Index Branch entry point for callers that cannot allocate device memory.

msa_index_select_static serves callers that hold only a stream and raw pointers (a plugin
inside another framework's engine, a serving loop that forbids allocations after start-up)
and so cannot provide the workspace msa_index_select needs. Its scratch is a fixed array in
the library's device image. It must give the same selection as msa_index_select, call after
call, and reject problems whose scratch would not fit.

This file is collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_tcgen05_b200 import msa, synth


def _call_static(lib, q_idx, k_idx, k, out):
    N, G, d_idx = q_idx.shape
    return lib.msa_index_select_static(q_idx.data_ptr(), k_idx.data_ptr(), N, G, d_idx, 128, k, out.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)


def test_static_entry_rejects_problems_beyond_its_scratch():
    """Validation runs before any device work: a last query block needing more than the
    32 MiB scratch (here g = 64 groups at 1M tokens, k = 12, which takes the two-kernel
    path) is refused, not truncated; so is a sequence just above the two-kernel path's
    32768-block limit (g = 1, whose last block alone would still fit the scratch)."""
    lib = msa.load_library()
    P = 1 << 12   # aligned stand-in pointers; never dereferenced because validation fails first
    st = lib.msa_index_select_static(P, P, 1 << 20, 64, 128, 128, 12, P, None)
    assert st == 2, msa.STATUS.get(st)
    assert b"static scratch" in lib.msa_last_error_detail()
    st = lib.msa_index_select_static(P, P, 32768 * 128 + 1, 1, 128, 128, 12, P, None)
    assert st == 2, msa.STATUS.get(st)
    assert b"two-kernel" in lib.msa_last_error_detail()
    assert lib.msa_index_select_static(None, P, 1000, 2, 32, 128, 4, P, None) == 1


@pytest.mark.gpu
def test_static_entry_matches_workspace_entry_on_two_calls(cuda_ok):
    """Calls in a row, each compared with msa_index_select on the same inputs. The first two
    take the two-kernel path and so use the static scratch: the first (N = 40000 tokens,
    8 groups, k = 12) needs more maxima than the scratch holds in one launch, so it also
    exercises the cut into several launches; the second is a different shape whose stale
    scratch contents from the first call must not matter. The third (k = 16) takes the
    one-kernel path, which needs no scratch. Once the entry's set-up has run, further calls
    leave the device's free memory unchanged."""
    lib = msa.load_library()
    cases = [
        synth.PrefillConfig("a", N=40000, Hq=8, G=8, d=64, d_idx=128, k=12, hot_frac=0.05, seed=501),
        synth.PrefillConfig("b", N=3000 + 77, Hq=4, G=2, d=64, d_idx=32, k=5, idx_range=3, seed=502),
        synth.PrefillConfig("c", N=5000, Hq=4, G=2, d=64, d_idx=64, k=16, hot_frac=0.05, seed=503),
    ]
    for n_call, cfg in enumerate(cases):
        inp = synth.prefill_inputs(cfg, device="cuda")
        ref = msa.msa_index_select(inp["q_idx"], inp["k_idx"], cfg.k)
        out = torch.full_like(ref, -7)
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        st = _call_static(lib, inp["q_idx"], inp["k_idx"], cfg.k, out)
        assert st == 0, lib.msa_last_error_detail()
        assert msa.msa_get_device_error() == 0
        if n_call > 0:
            assert torch.cuda.mem_get_info()[0] == free0, "the static entry changed the device's free memory"
        np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())
