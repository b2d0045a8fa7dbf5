"""C ABI checks that need no GPU: the library loads, exports every declared symbol, and
rejects bad arguments synchronously (before any CUDA work)."""
import ctypes
import os
import re

import pytest

from block_sparse_long_tcgen05_b200 import build as msa_build
from block_sparse_long_tcgen05_b200 import msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.load_library()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    assert set(names) == set(msa.EXPORTS), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {msa.LIB_PATH}").read()
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == sorted(declared_functions())


def test_status_strings(lib):
    for code, name in msa.STATUS.items():
        assert lib.msa_status_string(code).decode() == name


def test_validation_rejects_bad_arguments_without_cuda(lib):
    P = 1 << 12  # an aligned fake address: never dereferenced, validation fails first
    # NULL pointer
    assert lib.msa_index_select(None, P, 256, 2, 32, 128, 4, P, P, 1 << 30, None) == 1
    assert b"q_idx" in lib.msa_last_error_detail()
    # misaligned pointer
    assert lib.msa_index_select(P + 2, P, 256, 2, 32, 128, 4, P, P, 1 << 30, None) == 1
    # unsupported block size, d_idx, k
    assert lib.msa_index_select(P, P, 256, 2, 32, 96, 4, P, P, 1 << 30, None) == 2
    # block sizes below 128 take the one-kernel Index Branch only (k in 4, 8, 16, 32)
    assert lib.msa_index_select(P, P, 256, 2, 32, 64, 5, P, P, 1 << 30, None) == 2
    assert lib.msa_index_select_workspace(256, 2, 32, 64, 5) == 0
    assert lib.msa_index_select_workspace(256, 2, 32, 32, 8) > 0
    assert lib.msa_index_select(P, P, 256, 2, 48, 128, 4, P, P, 1 << 30, None) == 2
    assert lib.msa_index_select(P, P, 256, 2, 32, 128, 33, P, P, 1 << 30, None) == 2
    # bad n
    assert lib.msa_index_select(P, P, 0, 2, 32, 128, 4, P, P, 1 << 30, None) == 1
    # workspace too small
    need = lib.msa_index_select_workspace(4096, 2, 32, 128, 4)
    assert need > 0
    assert lib.msa_index_select(P, P, 4096, 2, 32, 128, 4, P, P, need - 1, None) == 3
    # heads not a multiple of groups / unsupported ratio / unsupported d
    assert lib.msa_sparse_attn(P, P, P, P, 256, 6, 4, 64, 128, 4, 0.0, P, P, 1 << 30, None) == 1
    assert lib.msa_sparse_attn(P, P, P, P, 256, 12, 4, 64, 128, 4, 0.0, P, P, 1 << 30, None) == 2
    assert lib.msa_sparse_attn(P, P, P, P, 256, 8, 2, 96, 128, 4, 0.0, P, P, 1 << 30, None) == 2
    assert lib.msa_sparse_attn(P, P, P, P, 256, 8, 2, 64, 128, 4, -1.0, P, P, 1 << 30, None) == 1
    assert lib.msa_sparse_attn(P, P, P, P, 256, 8, 2, 64, 128, 4, float("nan"), P, P, 1 << 30, None) == 1


def test_forward_param_validation(lib):
    P = 1 << 12
    p = msa.prefill_params(1000, 8, 2, 64, 32, 4)
    need = lib.msa_forward_workspace(ctypes.byref(p))
    assert need > 0
    p.query_chunk = 100   # not a multiple of 128
    assert lib.msa_forward_workspace(ctypes.byref(p)) == 0
    assert lib.msa_forward(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 1
    p.query_chunk = 0
    p.mode = 7
    assert lib.msa_forward(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 1
    d = msa.MsaParams(mode=1, hq=64, g=8, d=128, d_idx=128, bk=128, k=16, scale=0.0, n=4, lmax=1000,
                      seqlens=None, query_chunk=0)
    assert lib.msa_forward_workspace(ctypes.byref(d)) > 0
    assert lib.msa_forward(ctypes.byref(d), P, P, P, P, P, None, P, P, 1 << 40, None) == 1   # seqlens NULL
    d.lse_out = P
    assert lib.msa_forward(ctypes.byref(d), P, P, P, P, P, None, P, P, 1 << 40, None) == 2   # lse: prefill only
    p = msa.prefill_params(1000, 8, 2, 64, 32, 4)
    p.lse_out = P + 4                                                                       # unaligned
    assert lib.msa_forward(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 1


def test_index_kl_validation_without_cuda(lib):
    """msa_index_kl checks its shapes and pointers before anything is enqueued: prefill shapes,
    at most 8 heads per group, the Main Branch's sequence limit, a workspace large enough."""
    P = 1 << 12
    p = msa.prefill_params(3000, 16, 2, 128, 64, 8)
    need = lib.msa_index_kl_workspace(ctypes.byref(p))
    assert need > 0
    assert lib.msa_index_kl(ctypes.byref(p), P, P, P, P, P, P, 0.0, P, P, need - 1, None) == 3
    assert lib.msa_index_kl(ctypes.byref(p), P, P, P, P, P, None, 0.0, P, P, need, None) == 1   # lse NULL
    assert lib.msa_index_kl(ctypes.byref(p), P, P, P, P, P, P, -1.0, P, P, need, None) == 1     # idx_scale
    r16 = msa.prefill_params(3000, 32, 2, 128, 64, 8)                                          # 16 heads per group
    assert lib.msa_index_kl_workspace(ctypes.byref(r16)) == 0
    assert lib.msa_index_kl(ctypes.byref(r16), P, P, P, P, P, P, 0.0, P, P, 1 << 40, None) == 2
    dec = msa.MsaParams(mode=1, hq=16, g=2, d=128, d_idx=64, bk=128, k=8, scale=0.0, n=4, lmax=1000,
                        seqlens=P, query_chunk=0)
    assert lib.msa_index_kl(ctypes.byref(dec), P, P, P, P, P, P, 0.0, P, P, 1 << 40, None) == 2


def test_forward_host_validation_without_cuda(lib):
    """msa_forward_host checks everything before it touches a stream: prefill only, pointers,
    chunking, and the size of the device buffer (inputs + output + the forward workspace)."""
    P = 1 << 12
    p = msa.prefill_params(1000, 8, 2, 64, 32, 4)
    need = lib.msa_forward_host_device_bytes(ctypes.byref(p))
    io = 1000 * 8 * 64 * 2 * 2 + 2 * 1000 * 2 * 64 * 2 + 2 * 1000 * 2 * 32 * 2   # q, o, k, v, q_idx, k_idx
    assert need >= io + lib.msa_forward_workspace(ctypes.byref(p))
    assert lib.msa_forward_host(ctypes.byref(p), P, P, P, P, P, None, P, P, need - 1, None) == 3
    assert lib.msa_forward_host(ctypes.byref(p), P, None, P, P, P, None, P, P, need, None) == 1
    assert lib.msa_forward_host(ctypes.byref(p), P, P, P, P, P, None, P + 8, P, need, None) == 1   # unaligned o
    p.query_chunk = 100
    assert lib.msa_forward_host_device_bytes(ctypes.byref(p)) == 0
    assert lib.msa_forward_host(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 1
    d = msa.MsaParams(mode=1, hq=64, g=8, d=128, d_idx=128, bk=128, k=16, scale=0.0, n=4, lmax=1000,
                      seqlens=None, query_chunk=0)
    assert lib.msa_forward_host_device_bytes(ctypes.byref(d)) == 0
    assert lib.msa_forward_host(ctypes.byref(d), P, P, P, P, P, None, P, P, 1 << 40, None) == 2   # decode


def test_workspace_sizes_grow_with_problem(lib):
    a = lib.msa_sparse_attn_workspace(32768, 64, 8, 128, 128, 16)
    b = lib.msa_sparse_attn_workspace(131072, 64, 8, 128, 128, 16)
    assert 0 < a <= b
    # k = 16 at 128K takes the one-kernel Index Branch: no block maxima in memory
    assert 0 < lib.msa_index_select_workspace(131072, 8, 128, 128, 16) <= 4096
    # k = 5 takes the two-kernel path: the packed maxima triangle lives in the workspace
    assert lib.msa_index_select_workspace(131072, 8, 128, 128, 5) >= 4 * 8 * 128 * (1024 * 1023 // 2)
    # the one-kernel path serves k = 16 at every length (1M tokens: no maxima either)
    assert 0 < lib.msa_index_select_workspace(1 << 20, 8, 128, 128, 16) <= 4096
    assert lib.msa_index_select_workspace(524288, 8, 128, 128, 12) >= 4 * 8 * 128 * (4096 * 4095 // 2) // 8


def test_sequence_length_limits_are_checked_before_any_launch(lib):
    """Each path's longest sequence is validated with the other arguments, so nothing is
    enqueued for a problem that would fail part-way: the two-kernel Index Branch (odd k, or
    long sequences) takes at most 32768 query blocks (its key-run table), the Main Branch at
    most 14528 blocks (the CSR build's shared-memory masks)."""
    P = 1 << 12
    two_kernel_max = 32768 * 128
    csr_max = 14528 * 128
    # just above the two-kernel limit (g = 1): refused, and so is its workspace query
    assert lib.msa_index_select_workspace(two_kernel_max + 1, 1, 32, 128, 5) == 0
    assert lib.msa_index_select(P, P, two_kernel_max + 1, 1, 32, 128, 5, P, P, 1 << 40, None) == 2
    assert b"two-kernel" in lib.msa_last_error_detail()
    assert lib.msa_index_select_static(P, P, 5_000_000, 1, 32, 128, 5, P, None) == 2
    assert b"two-kernel" in lib.msa_last_error_detail()
    # at the limit the workspace query still answers
    assert lib.msa_index_select_workspace(two_kernel_max, 1, 32, 128, 5) > 0
    # Main Branch: the limit counts blocks, so it is 4x shorter in tokens at bk = 32
    assert lib.msa_sparse_attn_workspace(14528 * 32, 8, 2, 64, 32, 4) > 0
    assert lib.msa_sparse_attn_workspace(14528 * 32 + 1, 8, 2, 64, 32, 4) == 0
    assert lib.msa_sparse_attn_workspace(csr_max, 8, 2, 64, 128, 4) > 0
    assert lib.msa_sparse_attn_workspace(csr_max + 1, 8, 2, 64, 128, 4) == 0
    assert lib.msa_sparse_attn(P, P, P, P, csr_max + 1, 8, 2, 64, 128, 4, 0.0, P, P, 1 << 40, None) == 2
    assert b"Main Branch" in lib.msa_last_error_detail()
    p = msa.prefill_params(csr_max + 1, 8, 2, 64, 32, 4)
    assert lib.msa_forward_workspace(ctypes.byref(p)) == 0
    assert lib.msa_forward(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 2
    assert lib.msa_forward_host(ctypes.byref(p), P, P, P, P, P, None, P, P, 1 << 40, None) == 2
