"""The work counts behind the benchmark's TFLOP/s and GB/s figures, checked against closed
forms (CPU only)."""
import pytest

from block_sparse_long_tcgen05_b200 import accounting


def test_index_flops_closed_form():
    # 2 * d_idx per visible token per (query, group): sum_{i < N} (i + 1) = N (N + 1) / 2
    N, G, d_idx = 131072, 8, 128
    idx, _ = accounting.prefill_useful_flops(N, 64, G, 128, d_idx, 128, 16)
    assert idx == 2 * d_idx * G * N * (N + 1) // 2
    assert idx == pytest.approx(17.59e12, rel=1e-3)


def test_main_flops_at_128k():
    # queries past the first k blocks select (k - 1) * Bk earlier tokens plus their own prefix
    # of the local block: on average 1969.5 tokens per query at 128K
    N, Hq, d, Bk, k = 131072, 64, 128, 128, 16
    _, main = accounting.prefill_useful_flops(N, Hq, 8, d, 128, Bk, k)
    first = sum(i + 1 for i in range(k * Bk))                      # rows whose blocks all fit
    rest = sum((k - 1) * Bk + (i % Bk) + 1 for i in range(k * Bk, N))
    assert main == 4 * d * Hq * (first + rest)
    assert (first + rest) / N == pytest.approx(1969.5, abs=0.5)
    assert main == pytest.approx(8.46e12, rel=1e-3)


def test_kernel_work_bounds_the_useful_work():
    N, Hq, G, d, Bk, k = 131072, 64, 8, 128, 128, 16
    _, main = accounting.prefill_useful_flops(N, Hq, G, d, 128, Bk, k)
    kv = accounting.kvouter_flops(N, Hq, d, Bk, k)
    assert main <= kv <= main * 1.07          # whole 128-key blocks: the local block's masked part
    nb = N // Bk
    assert accounting.index_kernel_flops(0, nb, G, 128) == 2 * 128 * G * Bk * Bk * nb * (nb - 1) // 2
    byts = accounting.main_branch_bytes(N, Hq, G, d, Bk, k)
    nsel = sum(min(i // Bk + 1, k) for i in range(N))
    R = Hq // G
    assert byts["merge"] == nsel * G * R * (2 * d + 8) + N * G * k * 4 + N * Hq * d * 2


def test_decode_flops():
    L, B = 131073, 64
    idx, main = accounting.decode_useful_flops([L] * B, 64, 8, 128, 128, 128, 16)
    assert idx == 2 * 128 * 8 * L * B
    assert idx == pytest.approx(17.2e9, rel=1e-2)
    assert main == 4 * 128 * 64 * B * (15 * 128 + ((L - 1) % 128) + 1)
