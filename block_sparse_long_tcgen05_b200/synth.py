"""Seeded synthetic workloads for MiniMax Sparse Attention (MSA).

This module only draws numbers. It holds none of the method's arithmetic, and both
the CUDA path (tests, bench) and the CPU oracle take their inputs from here.

Every value comes from a counter-based generator: splitmix64 applied to
``seed * 2**40 + tensor_id * 2**34 + flat_index`` (Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014), written with torch int64
ops, so a tensor is the same on the CPU and on a GPU. Integer draws are exact there.
The Box-Muller normals are computed in fp64 and rounded to bf16 (round to nearest
even), so a 1-ulp difference in a device's fp64 log/cos would change a bf16 only
with negligible probability.

Workloads (the five synthetic configurations of the prefill/decode study):
  * Q, K, V: bf16 N(0, 1).
  * index q / index k: integers uniform in [-a, a] stored as bf16 (a = 3 tiny, 4 else).
  * "hot" blocks: a seeded set of floor(frac * nb) blocks per sequence. For each
    GQA group g, one integer direction h_g (entries uniform in [-2, 2]) is added to
    the index keys of every token of every hot block, so block popularity is skewed.
    Index keys stay integers in [-6, 6], exact in bf16.
"""
from __future__ import annotations

import dataclasses
import math

import torch

_M64 = (1 << 64) - 1


def _s64(x: int) -> int:
    """Reinterpret an unsigned 64-bit constant as a signed int64."""
    x &= _M64
    return x - (1 << 64) if x >= (1 << 63) else x


_GOLDEN = _s64(0x9E3779B97F4A7C15)
_MUL1 = _s64(0xBF58476D1CE4E5B9)
_MUL2 = _s64(0x94D049BB133111EB)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 lanes."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def splitmix64(x: torch.Tensor) -> torch.Tensor:
    """splitmix64 finaliser on int64 lanes (wrapping arithmetic)."""
    z = x + _GOLDEN
    z = (z ^ _srl(z, 30)) * _MUL1
    z = (z ^ _srl(z, 27)) * _MUL2
    return z ^ _srl(z, 31)


def _counters(seed: int, tensor_id: int, start: int, n: int, device) -> torch.Tensor:
    base = _s64((seed << 40) + (tensor_id << 34) + start)
    return torch.arange(n, dtype=torch.int64, device=device) + base


_CHUNK = 1 << 26  # lanes per generator pass, bounds temporaries to ~1.5 GB


def uniform_int(seed: int, tensor_id: int, shape, a: int, device="cpu",
                dtype=torch.bfloat16) -> torch.Tensor:
    """Integers uniform in [-a, a] (tiny modulo bias, 2a+1 << 2**53)."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=dtype, device=device)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        h = _srl(splitmix64(_counters(seed, tensor_id, s, m, device)), 11)
        out[s:s + m] = (torch.remainder(h, 2 * a + 1) - a).to(dtype)
    return out.view(*shape)


def normal_bf16(seed: int, tensor_id: int, shape, device="cpu") -> torch.Tensor:
    """N(0, 1) by Box-Muller in fp64, rounded to bf16."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    two53 = float(1 << 53)
    for s in range(0, n, _CHUNK):
        m = min(_CHUNK, n - s)
        c = _counters(seed, tensor_id, 2 * s, 2 * m, device)
        h = _srl(splitmix64(c), 11).to(torch.float64).view(m, 2)
        u1 = (h[:, 0] + 0.5) / two53
        u2 = (h[:, 1] + 0.5) / two53
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)
        out[s:s + m] = z.to(torch.bfloat16)
    return out.view(*shape)


def hot_block_ids(seed: int, tensor_id: int, nb: int, frac: float, device="cpu") -> torch.Tensor:
    """floor(frac * nb) distinct block ids, seeded, ascending."""
    m = int(math.floor(frac * nb))
    if m == 0:
        return torch.empty(0, dtype=torch.int64, device=device)
    keys = splitmix64(_counters(seed, tensor_id, 0, nb, device))
    order = torch.argsort(keys, stable=True)
    return torch.sort(order[:m]).values


# tensor ids (fixed: changing them changes every workload)
TID_Q, TID_K, TID_V, TID_QIDX, TID_KIDX, TID_HOTSET, TID_HOTDIR = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class PrefillConfig:
    name: str
    N: int
    Hq: int
    G: int
    d: int
    d_idx: int
    k: int
    Bk: int = 128
    idx_range: int = 4
    hot_frac: float = 0.0
    seed: int = 1000

    @property
    def R(self) -> int:
        return self.Hq // self.G

    @property
    def nb(self) -> int:
        return -(-self.N // self.Bk)


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    L: int          # tokens per sequence, including the new one
    Hq: int
    G: int
    d: int
    d_idx: int
    k: int
    Bk: int = 128
    idx_range: int = 4
    hot_frac: float = 0.05
    seed: int = 1003

    @property
    def R(self) -> int:
        return self.Hq // self.G


TINY = PrefillConfig("prefill-2k-tiny", N=2048, Hq=8, G=2, d=64, d_idx=32, k=4,
                     idx_range=3, hot_frac=0.0, seed=1000)
P32K = PrefillConfig("prefill-32k", N=32768, Hq=64, G=8, d=128, d_idx=128, k=16,
                     hot_frac=0.05, seed=1001)
P128K = PrefillConfig("prefill-128k", N=131072, Hq=64, G=8, d=128, d_idx=128, k=16,
                      hot_frac=0.05, seed=1002)
DEC128K = DecodeConfig("decode-b64-128k", B=64, L=131073, Hq=64, G=8, d=128, d_idx=128,
                       k=16, hot_frac=0.05, seed=1003)
P1M = PrefillConfig("prefill-1m", N=1048576, Hq=64, G=8, d=128, d_idx=128, k=16,
                    hot_frac=0.02, seed=1004)

CONFIGS = {c.name: c for c in (TINY, P32K, P128K, DEC128K, P1M)}


def _add_hot(k_idx: torch.Tensor, seed: int, seq: int, Bk: int, frac: float) -> None:
    """Add each group's hot direction to the index keys of the hot blocks (in place).

    k_idx: [L, G, d_idx] of one sequence.
    """
    L, G, d_idx = k_idx.shape
    nb = -(-L // Bk)
    hot = hot_block_ids(seed + 7919 * seq, TID_HOTSET, nb, frac, device=k_idx.device)
    if hot.numel() == 0:
        return
    hdir = uniform_int(seed + 7919 * seq, TID_HOTDIR, (G, d_idx), 2,
                       device=k_idx.device, dtype=torch.float32)
    for b in hot.tolist():
        lo, hi = b * Bk, min(L, (b + 1) * Bk)
        k_idx[lo:hi] = (k_idx[lo:hi].float() + hdir).to(k_idx.dtype)


def prefill_inputs(cfg: PrefillConfig, device="cpu", seed: int | None = None,
                   N: int | None = None) -> dict:
    """q [N,Hq,d], k/v [N,G,d], q_idx/k_idx [N,G,d_idx], all bf16.

    ``N`` overrides the configuration's length (ragged-tail tests); ``seed`` its seed.
    """
    seed = cfg.seed if seed is None else seed
    N = cfg.N if N is None else N
    q = normal_bf16(seed, TID_Q, (N, cfg.Hq, cfg.d), device)
    k = normal_bf16(seed, TID_K, (N, cfg.G, cfg.d), device)
    v = normal_bf16(seed, TID_V, (N, cfg.G, cfg.d), device)
    q_idx = uniform_int(seed, TID_QIDX, (N, cfg.G, cfg.d_idx), cfg.idx_range, device)
    k_idx = uniform_int(seed, TID_KIDX, (N, cfg.G, cfg.d_idx), cfg.idx_range, device)
    if cfg.hot_frac > 0:
        _add_hot(k_idx, seed, 0, cfg.Bk, cfg.hot_frac)
    return dict(q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx)


def decode_inputs(cfg: DecodeConfig, device="cpu", seed: int | None = None,
                  B: int | None = None, lengths=None, Lmax: int | None = None) -> dict:
    """One new token per sequence plus its contiguous cache.

    q [B,Hq,d], q_idx [B,G,d_idx]; caches k/v [B,Lmax,G,d], k_idx [B,Lmax,G,d_idx];
    seqlens [B] int32 counts the cached tokens plus the new one (whose k/v/k_idx sit
    at position seqlens-1). Cache rows at or beyond seqlens are zero.
    """
    seed = cfg.seed if seed is None else seed
    B = cfg.B if B is None else B
    if lengths is None:
        lengths = [cfg.L] * B
    lengths = [int(x) for x in lengths]
    Lmax = max(lengths) if Lmax is None else Lmax
    q = normal_bf16(seed, TID_Q, (B, cfg.Hq, cfg.d), device)
    q_idx = uniform_int(seed, TID_QIDX, (B, cfg.G, cfg.d_idx), cfg.idx_range, device)
    kc = torch.zeros(B, Lmax, cfg.G, cfg.d, dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    kic = torch.zeros(B, Lmax, cfg.G, cfg.d_idx, dtype=torch.bfloat16, device=device)
    for b, L in enumerate(lengths):
        s = seed + 104729 * (b + 1)
        kc[b, :L] = normal_bf16(s, TID_K, (L, cfg.G, cfg.d), device)
        vc[b, :L] = normal_bf16(s, TID_V, (L, cfg.G, cfg.d), device)
        kb = uniform_int(s, TID_KIDX, (L, cfg.G, cfg.d_idx), cfg.idx_range, device)
        if cfg.hot_frac > 0:
            _add_hot(kb, seed, b, cfg.Bk, cfg.hot_frac)
        kic[b, :L] = kb
    seqlens = torch.tensor(lengths, dtype=torch.int32, device=device)
    return dict(q=q, q_idx=q_idx, k_cache=kc, v_cache=vc, k_idx_cache=kic, seqlens=seqlens)
