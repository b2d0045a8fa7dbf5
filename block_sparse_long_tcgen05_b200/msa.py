"""Python binding of the MSA C ABI (include/msa.h): argument marshalling only.

Every computation runs in libmsa.so's CUDA kernels. PyTorch supplies device memory
(outputs and workspace) and the current stream. There is no fallback: if the library
is missing or a call fails, these functions raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

MSA_OK = 0
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
          4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_DEVICE_BOUNDS"}
MODE_PREFILL, MODE_DECODE = 0, 1

# Every symbol include/msa.h declares.
EXPORTS = ("msa_index_select_workspace", "msa_index_select", "msa_sparse_attn_workspace", "msa_sparse_attn",
           "msa_forward_workspace", "msa_forward", "msa_get_device_error", "msa_status_string",
           "msa_last_error_detail", "msa_profile_start", "msa_profile_stop", "msa_index_select_static",
           "msa_forward_host_device_bytes", "msa_forward_host", "msa_index_kl_workspace", "msa_index_kl",
           "msa_set_wait_limit_ns")


class MsaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class MsaParams(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("hq", ctypes.c_int32), ("g", ctypes.c_int32),
                ("d", ctypes.c_int32), ("d_idx", ctypes.c_int32), ("bk", ctypes.c_int32),
                ("k", ctypes.c_int32), ("scale", ctypes.c_float), ("n", ctypes.c_int64),
                ("lmax", ctypes.c_int64), ("seqlens", ctypes.c_void_p), ("query_chunk", ctypes.c_int64),
                ("lse_out", ctypes.c_void_p)]


class MsaKernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsa.so and declare its signatures. Raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} (run block_sparse_long_tcgen05_b200/build.py)")
    lib = ctypes.CDLL(path)
    c_i32, c_i64, c_sz, c_p, c_f = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
    pp = ctypes.POINTER(MsaParams)
    sig = {
        "msa_index_select_workspace": (c_sz, [c_i64, c_i32, c_i32, c_i32, c_i32]),
        "msa_index_select": (c_i32, [c_p, c_p, c_i64, c_i32, c_i32, c_i32, c_i32, c_p, c_p, c_sz, c_p]),
        "msa_sparse_attn_workspace": (c_sz, [c_i64, c_i32, c_i32, c_i32, c_i32, c_i32]),
        "msa_sparse_attn": (c_i32, [c_p, c_p, c_p, c_p, c_i64, c_i32, c_i32, c_i32, c_i32, c_i32, c_f, c_p,
                                    c_p, c_sz, c_p]),
        "msa_forward_workspace": (c_sz, [pp]),
        "msa_forward": (c_i32, [pp, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "msa_get_device_error": (c_i32, [c_p]),
        "msa_status_string": (ctypes.c_char_p, [c_i32]),
        "msa_last_error_detail": (ctypes.c_char_p, []),
        "msa_profile_start": (c_i32, []),
        "msa_profile_stop": (c_i32, [ctypes.POINTER(MsaKernelStat), c_i32]),
        "msa_index_select_static": (c_i32, [c_p, c_p, c_i64, c_i32, c_i32, c_i32, c_i32, c_p, c_p]),
        "msa_forward_host_device_bytes": (c_sz, [pp]),
        "msa_forward_host": (c_i32, [pp, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "msa_index_kl_workspace": (c_sz, [pp]),
        "msa_index_kl": (c_i32, [pp, c_p, c_p, c_p, c_p, c_p, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "msa_set_wait_limit_ns": (c_i32, [ctypes.c_uint64]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != MSA_OK:
        lib = load_library()
        raise MsaError(status, lib.msa_last_error_detail().decode())


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _bf16(t: torch.Tensor, name: str) -> int:
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16")
    return _ptr(t)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _workspace(nbytes: int, device, workspace: torch.Tensor | None) -> torch.Tensor:
    if workspace is not None and workspace.numel() * workspace.element_size() >= nbytes:
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def msa_index_select_workspace(n: int, g: int, d_idx: int, k: int, bk: int = 128) -> int:
    return load_library().msa_index_select_workspace(n, g, d_idx, bk, k)


def msa_index_select(q_idx: torch.Tensor, k_idx: torch.Tensor, k: int, bk: int = 128,
                     block_ids: torch.Tensor | None = None, workspace: torch.Tensor | None = None
                     ) -> torch.Tensor:
    """Index Branch: q_idx, k_idx [N, G, d_idx] bf16 -> block_ids [N, G, k] int32."""
    lib = load_library()
    N, G, d_idx = q_idx.shape
    if tuple(k_idx.shape) != (N, G, d_idx):
        raise ValueError("k_idx shape must equal q_idx shape")
    if block_ids is None:
        block_ids = torch.empty(N, G, k, dtype=torch.int32, device=q_idx.device)
    need = lib.msa_index_select_workspace(N, G, d_idx, bk, k)
    ws = _workspace(need, q_idx.device, workspace)
    _check(lib.msa_index_select(_bf16(q_idx, "q_idx"), _bf16(k_idx, "k_idx"), N, G, d_idx, bk, k,
                                _ptr(block_ids), _ptr(ws), ws.numel(), _stream(q_idx.device)))
    return block_ids


def msa_sparse_attn_workspace(n: int, hq: int, g: int, d: int, k: int, bk: int = 128) -> int:
    return load_library().msa_sparse_attn_workspace(n, hq, g, d, bk, k)


def msa_sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_ids: torch.Tensor,
                    bk: int = 128, scale: float = 0.0, o: torch.Tensor | None = None,
                    workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Main Branch (KV-outer): q [N,Hq,d], k/v [N,G,d], block_ids [N,G,k] -> o [N,Hq,d]."""
    lib = load_library()
    N, Hq, d = q.shape
    G = k.shape[1]
    topk = block_ids.shape[2]
    if block_ids.dtype != torch.int32:
        raise ValueError("block_ids must be int32")
    if o is None:
        o = torch.empty_like(q)
    need = lib.msa_sparse_attn_workspace(N, Hq, G, d, bk, topk)
    ws = _workspace(need, q.device, workspace)
    _check(lib.msa_sparse_attn(_bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v"), _ptr(block_ids), N, Hq, G, d, bk,
                               topk, scale, _ptr(o), _ptr(ws), ws.numel(), _stream(q.device)))
    return o


def prefill_params(N: int, Hq: int, G: int, d: int, d_idx: int, k: int, bk: int = 128, scale: float = 0.0,
                   query_chunk: int = 0) -> MsaParams:
    return MsaParams(mode=MODE_PREFILL, hq=Hq, g=G, d=d, d_idx=d_idx, bk=bk, k=k, scale=scale, n=N, lmax=0,
                     seqlens=None, query_chunk=query_chunk)


def decode_params(B: int, Lmax: int, seqlens: torch.Tensor, Hq: int, G: int, d: int, d_idx: int, k: int,
                  bk: int = 128, scale: float = 0.0) -> MsaParams:
    return MsaParams(mode=MODE_DECODE, hq=Hq, g=G, d=d, d_idx=d_idx, bk=bk, k=k, scale=scale, n=B, lmax=Lmax,
                     seqlens=_ptr(seqlens), query_chunk=0)


def msa_forward_workspace(p: MsaParams) -> int:
    return load_library().msa_forward_workspace(ctypes.byref(p))


def msa_forward(p: MsaParams, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_idx: torch.Tensor,
                k_idx: torch.Tensor, o: torch.Tensor | None = None, block_ids: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Both branches (prefill or decode, per p.mode); returns o. See include/msa.h."""
    lib = load_library()
    if o is None:
        o = torch.empty_like(q)
    need = lib.msa_forward_workspace(ctypes.byref(p))
    if need == 0:
        raise MsaError(1, "unsupported or invalid msa_params")
    ws = _workspace(need, q.device, workspace)
    _check(lib.msa_forward(ctypes.byref(p), _bf16(q, "q"), _bf16(k, "k"), _bf16(v, "v"), _bf16(q_idx, "q_idx"),
                           _bf16(k_idx, "k_idx"), _ptr(block_ids), _ptr(o), _ptr(ws), ws.numel(),
                           _stream(q.device)))
    return o


def _host(t: torch.Tensor | None, name: str, dtype=torch.bfloat16) -> int | None:
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} host tensor")
    return t.data_ptr()


def msa_forward_host_device_bytes(p: MsaParams) -> int:
    return load_library().msa_forward_host_device_bytes(ctypes.byref(p))


def forward_host(p: MsaParams, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_idx: torch.Tensor,
                 k_idx: torch.Tensor, o: torch.Tensor, block_ids: torch.Tensor | None = None,
                 device_buf: torch.Tensor | None = None, device=None) -> torch.Tensor:
    """Prefill with host tensors in and out (page-locked for the copies to overlap the
    kernels); see msa_forward_host in include/msa.h. Enqueued on the current stream of
    `device`: o (and block_ids) are complete once that stream is."""
    lib = load_library()
    device = torch.device("cuda") if device is None else torch.device(device)
    need = lib.msa_forward_host_device_bytes(ctypes.byref(p))
    if need == 0:
        raise MsaError(1, "unsupported or invalid msa_params for msa_forward_host")
    buf = _workspace(need, device, device_buf)
    _check(lib.msa_forward_host(ctypes.byref(p), _host(q, "q"), _host(k, "k"), _host(v, "v"), _host(q_idx, "q_idx"),
                                _host(k_idx, "k_idx"), _host(block_ids, "block_ids", torch.int32), _host(o, "o"),
                                _ptr(buf), buf.numel() * buf.element_size(), _stream(device)))
    return o


def prefill(q, k, v, q_idx, k_idx, topk: int, bk: int = 128, scale: float = 0.0, query_chunk: int = 0,
            block_ids: torch.Tensor | None = None, o: torch.Tensor | None = None,
            workspace: torch.Tensor | None = None, lse: torch.Tensor | None = None) -> torch.Tensor:
    """Both branches of one sequence; with `lse` (float32 [N, Hq]) also the log-sum-exp of
    every (query, head)'s logits over its selected tokens, as index_kl takes it."""
    N, Hq, d = q.shape
    G, d_idx = q_idx.shape[1], q_idx.shape[2]
    p = prefill_params(N, Hq, G, d, d_idx, topk, bk, scale, query_chunk)
    if lse is not None:
        if lse.dtype != torch.float32 or tuple(lse.shape) != (N, Hq):
            raise ValueError("lse must be float32 [N, Hq]")
        p.lse_out = _ptr(lse)
    return msa_forward(p, q, k, v, q_idx, k_idx, o=o, block_ids=block_ids, workspace=workspace)


def index_kl(q, k, q_idx, k_idx, block_ids: torch.Tensor, lse: torch.Tensor, bk: int = 128, scale: float = 0.0,
             idx_scale: float = 0.0, query_chunk: int = 0, kl: torch.Tensor | None = None,
             workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Index-branch KL loss forward (msa_index_kl): KL(P_main || P_idx) per (query, group) ->
    float32 [N, G]; block_ids and lse as the prefill forward produced them."""
    lib = load_library()
    N, Hq, d = q.shape
    G, d_idx = q_idx.shape[1], q_idx.shape[2]
    topk = block_ids.shape[2]
    if block_ids.dtype != torch.int32 or lse.dtype != torch.float32:
        raise ValueError("block_ids must be int32 and lse float32")
    p = prefill_params(N, Hq, G, d, d_idx, topk, bk, scale, query_chunk)
    if kl is None:
        kl = torch.empty(N, G, dtype=torch.float32, device=q.device)
    need = lib.msa_index_kl_workspace(ctypes.byref(p))
    if need == 0:
        raise MsaError(2, "unsupported shape for msa_index_kl")
    ws = _workspace(need, q.device, workspace)
    _check(lib.msa_index_kl(ctypes.byref(p), _bf16(q, "q"), _bf16(k, "k"), _bf16(q_idx, "q_idx"),
                            _bf16(k_idx, "k_idx"), _ptr(block_ids), _ptr(lse), idx_scale, _ptr(kl), _ptr(ws),
                            ws.numel(), _stream(q.device)))
    return kl


def decode(q, k_cache, v_cache, q_idx, k_idx_cache, seqlens, topk: int, bk: int = 128, scale: float = 0.0,
           block_ids: torch.Tensor | None = None, o: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None) -> torch.Tensor:
    B, Hq, d = q.shape
    Lmax, G = k_cache.shape[1], k_cache.shape[2]
    d_idx = q_idx.shape[2]
    if seqlens.dtype != torch.int32:
        raise ValueError("seqlens must be int32")
    p = decode_params(B, Lmax, seqlens, Hq, G, d, d_idx, topk, bk, scale)
    return msa_forward(p, q, k_cache, v_cache, q_idx, k_idx_cache, o=o, block_ids=block_ids,
                       workspace=workspace)


def msa_get_device_error(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error status."""
    lib = load_library()
    dev = device if device is not None else torch.cuda.current_device()
    return lib.msa_get_device_error(_stream(dev))


def check_device_error(device=None) -> None:
    st = msa_get_device_error(device)
    if st != MSA_OK:
        raise MsaError(st, load_library().msa_last_error_detail().decode())


def set_wait_limit_ns(ns: int) -> None:
    """Time limit of the kernels' gating waits on the current device (0: the 2 s default)."""
    _check(load_library().msa_set_wait_limit_ns(int(ns)))


def msa_profile_start() -> None:
    """Start recording CUDA events around every launch of the library."""
    _check(load_library().msa_profile_start())


def msa_profile_stop() -> dict:
    """Stop recording; {kernel name: (launches, total device ms)} since msa_profile_start."""
    lib = load_library()
    buf = (MsaKernelStat * 32)()
    n = lib.msa_profile_stop(buf, 32)
    if n < 0:
        raise MsaError(4, "profile events failed")
    return {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n, 32))}
