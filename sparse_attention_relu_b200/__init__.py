"""Python binding of libdsa.so, the sm_100a DSA hot path.

Thin marshalling over the C ABI declared in include/dsa.h: every function
here has the name of the C entry point it calls, takes torch tensors that
already live on the GPU, passes their device pointers and the current CUDA
stream, and raises DSAError on a non-zero status.  All computation happens
in the library's CUDA kernels; there is no fallback of any kind -- a missing
or unloadable libdsa.so raises at import of the first call.

Storage conventions: bf16 tensors are torch.bfloat16, e4m3 tensors
torch.float8_e4m3fn, scales and weights torch.float32, indices torch.int32.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARGUMENT, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE = 0, 1, 2, 3
DSA_ERR_CUDA, DSA_ERR_TIMEOUT, DSA_ERR_DEVICE_DATA = 4, 5, 6
DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
DSA_PREFILL, DSA_DECODE, DSA_CHUNKED = 0, 1, 2

_DTYPE_CODE = {torch.float32: DSA_F32, torch.bfloat16: DSA_BF16, torch.float8_e4m3fn: DSA_E4M3}


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dsa_status_string(status)} (status {status})")


class dsa_layout_t(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("kv_offsets", ctypes.c_void_p), ("max_len", ctypes.c_int32),
                ("n_q", ctypes.c_int32), ("n_k", ctypes.c_int64),
                ("q_offsets", ctypes.c_void_p)]


class dsa_forward_args_t(ctypes.Structure):
    _fields_ = [("idx_dtype", ctypes.c_int32), ("H_I", ctypes.c_int32), ("D_I", ctypes.c_int32),
                ("q_idx", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("k_idx", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("H", ctypes.c_int32), ("D_K", ctypes.c_int32), ("D_V", ctypes.c_int32),
                ("sm_scale", ctypes.c_float), ("q", ctypes.c_void_p), ("kv", ctypes.c_void_p),
                ("k", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("kv_scale", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded libdsa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not built ({LIB_PATH}); run "
                               "python -m sparse_attention_relu_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        LP = ctypes.POINTER(dsa_layout_t)
        AP = ctypes.POINTER(dsa_forward_args_t)
        L.dsa_indexer_scores.argtypes = [LP, P, P, P, P, P, I32, I32, I32, P, P]
        L.dsa_topk.argtypes = [LP, P, I32, P, P]
        L.dsa_sparse_mla_attn.argtypes = [LP, P, P, P, I32, I32, I32, I32, ctypes.c_float, P, P,
                                          P, SZ, P]
        L.dsa_sparse_mla_attn_noalloc.argtypes = [LP, P, P, P, I32, I32, I32, I32,
                                                  ctypes.c_float, P, P, P]
        L.dsa_sparse_mla_attn_e4m3.argtypes = [LP, P, P, P, P, I32, I32, I32, I32,
                                               ctypes.c_float, P, P, P, SZ, P]
        L.dsa_sparse_mla_attn_workspace_size.argtypes = [LP, I32, I32, I32, I32]
        L.dsa_sparse_mla_attn_workspace_size.restype = SZ
        L.dsa_forward_workspace_size.argtypes = [LP, AP]
        L.dsa_forward_workspace_size.restype = SZ
        L.dsa_forward.argtypes = [LP, AP, P, P, P, P, SZ, P]
        L.dsa_forward_timed.argtypes = [LP, AP, P, P, P, P, SZ, P, P, I32, P, P]
        L.dsa_forward_host_workspace_size.argtypes = [LP, AP, I32]
        L.dsa_forward_host_workspace_size.restype = SZ
        L.dsa_forward_host.argtypes = [LP, AP, AP, P, P, P, P, I32, P, SZ, P]
        L.dsa_device_status.argtypes = [P]
        L.dsa_selftest_wait_timeout.argtypes = [I64, P]
        L.dsa_status_string.argtypes = [ctypes.c_int]
        L.dsa_status_string.restype = ctypes.c_char_p
        L.dsa_abi_version.restype = I32
        for name in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn",
                     "dsa_sparse_mla_attn_noalloc", "dsa_sparse_mla_attn_e4m3", "dsa_forward",
                     "dsa_forward_timed", "dsa_forward_host", "dsa_device_status",
                     "dsa_selftest_wait_timeout"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def dsa_status_string(status: int) -> str:
    return lib().dsa_status_string(int(status)).decode()


def dsa_abi_version() -> int:
    return lib().dsa_abi_version()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libdsa takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return t.data_ptr() or None


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != DSA_OK:
        raise DSAError(status, where)


class Layout:
    """The ragged layout of include/dsa.h, built from a device int32 offsets tensor."""

    def __init__(self, kv_offsets: torch.Tensor, mode: int, max_len: int, n_q: int, n_k: int,
                 q_offsets: torch.Tensor = None):
        self.kv_offsets = kv_offsets  # keeps the tensors alive
        self.q_offsets = q_offsets
        self.c = dsa_layout_t(int(mode), int(kv_offsets.numel() - 1), _ptr(kv_offsets),
                              int(max_len), int(n_q), int(n_k), _ptr(q_offsets))

    @classmethod
    def of(cls, wl, kv_offsets: torch.Tensor, q_offsets: torch.Tensor = None):
        """Layout of a workloads.Workload whose offsets already sit on the device
        (q_offsets: the chunked mode's query offsets, on the device too)."""
        mode = {"prefill": DSA_PREFILL, "decode": DSA_DECODE, "chunked": DSA_CHUNKED}[wl.cfg.mode]
        if mode == DSA_CHUNKED and q_offsets is None:
            raise ValueError("chunked layout needs the device q_offsets")
        return cls(kv_offsets, mode, wl.max_len, wl.n_q, wl.n_k, q_offsets)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def dsa_indexer_scores(layout: Layout, q_idx, q_scale, w, k_idx, k_scale, scores, stream=None):
    """Stage 1: scores[n_q, max_len] (fp32) of the lightning indexer."""
    n_q, H_I, D_I = q_idx.shape
    dt = _DTYPE_CODE[q_idx.dtype]
    _check(lib().dsa_indexer_scores(layout.ref, _ptr(q_idx), _ptr(q_scale), _ptr(w), _ptr(k_idx),
                                    _ptr(k_scale), dt, H_I, D_I, _ptr(scores), _stream(stream)),
           "dsa_indexer_scores")
    return scores


def dsa_topk(layout: Layout, scores, k: int, idx, stream=None):
    """Stage 2: idx[n_q, k] (int32, local positions, -1 padded)."""
    _check(lib().dsa_topk(layout.ref, _ptr(scores), int(k), _ptr(idx), _stream(stream)), "dsa_topk")
    return idx


def dsa_sparse_mla_attn_workspace_size(layout: Layout, k: int, H: int, D_K: int, D_V: int) -> int:
    return lib().dsa_sparse_mla_attn_workspace_size(layout.ref, k, H, D_K, D_V)


def dsa_sparse_mla_attn(layout: Layout, q, kv, idx, k: int, D_V: int, sm_scale: float, out,
                        lse=None, workspace=None, stream=None):
    """Stage 3: out[n_q, H, D_V] (bf16) and lse[n_q, H] (fp32)."""
    _, H, D_K = q.shape
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_sparse_mla_attn(layout.ref, _ptr(q), _ptr(kv), _ptr(idx), int(k), H, D_K,
                                     int(D_V), float(sm_scale), _ptr(out), _ptr(lse),
                                     _ptr(workspace), ws_bytes, _stream(stream)),
           "dsa_sparse_mla_attn")
    return out


def dsa_sparse_mla_attn_e4m3(layout: Layout, q, kv, kv_scale, idx, k: int, D_V: int,
                             sm_scale: float, out, lse=None, workspace=None, stream=None):
    """Stage 3 over an FP8 cache: kv[n_k, D_K] float8_e4m3fn codes with one fp32
    scale per token (kv_scale[n_k]); out and lse as dsa_sparse_mla_attn."""
    _, H, D_K = q.shape
    if kv.dtype != torch.float8_e4m3fn:
        raise ValueError("dsa_sparse_mla_attn_e4m3 takes a float8_e4m3fn cache")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_sparse_mla_attn_e4m3(layout.ref, _ptr(q), _ptr(kv), _ptr(kv_scale),
                                          _ptr(idx), int(k), H, D_K, int(D_V), float(sm_scale),
                                          _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                          _stream(stream)),
           "dsa_sparse_mla_attn_e4m3")
    return out


def dsa_sparse_mla_attn_noalloc(layout: Layout, q, kv, idx, k: int, D_V: int, sm_scale: float,
                                out, lse=None, stream=None):
    """Stage 3 without a workspace: the library's fixed device scratch holds
    the split partials (for callers that cannot allocate; see include/dsa.h)."""
    _, H, D_K = q.shape
    _check(lib().dsa_sparse_mla_attn_noalloc(layout.ref, _ptr(q), _ptr(kv), _ptr(idx), int(k), H,
                                             D_K, int(D_V), float(sm_scale), _ptr(out), _ptr(lse),
                                             _stream(stream)),
           "dsa_sparse_mla_attn_noalloc")
    return out


def _hptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("expected a host tensor")
    if not t.is_contiguous():
        raise ValueError("libdsa takes contiguous tensors")
    return t.data_ptr() or None


def forward_args(*, q_idx, q_scale, w, k_idx, k_scale, q, kv, D_V, sm_scale, k, host=False,
                 kv_scale=None, kv_dtype=None):
    """The argument block of dsa_forward; host=True takes host tensors (the
    `host` block of dsa_forward_host, where k_idx / k_scale / kv / kv_scale
    may be None).  The MLA cache is bf16, or float8_e4m3fn codes with their
    per-token kv_scale (kv_dtype is taken from kv, or given when kv is None)."""
    n_q, H_I, D_I = q_idx.shape
    _, H, D_K = q.shape
    f = _hptr if host else _ptr
    if kv_dtype is None:
        kv_dtype = DSA_E4M3 if kv is not None and kv.dtype == torch.float8_e4m3fn else DSA_BF16
    a = dsa_forward_args_t(_DTYPE_CODE[q_idx.dtype], H_I, D_I, f(q_idx), f(q_scale), f(w),
                           f(k_idx), f(k_scale), H, D_K, int(D_V), float(sm_scale), f(q),
                           f(kv), int(k), int(kv_dtype), f(kv_scale))
    a._keep = (q_idx, q_scale, w, k_idx, k_scale, q, kv, kv_scale)
    return a


def dsa_forward_workspace_size(layout: Layout, args: dsa_forward_args_t) -> int:
    return lib().dsa_forward_workspace_size(layout.ref, ctypes.byref(args))


def dsa_forward(layout: Layout, args: dsa_forward_args_t, out, lse=None, idx_out=None,
                workspace=None, stream=None):
    """The whole chain: indexer -> top-k -> sparse MLA attention."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_forward(layout.ref, ctypes.byref(args), _ptr(out), _ptr(lse), _ptr(idx_out),
                             _ptr(workspace), ws_bytes, _stream(stream)), "dsa_forward")
    return out


def dsa_forward_timed(layout: Layout, args: dsa_forward_args_t, out, lse, idx_out, workspace,
                      events, stream=None):
    """dsa_forward recording events[0] before and events[i+1] after kernel i.

    events: list of torch.cuda.Event(enable_timing=True), already created.
    Returns the list of stage kinds of the kernels launched (0 indexer,
    1 top-k, 2 attention, 3 combine).
    """
    n = len(events)
    for e in events:  # materialise the underlying cudaEvent_t
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in events])
    kinds = (ctypes.c_int32 * max(n, 1))()
    nl = ctypes.c_int32(0)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_forward_timed(layout.ref, ctypes.byref(args), _ptr(out), _ptr(lse),
                                   _ptr(idx_out), _ptr(workspace), ws_bytes, _stream(stream), arr,
                                   n, kinds, ctypes.byref(nl)), "dsa_forward_timed")
    return [kinds[i] for i in range(min(nl.value, max(n - 1, 0)))], nl.value


def dsa_forward_host_workspace_size(layout: Layout, args: dsa_forward_args_t,
                                    rows_per_slab: int = 0) -> int:
    return lib().dsa_forward_host_workspace_size(layout.ref, ctypes.byref(args),
                                                 int(rows_per_slab))


def dsa_forward_host(layout: Layout, host: dsa_forward_args_t, dev: dsa_forward_args_t, host_out,
                     host_lse, dev_out, dev_lse, workspace, rows_per_slab: int = 0, stream=None):
    """The whole chain from host inputs to host results, copies and kernels
    overlapped slab by slab; `stream` is done once host_out is written."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().dsa_forward_host(layout.ref, ctypes.byref(host), ctypes.byref(dev),
                                  _hptr(host_out), _hptr(host_lse), _ptr(dev_out), _ptr(dev_lse),
                                  int(rows_per_slab), _ptr(workspace), ws_bytes, _stream(stream)),
           "dsa_forward_host")
    return host_out


def dsa_selftest_wait_timeout(cycles: int, stream=None):
    """Enqueues a wait on a barrier nothing completes, giving up after `cycles`."""
    _check(lib().dsa_selftest_wait_timeout(int(cycles), _stream(stream)),
           "dsa_selftest_wait_timeout")


def dsa_device_status(stream=None) -> int:
    """Synchronises the stream and returns (then clears) the device status word."""
    return lib().dsa_device_status(_stream(stream))
