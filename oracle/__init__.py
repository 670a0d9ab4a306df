"""Plain fp64 CPU oracle for the DSA hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never calls it and
shares no code with it.  The arithmetic lives in ``dsa_oracle.c`` (scalar
loops, fp64 accumulation); this module only builds it with gcc, marshals numpy
arrays and converts the results.

Functions (each cites, in ``dsa_oracle.c``, the passage of the pages it
follows):
  indexer_scores   lightning indexer with per-head ReLU and weighted head sum
  topk             k best candidates, ties to the lower position, -1 padded
  sparse_mla_attn  exact softmax attention over the selected cached rows
  dense_mla_attn   the same over every causal position (k >= t+1 check)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16, E4M3 = 0, 1, 2
_DT = {"f32": F32, "bf16": BF16, "e4m3": E4M3}


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.oracle_num_threads.restype = I
        lib.oracle_set_num_threads.argtypes = [I]
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_indexer_scores.argtypes = [I64, P, P, P, I, I, I, P, P, P, P, P, I64, P, P]
        lib.oracle_topk_f32.argtypes = [I64, P, I64, P, I, P]
        lib.oracle_topk_f64.argtypes = [I64, P, I64, P, I, P]
        lib.oracle_sparse_mla_attn.argtypes = [I64, P, P, P, I, I, I, I, ctypes.c_double, P, P, P, P]
        lib.oracle_dense_mla_attn.argtypes = [I64, P, P, P, I, I, I, ctypes.c_double, P, P, P, P]
        lib.oracle_sparse_mla_attn_kv.argtypes = [I64, P, P, P, I, I, I, I, ctypes.c_double, P, P,
                                                  I, P, P, P]
        lib.oracle_dense_mla_attn_kv.argtypes = [I64, P, P, P, I, I, I, ctypes.c_double, P, P, I,
                                                 P, P, P]
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _raw(a):
    """Contiguous numpy view of raw storage (bf16/e4m3 arrive as uint16/uint8)."""
    if a is None:
        return None, None
    a = np.ascontiguousarray(a)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def bf16_to_f64(bits: int) -> float:
    return _load().oracle_bf16_to_f64(int(bits))


def e4m3_to_f64(code: int) -> float:
    return _load().oracle_e4m3_to_f64(int(code))


def indexer_scores(qrow, kbase, tpos, q_I, w, k_I, *, dtype, ld, q_scale=None, k_scale=None,
                   with_abs=False):
    """I[i, s] for s <= tpos[i] (else -inf), shape [n_rows, ld], fp64.

    q_I: [n_q, H_I, D_I] raw storage (float32 / uint16 bf16 bits / uint8 e4m3)
    k_I: [N_k, D_I] raw storage; w: [n_q, H_I] float32
    q_scale: [n_q, H_I] float32 or None; k_scale: [N_k] float32 or None
    """
    lib = _load()
    dt = _DT[dtype] if isinstance(dtype, str) else int(dtype)
    n_q, H_I, D_I = q_I.shape
    qrow, pq = _c(qrow, np.int64)
    kbase, pk = _c(kbase, np.int64)
    tpos, pt = _c(tpos, np.int64)
    q_I, pqi = _raw(q_I)
    k_I, pki = _raw(k_I)
    w, pw = _c(w, np.float32)
    qs, pqs = (None, None) if q_scale is None else _c(q_scale, np.float32)
    ks, pks = (None, None) if k_scale is None else _c(k_scale, np.float32)
    n = len(qrow)
    out = np.empty((n, ld), np.float64)
    A = np.empty((n, ld), np.float64) if with_abs else None
    lib.oracle_indexer_scores(n, pq, pk, pt, H_I, D_I, dt, pqi, pqs, pw, pki, pks, int(ld),
                              out.ctypes.data_as(ctypes.c_void_p),
                              None if A is None else A.ctypes.data_as(ctypes.c_void_p))
    return (out, A) if with_abs else out


def topk(scores, n_valid, k):
    """int32 [n_rows, k]: best first (score desc, position asc), -1 padded.

    float32 scores are ranked in float32 values, float64 ones in float64.
    """
    lib = _load()
    scores = np.ascontiguousarray(scores)
    n, ld = scores.shape
    nv, pn = _c(n_valid, np.int64)
    out = np.empty((n, k), np.int32)
    fn = lib.oracle_topk_f64 if scores.dtype == np.float64 else lib.oracle_topk_f32
    if scores.dtype not in (np.float64, np.float32):
        scores = scores.astype(np.float32)
    fn(n, scores.ctypes.data_as(ctypes.c_void_p), ld, pn, int(k),
       out.ctypes.data_as(ctypes.c_void_p))
    return out


def sparse_mla_attn(qrow, kbase, idx, q, kv, *, D_V, sm_scale, kv_scale=None):
    """(out [n, H, D_V], lse [n, H]) fp64; q: uint16 [n_q, H, D_K] (bf16 bits);
    kv: uint16 [N_k, D_K] bf16 bits, or uint8 e4m3 codes with kv_scale [N_k]."""
    lib = _load()
    _, H, D_K = q.shape
    qrow, pq = _c(qrow, np.int64)
    kbase, pk = _c(kbase, np.int64)
    idx, pi = _c(idx, np.int32)
    q, pqq = _raw(q)
    kv, pkv = _raw(kv)
    kdt, ks, pks = _cache(kv, kv_scale)
    n, k = idx.shape
    out = np.empty((n, H, D_V), np.float64)
    lse = np.empty((n, H), np.float64)
    lib.oracle_sparse_mla_attn_kv(n, pq, pk, pi, k, H, D_K, D_V, float(sm_scale), pqq, pkv, kdt,
                                  pks, out.ctypes.data_as(ctypes.c_void_p),
                                  lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def dense_mla_attn(qrow, kbase, tpos, q, kv, *, D_V, sm_scale, kv_scale=None):
    """Dense causal attention over positions 0..tpos[i]; same shapes as sparse."""
    lib = _load()
    _, H, D_K = q.shape
    qrow, pq = _c(qrow, np.int64)
    kbase, pk = _c(kbase, np.int64)
    tpos, pt = _c(tpos, np.int64)
    q, pqq = _raw(q)
    kv, pkv = _raw(kv)
    kdt, ks, pks = _cache(kv, kv_scale)
    n = len(qrow)
    out = np.empty((n, H, D_V), np.float64)
    lse = np.empty((n, H), np.float64)
    lib.oracle_dense_mla_attn_kv(n, pq, pk, pt, H, D_K, D_V, float(sm_scale), pqq, pkv, kdt, pks,
                                 out.ctypes.data_as(ctypes.c_void_p),
                                 lse.ctypes.data_as(ctypes.c_void_p))
    return out, lse


def _cache(kv, kv_scale):
    """Storage type code of the MLA cache and its scale array (e4m3 only)."""
    if kv.dtype == np.uint8:
        if kv_scale is None:
            raise ValueError("an e4m3 cache needs its per-token kv_scale")
        ks, pks = _c(kv_scale, np.float32)
        return E4M3, ks, pks
    if kv.dtype != np.uint16 or kv_scale is not None:
        raise ValueError("the cache is bf16 bits (uint16) or e4m3 codes (uint8) with kv_scale")
    return BF16, None, None
