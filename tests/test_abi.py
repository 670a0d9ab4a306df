"""The C ABI loads, exports every declared entry point and rejects bad
arguments before touching a device (no GPU needed)."""
import ctypes
import os
import re

import pytest

import sparse_attention_relu_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(dsa_\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_relu_b200 import build

    build.build()
    return dsa.lib()


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert {"dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_forward"} <= declared
    for name in declared:
        assert hasattr(lib, name), name


def test_trace_entry_points_only_in_the_diagnostic_build(lib):
    """The per-tile trace of the attention kernel is a separate library
    (attn_tc.cu under -DDSA_ATTN_TRACE); the product library has none of it."""
    from sparse_attention_relu_b200 import build

    for name in ("dsa_attn_trace_select", "dsa_attn_trace_copy"):
        assert not hasattr(lib, name), name
    trace = ctypes.CDLL(build.build_trace())
    for name in ("dsa_attn_trace_select", "dsa_attn_trace_copy"):
        assert hasattr(trace, name), name
    assert os.path.realpath(build.TRACE_LIB) != os.path.realpath(dsa.LIB_PATH)


def test_fused_decode_selection_is_opt_in(lib, monkeypatch):
    """dsa_forward plans the fused decode indexer + selection (candidate lists
    instead of a score slab) only with DSA_FUSED_DECODE_SELECT=1; prefill
    never takes it."""
    P = 4096  # fake device addresses: the size query dereferences nothing
    d = dict(idx_dtype=dsa.DSA_BF16, H_I=64, D_I=128, q_idx=P, q_scale=None, w=P, k_idx=P,
             k_scale=None, H=128, D_K=576, D_V=512, sm_scale=0.1, q=P, kv=P, k=2048,
             kv_dtype=dsa.DSA_BF16, kv_scale=None)
    a = dsa.dsa_forward_args_t(*d.values())
    lib.dsa_forward_workspace_size.restype = ctypes.c_size_t

    def size(mode, env):
        if env is None:
            monkeypatch.delenv("DSA_FUSED_DECODE_SELECT", raising=False)
        else:
            monkeypatch.setenv("DSA_FUSED_DECODE_SELECT", env)
        L = _layout(mode=mode, batch=4, max_len=4096, n_q=4 if mode == dsa.DSA_DECODE else 4096,
                    n_k=4 * 4096)
        return lib.dsa_forward_workspace_size(ctypes.byref(L), ctypes.byref(a))

    off = size(dsa.DSA_DECODE, None)
    assert off > 0 and size(dsa.DSA_DECODE, "0") == off and size(dsa.DSA_DECODE, "11") == off
    assert size(dsa.DSA_DECODE, "1") != off
    assert size(dsa.DSA_PREFILL, "1") == size(dsa.DSA_PREFILL, None)


def test_status_strings(lib):
    for s in range(7):
        assert dsa.dsa_status_string(s) and dsa.dsa_status_string(s) != "unknown status"
    assert dsa.dsa_status_string(99) == "unknown status"
    assert dsa.dsa_abi_version() >= 1


def _layout(**kw):
    d = dict(mode=0, batch=1, kv_offsets=16, max_len=8, n_q=8, n_k=8)
    d.update(kw)
    return dsa.dsa_layout_t(d["mode"], d["batch"], d["kv_offsets"], d["max_len"], d["n_q"],
                            d["n_k"])


def test_argument_validation_without_device(lib):
    E = dsa.DSA_ERR_INVALID_ARGUMENT
    P = 4096  # a fake, 16-byte aligned "device pointer": never dereferenced
    assert lib.dsa_topk(None, P, 4, P, None) == E
    L = _layout()
    assert lib.dsa_topk(ctypes.byref(L), P, 0, P, None) == E  # k < 1
    assert lib.dsa_topk(ctypes.byref(L), P, 16385, P, None) == E
    assert lib.dsa_topk(ctypes.byref(L), P + 4, 4, P, None) == E  # misaligned
    assert lib.dsa_topk(ctypes.byref(L), None, 4, P, None) == E
    bad = _layout(n_q=7)  # prefill needs n_q == n_k
    assert lib.dsa_topk(ctypes.byref(bad), P, 4, P, None) == E
    bad = _layout(mode=1, batch=2, n_q=3)  # decode needs n_q == batch
    assert lib.dsa_topk(ctypes.byref(bad), P, 4, P, None) == E
    bad = _layout(kv_offsets=None)
    assert lib.dsa_topk(ctypes.byref(bad), P, 4, P, None) == E
    # indexer: dtype, head sizes, scales only with e4m3
    assert lib.dsa_indexer_scores(ctypes.byref(L), P, None, P, P, None, 7, 4, 32, P, None) == E
    assert lib.dsa_indexer_scores(ctypes.byref(L), P, P, P, P, P, dsa.DSA_BF16, 4, 32, P, None) == E
    assert lib.dsa_indexer_scores(ctypes.byref(L), P, None, P, P, None, dsa.DSA_E4M3, 4, 32, P,
                                  None) == E
    assert lib.dsa_indexer_scores(ctypes.byref(L), P, None, P, P, None, dsa.DSA_F32, 4, 3, P,
                                  None) == E  # row not a multiple of 16 bytes
    # attention: shape limits
    f = lib.dsa_sparse_mla_attn
    assert f(ctypes.byref(L), P, P, P, 4, 129, 576, 512, 0.1, P, None, None, 0, None) == E
    assert f(ctypes.byref(L), P, P, P, 4, 128, 576, 580, 0.1, P, None, None, 0, None) == E
    assert f(ctypes.byref(L), P, P, P, 4, 8, 80, 64, float("nan"), P, None, None, 0, None) == E
    # attention over an FP8 cache: scales required and aligned, D_K a multiple of 16
    g = lib.dsa_sparse_mla_attn_e4m3
    assert g(ctypes.byref(L), P, P, None, P, 4, 8, 80, 64, 0.1, P, None, None, 0, None) == E
    assert g(ctypes.byref(L), P, P, P + 4, P, 4, 8, 80, 64, 0.1, P, None, None, 0, None) == E
    assert g(ctypes.byref(L), P, P, P, P, 4, 8, 72, 64, 0.1, P, None, None, 0, None) == E
    assert g(ctypes.byref(L), P, P, P, P, 0, 8, 80, 64, 0.1, P, None, None, 0, None) == E
    # chunked prefill: query offsets required, and no more queries than cache rows
    ch = _layout(mode=dsa.DSA_CHUNKED, n_q=4)
    assert lib.dsa_topk(ctypes.byref(ch), P, 4, P, None) == E  # q_offsets missing
    ch_bad = _layout(mode=dsa.DSA_CHUNKED, n_q=9)
    ch_bad.q_offsets = P
    assert lib.dsa_topk(ctypes.byref(ch_bad), P, 4, P, None) == E  # n_q > n_k
    ch_mis = _layout(mode=dsa.DSA_CHUNKED, n_q=4)
    ch_mis.q_offsets = P + 4
    assert lib.dsa_indexer_scores(ctypes.byref(ch_mis), P, None, P, P, None, dsa.DSA_BF16, 64,
                                  128, P, None) == E  # misaligned offsets
    assert lib.dsa_topk(ctypes.byref(_layout(mode=3)), P, 4, P, None) == E  # unknown mode
    # the wait-timeout self-test takes limits in 0 .. 2e9 cycles only
    assert lib.dsa_selftest_wait_timeout(-1, None) == E
    assert lib.dsa_selftest_wait_timeout(2_000_000_001, None) == E
    # empty problems succeed without launching anything
    empty = _layout(batch=0, kv_offsets=None, max_len=0, n_q=0, n_k=0)
    assert lib.dsa_topk(ctypes.byref(empty), None, 4, None, None) == dsa.DSA_OK


def test_forward_host_validation_without_device(lib):
    """dsa_forward_host checks its host block against the device block before
    any copy or launch."""
    E = dsa.DSA_ERR_INVALID_ARGUMENT
    P, H = 4096, 8192  # fake device / host addresses: never dereferenced
    L = _layout()

    def args(ptr, **kw):
        d = dict(idx_dtype=dsa.DSA_BF16, H_I=64, D_I=128, q_idx=ptr, q_scale=None, w=ptr,
                 k_idx=ptr, k_scale=None, H=128, D_K=576, D_V=512, sm_scale=0.1, q=ptr, kv=ptr,
                 k=4, kv_dtype=dsa.DSA_BF16, kv_scale=None)
        d.update(kw)
        return dsa.dsa_forward_args_t(*d.values())

    dev = args(P)

    def call(host, rows=0, host_lse=None, dev_lse=None, dev_args=dev):
        return lib.dsa_forward_host(ctypes.byref(L), None if host is None else ctypes.byref(host),
                                    ctypes.byref(dev_args), H, host_lse, P, dev_lse, rows, P,
                                    1 << 30, None)

    assert call(None) == E
    assert call(args(H), rows=-1) == E
    assert call(args(H, H_I=32)) == E  # scalars differ from the device block
    assert call(args(H, sm_scale=0.2)) == E
    assert call(args(H, q=None)) == E  # a per-query input missing
    assert call(args(H, w=None)) == E
    assert call(args(H, k_scale=H)) == E  # scales only with e4m3
    assert call(args(H), host_lse=H) == E  # host lse without a device lse
    e4 = args(P, idx_dtype=dsa.DSA_E4M3, q_scale=P, k_scale=P)
    assert call(args(H, idx_dtype=dsa.DSA_E4M3, k_scale=H), dev_args=e4) == E  # q_scale missing
    # FP8 MLA cache: the host block's cache type must match; a bf16 cache has no scales
    f8 = args(P, kv_dtype=dsa.DSA_E4M3, kv_scale=P)
    assert call(args(H), dev_args=f8) == E
    assert call(args(H, kv_scale=H)) == E
    assert call(args(H, kv_dtype=dsa.DSA_E4M3, kv_scale=H), dev_args=args(P, kv_dtype=dsa.DSA_E4M3)) == E
    assert lib.dsa_forward_host_workspace_size(ctypes.byref(L), ctypes.byref(dev), -1) == 0


def test_binding_fails_loudly_without_device_or_library(monkeypatch, lib):
    """No CPU fallback: host tensors are refused where the ABI takes device
    pointers, and a missing library is an error, not a silent substitute."""
    import torch

    offs = torch.tensor([0, 8], dtype=torch.int32)  # a host tensor
    with pytest.raises(ValueError, match="device tensors"):
        dsa.Layout(offs, dsa.DSA_PREFILL, 8, 8, 8)
    with pytest.raises(ValueError, match="device tensors"):
        dsa.forward_args(q_idx=torch.zeros(8, 4, 32), q_scale=None, w=torch.zeros(8, 4),
                         k_idx=torch.zeros(8, 32), k_scale=None, q=torch.zeros(8, 8, 80),
                         kv=torch.zeros(8, 80), D_V=64, sm_scale=0.1, k=4)
    with pytest.raises(ValueError, match="contiguous"):  # the host block of dsa_forward_host
        dsa.forward_args(q_idx=torch.zeros(8, 32, 4).transpose(1, 2), q_scale=None,
                         w=torch.zeros(8, 4), k_idx=None, k_scale=None, q=torch.zeros(8, 8, 80),
                         kv=None, D_V=64, sm_scale=0.1, k=4, host=True)
    monkeypatch.setattr(dsa, "_lib", None)
    monkeypatch.setattr(dsa, "LIB_PATH", os.path.join(ROOT, "no_such_libdsa.so"))
    with pytest.raises(RuntimeError, match="not built"):
        dsa.lib()
