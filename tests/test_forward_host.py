"""dsa_forward_host: host inputs to host results, copies overlapped with the
kernels slab by slab.

The kernels are dsa_forward's; the selected set of a row is deterministic
but its order is not, so results are compared within the attention
tolerance: against the oracle re-run on dsa_forward's own selection, and
against dsa_forward's output.  Default slabs, smaller slabs (several, the
last one ragged), resident caches (key-side host pointers NULL) and pageable
host memory are covered.
"""
import numpy as np
import pytest
import torch

import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import Dev, assert_attn_close, ref_attn

pytestmark = pytest.mark.gpu


def _host_call(dev, rows_per_slab=0, resident=False, pin=True, with_lse=True):
    wl, d = dev.wl, dev.d
    c = wl.cfg

    def h(t):
        if t is None:
            return None
        return t.contiguous().pin_memory() if pin else t.contiguous()

    kv_dtype = dsa.DSA_E4M3 if d.kv_scale is not None else dsa.DSA_BF16
    host = dsa.forward_args(q_idx=h(wl.q_idx), q_scale=h(wl.q_scale), w=h(wl.w),
                            k_idx=None if resident else h(wl.k_idx),
                            k_scale=None if resident else h(wl.k_scale), q=h(wl.q),
                            kv=None if resident else h(wl.kv), D_V=c.D_V, sm_scale=c.sm_scale,
                            k=c.k, host=True,
                            kv_scale=None if resident else h(wl.kv_scale), kv_dtype=kv_dtype)
    # device buffers: queries start as garbage; the cache is current only when resident
    bufs = {n: torch.empty_like(getattr(d, n)) for n in ("q_idx", "w", "q")}
    bufs["q_scale"] = None if d.q_scale is None else torch.empty_like(d.q_scale)
    for n in ("k_idx", "k_scale", "kv", "kv_scale"):
        t = getattr(d, n)
        bufs[n] = None if t is None else (t.clone() if resident else torch.zeros_like(t))
    devargs = dsa.forward_args(D_V=c.D_V, sm_scale=c.sm_scale, k=c.k, **bufs)
    nws = dsa.dsa_forward_host_workspace_size(dev.layout, devargs, rows_per_slab)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    out_d = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device="cuda")
    lse_d = torch.empty(wl.n_q, c.H, dtype=torch.float32, device="cuda") if with_lse else None
    out_h = torch.full((wl.n_q, c.H, c.D_V), float("nan"), dtype=torch.bfloat16)
    lse_h = torch.full((wl.n_q, c.H), float("nan")) if with_lse else None
    if pin:
        out_h = out_h.pin_memory()
        lse_h = None if lse_h is None else lse_h.pin_memory()
    stream = torch.cuda.current_stream()
    dsa.dsa_forward_host(dev.layout, host, devargs, out_h, lse_h, out_d, lse_d, ws,
                         rows_per_slab)
    stream.synchronize()  # the call's contract: the stream done => host results written
    return out_h, lse_h


def _check(dev, out_h, lse_h, ref, idx, n_sample=None, must=()):
    """out_h / lse_h against the oracle on idx's selection and against ref."""
    wl = dev.wl
    rows = (np.arange(wl.n_q) if n_sample is None
            else workloads.sample_rows(wl.n_q, n_sample, list(must) + [0, wl.n_q - 1]))
    o_ref, l_ref = ref_attn(wl, rows, idx.cpu().numpy()[rows])
    o = out_h[rows].float().numpy()
    l = None if lse_h is None else lse_h[rows].numpy()
    assert_attn_close(o, l if l is not None else l_ref, o_ref, l_ref)
    o_dev, l_dev = ref
    assert_attn_close(o, l if l is not None else l_dev[rows].cpu().numpy(),
                      o_dev[rows].float().cpu().numpy(), l_dev[rows].cpu().numpy())


def _prefill(kv_dtype="bf16"):
    return Dev(workloads.generate(workloads.custom("prefill", [700, 300], idx_dtype="e4m3", k=64,
                                                   seed=11, kv_dtype=kv_dtype)))


def test_default_slabs_match_forward_and_oracle():
    dev = _prefill()
    out, lse, idx = dev.forward()
    out_h, lse_h = _host_call(dev)
    assert dev.status() == dsa.DSA_OK
    _check(dev, out_h, lse_h, (out, lse), idx, n_sample=32)


@pytest.mark.parametrize("pin,kv_dtype", [(True, "bf16"), (False, "bf16"), (True, "e4m3")])
def test_small_slabs_match_forward_and_oracle(pin, kv_dtype):
    """256-row slabs over 1000 queries: four slabs, the last one 232 rows
    (with a bf16 MLA cache, and with an FP8 one whose scales travel too)."""
    dev = _prefill(kv_dtype)
    out, lse, idx = dev.forward()
    out_h, lse_h = _host_call(dev, rows_per_slab=256, pin=pin)
    assert dev.status() == dsa.DSA_OK
    _check(dev, out_h, lse_h, (out, lse), idx, n_sample=24, must=[255, 256, 511, 767, 768])


@pytest.mark.parametrize("mode,lens,kv_dtype", [("decode", [700, 300, 129], "bf16"),
                                                ("chunked", [900, 400], "bf16"),
                                                ("decode", [700, 300, 129], "e4m3")])
def test_resident_cache_matches_forward_and_oracle(mode, lens, kv_dtype):
    kw = dict(chunks=[128, 64]) if mode == "chunked" else {}
    dev = Dev(workloads.generate(workloads.custom(mode, lens, idx_dtype="bf16", k=128, seed=3,
                                                  kv_dtype=kv_dtype, **kw)))
    out, lse, idx = dev.forward()
    out_h, lse_h = _host_call(dev, resident=True)
    assert dev.status() == dsa.DSA_OK
    _check(dev, out_h, lse_h, (out, lse), idx)


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_decode_in_slabs_of_rows(kv_dtype):
    """Decode through dsa_forward_host in slabs of 16 rows: every kernel of the
    path (the persistent decode indexer, the split top-k, the split attention
    and its merge) starts at a row offset, with the caches resident."""
    lens = [3000 + 977 * i for i in range(37)]
    dev = Dev(workloads.generate(workloads.custom("decode", lens, idx_dtype="e4m3", k=2048,
                                                  seed=17, kv_dtype=kv_dtype)))
    out, lse, idx = dev.forward()
    out_h, lse_h = _host_call(dev, rows_per_slab=16, resident=True)
    assert dev.status() == dsa.DSA_OK
    _check(dev, out_h, lse_h, (out, lse), idx)


def test_without_lse_and_repeated_calls():
    """No lse; two calls back to back on one stream, every row written."""
    dev = _prefill()
    out, lse, idx = dev.forward()
    a, _ = _host_call(dev, rows_per_slab=300, with_lse=False)
    b, _ = _host_call(dev, rows_per_slab=300, with_lse=False)
    assert dev.status() == dsa.DSA_OK
    assert not np.isnan(a.float().numpy()).any() and not np.isnan(b.float().numpy()).any()
    _check(dev, a, None, (out, lse), idx, n_sample=16)
    _check(dev, b, None, (out, lse), idx, n_sample=16)
