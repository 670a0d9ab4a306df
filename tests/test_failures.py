"""Failures the device alone can see, made on the host side and read back
through the status word, with the context still usable afterwards.

Nothing here faults, traps or hangs the GPU: the timeout comes from a wait
given a short limit on a barrier that nothing completes (the self-test entry
point, which uses the kernels' own bounded wait), and the bad data cases are
rows or indices that the kernels check and skip.
"""
import numpy as np
import pytest
import torch

import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import Dev, assert_attn_close, ref_attn

pytestmark = pytest.mark.gpu


def _small():
    return Dev(workloads.generate(workloads.custom("decode", [700, 300, 129], idx_dtype="bf16",
                                                   k=128, seed=5)))


def test_bounded_wait_runs_out_and_reports_timeout():
    assert dsa.dsa_device_status() in (dsa.DSA_OK, dsa.DSA_ERR_TIMEOUT, dsa.DSA_ERR_DEVICE_DATA)
    dsa.dsa_selftest_wait_timeout(200_000)  # about 0.1 ms
    assert dsa.dsa_device_status() == dsa.DSA_ERR_TIMEOUT
    assert dsa.dsa_device_status() == dsa.DSA_OK  # reading clears the word
    # the context is still usable: a full call afterwards is clean and correct
    dev = _small()
    idx = dev.topk(dev.scores())
    out, lse = dev.attn(idx)
    assert dsa.dsa_device_status() == dsa.DSA_OK
    rows = np.arange(dev.wl.n_q)
    o_ref, l_ref = ref_attn(dev.wl, rows, idx.cpu().numpy())
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_index_outside_its_sequence_is_skipped_and_reported():
    """Row 1 (length 300) gets one index past its end: that slot is dropped
    (as -1 would be), DSA_ERR_DEVICE_DATA is raised, other rows are exact."""
    dev = _small()
    idx = dev.topk(dev.scores())
    assert dsa.dsa_device_status() == dsa.DSA_OK
    bad = idx.clone()
    bad[1, 0] = 300  # sequence 1 has positions 0..299
    out, lse = dev.attn(bad)
    assert dsa.dsa_device_status() == dsa.DSA_ERR_DEVICE_DATA
    ref_idx = bad.cpu().numpy().copy()
    ref_idx[1, 0] = -1
    rows = np.arange(dev.wl.n_q)
    o_ref, l_ref = ref_attn(dev.wl, rows, ref_idx)
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("shape", ["tensor_core", "generic"])
def test_future_position_is_skipped_and_reported(shape):
    """A prefill query may only attend to positions s <= t (the causal mask of
    the indexer, "GLM sparse attention").  An index past t but inside the
    sequence is dropped like -1 and raises DSA_ERR_DEVICE_DATA; both the
    tensor-core kernel and the generic one check it."""
    kw = {} if shape == "tensor_core" else dict(H_I=16, D_I=64, idx_dtype="f32", H=20, D_K=96,
                                                D_V=32)
    cfg = workloads.custom("prefill", [400], k=64, seed=9, **kw)
    dev = Dev(workloads.generate(cfg))
    idx = dev.topk(dev.scores())
    assert dsa.dsa_device_status() == dsa.DSA_OK
    bad = idx.clone()
    bad[10, 0] = 11  # row 10 sees 0..10
    bad[300, 5] = 399
    out, lse = dev.attn(bad)
    assert dsa.dsa_device_status() == dsa.DSA_ERR_DEVICE_DATA
    ref_idx = bad.cpu().numpy().copy()
    ref_idx[10, 0] = -1
    ref_idx[300, 5] = -1
    rows = np.arange(dev.wl.n_q)
    o_ref, l_ref = ref_attn(dev.wl, rows, ref_idx)
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_offsets_past_the_cache_are_reported_and_the_rows_skipped():
    """A layout whose last offset runs past n_k: the indexer, top-k and
    attention skip that sequence (scores -inf, indices -1, output 0) and raise
    DSA_ERR_DEVICE_DATA; the other sequences are unaffected."""
    dev = _small()
    wl = dev.wl
    good = dev.scores()
    assert dsa.dsa_device_status() == dsa.DSA_OK
    offs = dev.d.kv_offsets.clone()
    offs[-1] = wl.n_k + 64  # past the cache (checked on the device only)
    lay = dsa.Layout(offs, dsa.DSA_DECODE, wl.max_len, wl.n_q, wl.n_k)
    s = torch.empty_like(good)
    d = dev.d
    dsa.dsa_indexer_scores(lay, d.q_idx, d.q_scale, d.w, d.k_idx, d.k_scale, s)
    assert dsa.dsa_device_status() == dsa.DSA_ERR_DEVICE_DATA
    assert torch.isneginf(s[2]).all()
    assert torch.equal(s[:2, :300], good[:2, :300])
    idx = torch.empty(wl.n_q, 128, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(lay, s, 128, idx)
    assert dsa.dsa_device_status() == dsa.DSA_ERR_DEVICE_DATA
    assert (idx[2] == -1).all()
    c = wl.cfg
    out = torch.full((wl.n_q, c.H, c.D_V), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device="cuda")
    nws = dsa.dsa_sparse_mla_attn_workspace_size(lay, 128, c.H, c.D_K, c.D_V)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    dsa.dsa_sparse_mla_attn(lay, d.q, d.kv, idx, 128, c.D_V, c.sm_scale, out, lse, ws)
    assert dsa.dsa_device_status() == dsa.DSA_ERR_DEVICE_DATA
    assert torch.count_nonzero(out[2].float()).item() == 0
    assert torch.isneginf(lse[2]).all()
