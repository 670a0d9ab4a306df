"""The allocation-free attention entry point against the regular one.

dsa_sparse_mla_attn_noalloc serves callers that cannot allocate device
memory (strict stream capture, a framework pool that owns the device,
plug-ins handed tensors without an allocator): it keeps its decode split
partials in a fixed array owned by the library instead of a caller
workspace.  This file is collected last so that a run stopping at the first
failure has already run every other test; it passes alone in a fresh
process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import ATTN_MAX_ABS, ATTN_MEAN_ABS, LSE_ABS, Dev

pytestmark = pytest.mark.gpu


def _compare(out_a, lse_a, out_b, lse_b):
    err = (out_a.float() - out_b.float()).abs()
    assert err.max().item() <= ATTN_MAX_ABS and err.mean().item() <= ATTN_MEAN_ABS
    fin = torch.isfinite(lse_b)
    assert torch.equal(fin, torch.isfinite(lse_a))
    if fin.any():
        assert (lse_a[fin] - lse_b[fin]).abs().max().item() <= LSE_ABS


@pytest.mark.parametrize("lens,k", [([3000, 5000, 2049, 700], 2048), ([900] * 20, 512)])
def test_noalloc_matches_workspace_call_twice(lens, k):
    """Two calls in a row (the second runs on the scratch the first left
    behind) both match the workspace-based entry point."""
    cfg = workloads.custom("decode", lens, idx_dtype="bf16", k=k, seed=11)
    dev = Dev(workloads.generate(cfg))
    wl, d = dev.wl, dev.d
    idx = dev.topk(dev.scores())
    ref_out, ref_lse = dev.attn(idx)
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        dsa.dsa_sparse_mla_attn_noalloc(dev.layout, d.q, d.kv, idx, k, cfg.D_V, cfg.sm_scale, out,
                                        lse)
        torch.cuda.synchronize()
        assert dsa.dsa_device_status() == dsa.DSA_OK
        _compare(out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("nrows", [37, 64])
def test_noalloc_largest_split_and_no_split(nrows):
    """37 rows at k = 2048 split in two: 74 (row, split) blocks, one per CTA
    pair on 148 SMs, the most any plan uses.  64 rows run unsplit in one
    wave and need no scratch.  Both match the workspace entry point."""
    cfg = workloads.custom("decode", [2600 + 40 * i for i in range(nrows)], idx_dtype="bf16",
                           k=2048, seed=3)
    dev = Dev(workloads.generate(cfg))
    d = dev.d
    idx = dev.topk(dev.scores())
    ref_out, ref_lse = dev.attn(idx)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    dsa.dsa_sparse_mla_attn_noalloc(dev.layout, d.q, d.kv, idx, 2048, cfg.D_V, cfg.sm_scale, out,
                                    lse)
    torch.cuda.synchronize()
    assert dsa.dsa_device_status() == dsa.DSA_OK
    _compare(out, lse, ref_out, ref_lse)
