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
from dsa_testutil import Dev, assert_attn_close, ref_attn

pytestmark = pytest.mark.gpu


def _compare(out_a, lse_a, out_b, lse_b):
    """The two entry points run the same kernels on the same indices, so their
    results are bit-identical (outputs compared as raw bf16 bits)."""
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    assert torch.equal(lse_a, lse_b)


def _against_oracle(dev, idx, out, lse):
    rows = np.arange(dev.wl.n_q)
    o_ref, l_ref = ref_attn(dev.wl, rows, idx.cpu().numpy())
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


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
    _against_oracle(dev, idx, out, lse)


def test_noalloc_generic_shape():
    """A shape outside the tensor-core kernel (the tiny prefill's 8 heads,
    80-d keys, 64-d values) takes the generic kernel, which needs no scratch;
    the no-alloc call gives the workspace call's result there too."""
    dev = Dev(workloads.generate(workloads.config(1)))
    cfg, d = dev.wl.cfg, dev.d
    idx = dev.topk(dev.scores())
    ref_out, ref_lse = dev.attn(idx)
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        dsa.dsa_sparse_mla_attn_noalloc(dev.layout, d.q, d.kv, idx, cfg.k, cfg.D_V, cfg.sm_scale,
                                        out, lse)
        torch.cuda.synchronize()
        assert dsa.dsa_device_status() == dsa.DSA_OK
        _compare(out, lse, ref_out, ref_lse)
    _against_oracle(dev, idx, out, lse)


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
