"""Index reuse across layers (IndexCache).

"Linear and Sparse Attention" (yuxiangdai.com), GLM 5.2 / IndexCache passage:
one lightning indexer serves four attention layers; layers 2-4 reuse the
top-k indices of layer 1 and run only the sparse attention.  Through the C
ABI that is dsa_forward on layer 1 with idx_out, then dsa_sparse_mla_attn on
each later layer's own (q, kv) with those indices.  Every layer is checked
against the oracle's attention on the same indices.
"""
import numpy as np
import pytest
import torch

import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import Dev, assert_attn_close, assert_selection_ok, ref_attn, ref_scores

pytestmark = pytest.mark.gpu

LAYERS = 4


@pytest.mark.parametrize("mode,lens,chunks,k", [
    ("prefill", [1500, 700], None, 256),
    ("decode", [3000, 4100, 129, 2049], None, 2048),
    ("chunked", [2000, 900], [300, 900], 128),
])
def test_one_indexer_serves_four_layers(mode, lens, chunks, k):
    cfg1 = workloads.custom(mode, lens, idx_dtype="bf16", k=k, seed=31, chunks=chunks)
    dev1 = Dev(workloads.generate(cfg1))
    wl1 = dev1.wl
    out1, lse1, idx = dev1.forward()
    assert dsa.dsa_device_status() == dsa.DSA_OK
    rows = np.arange(wl1.n_q)
    sel = idx.cpu().numpy()
    I, A = ref_scores(wl1, rows)
    assert_selection_ok(sel, I, A, wl1.tpos, k)
    o_ref, l_ref = ref_attn(wl1, rows, sel)
    assert_attn_close(out1.float().cpu().numpy(), lse1.cpu().numpy(), o_ref, l_ref)
    # the stage call on layer 1's own inputs and indices gives dsa_forward's result
    o, l = dev1.attn(idx)
    assert torch.equal(o.view(torch.int16), out1.view(torch.int16)) and torch.equal(l, lse1)

    for layer in range(2, LAYERS + 1):
        # the same sequences (same layout); this layer's own queries and cache
        cfg = workloads.custom(mode, lens, idx_dtype="bf16", k=k, seed=31 + 100 * layer,
                               chunks=chunks)
        wl = workloads.generate(cfg)
        assert np.array_equal(wl.tpos, wl1.tpos)
        q, kv = wl.q.cuda(), wl.kv.cuda()
        assert not torch.equal(kv, dev1.d.kv)
        c = cfg
        out = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device="cuda")
        nws = dsa.dsa_sparse_mla_attn_workspace_size(dev1.layout, k, c.H, c.D_K, c.D_V)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
        dsa.dsa_sparse_mla_attn(dev1.layout, q, kv, idx, k, c.D_V, c.sm_scale, out, lse, ws)
        assert dsa.dsa_device_status() == dsa.DSA_OK
        o_ref, l_ref = ref_attn(wl, rows, sel)
        assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)
