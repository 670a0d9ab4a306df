"""Sparse MLA attention over an FP8 MLA cache, against the oracle.

The cache holds e4m3 codes with one fp32 scale per token ("GLM sparse
attention", ReLU paragraph: FP8 for the indexer, applied here to the cached
latent + rotary rows).  The oracle decodes the same codes exactly in fp64;
the tolerances are those of the bf16 cache (the kernel decodes the codes
exactly and rounds only what it rounds for a bf16 cache: p * scale to bf16
where the bf16 path rounds p).
"""
import numpy as np
import pytest
import torch

import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import Dev, assert_attn_close, assert_selection_ok, ref_attn, ref_scores

pytestmark = pytest.mark.gpu

CASES = {
    "prefill_ragged": workloads.custom("prefill", [300, 45, 129], k=64, kv_dtype="e4m3"),
    "decode_split": workloads.custom("decode", [2049, 5, 4100], idx_dtype="e4m3", k=2048,
                                     kv_dtype="e4m3"),
    "decode_many": workloads.custom("decode", [900 + 37 * i for i in range(48)], k=256,
                                    kv_dtype="e4m3"),
    "chunked": workloads.custom("chunked", [700, 300, 2049, 129], k=128, chunks=[100, 300, 37, 1],
                                kv_dtype="e4m3"),
    "generic_shape": workloads.custom("prefill", [150], H_I=16, D_I=64, idx_dtype="f32", k=20,
                                      H=20, D_K=96, D_V=32, kv_dtype="e4m3"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_cache_attention_matches_oracle(name):
    dev = Dev(workloads.generate(CASES[name]))
    wl = dev.wl
    assert dev.d.kv.dtype == torch.float8_e4m3fn and dev.d.kv_scale is not None
    idx = dev.topk(dev.scores())
    out, lse = dev.attn(idx)
    assert dev.status() == dsa.DSA_OK
    rows = np.arange(wl.n_q)
    o_ref, l_ref = ref_attn(wl, rows, idx.cpu().numpy())
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("name", ["prefill_ragged", "decode_split"])
def test_fp8_cache_forward_matches_oracle(name):
    """The whole chain with an FP8 cache: dsa_forward's selection against the
    oracle's scores, its output against the oracle on that selection."""
    dev = Dev(workloads.generate(CASES[name]))
    wl = dev.wl
    out, lse, idx = dev.forward()
    assert dev.status() == dsa.DSA_OK
    rows = np.arange(wl.n_q)
    I, A = ref_scores(wl, rows)
    sel = idx.cpu().numpy()
    assert_selection_ok(sel, I, A, wl.tpos, wl.cfg.k)
    o_ref, l_ref = ref_attn(wl, rows, sel)
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("shape", ["tensor_core", "generic"])
def test_every_code_decodes_exactly(shape):
    """Each query selects one token: its output is that token's decoded latent
    (softmax weight 1).  With a scale of 1 (and 2^-3) the decoded values are
    exact in bf16, so the output must equal them bit for bit; the cache rows
    hold every non-NaN e4m3 code, subnormals and both zeros included."""
    H, D_K, D_V = (128, 576, 512) if shape == "tensor_core" else (8, 80, 64)
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    codes = codes[(codes & 0x7F) != 0x7F]  # 254 codes, no NaN
    n_k = 8
    flat = codes.repeat((n_k * D_K + len(codes) - 1) // len(codes))[: n_k * D_K]
    kv8 = flat.roll(3).reshape(n_k, D_K).contiguous()
    kv8[1] = codes[torch.arange(D_K) % len(codes)]
    scale = torch.tensor([1.0, 0.125] * (n_k // 2), dtype=torch.float32)
    offs = torch.tensor([0, n_k], dtype=torch.int32, device="cuda")
    lay = dsa.Layout(offs, dsa.DSA_PREFILL, n_k, n_k, n_k)
    q = (torch.randn(n_k, H, D_K, generator=torch.Generator().manual_seed(1)) / 24).to(
        torch.bfloat16).cuda()
    k = 4
    idx = torch.full((n_k, k), -1, dtype=torch.int32)
    for t in range(n_k):
        idx[t, t % k] = t  # one causal position per row: itself
    kv_d = kv8.view(torch.float8_e4m3fn).cuda()
    out = torch.empty(n_k, H, D_V, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_k, H, dtype=torch.float32, device="cuda")
    nws = dsa.dsa_sparse_mla_attn_workspace_size(lay, k, H, D_K, D_V)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
    dsa.dsa_sparse_mla_attn_e4m3(lay, q, kv_d, scale.cuda(), idx.cuda(), k, D_V, 0.05, out, lse,
                                 ws)
    assert dsa.dsa_device_status() == dsa.DSA_OK
    dec = kv8.view(torch.float8_e4m3fn).float() * scale[:, None]
    exp = dec[:, :D_V].to(torch.bfloat16)
    assert torch.equal(exp.float(), dec[:, :D_V])  # exact in bf16
    got = out.cpu()
    for t in range(n_k):  # compared as values: +0 and -0 alike
        assert torch.equal(got[t].float(), exp[t].float().expand(H, D_V)), f"row {t}"
