"""Per-stage parity of the CUDA path against the oracle, through the C ABI.

Small workloads that the oracle finishes in seconds but that still span
several key tiles, ragged tails and multiple sequences are compared element
by element; the tolerances are the ones written in dsa_testutil.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import (Dev, assert_attn_close, assert_scores_close, ref_attn, ref_scores)

pytestmark = pytest.mark.gpu

# 48 decode rows: lengths 1..3000 with a run of rows of at most one key tile
_MANY = [(i * 2654435761) % 2999 + 1 for i in range(32)] + [1, 7, 128, 129, 64, 2, 100, 3] * 2

SMALL = {
    "c1_tiny_f32": workloads.config(1),
    "prefill_bf16_ragged": workloads.custom("prefill", [300, 45, 129], idx_dtype="bf16", k=64),
    "prefill_e4m3": workloads.custom("prefill", [333], idx_dtype="e4m3", k=100),
    "decode_bf16": workloads.custom("decode", [1, 200, 700, 129], idx_dtype="bf16", k=128),
    "decode_e4m3": workloads.custom("decode", [2049, 5, 4100], idx_dtype="e4m3", k=2048),
    # enough key tiles that the persistent decode indexer gives each CTA a
    # range crossing several rows, runs of one-tile rows among them
    "decode_bf16_many_rows": workloads.custom("decode", _MANY, idx_dtype="bf16", k=64),
    "decode_e4m3_many_rows": workloads.custom("decode", _MANY[::-1], idx_dtype="e4m3", k=96),
    # chunked prefill against a prefix cache: the last C_b positions of each
    # sequence are new queries (a whole sequence, and one-token chunks, included)
    "chunked_bf16": workloads.custom("chunked", [700, 300, 2049, 129], idx_dtype="bf16", k=128,
                                     chunks=[100, 300, 37, 1]),
    "chunked_e4m3": workloads.custom("chunked", [3000, 130], idx_dtype="e4m3", k=256,
                                     chunks=[260, 130]),
    "prefill_f32_generic_dims": workloads.custom("prefill", [150], H_I=16, D_I=64,
                                                 idx_dtype="f32", k=20, H=20, D_K=96, D_V=32),
}


@pytest.fixture(scope="module")
def small():
    return {name: Dev(workloads.generate(cfg)) for name, cfg in SMALL.items()}


@pytest.mark.parametrize("name", list(SMALL))
def test_indexer_matches_oracle(small, name):
    dev = small[name]
    wl = dev.wl
    got = dev.scores().cpu().numpy()
    assert dev.status() == dsa.DSA_OK
    rows = np.arange(wl.n_q)
    ref, A = ref_scores(wl, rows)
    assert_scores_close(got, ref, A, wl.tpos)


@pytest.mark.parametrize("name", list(SMALL))
def test_topk_bit_exact_on_gpu_scores(small, name):
    dev = small[name]
    wl = dev.wl
    s = dev.scores()
    idx = dev.topk(s).cpu().numpy()
    ref = oracle.topk(s.cpu().numpy(), wl.tpos + 1, wl.cfg.k)
    for i in range(wl.n_q):
        g = idx[i]
        assert sorted(g[g >= 0].tolist()) == sorted(ref[i][ref[i] >= 0].tolist()), f"row {i}"
        assert (g == -1).sum() == (ref[i] == -1).sum()


@pytest.mark.parametrize("name", list(SMALL))
def test_attention_matches_oracle_on_same_indices(small, name):
    dev = small[name]
    wl = dev.wl
    idx = dev.topk(dev.scores())
    out, lse = dev.attn(idx)
    assert dev.status() == dsa.DSA_OK
    rows = np.arange(wl.n_q)
    o_ref, l_ref = ref_attn(wl, rows, idx.cpu().numpy())
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def _decode_layout(lens):
    offs = np.zeros(len(lens) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    d = torch.from_numpy(offs).cuda()
    return dsa.Layout(d, dsa.DSA_DECODE, max(lens), len(lens), int(offs[-1]))


@pytest.mark.parametrize("odd_stride", [False, True])
def test_topk_edge_rows(odd_stride):
    """Rows shorter than, equal to and one longer than k; all-equal rows;
    -0/+0 ties; NaN; rows of 131072.  With odd_stride a last row of 131075
    makes the row stride 131075 floats, so no row after the first starts on
    a 16-byte boundary."""
    k = 2048
    lens = [1, 100, k, k + 1, 5000, 5000, 5000, 60000, 131072, 131072]
    if odd_stride:
        lens.append(131075)
    L = _decode_layout(lens)
    g = torch.Generator().manual_seed(5)
    S = torch.randn(len(lens), max(lens), generator=g)
    S[3, :] = 1.0  # k + 1 equal scores: the last position is dropped
    S[4] = torch.round(S[4] * 3)  # heavy ties
    S[5, :] = 0.0
    S[5, ::2] = -0.0  # +0 and -0 everywhere: lowest positions win
    S[6, 100:200] = float("nan")
    S[9, :131072] = torch.arange(131072, dtype=torch.float32).flip(0) * 1e-3  # decreasing
    dS = S.cuda()
    idx = torch.empty(len(lens), k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(L, dS, k, idx)
    got = idx.cpu().numpy()
    ref = oracle.topk(S.numpy(), np.array(lens) - 0, k)  # decode: t = L-1, n = L
    for i in range(len(lens)):
        gi, ri = got[i], ref[i]
        assert sorted(gi[gi >= 0].tolist()) == sorted(ri[ri >= 0].tolist()), f"row {i}"
    assert sorted(got[3].tolist()) == list(range(k))
    assert sorted(got[5].tolist()) == list(range(k))
    assert sorted(got[9].tolist()) == list(range(k))
    assert (got[1] == -1).sum() == k - 100


def test_attention_edge_cases():
    """An all-empty row (out 0, lse -inf); a single selected row (out equals
    the cached latent exactly); the -1 slots are skipped wherever they sit."""
    cfg = workloads.custom("decode", [50, 60, 70], idx_dtype="bf16", k=16)
    dev = Dev(workloads.generate(cfg))
    wl = dev.wl
    idx = torch.full((3, 16), -1, dtype=torch.int32)
    idx[1, 7] = 33
    idx[2, ::3] = torch.tensor([0, 5, 69, 12, 40, 41])
    out, lse = dev.attn(idx.cuda())
    out, lse = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    latent = wl.kv[wl.kv_offsets[1].item() + 33, : cfg.D_V].float().numpy()
    assert np.array_equal(out[1], np.broadcast_to(latent, out[1].shape))
    o_ref, l_ref = ref_attn(wl, np.arange(3), idx.numpy())
    assert_attn_close(out, lse, o_ref, l_ref)


def test_unselected_rows_do_not_contribute():
    """Poisoning every unselected cache row with NaN leaves the output
    bit-identical ("DeepSeek Sparse Attention", section on the risk: a token
    left out of the selection adds nothing to the output)."""
    cfg = workloads.custom("prefill", [400], idx_dtype="bf16", k=64)
    dev = Dev(workloads.generate(cfg))
    idx = dev.topk(dev.scores())
    out1, lse1 = dev.attn(idx)
    sel = torch.zeros(dev.wl.n_k, dtype=torch.bool, device="cuda")
    flat = idx[idx >= 0].long()
    sel[flat] = True  # one sequence: local == global positions
    kv_saved = dev.d.kv.clone()
    dev.d.kv[~sel] = float("nan")
    out2, lse2 = dev.attn(idx)
    dev.d.kv.copy_(kv_saved)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)


def test_full_selection_equals_dense_attention():
    """k >= t+1 for every row: DSA reduces to dense causal attention."""
    cfg = workloads.custom("prefill", [96], idx_dtype="bf16", k=128)
    dev = Dev(workloads.generate(cfg))
    wl = dev.wl
    out, lse, idx = dev.forward()
    rows = np.arange(wl.n_q)
    o_ref, l_ref = oracle.dense_mla_attn(wl.qrow, wl.kbase, wl.tpos, wl.raw(wl.q), wl.raw(wl.kv),
                                         D_V=cfg.D_V, sm_scale=cfg.sm_scale)
    assert_attn_close(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


def test_index_order_does_not_matter():
    cfg = workloads.custom("decode", [3000, 2500], idx_dtype="bf16", k=512)
    dev = Dev(workloads.generate(cfg))
    idx = dev.topk(dev.scores())
    perm = idx[:, torch.randperm(512, device="cuda")].contiguous()
    o1, l1 = dev.attn(idx)
    o2, l2 = dev.attn(perm)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-3
    assert (l1 - l2).abs().max().item() <= 1e-4


def _scores_of(cfg):
    dev = Dev(workloads.generate(cfg))
    return dev, dev.scores()


def test_chunked_reduces_to_prefill_and_decode():
    """A chunk that is the whole sequence is a prefill; one-token chunks are a
    decode step.  Same seeded data, same scores (the prefill form runs the
    same kernel, so exactly; the decode form runs the decode kernel, so to
    rounding), and the same attention output on the same indices."""
    lens = [900, 333, 1500]
    pre_dev, pre = _scores_of(workloads.custom("prefill", lens, k=128, seed=21))
    ch_dev, ch = _scores_of(workloads.custom("chunked", lens, k=128, seed=21, chunks=lens))
    assert dsa.dsa_device_status() == dsa.DSA_OK
    assert torch.equal(torch.nan_to_num(ch, neginf=-1e30), torch.nan_to_num(pre, neginf=-1e30))
    idx = pre_dev.topk(pre)
    o_pre, l_pre = pre_dev.attn(idx)
    o_ch, l_ch = ch_dev.attn(idx)
    assert torch.equal(o_pre, o_ch) and torch.equal(l_pre, l_ch)

    dec_dev, dec = _scores_of(workloads.custom("decode", lens, k=128, seed=22))
    one_dev, one = _scores_of(workloads.custom("chunked", lens, k=128, seed=22,
                                               chunks=[1] * len(lens)))
    assert dsa.dsa_device_status() == dsa.DSA_OK
    fin = torch.isfinite(dec)
    assert torch.equal(fin, torch.isfinite(one))
    assert torch.allclose(one[fin], dec[fin], rtol=1e-5, atol=1e-6)
    idx = dec_dev.topk(dec)
    o_dec, l_dec = dec_dev.attn(idx)
    o_one, l_one = one_dev.attn(idx)
    assert torch.equal(o_dec, o_one) and torch.equal(l_dec, l_one)
