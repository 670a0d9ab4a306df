"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: a closed form, a
library routine (numpy matmul / stable argsort, torch scaled-dot-product
attention and logsumexp in fp64, torch's storage-format conversions), an
identity the method fixes, or a count the pages print.  The set is chosen so
that a plausible slip in the oracle -- a missing ReLU, the head weight inside
the ReLU, a wrong key base, a scale ignored or applied to the wrong token, a
transposed operand, a wrong tie rule, a value vector taken from the wrong
columns -- fails at least one test.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.double().numpy()


def _rows_single(T):
    return np.arange(T), np.zeros(T, np.int64), np.arange(T)


# ---------------------------------------------------------------- formats
def test_e4m3_decode_matches_torch_all_codes(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    mine = np.array([oracle_mod.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine)) and nan.sum() == 2  # 0x7F, 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])
    # closed forms from the format definition
    assert oracle_mod.e4m3_to_f64(0x7E) == 448.0
    assert oracle_mod.e4m3_to_f64(0x38) == 1.0
    assert oracle_mod.e4m3_to_f64(0x08) == 2.0 ** -6
    assert oracle_mod.e4m3_to_f64(0x01) == 2.0 ** -9
    assert oracle_mod.e4m3_to_f64(0x80) == 0.0 and math.copysign(1, oracle_mod.e4m3_to_f64(0x80)) < 0


def test_bf16_decode_matches_torch(oracle_mod):
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 16, 4096).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    mine = np.array([oracle_mod.bf16_to_f64(int(b)) for b in bits])
    assert np.array_equal(ref, mine)


def test_generator_e4m3_is_nearest_even_and_saturating(oracle_mod):
    """The generator's codes are the nearest e4m3 value to x/scale (ties to even)."""
    table = np.array([oracle_mod.e4m3_to_f64(c) for c in range(256)])
    finite = ~np.isnan(table)
    g = torch.Generator().manual_seed(3)
    x = torch.randn(64, 96, generator=g) * torch.logspace(-4, 3, 64)[:, None]
    codes, scale = workloads.quantize_e4m3_per_token(x)
    y = (x / scale[:, None]).double().numpy().ravel()
    got = table[codes.view(torch.uint8).numpy().ravel()]
    vals = table[finite]
    for yi, gi in zip(y, got):
        d = np.abs(vals - yi)
        best = vals[d == d.min()]
        assert gi in best
    # per-token scale is amax / 448: every row reaches +-448 exactly
    assert np.allclose(np.abs(got.reshape(64, 96)).max(1), 448.0)


# ---------------------------------------------------------------- indexer
def test_indexer_single_head_unit_weight_is_causal_gemm(oracle_mod):
    """H_I = 1, w = 1, positive inputs: I = q k^T on the causal triangle."""
    rng = np.random.default_rng(1)
    T, D = 40, 16
    q = rng.random((T, 1, D)).astype(np.float32)
    k = rng.random((T, D)).astype(np.float32)
    w = np.ones((T, 1), np.float32)
    I = oracle_mod.indexer_scores(*_rows_single(T), q, w, k, dtype="f32", ld=T)
    ref = q[:, 0, :].astype(np.float64) @ k.astype(np.float64).T
    tri = np.tril(np.ones((T, T), bool))
    assert np.allclose(I[tri], ref[tri], rtol=1e-13, atol=0)
    assert np.all(np.isneginf(I[~tri]))


def test_indexer_one_hot_weight_is_clipped_head(oracle_mod):
    rng = np.random.default_rng(2)
    T, H, D = 33, 4, 8
    q = rng.standard_normal((T, H, D)).astype(np.float32)
    k = rng.standard_normal((T, D)).astype(np.float32)
    for j in range(H):
        w = np.zeros((T, H), np.float32)
        w[:, j] = 1.0
        I = oracle_mod.indexer_scores(*_rows_single(T), q, w, k, dtype="f32", ld=T)
        ref = np.maximum(q[:, j, :].astype(np.float64) @ k.astype(np.float64).T, 0.0)
        tri = np.tril(np.ones((T, T), bool))
        assert np.allclose(I[tri], ref[tri], rtol=1e-13, atol=1e-300)
        assert (ref[tri] == 0).any() and (ref[tri] > 0).any()


def test_indexer_relu_odd_part_is_weighted_query_gemm(oracle_mod):
    """ReLU(x) - ReLU(-x) = x, so I(q) - I(-q) = (sum_j w_j q_j) . k and
    ReLU(x) + ReLU(-x) = |x| gives I(q) + I(-q) = A when w >= 0."""
    rng = np.random.default_rng(4)
    T, H, D = 48, 6, 12
    q = rng.standard_normal((T, H, D)).astype(np.float32)
    k = rng.standard_normal((T, D)).astype(np.float32)
    w = rng.standard_normal((T, H)).astype(np.float32)
    rows = _rows_single(T)
    Ip = oracle_mod.indexer_scores(*rows, q, w, k, dtype="f32", ld=T)
    In = oracle_mod.indexer_scores(*rows, -q, w, k, dtype="f32", ld=T)
    v = np.einsum("th,thd->td", w.astype(np.float64), q.astype(np.float64))
    ref = v @ k.astype(np.float64).T
    tri = np.tril(np.ones((T, T), bool))
    assert np.allclose(Ip[tri] - In[tri], ref[tri], rtol=1e-12, atol=1e-12)
    wa = np.abs(w)
    Ip, A = oracle_mod.indexer_scores(*rows, q, wa, k, dtype="f32", ld=T, with_abs=True)
    In = oracle_mod.indexer_scores(*rows, -q, wa, k, dtype="f32", ld=T)
    assert np.allclose((Ip + In)[tri], A[tri], rtol=1e-12, atol=1e-12)


def test_indexer_weight_linearity_and_dead_head(oracle_mod):
    """w sits outside the ReLU: I is linear in w (any sign).  A head whose
    similarities are all negative contributes nothing, whatever its weight."""
    rng = np.random.default_rng(5)
    T, H, D = 30, 5, 10
    q = rng.standard_normal((T, H, D)).astype(np.float32)
    k = np.abs(rng.standard_normal((T, D))).astype(np.float32) + 0.1
    q[:, 0, :] = -np.abs(q[:, 0, :]) - 0.1  # head 0: <q_0, k> < 0 everywhere
    w1 = rng.standard_normal((T, H)).astype(np.float32)
    w2 = rng.standard_normal((T, H)).astype(np.float32)
    rows = _rows_single(T)
    f = lambda w: oracle_mod.indexer_scores(*rows, q, w, k, dtype="f32", ld=T)
    tri = np.tril(np.ones((T, T), bool))
    assert np.allclose((f(w1) + f(w2))[tri], f(w1 + w2)[tri], rtol=1e-5, atol=1e-5)
    assert np.allclose((-2.0 * f(w1))[tri], f(-2.0 * w1)[tri], rtol=1e-12, atol=1e-12)
    wa, wb = w1.copy(), w1.copy()
    wa[:, 0], wb[:, 0] = 7.0, -7.0
    assert np.array_equal(f(wa)[tri], f(wb)[tri])
    assert np.all(f(np.abs(w1))[tri] >= 0)


def test_indexer_ragged_sequences_use_their_own_keys(oracle_mod):
    """Two sequences: zeroing the second sequence's keys zeroes exactly its rows."""
    rng = np.random.default_rng(6)
    lens = [11, 7]
    H, D = 3, 8
    n = sum(lens)
    q = rng.standard_normal((n, H, D)).astype(np.float32)
    k = rng.standard_normal((n, D)).astype(np.float32)
    k[lens[0]:] = 0.0
    w = np.abs(rng.standard_normal((n, H))).astype(np.float32) + 0.5
    seq = np.repeat([0, 1], lens)
    tpos = np.concatenate([np.arange(L) for L in lens])
    kbase = np.array([0, lens[0]])[seq]
    I = oracle_mod.indexer_scores(np.arange(n), kbase, tpos, q, w, k, dtype="f32", ld=max(lens))
    for r in range(n):
        row = I[r, : tpos[r] + 1]
        if seq[r] == 1:
            assert np.all(row == 0.0)
        else:
            assert np.all(np.isfinite(row))
        assert np.all(np.isneginf(I[r, tpos[r] + 1:]))
    assert (I[: lens[0]][np.isfinite(I[: lens[0]])] > 0).any()


def test_indexer_fp8_scales_fold(oracle_mod):
    """Dequantised value = code * scale of its own token: scaling one key's
    scale by c > 0 scales its column by c; scaling head j's query scale by
    c > 0 equals scaling w_j by c."""
    rng = np.random.default_rng(7)
    T, H, D = 20, 4, 16
    x = torch.from_numpy(rng.standard_normal((T, H, D)).astype(np.float32))
    y = torch.from_numpy(rng.standard_normal((T, D)).astype(np.float32))
    qc, qs = workloads.quantize_e4m3_per_token(x)
    kc, ks = workloads.quantize_e4m3_per_token(y)
    qs = qs[:, None].expand(T, H).contiguous().numpy()
    ks = ks.numpy()
    q8 = qc.view(torch.uint8).numpy()
    k8 = kc.view(torch.uint8).numpy()
    w = rng.standard_normal((T, H)).astype(np.float32)
    rows = _rows_single(T)
    f = lambda w_, qs_, ks_: oracle_mod.indexer_scores(*rows, q8, w_, k8, dtype="e4m3", ld=T,
                                                       q_scale=qs_, k_scale=ks_)
    base = f(w, qs, ks)
    tri = np.tril(np.ones((T, T), bool))
    ks2 = ks.copy()
    ks2[5] *= 4.0
    got = f(w, qs, ks2)
    exp = base.copy()
    exp[:, 5] *= 4.0
    assert np.allclose(got[tri], exp[tri], rtol=1e-12, atol=1e-12)
    qs2, w2 = qs.copy(), w.copy()
    qs2[:, 2] *= 2.0
    w2[:, 2] *= 2.0
    assert np.allclose(f(w, qs2, ks)[tri], f(w2, qs, ks)[tri], rtol=1e-12, atol=1e-12)
    # and the fp8 path equals the fp32 path on the exactly dequantised values
    table = np.array([oracle_mod.e4m3_to_f64(c) for c in range(256)])
    qf = (table[q8] * qs[:, :, None]).astype(np.float64)
    kf = (table[k8] * ks[:, None]).astype(np.float64)
    ref = np.zeros((T, T))
    for j in range(H):
        ref += w[:, j:j + 1] * np.maximum(qf[:, j, :] @ kf.T, 0)
    assert np.allclose(base[tri], ref[tri], rtol=1e-10, atol=1e-10)


# ---------------------------------------------------------------- top-k
def test_topk_matches_stable_argsort(oracle_mod):
    rng = np.random.default_rng(8)
    n, ld, k = 50, 300, 37
    s = np.round(rng.standard_normal((n, ld)) * 4).astype(np.float32)  # many ties
    nv = rng.integers(1, ld + 1, n)
    got = oracle_mod.topk(s, nv, k)
    for i in range(n):
        order = np.argsort(-s[i, : nv[i]], kind="stable")[:k]
        exp = np.full(k, -1, np.int32)
        exp[: len(order)] = order
        assert np.array_equal(got[i], exp)


def test_topk_f64_matches_stable_argsort(oracle_mod):
    """The fp64 ranking (used on the oracle's own scores by every end-to-end
    selection check) against numpy's stable argsort: ties to the lower
    position ("Sparse Attention Architecture Evolution in LLMs", Top-K
    Selection), rows shorter than the stride, values that differ below
    float32 resolution, +0/-0 and NaN (ranked as -inf)."""
    rng = np.random.default_rng(18)
    n, ld, k = 40, 257, 31
    s = np.round(rng.standard_normal((n, ld)) * 3).astype(np.float64)  # many ties
    # differences float32 cannot see: the fp64 path must keep them apart
    s[::3, ::5] += 1e-12 * rng.integers(1, 4, s[::3, ::5].shape)
    s[1, :] = 0.0
    s[1, 1::2] = -0.0  # +0 and -0 tie: position order
    s[2, :] = -2.0
    s[2, [3, 7, 100]] = np.nan  # NaN ranks as -inf: after every finite score
    s[3, :] = -np.inf
    s[3, [10, 20]] = np.nan  # NaN ties with -inf: position order
    nv = rng.integers(1, ld + 1, n)
    nv[1:4] = ld
    nv[4] = 1
    got = oracle_mod.topk(s, nv, k)
    assert got.dtype == np.int32 and got.shape == (n, k)
    for i in range(n):
        key = np.where(np.isnan(s[i, : nv[i]]), -np.inf, s[i, : nv[i]])
        order = np.argsort(-key, kind="stable")[:k]
        exp = np.full(k, -1, np.int32)
        exp[: len(order)] = order
        assert np.array_equal(got[i], exp), f"row {i}"
    assert list(got[1][:4]) == [0, 1, 2, 3]
    assert not {3, 7, 100} & set(got[2].tolist())
    assert list(got[3][:5]) == [0, 1, 2, 3, 4]
    # a row read at the wrong stride would pick up the neighbour's values
    t = np.full((3, 64), -5.0)
    t[1, :16] = np.arange(16.0)
    t[0, 16:] = 100.0  # past row 0's valid prefix: never read
    got = oracle_mod.topk(t, np.array([16, 16, 16]), 4)
    assert list(got[0]) == [0, 1, 2, 3] and list(got[1]) == [15, 14, 13, 12]
    # fp64 resolution: a float32 cast would tie these and pick position order
    u = np.array([[1.0, 1.0 + 1e-12, 1.0 + 2e-12, 1.0]])
    assert list(oracle_mod.topk(u, np.array([4]), 2)[0]) == [2, 1]
    assert list(oracle_mod.topk(u.astype(np.float32), np.array([4]), 2)[0]) == [0, 1]


def test_topk_special_rows(oracle_mod):
    k = 8
    rows = np.zeros((5, 20), np.float32)
    rows[1] = np.arange(20)  # strictly increasing -> last k
    rows[2, :] = 3.0  # all equal -> first k
    rows[3, :] = -1.0
    rows[3, [2, 9]] = [0.0, -0.0]  # -0 == +0: tie -> lower position first
    rows[3, 4] = np.nan  # NaN ranks as -inf
    nv = np.array([5, 20, 20, 20, 20])
    got = oracle_mod.topk(rows, nv, k)
    assert list(got[0]) == [0, 1, 2, 3, 4, -1, -1, -1]
    assert sorted(got[1]) == list(range(12, 20))
    assert list(got[2]) == list(range(8))
    assert list(got[3][:2]) == [2, 9] and 4 not in got[3]
    rows[4, :] = -np.inf
    rows[4, 7] = np.nan
    got = oracle_mod.topk(rows[4:5], np.array([20]), 20)
    assert list(got[0]) == list(range(20))  # NaN ties with -inf, position order


def test_golden_read_counts(oracle_mod):
    """Pages' read-count widget: at 65,536 context, full attention reads
    65,536 positions and DSA main attention 2,048 (a 32x reduction)."""
    with open(os.path.join(GOLDEN, "read_counts.json")) as f:
        g = json.load(f)
    L, k = g["context"], g["k"]
    s = np.random.default_rng(9).standard_normal((1, L)).astype(np.float32)
    sel = oracle_mod.topk(s, np.array([L]), k)[0]
    assert (sel >= 0).sum() == g["dsa_reads"] and len(np.unique(sel)) == k
    assert L == g["full_reads"] and L // k == g["reduction"]


# ---------------------------------------------------------------- attention
def _sdpa(q, kmat, v, scale, mask=None):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(kmat)[None], torch.from_numpy(v)[None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None], scale=scale)[0].numpy()


def _mla_inputs(rng, n_q, H, D_K, N_k):
    qb, qf = _bf16(rng.standard_normal((n_q, H, D_K)) / math.sqrt(D_K) * 8)
    cb, cf = _bf16(rng.standard_normal((N_k, D_K)) / math.sqrt(D_K) * 8)
    return qb, qf, cb, cf


def test_sparse_attn_matches_masked_sdpa(oracle_mod):
    """One gathered latent row serves every head (MQA at read time); the value
    is the first D_V columns.  Reference: torch SDPA in fp64 with the
    selection as a boolean mask."""
    rng = np.random.default_rng(10)
    H, D_K, D_V, L, k = 4, 80, 64, 50, 12
    qb, qf, cb, cf = _mla_inputs(rng, 3, H, D_K, L)
    idx = np.full((3, k), -1, np.int32)
    for i in range(3):
        sel = rng.choice(L, size=k - i, replace=False)
        idx[i, rng.permutation(k)[: k - i]] = sel
    sc = 1 / math.sqrt(D_K)
    out, lse = oracle_mod.sparse_mla_attn(np.arange(3), np.zeros(3, np.int64), idx, qb, cb,
                                          D_V=D_V, sm_scale=sc)
    for i in range(3):
        mask = np.zeros((H, L), bool)
        mask[:, idx[i][idx[i] >= 0]] = True
        ref = _sdpa(qf[i], cf, cf[:, :D_V].copy(), sc, mask)
        assert np.allclose(out[i], ref, rtol=1e-12, atol=1e-14)
        z = torch.from_numpy(qf[i] @ cf[idx[i][idx[i] >= 0]].T * sc)
        assert np.allclose(lse[i], torch.logsumexp(z, dim=1).numpy(), rtol=1e-13, atol=1e-13)


def test_dense_attn_matches_causal_sdpa(oracle_mod):
    rng = np.random.default_rng(11)
    H, D_K, D_V, T = 3, 24, 16, 17
    qb, qf, cb, cf = _mla_inputs(rng, T, H, D_K, T)
    out, lse = oracle_mod.dense_mla_attn(np.arange(T), np.zeros(T, np.int64), np.arange(T), qb, cb,
                                         D_V=D_V, sm_scale=0.3)
    for t in range(T):
        ref = _sdpa(qf[t], cf[: t + 1], cf[: t + 1, :D_V].copy(), 0.3)
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-14)


def test_attn_single_index_zero_query_and_order(oracle_mod):
    rng = np.random.default_rng(12)
    H, D_K, D_V, L = 2, 32, 16, 40
    qb, qf, cb, cf = _mla_inputs(rng, 1, H, D_K, L)
    one = np.array([[17, -1, -1]], np.int32)
    out, lse = oracle_mod.sparse_mla_attn([0], [0], one, qb, cb, D_V=D_V, sm_scale=0.5)
    assert np.array_equal(out[0], np.broadcast_to(cf[17, :D_V], (H, D_V)))
    assert np.allclose(lse[0], 0.5 * qf[0] @ cf[17], rtol=1e-14, atol=0)
    # zero query: uniform weights, output = mean of the selected values
    sel = np.array([[3, 9, -1, 31, 4]], np.int32)
    zq = np.zeros_like(qb)
    out, lse = oracle_mod.sparse_mla_attn([0], [0], sel, zq, cb, D_V=D_V, sm_scale=0.5)
    m = cf[[3, 9, 31, 4], :D_V].mean(0)
    assert np.allclose(out[0], m, rtol=1e-14, atol=1e-15) and np.allclose(lse[0], math.log(4))
    # a permutation of the index list changes nothing beyond rounding order
    a, la = oracle_mod.sparse_mla_attn([0], [0], sel, qb, cb, D_V=D_V, sm_scale=0.5)
    b, lb = oracle_mod.sparse_mla_attn([0], [0], sel[:, ::-1].copy(), qb, cb, D_V=D_V, sm_scale=0.5)
    assert np.allclose(a, b, rtol=1e-14, atol=1e-16) and np.allclose(la, lb, rtol=1e-14)


def test_full_selection_equals_dense(oracle_mod):
    """k >= t+1 selects every candidate, so DSA reduces to dense causal attention."""
    rng = np.random.default_rng(13)
    T, H_I, D_I, H, D_K, D_V, k = 24, 4, 8, 2, 24, 16, 32
    q = rng.standard_normal((T, H_I, D_I)).astype(np.float32)
    kk = rng.standard_normal((T, D_I)).astype(np.float32)
    w = rng.standard_normal((T, H_I)).astype(np.float32)
    rows = _rows_single(T)
    I = oracle_mod.indexer_scores(*rows, q, w, kk, dtype="f32", ld=T)
    idx = oracle_mod.topk(I, np.arange(T) + 1, k)
    qb, qf, cb, cf = _mla_inputs(rng, T, H, D_K, T)
    o_s, l_s = oracle_mod.sparse_mla_attn(rows[0], rows[1], idx, qb, cb, D_V=D_V, sm_scale=0.2)
    o_d, l_d = oracle_mod.dense_mla_attn(*rows, qb, cb, D_V=D_V, sm_scale=0.2)
    assert np.allclose(o_s, o_d, rtol=1e-12, atol=1e-15) and np.allclose(l_s, l_d, rtol=1e-13)


def _e4m3_cache(rng, N_k, D_K, pow2=False):
    """e4m3 codes [N_k, D_K] (uint8, never the NaN code) and per-token scales."""
    x = torch.from_numpy(rng.standard_normal((N_k, D_K)) / math.sqrt(D_K) * 8)
    codes, scale = workloads.quantize_e4m3_per_token(x.float())
    if pow2:  # scales that are powers of two: code * scale is exact in bf16
        scale = torch.exp2(torch.round(torch.log2(scale)))
    return codes.view(torch.uint8).numpy(), scale.numpy()


def test_fp8_cache_attn_matches_sdpa_on_decoded_values(oracle_mod):
    """FP8 MLA cache (e4m3 codes, one fp32 scale per token): the oracle's
    attention equals torch SDPA in fp64 on the decoded cache, table[code] *
    scale, with the selection as a mask; the value is the first D_V decoded
    columns.  The decode table is pinned to torch's own e4m3 cast above."""
    rng = np.random.default_rng(21)
    H, D_K, D_V, L, k = 4, 80, 64, 60, 15
    qb, qf, _, _ = _mla_inputs(rng, 3, H, D_K, L)
    codes, scale = _e4m3_cache(rng, L, D_K)
    table = torch.tensor([0.0] * 256, dtype=torch.float64)
    table[:] = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double()
    cf = (table[torch.from_numpy(codes).long()] * torch.from_numpy(scale).double()[:, None]).numpy()
    idx = np.full((3, k), -1, np.int32)
    for i in range(3):
        idx[i, rng.permutation(k)[: k - 2 * i]] = rng.choice(L, size=k - 2 * i, replace=False)
    sc = 1 / math.sqrt(D_K)
    out, lse = oracle_mod.sparse_mla_attn(np.arange(3), np.zeros(3, np.int64), idx, qb, codes,
                                          D_V=D_V, sm_scale=sc, kv_scale=scale)
    for i in range(3):
        mask = np.zeros((H, L), bool)
        mask[:, idx[i][idx[i] >= 0]] = True
        ref = _sdpa(qf[i], cf, cf[:, :D_V].copy(), sc, mask)
        assert np.allclose(out[i], ref, rtol=1e-12, atol=1e-14)
        z = torch.from_numpy(qf[i] @ cf[idx[i][idx[i] >= 0]].T * sc)
        assert np.allclose(lse[i], torch.logsumexp(z, dim=1).numpy(), rtol=1e-13, atol=1e-13)
    # a single selected token: the output is its decoded latent exactly
    one = np.array([[-1, 7, -1]], np.int32)
    o1, l1 = oracle_mod.sparse_mla_attn([0], [0], one, qb, codes, D_V=D_V, sm_scale=0.5,
                                        kv_scale=scale)
    assert np.array_equal(o1[0], np.broadcast_to(cf[7, :D_V], (H, D_V)))
    # dense over an fp8 cache equals sparse with every position selected
    T = 20
    od, ld = oracle_mod.dense_mla_attn(np.arange(T), np.zeros(T, np.int64), np.arange(T), qb[:1]
                                       .repeat(T, 0), codes, D_V=D_V, sm_scale=sc,
                                       kv_scale=scale)
    full = np.where(np.arange(T)[None, :] <= np.arange(T)[:, None], np.arange(T)[None, :], -1)
    os_, ls_ = oracle_mod.sparse_mla_attn(np.arange(T), np.zeros(T, np.int64),
                                          full.astype(np.int32), qb[:1].repeat(T, 0), codes,
                                          D_V=D_V, sm_scale=sc, kv_scale=scale)
    assert np.allclose(od, os_, rtol=1e-12, atol=1e-15) and np.allclose(ld, ls_, rtol=1e-13)


def test_fp8_cache_equals_bf16_cache_when_exact(oracle_mod):
    """With power-of-two scales every decoded element code * scale is exactly
    a bf16 value, so the fp8 path must equal the bf16 path on that cache."""
    rng = np.random.default_rng(22)
    H, D_K, D_V, L, k = 3, 48, 32, 30, 9
    qb, _, _, _ = _mla_inputs(rng, 2, H, D_K, L)
    codes, scale = _e4m3_cache(rng, L, D_K, pow2=True)
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).float() * torch.from_numpy(scale)[:, None]
    cb = dec.to(torch.bfloat16)
    assert torch.equal(cb.float(), dec)  # exact
    cbits = cb.view(torch.int16).numpy().view(np.uint16)
    idx = np.stack([rng.choice(L, size=k, replace=False) for _ in range(2)]).astype(np.int32)
    a = oracle_mod.sparse_mla_attn([0, 1], [0, 0], idx, qb, codes, D_V=D_V, sm_scale=0.4,
                                   kv_scale=scale)
    b = oracle_mod.sparse_mla_attn([0, 1], [0, 0], idx, qb, cbits, D_V=D_V, sm_scale=0.4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    with pytest.raises(ValueError):
        oracle_mod.sparse_mla_attn([0], [0], idx[:1], qb, codes, D_V=D_V, sm_scale=0.4)


# ---------------------------------------------------------------- workloads
@pytest.mark.slow
def test_config2_needles_rank_first(oracle_mod):
    wl = workloads.generate(2, with_mla=False)
    rows = np.array([t for t, _ in wl.planted])
    I = oracle_mod.indexer_scores(rows, wl.kbase[rows], wl.tpos[rows], wl.raw(wl.q_idx),
                                  wl.raw(wl.w), wl.raw(wl.k_idx), dtype="bf16", ld=wl.max_len)
    for r, (t, pos) in enumerate(wl.planted):
        assert int(np.argmax(I[r, : t + 1])) == pos[0]


@pytest.mark.slow
def test_config5_sinks_and_window_selected(oracle_mod):
    wl = workloads.generate(5, with_mla=False)
    for b in (0, 11):
        r = np.array([b])
        I = oracle_mod.indexer_scores(r, wl.kbase[r], wl.tpos[r], wl.raw(wl.q_idx),
                                      wl.raw(wl.w), wl.raw(wl.k_idx), dtype="e4m3",
                                      ld=wl.max_len, q_scale=wl.raw(wl.q_scale),
                                      k_scale=wl.raw(wl.k_scale))
        sel = set(oracle_mod.topk(I, wl.tpos[r] + 1, 2048)[0].tolist())
        assert set(wl.planted[b][1]) <= sel


def test_config_shapes():
    wl = workloads.generate(1)
    c = wl.cfg
    assert wl.q_idx.shape == (256, 4, 32) and wl.q_idx.dtype == torch.float32
    assert wl.q.shape == (256, 8, 80) and wl.kv.shape == (256, 80) and wl.q.dtype == torch.bfloat16
    assert c.k == 32 and abs(c.sm_scale - 1 / math.sqrt(80)) < 1e-15
    w3 = workloads.generate(3, with_mla=False)
    assert w3.B == 64 and all(4096 <= L <= 65536 for L in w3.lens)
    assert w3.n_q == 64 and list(w3.tpos) == [L - 1 for L in w3.lens]
    a = workloads.generate(1)
    assert torch.equal(a.q, wl.q) and torch.equal(a.q_idx, wl.q_idx)  # seeded
