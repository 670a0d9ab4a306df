"""Helpers shared by the GPU parity tests: device copies of workloads, calls
through the C ABI, and the tolerance checks written out once."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_attention_relu_b200 as dsa
import workloads

# Tolerances (see the oracle readings: indexer scores within 1e-3 relative to
# the error scale A = sum_j |w_j| |<q_j, k>|; attention 2e-2 max-abs, 2e-3
# mean-abs, 1e-2 relative L2 per row, lse 1e-3 absolute).
SCORE_RTOL = 1e-3
ATTN_MAX_ABS = 2e-2
ATTN_MEAN_ABS = 2e-3
ATTN_ROW_REL_L2 = 1e-2
LSE_ABS = 1e-3


class Dev:
    """A workload copied to cuda:0 with its layout."""

    def __init__(self, wl: workloads.Workload):
        self.wl = wl
        d = wl.to("cuda")
        self.d = d
        self.layout = dsa.Layout.of(wl, d.kv_offsets, d.q_offsets)
        torch.cuda.synchronize()

    def scores(self):
        wl, d = self.wl, self.d
        s = torch.empty(wl.n_q, wl.max_len, dtype=torch.float32, device="cuda")
        dsa.dsa_indexer_scores(self.layout, d.q_idx, d.q_scale, d.w, d.k_idx, d.k_scale, s)
        return s

    def topk(self, scores, k=None):
        k = k or self.wl.cfg.k
        idx = torch.empty(self.wl.n_q, k, dtype=torch.int32, device="cuda")
        dsa.dsa_topk(self.layout, scores, k, idx)
        return idx

    def attn(self, idx, k=None):
        wl, d = self.wl, self.d
        c = wl.cfg
        k = k or idx.shape[1]
        out = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device="cuda")
        nws = dsa.dsa_sparse_mla_attn_workspace_size(self.layout, k, c.H, c.D_K, c.D_V)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
        if d.kv_scale is not None:  # FP8 cache
            dsa.dsa_sparse_mla_attn_e4m3(self.layout, d.q, d.kv, d.kv_scale, idx, k, c.D_V,
                                         c.sm_scale, out, lse, ws)
        else:
            dsa.dsa_sparse_mla_attn(self.layout, d.q, d.kv, idx, k, c.D_V, c.sm_scale, out, lse,
                                    ws)
        return out, lse

    def forward(self, with_idx=True):
        wl, d = self.wl, self.d
        c = wl.cfg
        args = dsa.forward_args(q_idx=d.q_idx, q_scale=d.q_scale, w=d.w, k_idx=d.k_idx,
                                k_scale=d.k_scale, q=d.q, kv=d.kv, D_V=c.D_V,
                                sm_scale=c.sm_scale, k=c.k, kv_scale=d.kv_scale)
        nws = dsa.dsa_forward_workspace_size(self.layout, args)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device="cuda")
        out = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device="cuda")
        idx = torch.empty(wl.n_q, c.k, dtype=torch.int32, device="cuda") if with_idx else None
        dsa.dsa_forward(self.layout, args, out, lse, idx, ws)
        return out, lse, idx

    def status(self):
        return dsa.dsa_device_status()


def ref_scores(wl, rows, with_abs=True):
    c = wl.cfg
    return oracle.indexer_scores(wl.qrow[rows], wl.kbase[rows], wl.tpos[rows], wl.raw(wl.q_idx),
                                 wl.raw(wl.w), wl.raw(wl.k_idx), dtype=c.idx_dtype,
                                 ld=wl.max_len, q_scale=wl.raw(wl.q_scale),
                                 k_scale=wl.raw(wl.k_scale), with_abs=with_abs)


def ref_attn(wl, rows, idx_rows):
    c = wl.cfg
    return oracle.sparse_mla_attn(wl.qrow[rows], wl.kbase[rows], idx_rows, wl.raw(wl.q),
                                  wl.raw(wl.kv), D_V=c.D_V, sm_scale=c.sm_scale,
                                  kv_scale=wl.raw(getattr(wl, "kv_scale", None)))


def assert_scores_close(got, ref, A, tpos):
    """Element by element: -inf exactly above the diagonal; below it within
    SCORE_RTOL of max(|ref|, A)."""
    got = np.asarray(got, np.float64)
    for i in range(got.shape[0]):
        n = int(tpos[i]) + 1
        assert np.all(np.isneginf(got[i, n:])), f"row {i}: masked entries not -inf"
        g, r, a = got[i, :n], ref[i, :n], A[i, :n]
        bound = SCORE_RTOL * np.maximum(np.abs(r), a) + 1e-30
        bad = np.abs(g - r) > bound
        assert not bad.any(), (f"row {i}: {bad.sum()} scores off, worst at s={np.argmax(np.abs(g-r)-bound)}"
                               f" got {g[bad][:4]} ref {r[bad][:4]}")


def assert_attn_close(out, lse, out_ref, lse_ref):
    out = np.asarray(out, np.float64)
    lse = np.asarray(lse, np.float64)
    err = np.abs(out - out_ref)
    assert err.max() <= ATTN_MAX_ABS, f"max abs {err.max()}"
    assert err.mean() <= ATTN_MEAN_ABS, f"mean abs {err.mean()}"
    num = np.sqrt((err ** 2).reshape(out.shape[0], -1).sum(1))
    den = np.sqrt((out_ref ** 2).reshape(out.shape[0], -1).sum(1))
    nz = den > 0
    rel = num[nz] / den[nz]
    assert rel.size == 0 or rel.max() <= ATTN_ROW_REL_L2, f"row rel L2 {rel.max()}"
    assert np.all(num[~nz] == 0)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(fin, np.isfinite(lse)), "lse finiteness differs"
    if fin.any():
        assert np.abs(lse[fin] - lse_ref[fin]).max() <= LSE_ABS


def assert_selection_ok(sel_gpu, I_ref, A, tpos, k):
    """End-to-end top-k: the GPU set may differ from the oracle's only at
    positions whose oracle score lies within 1e-3 of the k-th best score."""
    for i in range(sel_gpu.shape[0]):
        n = int(tpos[i]) + 1
        g = sel_gpu[i]
        gs = set(g[g >= 0].tolist())
        assert len(gs) == min(n, k) and (g >= 0).sum() == min(n, k), f"row {i}: size"
        assert all(0 <= s < n for s in gs), f"row {i}: out of range"
        if n <= k:
            assert gs == set(range(n))
            continue
        r = I_ref[i, :n]
        ref = oracle.topk(r[None], np.array([n]), k)[0]
        rs = set(ref.tolist())
        tau = r[ref[-1]]
        for s in gs ^ rs:
            assert abs(r[s] - tau) <= SCORE_RTOL * max(abs(tau), A[i, s]), \
                f"row {i}: position {s} (score {r[s]}, k-th {tau}) differs"
