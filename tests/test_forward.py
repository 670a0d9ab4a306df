"""End-to-end parity of dsa_forward at the five workload sizes.

Each workload runs in full on the GPU in the same launch configuration the
benchmark times; the oracle checks every query row of the two decode
workloads and of the tiny prefill, and for the long prefills 64 evenly
spaced rows plus the rows on both sides of every slab boundary of
dsa_forward, the rows at t = k-1 and t = k, the last row and the planted
needles: the selected set against the oracle's (differences allowed only
within 1e-3 of the k-th score), the attention output against the oracle
re-run on the GPU's own selection, and the unit calls (indexer, top-k) on
the same rows.
"""
import types

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import (Dev, assert_attn_close, assert_scores_close, assert_selection_ok,
                          ref_attn, ref_scores)

# None: every query row
SAMPLES = {1: None, 2: 64, 3: None, 4: 64, 5: None, 6: 64}

# dsa_forward runs query rows in slabs holding at most 1 GiB of fp32 scores
# at max_len per row (include/dsa.h); a slab starts at a multiple of this.
SLAB_SCORE_BYTES = 1 << 30


def slab_boundary_rows(n_q, max_len):
    """The last row of every slab and the first row of the next."""
    slab = max(1, SLAB_SCORE_BYTES // (4 * max_len))
    out = []
    for r0 in range(slab, n_q, slab):
        out += [r0 - 1, r0]
    return out


def _rows(wl, n):
    if n is None:
        return np.arange(wl.n_q)
    must = [0, wl.n_q - 1] + slab_boundary_rows(wl.n_q, wl.max_len)
    if wl.cfg.mode == "prefill":
        must += [wl.cfg.k - 1, wl.cfg.k]  # t = k-1 (every candidate kept), t = k (one dropped)
    if wl.cfg.plant == "needles":
        must += [t for t, _ in wl.planted]
    return workloads.sample_rows(wl.n_q, n, must)


@pytest.mark.parametrize("cid", [4, 6])
def test_sampled_rows_cover_slab_boundaries(cid):
    cfg = workloads.config(cid)
    n_q = sum(cfg.chunks) if cfg.chunks else sum(cfg.lens)
    wl = types.SimpleNamespace(cfg=cfg, n_q=n_q, max_len=max(cfg.lens), planted=[])
    rows = set(_rows(wl, SAMPLES[cid]).tolist())
    assert {4095, 4096, n_q - 4097, n_q - 4096, n_q - 1} <= rows
    assert len(rows) >= 64 + 2 * (n_q // 4096 - 1)
    if cfg.mode == "prefill":
        assert {2047, 2048} <= rows


@pytest.mark.gpu
@pytest.mark.parametrize("cid,kv_dtype", [(1, "bf16"), (2, "bf16"), (3, "bf16"), (4, "bf16"),
                                          (5, "bf16"), (6, "bf16"), (2, "e4m3"), (3, "e4m3"),
                                          (4, "e4m3"), (5, "e4m3")])
def test_forward_matches_oracle(cid, kv_dtype):
    """kv_dtype e4m3: the same workload with an FP8 MLA cache (per-token scales)."""
    cfg = workloads.config(cid)
    cfg.kv_dtype = kv_dtype
    wl = workloads.generate(cfg)
    dev = Dev(wl)
    out, lse, idx = dev.forward()
    assert dev.status() == dsa.DSA_OK
    rows = _rows(wl, SAMPLES[cid])
    I, A = ref_scores(wl, rows)
    sel = idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    assert_selection_ok(sel, I, A, wl.tpos[rows], wl.cfg.k)
    o_ref, l_ref = ref_attn(wl, rows, sel)
    r = torch.from_numpy(rows).cuda()
    assert_attn_close(out[r].float().cpu().numpy(), lse[r].cpu().numpy(), o_ref, l_ref)
    # planted structure survives selection
    for qr, pos in wl.planted:
        got = set(idx[qr].cpu().tolist())
        assert set(pos) <= got, f"planted positions of row {qr} not selected"
    # unit calls on the same rows: indexer element by element, top-k bit-exact
    scores = dev.scores()
    s_rows = scores[r].cpu().numpy()
    assert_scores_close(s_rows, I, A, wl.tpos[rows])
    del scores
    srows = torch.from_numpy(s_rows).cuda()
    lay = _rows_layout(wl, rows)
    got = torch.empty(len(rows), wl.cfg.k, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(lay, srows, wl.cfg.k, got)
    ref = oracle.topk(s_rows, wl.tpos[rows] + 1, wl.cfg.k)
    got = got.cpu().numpy()
    for i in range(len(rows)):
        assert sorted(got[i][got[i] >= 0].tolist()) == sorted(ref[i][ref[i] >= 0].tolist())
    # the forward's own selection equals top-k of the indexer's scores
    assert all(sorted(sel[i][sel[i] >= 0].tolist()) == sorted(got[i][got[i] >= 0].tolist())
               for i in range(len(rows)))


def _rows_layout(wl, rows):
    """A decode layout whose row i has t = tpos[rows[i]] (for top-k on copied rows)."""
    lens = (wl.tpos[rows] + 1).astype(np.int64)
    offs = np.zeros(len(rows) + 1, np.int32)
    offs[1:] = np.cumsum(lens)
    d = torch.from_numpy(offs).cuda()
    return dsa.Layout(d, dsa.DSA_DECODE, wl.max_len, len(rows), int(offs[-1]))
