"""The decode path's fused indexer + top-k against the unit calls and the oracle.

With DSA_FUSED_DECODE_SELECT=1 (off by default: not yet faster than the two
kernels), dsa_forward in decode mode runs the indexer with the selection fused
in: no score row is written; each score is kept as a candidate only when it reaches
the row's running threshold (the k-th best counted so far), and the CTA that
finishes a row selects its k best from the candidates ("GLM sparse
attention", threshold figure).  The scores themselves are computed by the
same epilogue arithmetic as dsa_indexer_scores, so the fused selection must
equal -- as a set, bit for bit -- the oracle's top-k on the unit call's
scores, ties going to the lower position.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_relu_b200 as dsa
import workloads
from dsa_testutil import Dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _fused(monkeypatch):
    monkeypatch.setenv("DSA_FUSED_DECODE_SELECT", "1")


def _fused_vs_unit(dev):
    wl = dev.wl
    _, _, idx = dev.forward()
    scores = dev.scores()
    assert dev.status() == dsa.DSA_OK
    ref = oracle.topk(scores.cpu().numpy(), wl.tpos + 1, wl.cfg.k)
    got = idx.cpu().numpy()
    for i in range(wl.n_q):
        g, r = got[i], ref[i]
        assert sorted(g[g >= 0].tolist()) == sorted(r[r >= 0].tolist()), f"row {i}"
        assert (g == -1).sum() == (r == -1).sum(), f"row {i}"


@pytest.mark.parametrize("dtype,lens,k", [
    ("bf16", [1, 7, 128, 129, 2047, 2048, 2049, 3000, 40000, 65536], 2048),
    ("e4m3", [(i * 2654435761) % 30000 + 1 for i in range(64)], 2048),
    ("bf16", [900 + 61 * i for i in range(48)], 64),
    ("e4m3", [131072] * 3, 2048),
])
def test_fused_selection_is_the_topk_of_the_scores(dtype, lens, k):
    """Rows shorter than k, of one tile, exactly k and k+1 long, and long rows
    whose tiles several CTAs score (their thresholds shared)."""
    dev = Dev(workloads.generate(workloads.custom("decode", lens, idx_dtype=dtype, k=k,
                                                  seed=41)))
    _fused_vs_unit(dev)


def test_fused_selection_with_massive_ties():
    """Sequence 0: every key equal (one score repeated 9000 times: the k best
    are the lowest 2048 positions).  Sequence 1: keys from 16 distinct rows (a
    few hundred exact ties per value, straddling the k-th).  Sequence 2: every
    head's similarity <= 0, so every score is +-0 (ReLU clips them all): the
    lowest 2048 positions again."""
    lens = [9000, 7000, 5000]
    cfg = workloads.custom("decode", lens, idx_dtype="bf16", k=2048, seed=43)
    wl = workloads.generate(cfg)
    off = wl.kv_offsets.tolist()
    wl.k_idx[off[0]:off[1]] = wl.k_idx[off[0]]
    src = wl.k_idx[off[1]:off[1] + 16].clone()
    wl.k_idx[off[1]:off[2]] = src[torch.arange(lens[1]) % 16]
    wl.q_idx[2] = wl.q_idx[2].abs()
    wl.k_idx[off[2]:off[3]] = -wl.k_idx[off[2]:off[3]].abs()
    dev = Dev(wl)
    _fused_vs_unit(dev)
    got = dev.forward()[2].cpu().numpy()
    assert sorted(got[0].tolist()) == list(range(2048))
    assert sorted(got[2].tolist()) == list(range(2048))
