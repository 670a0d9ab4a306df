"""The seeded input generator's query layouts, against their definitions.

The oracle takes each query row's sequence and position as given, so the
mapping from a layout to (sequence, position, first cache row) is pinned
here: prefill puts query r of sequence b at position r - offset[b]; decode
puts sequence b's one query at its last position; a chunk of C_b queries
occupies the last C_b positions, so chunks of the full lengths are the
prefill and chunks of one are the decode.
"""
import numpy as np
import torch

import workloads


def _gen(mode, lens, **kw):
    return workloads.generate(workloads.custom(mode, lens, seed=3, **kw), with_mla=False)


def test_chunked_rows_are_the_last_positions():
    wl = _gen("chunked", [10, 7, 3], chunks=[4, 0, 3])
    np.testing.assert_array_equal(wl.seq, [0, 0, 0, 0, 2, 2, 2])
    np.testing.assert_array_equal(wl.tpos, [6, 7, 8, 9, 0, 1, 2])
    np.testing.assert_array_equal(wl.kbase, [0, 0, 0, 0, 17, 17, 17])
    assert wl.q_offsets.tolist() == [0, 4, 4, 7]
    assert wl.kv_offsets.tolist() == [0, 10, 17, 20]
    assert (wl.n_q, wl.n_k, wl.max_len) == (7, 20, 10)


def test_prefill_and_decode_positions():
    pre = _gen("prefill", [3, 2])
    np.testing.assert_array_equal(pre.seq, [0, 0, 0, 1, 1])
    np.testing.assert_array_equal(pre.tpos, [0, 1, 2, 0, 1])
    np.testing.assert_array_equal(pre.kbase, [0, 0, 0, 3, 3])
    dec = _gen("decode", [3, 2])
    np.testing.assert_array_equal(dec.seq, [0, 1])
    np.testing.assert_array_equal(dec.tpos, [2, 1])
    np.testing.assert_array_equal(dec.kbase, [0, 3])
    assert pre.q_offsets is None and dec.q_offsets is None


def test_chunked_reduces_to_prefill_and_decode():
    lens = [37, 5, 64]
    pre, full = _gen("prefill", lens), _gen("chunked", lens, chunks=lens)
    for name in ("seq", "tpos", "kbase"):
        np.testing.assert_array_equal(getattr(full, name), getattr(pre, name))
    assert full.q_offsets.tolist() == pre.kv_offsets.tolist()
    # same seed, same row count: the same inputs, so the same problem
    assert torch.equal(full.q_idx.float(), pre.q_idx.float())
    assert torch.equal(full.k_idx.float(), pre.k_idx.float())
    assert torch.equal(full.w, pre.w)
    dec, one = _gen("decode", lens), _gen("chunked", lens, chunks=[1, 1, 1])
    for name in ("seq", "tpos", "kbase"):
        np.testing.assert_array_equal(getattr(one, name), getattr(dec, name))
    assert one.q_offsets.tolist() == [0, 1, 2, 3]
