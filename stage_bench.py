"""Times one stage of the hot path through its C ABI call on a synthetic case.

    python stage_bench.py --stage attn --case prefill --reps 4
    python stage_bench.py --stage indexer --case prefill --tokens 16384

Small, fixed cases meant for profiler captures of a single kernel:
  attn/prefill   one sequence of T tokens (cache L2-resident); row t selects
                 min(t+1, k) distinct random positions in 0..t
  attn/decode    64 sequences x 16384 tokens (cache from HBM), k scattered positions
  indexer|topk   e4m3 prefill of T tokens (the unit calls write full score rows)
Prints one line with the last repetition's time and throughput.

    python stage_bench.py --stage attn --case prefill --trace [--trace-row 3000]

runs attn/prefill on libdsa_trace.so (built on demand: the attention kernel
with per-tile clock64 stamps) and prints, for the two CTAs of one query row,
the steady-state cycles between the events of a tile (medians over the middle
tiles): the MMA thread's issue of QK-A, QK-B and PV, the softmax thread's
waits, producer thread 0's copies.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sparse_attention_relu_b200 as dsa  # noqa: E402


def _timed(fn):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1)


def attn(case: str, reps: int, T: int, k: int = 2048, kv_dtype: str = "bf16"):
    dev = "cuda"
    torch.manual_seed(0)
    if case == "prefill":
        offs = torch.tensor([0, T], dtype=torch.int32, device=dev)
        lay = dsa.Layout(offs, dsa.DSA_PREFILL, T, T, T)
        n_q, n_k = T, T
        # the k best of random causal scores: scattered positions, as the
        # indexer selects them
        idx = torch.empty(T, k, dtype=torch.int64, device=dev)
        pos = torch.arange(T, device=dev)
        for r0 in range(0, T, 1024):
            r1 = min(T, r0 + 1024)
            sc = torch.rand(r1 - r0, T, device=dev)
            sc.masked_fill_(pos[None, :] > pos[r0:r1, None], -1.0)
            v, i = torch.topk(sc, k, dim=1)
            idx[r0:r1] = torch.where(v >= 0, i, -1)
    else:
        B, L = 64, 16384
        offs = torch.arange(0, (B + 1) * L, L, dtype=torch.int32, device=dev)
        lay = dsa.Layout(offs, dsa.DSA_DECODE, L, B, B * L)
        n_q, n_k = B, B * L
        j = torch.arange(k, device=dev)[None, :]
        idx = (j * 7 + 131 * torch.arange(B, device=dev)[:, None]) % L
    idx = idx.to(torch.int32).contiguous()
    kv32 = torch.randn(n_k, 576, device=dev) / 24
    kv_scale = None
    if kv_dtype == "e4m3":
        import workloads

        kv, kv_scale = workloads.quantize_e4m3_per_token(kv32)
    else:
        kv = kv32.to(torch.bfloat16)
    del kv32
    q = (torch.randn(n_q, 128, 576, device=dev) / 24).to(torch.bfloat16)
    out = torch.empty(n_q, 128, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(n_q, 128, dtype=torch.float32, device=dev)
    nws = dsa.dsa_sparse_mla_attn_workspace_size(lay, k, 128, 576, 512)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    if kv_scale is None:
        run = lambda: dsa.dsa_sparse_mla_attn(lay, q, kv, idx, k, 512, 1 / 24, out, lse, ws)
    else:
        run = lambda: dsa.dsa_sparse_mla_attn_e4m3(lay, q, kv, kv_scale, idx, k, 512, 1 / 24, out,
                                                   lse, ws)
    for _ in range(reps):
        run()
    torch.cuda.synchronize()
    assert dsa.dsa_device_status() == 0
    ms = _timed(run)
    sel = (idx >= 0).sum().item()
    row_bytes = 1152 if kv_scale is None else 580
    print(f"attn/{case} ({kv_dtype} cache): rows={n_q} selected={sel} ms={ms:.3f} "
          f"TFLOP/s={sel * 278528 / ms / 1e9:.1f} gather GB/s={sel * row_bytes / ms / 1e6:.1f}")


def indexer_topk(stage: str, reps: int, T: int, k: int = 2048):
    import workloads

    cfg = workloads.custom("prefill", [T], idx_dtype="e4m3", k=k)
    wl = workloads.generate(cfg, with_mla=False)
    d = wl.to("cuda")
    lay = dsa.Layout.of(wl, d.kv_offsets, d.q_offsets)
    scores = torch.empty(T, T, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    ind = lambda: dsa.dsa_indexer_scores(lay, d.q_idx, d.q_scale, d.w, d.k_idx, d.k_scale, scores)
    top = lambda: dsa.dsa_topk(lay, scores, k, idx)
    for _ in range(reps):
        ind()
        top()
    torch.cuda.synchronize()
    assert dsa.dsa_device_status() == 0
    pairs = T * (T + 1) / 2
    if stage == "indexer":
        ms = _timed(ind)
        print(f"indexer/e4m3 T={T}: ms={ms:.3f} TFLOP/s={pairs * 16384 / ms / 1e9:.1f}")
    else:
        ms = _timed(top)
        print(f"topk T={T}: ms={ms:.3f} score read GB/s={pairs * 4 / ms / 1e6:.1f}")


# event fields of the trace build (attn_tc.cu, DSA_STAMP)
_EV = {"qka_b": 0, "qka_e": 1, "qkb_b": 2, "qkb_e": 3, "pv_b": 4, "pv_e": 5, "s_seen": 6,
       "s_free": 7, "pv_prev_done": 8, "p_pub": 9, "a_empty": 10, "a_issued": 11, "v_issued": 12}


def trace_attn(T: int, row: int, k: int = 2048):
    import ctypes

    import numpy as np

    from sparse_attention_relu_b200 import build as B

    dsa.LIB_PATH = B.build_trace()
    L = dsa.lib()
    L.dsa_attn_trace_select.argtypes = [ctypes.c_int]
    L.dsa_attn_trace_copy.argtypes = [ctypes.c_void_p]
    assert L.dsa_attn_trace_select(row) == 0
    attn("prefill", 2, T, k)
    torch.cuda.synchronize()
    tiles, nev = 64, 16
    buf = np.zeros(2 * tiles * nev + 2, np.int64)
    assert L.dsa_attn_trace_copy(buf.ctypes.data_as(ctypes.c_void_p)) == 0
    st = buf[: 2 * tiles * nev].reshape(2, tiles, nev)
    t0 = buf[2 * tiles * nev:]
    e = _EV
    rows = [
        ("tile period (QK-A issue to the next)", lambda a, n: a[n + 1, e["qka_b"]] - a[n, e["qka_b"]]),
        ("QK-A issue, 20 K steps", lambda a, n: a[n, e["qka_e"]] - a[n, e["qka_b"]]),
        ("QK-A issued -> QK-B issue starts", lambda a, n: a[n, e["qkb_b"]] - a[n, e["qka_e"]]),
        ("QK-B issue, 16 K steps", lambda a, n: a[n, e["qkb_e"]] - a[n, e["qkb_b"]]),
        ("QK-B issued -> softmax sees S", lambda a, n: a[n, e["s_seen"]] - a[n, e["qkb_e"]]),
        ("softmax: S seen -> read and released", lambda a, n: a[n, e["s_free"]] - a[n, e["s_seen"]]),
        ("S released -> next QK-A issue starts", lambda a, n: a[n + 1, e["qka_b"]] - a[n, e["s_free"]]),
        ("softmax: released -> PV(n-1) retired", lambda a, n: a[n, e["pv_prev_done"]] - a[n, e["s_free"]]),
        ("softmax: PV(n-1) retired -> P(n) published", lambda a, n: a[n, e["p_pub"]] - a[n, e["pv_prev_done"]]),
        ("P(n) published -> PV(n) issue starts", lambda a, n: a[n, e["pv_b"]] - a[n, e["p_pub"]]),
        ("PV issue, 4 K steps", lambda a, n: a[n, e["pv_e"]] - a[n, e["pv_b"]]),
        ("producers: stage free -> group A issued", lambda a, n: a[n, e["a_issued"]] - a[n, e["a_empty"]]),
    ]
    for c in range(2):
        a = st[c]
        nt = int(np.count_nonzero(a[:, e["qka_b"]]))
        if nt < 12:
            print(f"CTA {c}: {nt} tiles traced, too few")
            continue
        mid = range(4, nt - 4)
        print(f"row {row}, CTA {c} (output columns {256 * c}..{256 * c + 255}), {nt} tiles; "
              f"first score tile seen {a[0, e['s_seen']] - t0[c]} cycles after the CTA starts")
        for name, f in rows:
            v = np.array([f(a, n) for n in mid])
            print(f"  {name:44s} median {int(np.median(v)):6d}  min {int(v.min()):6d}  max {int(v.max()):6d}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", choices=["attn", "indexer", "topk"], required=True)
    ap.add_argument("--case", choices=["prefill", "decode"], default="prefill")
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--kv", choices=["bf16", "e4m3"], default="bf16", help="MLA cache storage")
    ap.add_argument("--trace", action="store_true",
                    help="attn/prefill on the trace build: per-tile event table of one row")
    ap.add_argument("--trace-row", type=int, default=3000)
    a = ap.parse_args()
    if a.trace:
        trace_attn(a.tokens or 4096, a.trace_row)
    elif a.stage == "attn":
        attn(a.case, a.reps, a.tokens or 4096, kv_dtype=a.kv)
    else:
        indexer_topk(a.stage, a.reps, a.tokens or 16384)


if __name__ == "__main__":
    main()
