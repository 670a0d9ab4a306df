"""Times one stage of the hot path through its C ABI call on a synthetic case.

    python stage_bench.py --stage attn --case prefill --reps 4
    python stage_bench.py --stage indexer --case prefill --tokens 16384

Small, fixed cases meant for profiler captures of a single kernel:
  attn/prefill   one sequence of T tokens (cache L2-resident); row t selects
                 min(t+1, k) distinct random positions in 0..t
  attn/decode    64 sequences x 16384 tokens (cache from HBM), k scattered positions
  indexer|topk   e4m3 prefill of T tokens (the unit calls write full score rows)
Prints one line with the last repetition's time and throughput.
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", choices=["attn", "indexer", "topk"], required=True)
    ap.add_argument("--case", choices=["prefill", "decode"], default="prefill")
    ap.add_argument("--reps", type=int, default=4)
    ap.add_argument("--tokens", type=int, default=None)
    ap.add_argument("--kv", choices=["bf16", "e4m3"], default="bf16", help="MLA cache storage")
    a = ap.parse_args()
    if a.stage == "attn":
        attn(a.case, a.reps, a.tokens or 4096, kv_dtype=a.kv)
    else:
        indexer_topk(a.stage, a.reps, a.tokens or 16384)


if __name__ == "__main__":
    main()
