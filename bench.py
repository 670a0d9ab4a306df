"""Throughput of the DSA hot path (indexer -> top-k -> sparse MLA attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dsa|reference]
                    [--workload prefill64k|decode64k|prefill8k|decode128k|chunked64k|tiny]

One JSON line on rank 0.  A step is one dsa_forward over the whole workload
(every stage of the path).  The default workload is the 64K-token prefill
(e4m3 indexer); the same line carries a `decode` object for the 64K-context
decode batch (64 sequences, lengths 4K..64K, bf16 indexer), measured the same
way.

Timing: W untimed warm-up steps, then K steps, each preceded by an L2 flush
outside its CUDA-event interval: a 512 MB write, then a read of 256 MB of
it, so that the step starts with none of the previous step's lines in L2
and no dirty line either (write-backs of the flush would otherwise take
about 20 us of HBM time from the first kernel of the step); then a 0.5 ms
spin kernel, during which the host queues the step, so that the interval
times the step's kernels and not the host's launch latency (a decode step
is a quarter of a millisecond; serving replays it from a CUDA graph); barrier + synchronize
around the timed region; the max over ranks.  Multi-GPU runs are weak
scaling: every rank processes its own copy of the workload (independent
sequences), no collective on the data path.

`--impl reference` times the fp64 CPU oracle on the host cores (a bounded
sample of query rows per step): the only place besides `cpu_baseline` where
this script executes the oracle.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "DSA prefill & decode tokens/s at 64K ctx, k=2048; % of TC/HBM roofline"

WORKLOADS = {
    "tiny": 1, "prefill8k": 2, "decode64k": 3, "prefill64k": 4, "decode128k": 5, "chunked64k": 6,
}
DESCR = {
    1: "DSA prefill, 1 x 256 tokens, fp32 indexer 4x32, k=32, MLA 8 heads 80/64 bf16",
    2: "DSA prefill, 1 x 8192 tokens, bf16 indexer 64x128, k=2048, MLA 128 heads 576/512 bf16",
    3: "DSA decode, 64 sequences x 1 query, cache 4K..64K (seeded), bf16 indexer 64x128, k=2048, "
       "MLA 128 heads 576/512 bf16",
    4: "DSA prefill, 1 x 65536 tokens, e4m3 indexer 64x128 (per-token scales), k=2048, "
       "MLA 128 heads 576/512 bf16",
    5: "DSA decode, 16 sequences x 1 query, cache 131072, e4m3 indexer, k=2048, MLA 128 heads "
       "576/512 bf16",
    6: "DSA chunked prefill, 4 sequences x 65536 cached tokens, the last 4096 of each new "
       "(16384 query rows), e4m3 indexer 64x128, k=2048, MLA 128 heads 576/512 bf16",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# --------------------------------------------------------------- work model
def algorithmic_work(wl):
    """Per-row units of the method's own work (not the dense work it skips).

    indexer: 2*H_I*D_I flop per causal (t, s) pair; key bytes D_I*esize
             (+4 for an fp8 scale) per key a decode row scans;
    top-k:   4 B read per candidate + 4k B written per row;
    attention: H*(2*D_K + 2*D_V) flop and D_K*2 gathered bytes (D_K + 4 for
             an e4m3 cache with its scale) per (row, selected position).
    """
    c = wl.cfg
    n = (wl.tpos + 1).astype(np.float64)
    sel = np.minimum(n, c.k)
    esz = {"f32": 4, "bf16": 2, "e4m3": 1}[c.idx_dtype]
    return {
        "idx_flop": 2.0 * c.H_I * c.D_I * n,
        "idx_bytes": n * (c.D_I * esz + (4 if c.idx_dtype == "e4m3" else 0)),
        "topk_bytes": 4.0 * n + 4.0 * c.k,
        "attn_flop": c.H * (2.0 * c.D_K + 2.0 * c.D_V) * sel,
        # gathered bytes per selected token: a bf16 row, or e4m3 codes + a fp32 scale
        "attn_bytes": (2.0 * c.D_K if c.kv_dtype == "bf16" else c.D_K + 4.0) * sel,
    }


# decode end to end: rows per slab of dsa_forward_host (the copies of one slab
# overlap the kernels of another)
DECODE_SLAB_ROWS = 32

SPIN_CYCLES = 1_000_000  # about 0.5 ms at 1.9-2 GHz, longer than the host takes to queue a step


def slab_rows(wl):
    """Rows per slab of dsa_forward (scores slab capped at 1 GiB)."""
    rows = max(1, (1 << 30) // (wl.max_len * 4))
    return min(rows, wl.n_q)


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of this GPU's SM clock and throttle reasons."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        uuid = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
        except Exception:
            pass
        sel = ["-i", uuid] if uuid else []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- device run
def workload_config(cid, kv_dtype="bf16"):
    cfg = workloads.config(cid)
    if kv_dtype != "bf16":
        cfg.kv_dtype = kv_dtype
    return cfg


def describe(cfg):
    d = DESCR[cfg.cid]
    if cfg.kv_dtype == "e4m3":
        d = d.replace("576/512 bf16", "576/512, FP8 e4m3 MLA cache with per-token fp32 scales")
    return d


def run_device(cid, steps, warmup, rank, world, do_e2e=True, index_reuse=1, kv_dtype="bf16",
               decode_slab_rows=None):
    import sparse_attention_relu_b200 as dsa

    dev = torch.device("cuda", torch.cuda.current_device())
    wl = workloads.generate(workload_config(cid, kv_dtype), pin=do_e2e)
    c = wl.cfg
    d = wl.to(dev)
    lay = dsa.Layout.of(wl, d.kv_offsets, d.q_offsets)
    args = dsa.forward_args(q_idx=d.q_idx, q_scale=d.q_scale, w=d.w, k_idx=d.k_idx,
                            k_scale=d.k_scale, q=d.q, kv=d.kv, D_V=c.D_V, sm_scale=c.sm_scale,
                            k=c.k, kv_scale=d.kv_scale)
    nws = dsa.dsa_forward_workspace_size(lay, args)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    out = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device=dev)
    flush = torch.empty(128 << 20, dtype=torch.float32, device=dev)  # 512 MB > L2
    n_slab = math.ceil(wl.n_q / slab_rows(wl))
    n_ev = 1 + 4 * n_slab + 1
    stream = torch.cuda.current_stream()

    def step(evs):
        return dsa.dsa_forward_timed(lay, args, out, lse, None, ws, evs)

    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    for _ in range(warmup):
        step(evs)
    torch.cuda.synchronize()
    st = dsa.dsa_device_status()
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status after warm-up: {dsa.dsa_status_string(st)}")

    step_ms, stage_ms, launches = [], {}, 0
    sampler = ClockSampler(torch.cuda.current_device())
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    for i in range(steps):
        flush.fill_(float(i))
        flush[: 64 << 20].sum()  # 256 MB read: the write-backs happen here
        # a spin kernel keeps the GPU busy while the host queues the step, so
        # the timed interval holds the step's kernels and not host launch
        # latency (the e2e figure, which calls the API per step, includes it)
        torch.cuda._sleep(SPIN_CYCLES)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kinds, nl = step(evs)
        e1.record(stream)
        e1.synchronize()
        step_ms.append(e0.elapsed_time(e1))
        launches += nl
        for j, kd in enumerate(kinds):
            stage_ms.setdefault(kd, []).append(evs[j].elapsed_time(evs[j + 1]))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    ms = sum(step_ms) / steps
    st = dsa.dsa_device_status()
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status after timing: {dsa.dsa_status_string(st)}")

    e2e = None
    if do_e2e:
        e2e = run_e2e(dsa, wl, lay, c, dev, steps, d, ws, stream, decode_slab_rows)
    reuse = None
    if index_reuse > 1:
        reuse = run_index_reuse(dsa, wl, lay, args, out, lse, ws, flush, stream, steps, warmup,
                                index_reuse, world)
    return wl, ms, stage_ms, launches, clocks, e2e, reuse


def run_index_reuse(dsa, wl, lay, args, out, lse, ws, flush, stream, steps, warmup, layers,
                    world):
    """IndexCache ("Linear and Sparse Attention", GLM 5.2 / IndexCache
    passage): one indexer serves `layers` attention layers.  A step is
    dsa_forward on layer 1 (indexer, top-k, attention; the indices kept in
    idx_out), then dsa_sparse_mla_attn on each later layer's own absorbed
    queries and MLA cache with those indices.  The later layers' inputs are
    drawn on the device (seeded, the workload's shapes and distribution:
    N(0, 1/D_K) rounded to bf16); timing as for the main step."""
    c = wl.cfg
    dev = out.device
    idx = torch.empty(wl.n_q, c.k, dtype=torch.int32, device=dev)
    g = torch.Generator(device=dev)
    extra = []
    for layer in range(2, layers + 1):
        g.manual_seed(c.seed * 100 + layer)
        q = (torch.randn(wl.n_q, c.H, c.D_K, generator=g, device=dev) * c.mla_std).to(
            torch.bfloat16)
        kv32 = torch.randn(wl.n_k, c.D_K, generator=g, device=dev) * c.mla_std
        if c.kv_dtype == "e4m3":
            extra.append((q, *workloads.quantize_e4m3_per_token(kv32)))
        else:
            extra.append((q, kv32.to(torch.bfloat16), None))
        del kv32
    nws = dsa.dsa_sparse_mla_attn_workspace_size(lay, c.k, c.H, c.D_K, c.D_V)
    aws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    o2 = torch.empty_like(out)
    l2 = torch.empty_like(lse)

    def step(ev_mid):
        dsa.dsa_forward(lay, args, out, lse, idx, ws)
        ev_mid.record(stream)
        for q, kv, kv_scale in extra:
            if kv_scale is None:
                dsa.dsa_sparse_mla_attn(lay, q, kv, idx, c.k, c.D_V, c.sm_scale, o2, l2, aws)
            else:
                dsa.dsa_sparse_mla_attn_e4m3(lay, q, kv, kv_scale, idx, c.k, c.D_V, c.sm_scale,
                                             o2, l2, aws)

    for _ in range(warmup):
        step(torch.cuda.Event())
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    first, total = [], []
    for i in range(steps):
        flush.fill_(float(i))
        flush[: 64 << 20].sum()
        torch.cuda._sleep(SPIN_CYCLES)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        step(e1)
        e2.record(stream)
        e2.synchronize()
        first.append(e0.elapsed_time(e1))
        total.append(e0.elapsed_time(e2))
    if world > 1:
        torch.distributed.barrier()
    st = dsa.dsa_device_status()
    if st != dsa.DSA_OK:
        raise RuntimeError(f"device status after index reuse: {dsa.dsa_status_string(st)}")
    ms, ms1 = sum(total) / steps, sum(first) / steps
    return {"layers": layers, "ms_per_step": ms, "layer1_ms": ms1,
            "later_layer_ms": (ms - ms1) / (layers - 1)}


def run_e2e(dsa, wl, lay, c, dev, steps, d, ws, stream, decode_slab_rows=None):
    """Same metric through the public API with host buffers: every step copies
    the step's inputs from pinned host memory and reads the result back.

    Prefill: the step's inputs are the whole sequence (queries, indexer keys,
    MLA cache), all copied every step.  Decode and chunked prefill: the caches
    are state that earlier steps built and that stays in HBM (copied once,
    untimed); a step's inputs are the new queries and the cache rows of the
    new tokens (indexer key, its scale, latent + rotary row: one per sequence
    in decode, the chunk's in chunked prefill), written in place every step."""
    names = ["q_idx", "q_scale", "w", "k_idx", "k_scale", "q", "kv", "kv_scale", "kv_offsets",
             "q_offsets"]
    resident = c.mode in ("decode", "chunked")
    cache = ("k_idx", "k_scale", "kv", "kv_scale") if resident else ()
    host = {n: getattr(wl, n) for n in names if getattr(wl, n) is not None}
    dbuf = {n: torch.empty_like(t, device=dev) for n, t in host.items()}
    for n in cache + ("kv_offsets", "q_offsets") if resident else ():
        if n in host:
            dbuf[n].copy_(host.pop(n))  # resident state, outside the timed region
    if not resident:  # the layout (sequence offsets) is set up once, like the workspace
        dbuf["kv_offsets"].copy_(host.pop("kv_offsets"))
    new_rows = {}
    if cache:
        ends = wl.kv_offsets.numpy()[1:].astype("int64")
        fresh = [1] * wl.B if c.mode == "decode" else list(c.chunks)
        last = torch.from_numpy(np.concatenate(
            [np.arange(e - f, e) for e, f in zip(ends, fresh)]).astype("int64"))
        last_dev = last.to(dev)
        for n in cache:
            if n in dbuf:
                src = getattr(wl, n)
                new_rows[n] = (src[last].contiguous().pin_memory(),
                               torch.empty((len(last),) + tuple(src.shape[1:]), dtype=src.dtype,
                                           device=dev))
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + sum(
        h.numel() * h.element_size() for h, _ in new_rows.values())
    out_h = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, pin_memory=True)
    lse_h = torch.empty(wl.n_q, c.H, dtype=torch.float32, pin_memory=True)
    d2h = out_h.numel() * 2 + lse_h.numel() * 4
    lay2 = dsa.Layout.of(wl, dbuf["kv_offsets"], dbuf.get("q_offsets"))
    args = dsa.forward_args(q_idx=dbuf["q_idx"], q_scale=dbuf.get("q_scale"), w=dbuf["w"],
                            k_idx=dbuf["k_idx"], k_scale=dbuf.get("k_scale"), q=dbuf["q"],
                            kv=dbuf["kv"], D_V=c.D_V, sm_scale=c.sm_scale, k=c.k,
                            kv_scale=dbuf.get("kv_scale"))
    out = torch.empty(wl.n_q, c.H, c.D_V, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wl.n_q, c.H, dtype=torch.float32, device=dev)
    # dsa_forward_host overlaps the query uploads, the kernels and the output
    # downloads slab by slab (a resident cache is passed as NULL on the host
    # side); decode rows run in slabs of DECODE_SLAB_ROWS so that its copies
    # overlap too
    use_host = True
    slab_cap = (decode_slab_rows or DECODE_SLAB_ROWS) if c.mode == "decode" else 0
    if use_host:
        hargs = dsa.forward_args(q_idx=host["q_idx"], q_scale=host.get("q_scale"), w=host["w"],
                                 k_idx=host.get("k_idx"), k_scale=host.get("k_scale"),
                                 q=host["q"], kv=host.get("kv"), D_V=c.D_V, sm_scale=c.sm_scale,
                                 k=c.k, host=True, kv_scale=host.get("kv_scale"),
                                 kv_dtype=args.kv_dtype)
        nws = dsa.dsa_forward_host_workspace_size(lay2, args, slab_cap)
        if nws > ws.numel():
            ws = torch.empty(nws, dtype=torch.uint8, device=dev)

    def one():
        if not use_host:
            for n, t in host.items():
                dbuf[n].copy_(t, non_blocking=True)
        for n, (h, stage) in new_rows.items():  # the new tokens' cache rows, in place
            stage.copy_(h, non_blocking=True)
            if stage.dtype == torch.float8_e4m3fn:  # no fp8 index_copy: move the bytes
                dbuf[n].view(torch.uint8).index_copy_(0, last_dev, stage.view(torch.uint8))
            else:
                dbuf[n].index_copy_(0, last_dev, stage)
        if use_host:
            dsa.dsa_forward_host(lay2, hargs, args, out_h, lse_h, out, lse, ws, slab_cap)
            return
        dsa.dsa_forward(lay2, args, out, lse, None, ws)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    one()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        one()
    e1.record(stream)
    e1.synchronize()
    ms = e0.elapsed_time(e1) / steps
    inputs = ("new queries + the new tokens' cache rows per step (caches resident in HBM)"
              if cache else "every input of the step (queries, indexer keys, MLA cache)")
    if use_host:
        inputs += "; copies overlapped with the kernels slab by slab (dsa_forward_host"
        inputs += f", {slab_cap} rows per slab)" if slab_cap else ")"
    return {"ms_per_step": ms, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "inputs": inputs}


KERNEL_SOURCES = {"indexer": "indexer_tc.cu", "topk": "topk.cu", "sparse_mla_attn": "attn_tc.cu"}


def measured_traffic(kernel, cfg):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    `kernel` on workload `cfg` (its id, and its cache type when not bf16), from
    the ncu capture recorded in profiles/dram_traffic.json -- or None when
    there is none, or when the kernel's source has changed since (the record
    keeps its SHA-256)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    key = f"{kernel}/{cfg.cid}" + ("" if cfg.kv_dtype == "bf16" else f"/{cfg.kv_dtype}")
    with open(path) as f:
        rec = json.load(f).get(key)
    if not rec:
        return None
    src = os.path.join(ROOT, "sparse_attention_relu_b200", "csrc", KERNEL_SOURCES[kernel])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
            return None
    return rec["bytes_per_launch"]


STAGE_NAMES = {0: "indexer", 1: "topk", 2: "sparse_mla_attn", 3: "split_combine"}


def stage_roof(wl, kind, peaks):
    """The roofline of one stage on workload wl: its algorithmic work per
    step (all rows), the bound that applies (tensor or HBM), the unit and the
    peak.  None for a stage with no work of its own (the split merge)."""
    w = algorithmic_work(wl)
    c = wl.cfg
    if kind == 2:
        if c.mode == "decode":  # gather-bound: HBM roofline of the gathered rows
            return w["attn_bytes"].sum(), "hbm", "GB/s", peaks["hbm"]
        return w["attn_flop"].sum(), "tensor", "TFLOP/s", peaks["bf16_sustained"]
    if kind == 0:
        if c.mode == "decode":
            return w["idx_bytes"].sum(), "hbm", "GB/s", peaks["hbm"]
        return (w["idx_flop"].sum(), "tensor", "TFLOP/s",
                peaks["bf16_sustained"] * (2.0 if c.idx_dtype == "e4m3" else 1.0))
    if kind == 1:
        return w["topk_bytes"].sum(), "hbm", "GB/s", peaks["hbm"]
    return None


def _rate(work, ms, unit):
    """work per ms in the unit's scale (TFLOP/s or GB/s)."""
    return work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)


def roofline(wl, stage_ms, peaks):
    """Dominant kernel (largest share of the step) against its roofline."""
    tot = {k: sum(v) for k, v in stage_ms.items()}
    if not tot:
        return None, {}
    kind = max(tot, key=tot.get)
    per_launch_ms = statistics.mean(stage_ms[kind])
    c = wl.cfg
    slabs = math.ceil(wl.n_q / slab_rows(wl))
    # every launch of a kind processes one slab; average work per launch
    work, bound, unit, peak = stage_roof(wl, kind, peaks)
    work /= slabs
    achieved = _rate(work, per_launch_ms, unit)
    shares = {STAGE_NAMES[k]: round(v / sum(tot.values()), 4) for k, v in tot.items()}
    return {"kernel": STAGE_NAMES[kind], "bound": bound, "achieved": round(achieved, 2),
            "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": measured_traffic(STAGE_NAMES[kind], c),
            "peak_source": peaks["source"] + (" (x2 nominal fp8/bf16 ratio)" if
                                             unit == "TFLOP/s" and kind == 0 and
                                             c.idx_dtype == "e4m3" else ""),
            "launch_ms": round(per_launch_ms, 4)}, shares


def stage_rooflines(wl, stage_ms, steps, ms_per_step, peaks):
    """Every stage against its roofline, and the step's roofline fraction:
    the sum of the stages' roofline times (algorithmic work / peak) over the
    measured step time.  stage_ms holds the launches of `steps` timed steps."""
    stages, bound_ms = {}, 0.0
    for kind, launches in sorted(stage_ms.items()):
        r = stage_roof(wl, kind, peaks)
        if r is None or not launches:
            continue
        work, bound, unit, peak = r
        ms = sum(launches) / steps  # this stage's device time per step
        achieved = _rate(work, ms, unit)
        floor_ms = work / (peak * (1e12 if unit == "TFLOP/s" else 1e9)) * 1e3
        bound_ms += floor_ms
        stages[STAGE_NAMES[kind]] = {"bound": bound, "unit": unit, "achieved": round(achieved, 2),
                                     "peak": peak, "frac": round(achieved / peak, 4),
                                     "ms_per_step": round(ms, 4),
                                     "roofline_ms": round(floor_ms, 4)}
    return stages, (round(bound_ms / ms_per_step, 4) if ms_per_step > 0 else None)


# --------------------------------------------------------------- ranks
def max_over_ranks(x, world, device):
    """The largest of every rank's x (all ranks call it, in the same order)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_throughput(units_per_rank, ms_max, world):
    """Whole-job units/s: every rank processes its own replica of the workload
    (weak scaling), and the job takes as long as its slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


# --------------------------------------------------------------- oracle runs
def oracle_rows(wl, rows):
    """Runs the whole oracle path (indexer, top-k, attention) on `rows`."""
    import oracle

    c = wl.cfg
    I = oracle.indexer_scores(wl.qrow[rows], wl.kbase[rows], wl.tpos[rows], wl.raw(wl.q_idx),
                              wl.raw(wl.w), wl.raw(wl.k_idx), dtype=c.idx_dtype, ld=wl.max_len,
                              q_scale=wl.raw(wl.q_scale), k_scale=wl.raw(wl.k_scale))
    idx = oracle.topk(I, wl.tpos[rows] + 1, c.k)
    oracle.sparse_mla_attn(wl.qrow[rows], wl.kbase[rows], idx, wl.raw(wl.q), wl.raw(wl.kv),
                           D_V=c.D_V, sm_scale=c.sm_scale, kv_scale=wl.raw(wl.kv_scale))


def cpu_baseline(cid, budget_s=20.0, wl=None):
    """The oracle as it stands on this host's cores, over an evenly spaced
    sample of query rows (an unbiased estimate of the per-row mean cost),
    grown until about `budget_s` seconds of work."""
    import oracle

    oracle.build()
    wl = wl or workloads.generate(cid)
    n = 2
    done_rows, t_used = 0, 0.0
    while t_used < budget_s and done_rows < wl.n_q:
        rows = workloads.sample_rows(wl.n_q, n)
        t0 = time.perf_counter()
        oracle_rows(wl, rows)
        dt = time.perf_counter() - t0
        done_rows, t_used = len(rows), dt
        if dt > budget_s / 3:
            break
        n *= 2
    return {"value": round(done_rows / t_used, 3), "unit": "tokens/s",
            "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done_rows} evenly spaced query rows of the same workload "
                      f"(all three stages, fp64), {t_used:.1f} s"}


def run_reference(cid, steps, warmup, n_gpus, kv_dtype="bf16"):
    import oracle

    oracle.build()
    wl = workloads.generate(workload_config(cid, kv_dtype))
    # four rows per oracle thread each step: every core works, and the dynamic
    # row schedule evens out the rows' different causal lengths
    rows_per_step = min(wl.n_q, 4 * oracle.num_threads())
    offsets = np.linspace(0, wl.n_q - 1, num=max(1, (steps + warmup) * rows_per_step)).round()
    all_rows = np.unique(offsets.astype(np.int64))
    chunks = np.array_split(all_rows, steps + warmup)
    for ch in chunks[:warmup]:
        oracle_rows(wl, ch)
    t0 = time.perf_counter()
    done = 0
    for ch in chunks[warmup:]:
        oracle_rows(wl, ch)
        done += len(ch)
    dt = time.perf_counter() - t0
    value = done / dt
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
            "n_gpus": n_gpus, "steps": steps, "warmup": warmup,
            "ms_per_step": round(dt / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(wl.cfg), "sample_rows_per_step": rows_per_step},
            "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "value": round(value, 3),
                             "sample": f"{done} evenly spaced query rows over {steps} steps "
                                       f"({rows_per_step} per step, all three stages, fp64)"},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _reuse_line(r, ms_max, tokens, world):
    return {"layers": r["layers"], "value": round(job_throughput(tokens, ms_max, world), 1),
            "unit": "tokens/s (all layers of the step)", "ms_per_step": round(ms_max, 4),
            "layer1_ms": round(r["layer1_ms"], 4),
            "later_layer_ms": round(r["later_layer_ms"], 4),
            "note": "layer 1: dsa_forward (indexer, top-k, attention); layers 2..L: "
                    "dsa_sparse_mla_attn on their own q and MLA cache with layer 1's indices"}


# --------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--workload", default="prefill64k", choices=list(WORKLOADS))
    ap.add_argument("--decode-workload", default="decode64k", choices=list(WORKLOADS) + ["none"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-dtype", default="bf16", choices=["bf16", "e4m3"],
                    help="storage of the MLA cache: bf16, or FP8 e4m3 codes with per-token "
                         "scales (dsa_sparse_mla_attn_e4m3)")
    ap.add_argument("--decode-slab-rows", type=int, default=None,
                    help=f"decode end to end: rows per slab of dsa_forward_host "
                         f"(default {DECODE_SLAB_ROWS})")
    ap.add_argument("--index-reuse", type=int, default=1,
                    help="L > 1 adds an `index_reuse` object: one indexer serving L attention "
                         "layers (IndexCache), tokens/s of the L-layer step")
    a = ap.parse_args()
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cid = WORKLOADS[a.workload]

    if a.impl == "reference":
        if rank == 0:
            run_reference(cid, a.steps, a.warmup, a.gpus, a.kv_dtype)
        return

    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    peaks = load_peaks()
    wl, ms, stage_ms, launches, clocks, e2e, reuse = run_device(
        cid, a.steps, a.warmup, rank, world, not a.no_e2e, a.index_reuse, a.kv_dtype,
        a.decode_slab_rows)
    dec = None
    if a.decode_workload != "none":
        dcid = WORKLOADS[a.decode_workload]
        dwl, dms, dstage, dlaunch, _, de2e, dreuse = run_device(
            dcid, a.steps, a.warmup, rank, world, not a.no_e2e, a.index_reuse, a.kv_dtype,
            a.decode_slab_rows)
        dec = (dwl, dms, dstage, dlaunch, de2e, dreuse)

    ms = max_over_ranks(ms, world, "cuda")
    e2e_ms = max_over_ranks(e2e["ms_per_step"], world, "cuda") if e2e else None
    reuse_ms = max_over_ranks(reuse["ms_per_step"], world, "cuda") if reuse else None
    if dec:
        dreuse_ms = max_over_ranks(dec[5]["ms_per_step"], world, "cuda") if dec[5] else None
        dms = max_over_ranks(dec[1], world, "cuda")
        de2e_ms = max_over_ranks(dec[4]["ms_per_step"], world, "cuda") if dec[4] else None
    tokens = wl.n_q
    value = job_throughput(tokens, ms, world)
    roof, shares = roofline(wl, stage_ms, peaks)
    if rank == 0:
        cfg = wl.cfg
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"f32": "f32", "bf16": "bf16", "e4m3": "e4m3+bf16"}[cfg.idx_dtype]
                     + ("+e4m3 cache" if cfg.kv_dtype == "e4m3" else ""),
            "data": "synthetic",
            "config": {"workload": describe(cfg), "tokens_per_step_per_gpu": tokens,
                       "k": cfg.k, "l2": "flushed before every timed step (512 MB write, 256 MB of it read back)",
                       "queued": "step launches queued behind a 0.5 ms spin kernel outside the timed interval",
                       "parallelism": f"{world} independent replicas (weak scaling)"},
            "roofline": roof, "stage_share": shares,
            "gpu_launches": launches,
        }
        line["stage_roofline"], line["step_roofline_frac"] = stage_rooflines(
            wl, stage_ms, a.steps, ms, peaks)
        if e2e:
            line["e2e"] = {"value": round(job_throughput(tokens, e2e_ms, world), 1), "unit": "tokens/s",
                           "h2d_bytes_per_step": e2e["h2d_bytes_per_step"],
                           "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                           "inputs": e2e["inputs"]}
        if reuse:
            line["index_reuse"] = _reuse_line(reuse, reuse_ms, tokens, world)
        if clocks:
            line["clocks"] = clocks
        if dec:
            dwl = dec[0]
            droof, dshares = roofline(dwl, dec[2], peaks)
            line["decode"] = {"workload": describe(dwl.cfg),
                              "value": round(job_throughput(dwl.n_q, dms, world), 1),
                              "unit": "tokens/s", "ms_per_step": round(dms, 4),
                              "roofline": droof, "stage_share": dshares,
                              "gpu_launches": dec[3]}
            (line["decode"]["stage_roofline"],
             line["decode"]["step_roofline_frac"]) = stage_rooflines(dwl, dec[2], a.steps, dms,
                                                                     peaks)
            if dec[5]:
                line["decode"]["index_reuse"] = _reuse_line(dec[5], dreuse_ms, dwl.n_q, world)
            if dec[4]:
                line["decode"]["e2e"] = {
                    "value": round(job_throughput(dwl.n_q, de2e_ms, world), 1), "unit": "tokens/s",
                    "h2d_bytes_per_step": dec[4]["h2d_bytes_per_step"],
                    "d2h_bytes_per_step": dec[4]["d2h_bytes_per_step"],
                    "inputs": dec[4]["inputs"]}
        if world == 1 and not a.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(cid, wl=wl)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
