"""Seeded synthetic inputs for the DSA hot path.

This module is shared by the tests, the benchmark and the smoke check.  It
holds none of the method's arithmetic (no scores, no selection, no
attention): only the distributions, storage-format rounding (bf16, fp8 e4m3
with per-token scales) and the planted structure that the pages describe in
words:

* "GLM sparse attention" (thethings.ai), needle figure: a far-away relevant
  token that only the indexer can find -> ``needles`` plants keys aligned with
  chosen queries;
* same page, 56-token causal figure: attention mass sits on the first tokens
  (sinks) and a recent window -> ``sinks_window`` boosts those keys toward the
  decode query.

Planting adds ``alpha * u`` to a key row, ``u`` being the unit vector of the
target query's head-weighted indexer query sum_j w[t,j] q_I[t,j].  Adding
(rather than replacing) keeps every row distinct.  ``alpha`` is fixed; the
tests check with the oracle that every planted key is selected.

Generation is block-seeded: each tensor is drawn in row blocks, each block
from its own torch CPU generator seeded from (config seed, tensor name, block
index), so any size can be produced in bounded memory and the same seed gives
the same bytes on every machine.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import List, Optional

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclasses.dataclass
class Config:
    cid: int
    name: str
    mode: str  # "prefill" | "decode" | "chunked"
    lens: Optional[List[int]]  # per-sequence cache lengths (None: drawn, see len_range)
    B: int
    H_I: int
    D_I: int
    idx_dtype: str  # "f32" | "bf16" | "e4m3"
    k: int
    H: int
    D_K: int
    D_V: int
    sm_scale: float
    w_std: float
    mla_std: float
    plant: Optional[str] = None  # "needles" | "sinks_window" | None
    len_range: Optional[tuple] = None
    alpha: float = 64.0
    seed: int = 0
    chunks: Optional[List[int]] = None  # chunked: new query tokens per sequence (<= its length)
    kv_dtype: str = "bf16"  # MLA cache storage: "bf16" | "e4m3" (codes + one fp32 scale per token)

    def __post_init__(self):
        if not self.seed:
            self.seed = 1000 + self.cid


def config(cid: int) -> Config:
    """The five workloads, by number (1 = tiny prefill ... 5 = 128K decode), and 6: a
    chunked prefill against a prefix cache (beyond the five, for that mode)."""
    if cid == 1:
        return Config(1, "prefill_T256_tiny_f32", "prefill", [256], 1, 4, 32, "f32", 32, 8, 80,
                      64, 1 / math.sqrt(80), math.sqrt(1 / 4), 1 / math.sqrt(80))
    if cid == 2:
        return Config(2, "prefill_T8192_bf16_needles", "prefill", [8192], 1, 64, 128, "bf16",
                      2048, 128, 576, 512, 1 / math.sqrt(576), math.sqrt(1 / 64),
                      1 / math.sqrt(576), plant="needles")
    if cid == 3:
        return Config(3, "decode_B64_L4K-64K_bf16", "decode", None, 64, 64, 128, "bf16", 2048,
                      128, 576, 512, 1 / math.sqrt(576), math.sqrt(1 / 64), 1 / math.sqrt(576),
                      len_range=(4096, 65536))
    if cid == 4:
        return Config(4, "prefill_T65536_e4m3", "prefill", [65536], 1, 64, 128, "e4m3", 2048,
                      128, 576, 512, 1 / math.sqrt(576), math.sqrt(1 / 64), 1 / math.sqrt(576))
    if cid == 5:
        return Config(5, "decode_B16_L131072_e4m3_sinks", "decode", [131072] * 16, 16, 64, 128,
                      "e4m3", 2048, 128, 576, 512, 1 / math.sqrt(576), math.sqrt(1 / 64),
                      1 / math.sqrt(576), plant="sinks_window")
    if cid == 6:
        # chunked prefill with a prefix cache: 4 sequences of 65,536 cached tokens,
        # the last 4,096 of each new (16,384 query rows); e4m3 indexer as config 4
        return Config(6, "chunked_B4_L65536_C4096_e4m3", "chunked", [65536] * 4, 4, 64, 128,
                      "e4m3", 2048, 128, 576, 512, 1 / math.sqrt(576), math.sqrt(1 / 64),
                      1 / math.sqrt(576), chunks=[4096] * 4)
    raise ValueError(f"unknown config {cid}")


def custom(mode="prefill", lens=(300,), H_I=64, D_I=128, idx_dtype="bf16", k=64, H=128,
           D_K=576, D_V=512, sm_scale=None, w_std=None, mla_std=None, plant=None, seed=7,
           name=None, chunks=None, kv_dtype="bf16") -> Config:
    """A small workload with the structure of the big ones (tests).  For
    mode "chunked", chunks[b] new query tokens close sequence b."""
    lens = list(lens)
    return Config(0, name or f"custom_{mode}_{idx_dtype}", mode, lens, len(lens), H_I, D_I,
                  idx_dtype, k, H, D_K, D_V,
                  sm_scale if sm_scale is not None else 1 / math.sqrt(D_K),
                  w_std if w_std is not None else 1 / math.sqrt(H_I),
                  mla_std if mla_std is not None else 1 / math.sqrt(D_K), plant=plant, seed=seed,
                  chunks=list(chunks) if chunks is not None else None, kv_dtype=kv_dtype)


def _seed(*parts) -> int:
    h = hashlib.sha256("/".join(str(p) for p in parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _normal_blocks(seed, name, shape, std, out_dtype, block_rows, pin=False):
    """N(0, std^2) in fp32, rounded to ``out_dtype`` block by block."""
    out = torch.empty(shape, dtype=out_dtype, pin_memory=pin)
    rows = shape[0]
    for bi, r0 in enumerate(range(0, rows, block_rows)):
        r1 = min(rows, r0 + block_rows)
        g = torch.Generator().manual_seed(_seed(seed, name, bi))
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[r0:r1].copy_(x)
    return out


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token fp8 e4m3: scale = amax / 448 (amax == 0 -> 1), codes RNE, saturating.

    x: fp32 [rows, ...]; returns (codes float8_e4m3fn [rows, ...], scale fp32 [rows]).
    """
    flat = x.reshape(x.shape[0], -1)
    amax = flat.abs().amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (flat / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).reshape(x.shape)
    return codes, scale.to(torch.float32)


class Workload:
    """Host tensors of one workload (torch CPU, optionally pinned).

    kv_offsets int32 [B+1]; q_idx [n_q, H_I, D_I]; q_scale fp32 [n_q, H_I] or
    None; w fp32 [n_q, H_I]; k_idx [N_k, D_I]; k_scale fp32 [N_k] or None;
    q bf16 [n_q, H, D_K]; kv bf16 [N_k, D_K], or (cfg.kv_dtype "e4m3") fp8 codes
    [N_k, D_K] with kv_scale fp32 [N_k].
    Query row r belongs to sequence seq[r] at local position tpos[r]; its keys
    are rows kv_offsets[seq] ... kv_offsets[seq] + tpos[r].
    """

    def __init__(self, cfg: Config, pin: bool = False, with_mla: bool = True):
        self.cfg = cfg
        seed = cfg.seed
        if cfg.lens is None:
            g = torch.Generator().manual_seed(_seed(seed, "lens"))
            lo, hi = cfg.len_range
            lens = torch.randint(lo, hi + 1, (cfg.B,), generator=g).tolist()
        else:
            lens = list(cfg.lens)
        self.lens = lens
        self.B = len(lens)
        self.max_len = max(lens) if lens else 0
        offs = np.zeros(self.B + 1, np.int64)
        offs[1:] = np.cumsum(lens)
        self.kv_offsets = torch.from_numpy(offs.astype(np.int32))
        self.n_k = int(offs[-1])
        self.q_offsets = None
        if cfg.mode == "prefill":
            self.seq = np.repeat(np.arange(self.B), lens).astype(np.int64)
            self.tpos = np.concatenate([np.arange(L) for L in lens]).astype(np.int64) \
                if self.B else np.zeros(0, np.int64)
        elif cfg.mode == "chunked":
            chunks = list(cfg.chunks)
            assert len(chunks) == self.B and all(0 <= c <= L for c, L in zip(chunks, lens))
            self.seq = np.repeat(np.arange(self.B), chunks).astype(np.int64)
            self.tpos = np.concatenate([np.arange(L - c, L) for L, c in zip(lens, chunks)]) \
                .astype(np.int64) if self.B else np.zeros(0, np.int64)
            qo = np.zeros(self.B + 1, np.int64)
            qo[1:] = np.cumsum(chunks)
            self.q_offsets = torch.from_numpy(qo.astype(np.int32))
        else:
            self.seq = np.arange(self.B, dtype=np.int64)
            self.tpos = np.array([L - 1 for L in lens], np.int64)
        self.n_q = len(self.seq)
        self.kbase = offs[:-1][self.seq].astype(np.int64)
        self.qrow = np.arange(self.n_q, dtype=np.int64)

        H_I, D_I = cfg.H_I, cfg.D_I
        big = 1 << 16
        qI = _normal_blocks(seed, "q_I", (self.n_q, H_I, D_I), 1.0, torch.float32, big)
        kI = _normal_blocks(seed, "k_I", (self.n_k, D_I), 1.0, torch.float32, big * 4)
        self.w = _normal_blocks(seed, "w", (self.n_q, H_I), cfg.w_std, torch.float32, big)
        self.planted = self._plant(qI, kI)
        if cfg.idx_dtype == "f32":
            self.q_idx, self.k_idx = qI, kI
            self.q_scale = self.k_scale = None
        elif cfg.idx_dtype == "bf16":
            self.q_idx, self.k_idx = qI.to(torch.bfloat16), kI.to(torch.bfloat16)
            self.q_scale = self.k_scale = None
        elif cfg.idx_dtype == "e4m3":
            self.q_idx, qs = quantize_e4m3_per_token(qI)
            self.k_idx, self.k_scale = quantize_e4m3_per_token(kI)
            # one scale per query token, handed to the library per (token, head)
            self.q_scale = qs[:, None].expand(self.n_q, H_I).contiguous()
        else:
            raise ValueError(cfg.idx_dtype)
        del qI, kI
        if pin:
            for name in ("q_idx", "k_idx", "w", "q_scale", "k_scale", "kv_offsets", "q_offsets"):
                t = getattr(self, name)
                if t is not None:
                    setattr(self, name, t.pin_memory())
        if with_mla:
            rows_per_block = max(1, (1 << 24) // (cfg.H * cfg.D_K))
            self.q = _normal_blocks(seed, "q", (self.n_q, cfg.H, cfg.D_K), cfg.mla_std,
                                    torch.bfloat16, rows_per_block, pin)
            kv_rows = max(1, (1 << 24) // cfg.D_K)
            self.kv_scale = None
            if cfg.kv_dtype == "bf16":
                self.kv = _normal_blocks(seed, "kv", (self.n_k, cfg.D_K), cfg.mla_std,
                                         torch.bfloat16, kv_rows, pin)
            elif cfg.kv_dtype == "e4m3":
                # the same fp32 draws as the bf16 cache, quantised per token
                kv32 = _normal_blocks(seed, "kv", (self.n_k, cfg.D_K), cfg.mla_std,
                                      torch.float32, kv_rows)
                self.kv, self.kv_scale = quantize_e4m3_per_token(kv32)
                del kv32
                if pin:
                    self.kv, self.kv_scale = self.kv.pin_memory(), self.kv_scale.pin_memory()
            else:
                raise ValueError(cfg.kv_dtype)
        else:
            self.q = self.kv = self.kv_scale = None

    # -- planted structure -------------------------------------------------
    def _direction(self, qI, r):
        v = (self.w[r][:, None] * qI[r]).sum(0)
        return v / v.norm()

    def _plant(self, qI, kI):
        cfg = self.cfg
        planted = []  # (query row, [local positions])
        if cfg.plant == "needles":
            L = self.lens[0]
            g = torch.Generator().manual_seed(_seed(cfg.seed, "needles"))
            lo = L // 2
            for i in range(16):
                t = lo + (i * (L - 1 - lo)) // 15
                p = int(torch.randint(0, max(1, t - 1024), (1,), generator=g))
                kI[p] += cfg.alpha * self._direction(qI, t)
                planted.append((t, [p]))
        elif cfg.plant == "sinks_window":
            offs = self.kv_offsets.tolist()
            for b, L in enumerate(self.lens):
                u = self._direction(qI, b)
                pos = list(range(min(4, L))) + list(range(max(0, L - 128), L))
                pos = sorted(set(pos))
                for p in pos:
                    kI[offs[b] + p] += cfg.alpha * u
                planted.append((b, pos))
        return planted

    # -- raw views for the oracle ------------------------------------------
    @staticmethod
    def raw(t):
        """numpy view of a tensor's storage (bf16 -> uint16, e4m3 -> uint8)."""
        if t is None:
            return None
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()

    def to(self, device):
        """A shallow copy whose tensors live on ``device``."""
        other = object.__new__(Workload)
        other.__dict__.update(self.__dict__)
        for name in ("q_idx", "k_idx", "w", "q_scale", "k_scale", "kv_offsets", "q_offsets", "q",
                     "kv", "kv_scale"):
            t = getattr(self, name)
            if t is not None:
                setattr(other, name, t.to(device, non_blocking=True))
        return other


def generate(cid_or_cfg, pin=False, with_mla=True) -> Workload:
    cfg = config(cid_or_cfg) if isinstance(cid_or_cfg, int) else cid_or_cfg
    return Workload(cfg, pin=pin, with_mla=with_mla)


def sample_rows(n_q: int, n: int, must=()) -> np.ndarray:
    """Evenly spaced query rows plus the listed ones, sorted and unique."""
    base = np.linspace(0, n_q - 1, num=min(n, n_q)).round().astype(np.int64)
    extra = np.array([m for m in must if 0 <= m < n_q], np.int64)
    return np.unique(np.concatenate([base, extra]))
