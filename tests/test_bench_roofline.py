"""The bench's roofline arithmetic on CPU: each stage's algorithmic work over
its measured time against its peak, and the step's roofline fraction (the sum
of the stages' roofline times over the measured step time)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402

PEAKS = {"hbm": 5000.0, "bf16_sustained": 1000.0, "source": "test"}


@pytest.mark.parametrize("mode,idx_dtype", [("prefill", "bf16"), ("prefill", "e4m3"),
                                            ("decode", "bf16")])
def test_stage_rooflines_and_step_fraction(mode, idx_dtype):
    lens = [300, 170] if mode == "prefill" else [5000, 3000, 900]
    wl = workloads.generate(workloads.custom(mode, lens, idx_dtype=idx_dtype, k=128))
    assert bench.slab_rows(wl) >= wl.n_q  # one slab: a launch is a step's whole stage
    steps, ms_step = 2, 3.5
    stage_ms = {0: [1.0, 1.2], 1: [0.4, 0.4], 2: [1.5, 1.7]}
    stages, frac = bench.stage_rooflines(wl, stage_ms, steps, ms_step, PEAKS)
    w = bench.algorithmic_work(wl)
    # the work each stage must do, written out per stage
    if mode == "decode":
        want = {"indexer": (w["idx_bytes"].sum(), "GB/s", PEAKS["hbm"]),
                "sparse_mla_attn": (w["attn_bytes"].sum(), "GB/s", PEAKS["hbm"])}
    else:
        fp8 = 2.0 if idx_dtype == "e4m3" else 1.0
        want = {"indexer": (w["idx_flop"].sum(), "TFLOP/s", PEAKS["bf16_sustained"] * fp8),
                "sparse_mla_attn": (w["attn_flop"].sum(), "TFLOP/s", PEAKS["bf16_sustained"])}
    want["topk"] = (w["topk_bytes"].sum(), "GB/s", PEAKS["hbm"])
    per_step = {"indexer": 1.1, "topk": 0.4, "sparse_mla_attn": 1.6}
    total_floor = 0.0
    for name, (work, unit, peak) in want.items():
        s = stages[name]
        scale = 1e12 if unit == "TFLOP/s" else 1e9
        assert s["unit"] == unit and s["peak"] == peak
        assert s["ms_per_step"] == pytest.approx(per_step[name])
        achieved = work / (per_step[name] * 1e-3) / scale
        assert s["achieved"] == pytest.approx(achieved, rel=1e-3, abs=0.01)
        assert s["frac"] == pytest.approx(achieved / peak, rel=1e-3, abs=1e-4)
        floor = work / (peak * scale) * 1e3
        assert s["roofline_ms"] == pytest.approx(floor, rel=1e-3, abs=1e-4)
        total_floor += floor
    assert frac == pytest.approx(total_floor / ms_step, rel=1e-3, abs=1e-4)
    # with one slab per step, the dominant stage's launch roofline is its step roofline
    roof, shares = bench.roofline(wl, stage_ms, PEAKS)
    assert roof["kernel"] == "sparse_mla_attn"
    assert roof["frac"] == pytest.approx(stages["sparse_mla_attn"]["frac"], rel=1e-3, abs=1e-4)
    assert sum(shares.values()) == pytest.approx(1.0, abs=1e-3)


def test_a_stage_without_work_of_its_own_is_left_out():
    wl = workloads.generate(workloads.custom("decode", [5000, 3000], idx_dtype="bf16", k=128))
    slow = {"hbm": 0.5, "bf16_sustained": 1000.0, "source": "test"}  # floors of whole ms
    stages, frac = bench.stage_rooflines(wl, {2: [1.0], 3: [0.2]}, 1, 1.2, slow)
    assert set(stages) == {"sparse_mla_attn"}
    floor = bench.algorithmic_work(wl)["attn_bytes"].sum() / (0.5 * 1e9) * 1e3
    assert frac == pytest.approx(floor / 1.2, rel=1e-3)
