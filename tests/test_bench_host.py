"""Host-side checks of bench.py's accounting (no GPU): the algorithmic work it
divides by is the oracle's definition of the same operations, and the JSON
line's fixed parts are what the measurement contract asks for."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth_inputs as si  # noqa: E402
from oracle import ispa_oracle as orc  # noqa: E402


def test_step_work_matches_the_oracle_flop_definitions():
    sh = si.SHAPE_1P3B
    w = bench.step_work(sh)
    T = sh.B * sh.Lq
    # the split costs the dot products of full attention; the post-switch passes see
    # the local rows (L-layer) and every row (F-layer)
    assert w["attn_split"] == orc.attention_flops(T, sh.Lkv, sh.H, sh.d)
    assert w["attn_full"] == orc.attention_flops(T, sh.Lkv, sh.H, sh.d)
    assert w["attn_local"] == orc.attention_flops(T, len(sh.local_rows), sh.H, sh.d)
    assert abs(w["attn_split"] - 0.942e12) < 0.001e12          # the 0.942 TFLOP quoted for the layer
    D = sh.D
    assert w["stats"] == 2.0 * T * D * D + T * D * (D + 1) + 2.0 * T * D * D
    assert w["proj"] == 2 * 2.0 * T * D * D
    assert abs(w["total"] - sum(v for k, v in w.items() if k != "total")) < 1.0


def test_aggregate_value_is_whole_job_throughput():
    # value = work of all ranks / the slowest rank's time
    assert bench.aggregate_value(2e12, 4.0, 1) == 2e12 / 4e-3 / 1e12
    assert bench.aggregate_value(2e12, 4.0, 8) == 8 * 2e12 / 4e-3 / 1e12


def test_config_block_names_the_workload():
    c = bench.config_block(1)
    assert "1.3B" in c["workload"] and c["Lq"] == 4680 and c["Lkv"] == 32760 and c["D"] == 1536
    assert "l2" in c and "parallelism" in c


def test_kv_retained_fraction_of_the_model():
    # 15 of 30 layers keep sink + current (6 of 21 frames): 64.3 %, the pages' ISPA-0.5 figure
    sh = si.SHAPE_1P3B
    kept = len(orc._local_rows(sh)) // sh.tpf
    frac = ((30 - 15) * sh.kv_frames + 15 * kept) / (30 * sh.kv_frames)
    assert kept == 6 and abs(frac - 0.6428571) < 1e-6
    assert abs(orc.kv_retained_fraction(0.5, (sh.kv_frames - kept) / sh.kv_frames) - frac) < 1e-12


def test_clock_sampler_summary_maps_reasons():
    c = bench.ClockSampler(0)
    # NVML samples: (sm MHz, max MHz, clock-event reason bits); 0x4 = sw power cap, 0x8 = hw slowdown
    c.samples = [(1965.0, 1965.0, 0), (1900.0, 1965.0, 0x4), (1800.0, 1965.0, 0x4 | 0x8)]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    # nvidia-smi lines (the fallback): fields as queried, "Active" / "Not Active"
    c2 = bench.ClockSampler(0)
    c2.lines = ["1965, 1965, 800.0, Not Active, Not Active, Not Active, Active",
                "1950, 1965, 810.0, Not Active, Active, Not Active, Not Active"]
    s2 = c2.summary()
    assert s2["samples"] == 2 and s2["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert bench.ClockSampler(0).summary()["sm_mhz"] is None


def test_oracle_sample_work_scales_to_the_step():
    # a sample of all Lq rows is the whole step; the solve is counted once per sample
    sh = si.SHAPE_1P3B
    w = bench.step_work(sh)
    assert abs(bench.sample_work(sh.B * sh.Lq) - w["total"]) <= 1e-9 * w["total"]
    assert abs(bench.sample_work(0) - w["solve"]) <= 1e-9 * w["solve"]


def test_sweep_kv_retained_matches_the_oracle_accounting():
    # every sweep point: the bytes the bench reports as kept equal the oracle's
    # retained fraction 1 - (K/N) h, with K = floor(x N) and h the history share of the keys
    for name, H, N in bench.SWEEP_SHAPES:
        for B in (1, 2):
            for Hf in bench.SWEEP_HIST:
                sh = si.video_shape(H, Hf, B=B)
                h_frac = len(sh.hist_rows) / sh.Lkv
                for x in bench.SWEEP_X:
                    kv = bench.kv_retained(sh, B, N, x)
                    K = orc.num_selected(x, N)
                    assert kv["l_layers"] == K
                    assert abs(kv["fraction"] - orc.kv_retained_fraction(K / N, h_frac)) < 1e-12
                    assert kv["kv_bytes_full"] == B * N * sh.Lkv * sh.D * 4
    # the 30-layer 1.3B model at ISPA-0.5 keeps 64.3 % of its KV
    assert abs(bench.kv_retained(si.SHAPE_1P3B, 1, 30, 0.5)["fraction"] - 0.6428571428) < 1e-9
