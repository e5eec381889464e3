"""The measurement's accounting, on CPU: the algorithmic bytes and flops per call of the stated
workloads (the survey's figures, plus the two fp32 scalars alpha and lora_scale), the roofline
peaks derived from the measured copy bandwidth and bf16 GEMM rate, and the MoE and LoRA-delta byte
counts built from the generated problems."""

import math

import pytest

import bench
from workloads import BGMV, CONFIGS, MOE, make_bgmv_problem, make_grouped_problem


@pytest.mark.parametrize("name,want_bytes,want_flops", [
    ("cfg0", 133_120, 16_777_216),
    ("cfg1", 10_139_648, 536_870_912),
    ("cfg2", 52_699_136, 137_438_953_472),
    ("cfg3", 644_349_952, 3_848_290_697_216),
])
def test_algorithmic_bytes_and_flops_of_the_workloads(name, want_bytes, want_flops):
    nbytes, flops, lora_flops = bench.algorithmic(CONFIGS[name])
    assert nbytes == want_bytes + 8          # + alpha and lora_scale (fp32 device scalars)
    assert flops == want_flops
    c = CONFIGS[name]
    assert lora_flops == 2 * c["M"] * c["N"] * c["r"]


def test_roofline_peaks_follow_the_measured_figures(monkeypatch):
    monkeypatch.setattr(bench, "measured_peaks",
                        lambda: ({"hbm_gbs": 6539.2, "bf16_tflops": 1658.4, "bf16_tflops_sustained": 1402.6},
                                 "measured"))
    monkeypatch.setattr(bench, "recorded_traffic", lambda *a, **k: None)
    hbm = bench.roofline_block(None, "cfg1", 3269.6, "GB/s", 10, 5.0)
    assert hbm["bound"] == "hbm" and hbm["peak"] == 6539.2 and math.isclose(hbm["frac"], 0.5)
    burst = bench.roofline_block(None, "cfg3", 3316.8, "TFLOPS", 10, 16.0)        # 16 ms region
    assert burst["bound"] == "tensor" and math.isclose(burst["peak"], 4 * 1658.4) and math.isclose(burst["frac"], 0.5)
    sustained = bench.roofline_block(None, "cfg3", 2805.2, "TFLOPS", 10, 3000.0)  # 3 s region
    assert math.isclose(sustained["peak"], 4 * 1402.6) and math.isclose(sustained["frac"], 0.5)


def test_moe_and_delta_byte_counts():
    mp = make_grouped_problem(list(MOE["segments"]), MOE["N"], MOE["K"], MOE["r"], MOE["seed"], pad_rows=0)
    nbytes, flops = bench.moe_algorithmic(mp)
    rows, E, N, K, r = sum(MOE["segments"]), len(MOE["segments"]), MOE["N"], MOE["K"], MOE["r"]
    assert flops == 2 * rows * N * K
    want = (rows * K // 2 + E * N * K // 2 + rows * K // 16 + E * N * K // 16 + rows * r * 2 + E * N * r * 2
            + E * N * 2 + rows * N * 2 + 4 * E + 4 * (E + 1) + 4)
    assert nbytes == want
    bp = make_bgmv_problem(**BGMV)
    nb, fl = bench.bgmv_algorithmic(bp)
    act_rows = sum(1 for t in range(bp.T) if bp.lora_ids[t] >= 0
                   for j in range(bp.top_k) if bp.perm[t * bp.top_k + j] >= 0)
    pairs = {(int(bp.lora_ids[t]), int(bp.topk_ids[t, j])) for t in range(bp.T) if bp.lora_ids[t] >= 0
             for j in range(bp.top_k) if bp.perm[t * bp.top_k + j] >= 0}
    assert fl == 2 * act_rows * (bp.rank * bp.I + bp.H * bp.rank)
    assert nb == (act_rows * bp.I * 2 + len(pairs) * (bp.rank * bp.I + bp.H * bp.rank) * 2 + bp.T * bp.top_k * 12
                  + bp.T * 4 + 2 * bp.num_experts * 8 + bp.T * bp.H * 2)
    assert nb == 9_717_632
