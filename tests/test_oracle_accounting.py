"""Pins of the oracle's parameter and FLOP accounting against the numbers the pages print.

The golden fixture holds the printed figures with their page and section. The checks:
the Qwen3-1.7B-shaped model with an untied head has about 2B parameters; 6ND over the
1,398.83B tokens of both phases, at the median 238 TFLOP/s, lands near the 20,000
GPU-hours the walkthrough estimates and within 20% of the 22,514 GPU-hours spent; the
two phases of Table 1 add up to the total; and the FLOPs of the explicit list of GEMM
calls of one micro-step equal 6 x (linear parameters) x tokens.
"""

import json
import os

from oracle import accounting as acc
from tests.conftest import GOLDEN


def _gold():
    with open(os.path.join(GOLDEN, "paper_accounting.json")) as f:
        return {k: v["value"] for k, v in json.load(f).items()}


def test_param_count_is_about_2b():
    g = _gold()
    assert acc.linear_params() == 28 * 50_331_648 + 151_936 * 2048
    n = acc.total_params()
    assert abs(n - g["params_approx"]) / g["params_approx"] < 0.05


def test_6nd_matches_printed_gpu_hours():
    g = _gold()
    tokens = g["tokens_phase1"] + g["tokens_phase2"]
    c = acc.flops_6nd(acc.total_params(), tokens)
    est_hours = c / g["throughput_flops_per_gpu"] / 3600.0
    assert abs(est_hours - g["estimate_gpu_hours"]) / g["estimate_gpu_hours"] < 0.05
    spent = g["gpu_hours_total"] * 3600.0 * g["throughput_flops_per_gpu"]
    assert abs(c / spent - 1.0) < 0.2


def test_table1_phases_add_up():
    g = _gold()
    assert abs(g["gpu_hours_phase1"] + g["gpu_hours_phase2"] - g["gpu_hours_total"]) < 1.0


def test_microstep_gemm_flops_equal_6_params_tokens():
    g = _gold()
    tokens = 2 * int(g["seq_len"])
    assert acc.microstep_flops(tokens) == 6 * acc.linear_params() * tokens
    assert acc.microstep_flops(tokens) == 84_563_611_090_944
    assert len(acc.microstep_gemms(tokens)) == 3 * (4 * 28 + 1)
