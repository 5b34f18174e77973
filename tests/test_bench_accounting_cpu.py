"""bench.py's work accounting (the numerators of every roofline fraction it reports), checked
on the CPU against the closed forms of the layer's traffic and arithmetic:

* bytes of one forward = the weights of every expert some token chose, plus the shared
  expert's, each read once (gate + up + down = 3 d f elements), plus the router matrix, plus x
  read and out written once;
* flops = 2 (T k + T) 3 d f for the expert contractions (T k routed rows and T shared rows)
  plus 2 T d E for the router.

The expected values are written out from the shapes by hand, not from bench.py's formulas.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from sparse_moe_layer_warp_b200 import synth  # noqa: E402


def _counts(E, touched, total):
    c = np.zeros(E, dtype=np.int64)
    c[:touched] = total // touched
    c[0] += total - c.sum()
    return c


def test_decode_t16_bytes_and_flops():
    w = synth.WORKLOADS["decode_t16"]  # T=16, d=4096, E=288, k=8, f=1280, bf16, 1 shared
    a = bench.algorithmic(w, _counts(288, 104, 16 * 8), 16)
    assert a["touched"] == 105
    # 105 experts x 3 x 1280 x 4096 x 2 B, + W_r 288 x 4096 x 2 B, + x and out 2 x 16 x 4096 x 2 B
    assert a["layer_bytes"] == 105 * 31_457_280 + 2_359_296 + 262_144 == 3_305_635_840
    # (128 + 16) rows x 3 x 4096 x 1280 x 2, + 2 x 16 x 4096 x 288
    assert a["layer_flops"] == 2 * 144 * 3 * 4096 * 1280 + 2 * 16 * 4096 * 288
    # the up kernel: gate + up weights of the touched experts, its 144 operand rows of x,
    # and the 144 x 1280 bf16 rows of h it writes
    assert a["up_bytes"] == 105 * 2 * 1280 * 4096 * 2 + 144 * 4096 * 2 + 144 * 1280 * 2
    # the down kernel: down weights, h read, fp32 y rows written
    assert a["down_bytes"] == 105 * 4096 * 1280 * 2 + 144 * 1280 * 2 + 144 * 4096 * 4
    assert a["up_flops"] + a["down_flops"] == 2 * 144 * 3 * 4096 * 1280


def test_prefill_t8192_flops_match_the_ridge_arithmetic():
    w = synth.WORKLOADS["prefill_t8192"]
    a = bench.algorithmic(w, np.full(288, 8192 * 8 // 288 + 1), 8192)
    assert a["touched"] == 289
    assert a["layer_flops"] == pytest.approx(2.3386e12, rel=1e-4)  # 2.339 TFLOP
    assert a["layer_bytes"] == pytest.approx(9.23e9, rel=2e-3)      # weights once + x + out
    # arithmetic intensity on the measured ridge (about 251 flop/B on B200)
    assert 240 < a["layer_flops"] / a["layer_bytes"] < 260


def test_untouched_experts_cost_nothing_and_fp32_doubles_bytes():
    w = synth.WORKLOADS["tiny_fp32"]  # T=64, d=256, E=16, k=2, f=64, fp32, 1 shared
    a = bench.algorithmic(w, _counts(16, 3, 64 * 2), 64)
    assert a["touched"] == 4
    assert a["layer_bytes"] == 4 * 3 * 64 * 256 * 4 + 16 * 256 * 4 + 2 * 64 * 256 * 4
    wb = w.replace(dtype="bf16")
    b = bench.algorithmic(wb, _counts(16, 3, 64 * 2), 64)
    assert a["layer_bytes"] == 2 * b["layer_bytes"]
    assert a["layer_flops"] == b["layer_flops"]


def test_dense_ffn_has_no_shared_rows():
    w = synth.WORKLOADS["dense_ffn_t4096"]  # E=1, k=1, f=11264, no shared expert
    a = bench.algorithmic(w, np.array([4096]), 4096)
    assert a["touched"] == 1
    assert a["layer_flops"] == 2 * 4096 * 3 * 4096 * 11264 + 2 * 4096 * 4096
    assert a["layer_bytes"] == 3 * 11264 * 4096 * 2 + 4096 * 2 + 2 * 4096 * 4096 * 2


def test_layer_roofline_is_the_tensor_fraction_of_a_tensor_bound_forward():
    """prefill_t8192 (every expert touched: 289 x 3 x 1280 x 4096 x 2 B + W_r + x + out =
    9.23 GB, 2.34 TFLOP, 253 flop/B above the measured ridge of 1642.5 / 6554.2 = 250.6):
    the bench line's roofline is the forward's flops over the step time against the burst
    bf16 peak.  decode_t16 (1.4 flop/B) is HBM-bound: no layer tensor roofline."""
    peaks = {"hbm_gbs": 6554.2, "bf16_tflops": 1642.5}
    w = synth.WORKLOADS["prefill_t8192"]
    a = bench.algorithmic(w, _counts(288, 288, 8192 * 8), 8192)
    flops = 2 * (8192 * 8 + 8192) * 3 * 4096 * 1280 + 2 * 8192 * 4096 * 288
    assert a["layer_flops"] == flops
    r = bench.layer_roofline(a["layer_bytes"], a["layer_flops"], 2.85e-3, peaks)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["frac"] == round(flops / 2.85e-3 / 1e12 / 1642.5, 4)
    assert 0.499 < r["frac"] < 0.501  # 2.3386 TFLOP in 2.85 ms is half the burst peak
    d = synth.WORKLOADS["decode_t16"]
    b = bench.algorithmic(d, _counts(288, 104, 16 * 8), 16)
    assert bench.layer_roofline(b["layer_bytes"], b["layer_flops"], 0.5e-3, peaks) is None


def test_layer_roofline_peak_follows_the_measured_gemm_clock():
    """frac stays the burst fraction; the clock-regime fraction beside it uses the sustained
    peak only when the GEMMs' own effective clock is within 10 % of the sustained loop's
    median clock; otherwise (or unmeasured) the burst peak."""
    peaks = {"hbm_gbs": 6554.2, "bf16_tflops": 1642.5, "bf16_tflops_sustained": 1394.5,
             "clocks_under_load": {"sm_mhz_median": 1335.0}}
    w = synth.WORKLOADS["prefill_t8192"]
    a = bench.algorithmic(w, _counts(288, 288, 8192 * 8), 8192)
    args = (a["layer_bytes"], a["layer_flops"], 2.85e-3, peaks)
    ach = a["layer_flops"] / 2.85e-3 / 1e12
    r = bench.layer_roofline(*args, gemm_mhz=1370.0)
    assert r["peak"] == 1642.5 and r["frac"] == round(ach / 1642.5, 4)
    assert r["clock_regime"] == "sustained"
    assert r["frac_of_clock_regime_peak"] == round(ach / 1394.5, 4)
    for mhz in (None, 1900.0, 1100.0):
        r = bench.layer_roofline(*args, gemm_mhz=mhz)
        assert r["clock_regime"] == "burst" and r["frac_of_clock_regime_peak"] == r["frac"]
    del peaks["bf16_tflops_sustained"]
    assert bench.layer_roofline(*args, gemm_mhz=1370.0)["clock_regime"] == "burst"
