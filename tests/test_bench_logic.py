"""Host logic of bench.py that needs no GPU: the per-configuration table
built from whole-call timings (forward, forward+backward and paged-decode
fractions of the measured peaks) and the visible-pair count behind every
flop figure."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _FakeTracer:
    def __init__(self, per_call, per_unit):
        self.per_call = per_call
        self.per_unit = per_unit


PEAKS = {"bf16_tflops_sustained": 1000.0, "bf16_tflops": 2000.0, "hbm_gbs": 5000.0}


def test_per_config_fractions():
    # two steps of 1 ms forward (1 TFLOP) and 2.5 ms backward (2.5 TFLOP)
    per_call = {("fwd", "H16D128S4096n"): [2.0, 2, 2e12], ("bwd", "H16D128S4096n"): [5.0, 2, 5e12],
                ("fwd", "H16D128S8192c"): [4.0, 2, 2e12], ("bwd", "H16D128S8192c"): [10.0, 2, 5e12],
                ("fwd", "H32D64S4096n"): [1.0, 1, 1e12],
                ("decode", "decode-s4"): [0.2, 2, 1e9]}
    per_unit = {("decode", "decode-s4"): [0.1, 2, 1e9]}
    pts, summ = bench.per_config(_FakeTracer(per_call, per_unit), PEAKS)
    a = pts["H16D128S4096n"]
    assert abs(a["fwd_tflops"] - 1000.0) < 1e-6 and abs(a["fwd_frac"] - 1.0) < 1e-9
    assert abs(a["fwd_frac_burst"] - 0.5) < 1e-9
    assert abs(a["bwd_tflops"] - 1000.0) < 1e-6
    assert abs(a["fwdbwd_tflops"] - 1000.0) < 1e-6 and abs(a["fwdbwd_frac"] - 1.0) < 1e-9
    c = pts["H16D128S8192c"]
    assert abs(c["fwd_tflops"] - 500.0) < 1e-6 and abs(c["fwdbwd_frac"] - 0.5) < 1e-9
    d = pts["decode-s4"]
    assert abs(d["call_gbs"] - 5000.0) < 1e-6 and abs(d["call_frac"] - 1.0) < 1e-9
    assert abs(d["split_kernel_gbs"] - 10000.0) < 1e-6
    # the long head-dim-128 summary takes the worst of the S >= 4096 points
    assert summ["d128_s4k_plus"]["points"] == 2
    assert abs(summ["d128_s4k_plus"]["fwd_frac_min"] - 0.5) < 1e-9
    assert abs(summ["d128_s4k_plus"]["fwdbwd_frac_min"] - 0.5) < 1e-9
    assert abs(summ["decode_call_frac_min"] - 1.0) < 1e-9


def test_visible_pairs_closed_forms():
    S = 257
    assert bench.visible_pairs(S, S, False, -1, -1) == S * S
    assert bench.visible_pairs(S, S, True, -1, -1) == S * (S + 1) // 2
    # window (w, 0) with causal: row i sees min(i, w) + 1 keys
    w = 16
    assert bench.visible_pairs(S, S, True, w, 0) == sum(min(i, w) + 1 for i in range(S))
    # Sq < Sk, bottom-right aligned causal: row i sees Sk - Sq + i + 1 keys
    assert bench.visible_pairs(3, 10, True, -1, -1) == 8 + 9 + 10
