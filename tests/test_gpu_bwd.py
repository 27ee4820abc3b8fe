"""Backward parity: CUDA dQ/dK/dV vs the float64 oracle's chain rule, atomic
and deterministic (ordered) dQ modes; bit-identity of the deterministic mode."""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_grad, check_lse, check_out, f64
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# (B, Sq, Sk, Hq, Hkv, D, dtype, causal, window, softcap, scale, amp)
SMALL = [
    (2, 77, 77, 4, 4, 64, "bf16", True, (-1, -1), 0.0, None, 1.0),
    (1, 130, 200, 4, 2, 128, "fp16", False, (-1, -1), 5.0, None, 1.0),
    (2, 200, 130, 8, 2, 64, "bf16", True, (-1, -1), 0.0, None, 1.0),
    (1, 257, 257, 2, 1, 128, "bf16", False, (32, 16), 0.0, None, 1.0),
    (1, 1, 300, 4, 4, 64, "fp16", True, (-1, -1), 0.0, None, 1.0),
    (1, 300, 1, 2, 2, 128, "bf16", False, (-1, -1), 0.0, None, 1.0),
    (3, 190, 190, 6, 3, 128, "fp16", True, (50, 0), 10.0, None, 2.0),
    (1, 512, 512, 4, 1, 128, "bf16", True, (-1, -1), 30.0, 0.3, 2.0),
]


def _fwd_bwd(q, k, v, do, det, **kw):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    dq, dk, dv = api.fa_bwd(dod, qd, kd, vd, out, lse, deterministic=det, **kw)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    return out, lse, dq, dk, dv


@pytest.mark.parametrize("which", [0, 1], ids=["auto", "mma"])
@pytest.mark.parametrize("det", [False, True], ids=["atomic", "ordered"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B%dSq%dSk%dH%d-%dD%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], c[6], "c" if c[7] else ""))
def test_bwd_small_full_compare(case, det, which):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, scale, amp = case
    q, k, v, do = inputs.attention_inputs(B, Sq, Sk, Hq, Hkv, D, dt, seed=21, amp=amp)
    kw = dict(scale=scale, causal=causal, window=window, softcap=cap)
    _lib.load().fa_set_bwd_kernel(which)
    try:
        out, lse, dq, dk, dv = _fwd_bwd(q, k, v, do, det, **kw)
    finally:
        _lib.load().fa_set_bwd_kernel(0)
    sc = scale or 1 / math.sqrt(D)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(f64(do), f64(q), f64(k), f64(v), sc, causal, window[0], window[1], cap)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


@pytest.mark.parametrize("det", [False, True], ids=["atomic", "ordered"])
def test_fwd_bwd_512_full(det):
    cfg = inputs.fwd_bwd_512_config()
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"])
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, do, det, scale=cfg["scale"], causal=True)
    o_r, l_r = oracle.attn_fwd(f64(q), f64(k), f64(v), cfg["scale"], True)
    check_out(out, o_r, torch.float16)
    check_lse(lse, l_r)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(f64(do), f64(q), f64(k), f64(v), cfg["scale"], True)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


@pytest.mark.parametrize("det", [False, True], ids=["atomic", "ordered"])
def test_gqa_local_full_size_slices(det):
    """Full-size GQA + window + softcap workload; gradients of two kv-head groups
    (all their q-heads) in both batches are compared with the oracle."""
    cfg = inputs.gqa_local_config()
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"], amp=cfg["amp"])
    kw = dict(scale=cfg["scale"], causal=True, window=cfg["window"], softcap=cfg["softcap"])
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, do, det, **kw)
    G = cfg["Hq"] // cfg["Hkv"]
    for b in (0, 1):
        for g in (0, cfg["Hkv"] - 1):
            hs = slice(g * G, (g + 1) * G)
            sl = lambda t, heads: f64(t[b:b + 1, :, heads])
            dq_r, dk_r, dv_r, _ = oracle.attn_bwd(sl(do, hs), sl(q, hs), sl(k, slice(g, g + 1)),
                                                  sl(v, slice(g, g + 1)), cfg["scale"], True,
                                                  cfg["window"][0], 0, cfg["softcap"])
            check_grad(dq[b:b + 1, :, hs], dq_r, f"dQ b{b} g{g}")
            check_grad(dk[b:b + 1, :, g:g + 1], dk_r, f"dK b{b} g{g}")
            check_grad(dv[b:b + 1, :, g:g + 1], dv_r, f"dV b{b} g{g}")


@pytest.mark.parametrize("which", [0, 1], ids=["auto", "mma"])
def test_deterministic_is_bit_identical(which):
    cfg = inputs.gqa_local_config()
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"], amp=cfg["amp"])
    kw = dict(scale=cfg["scale"], causal=True, window=cfg["window"], softcap=cfg["softcap"])
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    runs = []
    _lib.load().fa_set_bwd_kernel(which)
    try:
        for _ in range(3):
            runs.append([t.clone() for t in api.fa_bwd(dod, qd, kd, vd, out, lse, deterministic=True, **kw)])
        torch.cuda.synchronize()
    finally:
        _lib.load().fa_set_bwd_kernel(0)
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert api.fa_last_device_status() == 0


@pytest.mark.parametrize("cfg", [c for c in inputs.seqlen_sweep_configs() if c["Sq"] <= 2048],
                         ids=lambda c: "H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n"))
def test_bwd_seqlen_sweep_head_slices(cfg):
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"])
    out, lse, dq, dk, dv = _fwd_bwd(q, k, v, do, False, scale=cfg["scale"], causal=cfg["causal"])
    for b, h in ((0, 0), (cfg["B"] - 1, cfg["Hq"] - 1)):
        sl = lambda t: f64(t[b:b + 1, :, h:h + 1])
        dq_r, dk_r, dv_r, _ = oracle.attn_bwd(sl(do), sl(q), sl(k), sl(v), cfg["scale"], cfg["causal"])
        check_grad(dq[b:b + 1, :, h:h + 1], dq_r, "dQ")
        check_grad(dk[b:b + 1, :, h:h + 1], dk_r, "dK")
        check_grad(dv[b:b + 1, :, h:h + 1], dv_r, "dV")


def _sample(S, rng, n):
    idx = set([0, 1, S // 2, S - 2, S - 1]) | set(rng.integers(0, S, n).tolist())
    return np.array(sorted(i for i in idx if 0 <= i < S))


@pytest.mark.parametrize("cfg", [c for c in inputs.seqlen_sweep_configs() if c["Sq"] >= 4096],
                         ids=lambda c: "H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n"))
def test_bwd_seqlen_sweep_sampled(cfg):
    """Long sweep points (S = 4k, 8k, 16k) in the benchmark's launch
    configuration: dQ of sampled query rows of two (batch, head) slices and
    dK/dV of sampled key rows of one, against the oracle's per-row chain
    rule, for the atomic and the ordered dQ accumulation."""
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"])
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    kw = dict(scale=cfg["scale"], causal=cfg["causal"])
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    grads = {}
    for det in (False, True):
        grads[det] = [t.cpu() for t in api.fa_bwd(dod, qd, kd, vd, out, lse, deterministic=det, **kw)]
        torch.cuda.synchronize()
        assert api.fa_last_device_status() == 0
    Q, K, V, DO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    rng = np.random.default_rng(cfg["seed"])
    B, Hq, S = cfg["B"], cfg["Hq"], cfg["Sq"]
    for b, h in ((0, 0), (B - 1, Hq - 1)):
        rows = _sample(S, rng, 24)
        dq_r, _, _ = oracle.attn_bwd_rows(DO, Q, K, V, b, h, rows, cfg["scale"], cfg["causal"])
        for det, (dq, _, _) in grads.items():
            check_grad(dq[b, rows, h], dq_r, f"dQ b{b} h{h} det={det}")
    b, g = B - 1, cfg["Hkv"] - 1
    cols = _sample(S, rng, 12)
    dk_r, dv_r = oracle.attn_bwd_cols(DO, Q, K, V, b, g, cols, cfg["scale"], cfg["causal"])
    for det, (_, dk, dv) in grads.items():
        check_grad(dk[b, cols, g], dk_r, f"dK b{b} g{g} det={det}")
        check_grad(dv[b, cols, g], dv_r, f"dV b{b} g{g} det={det}")


@pytest.mark.parametrize("cfg", inputs.long_context_configs(),
                         ids=lambda c: "H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n"))
def test_bwd_long_context_sampled(cfg):
    """32k tokens in one sequence, atomic dQ: dQ of sampled query rows of
    the first and last head and dK/dV of sampled key rows of the last kv-head
    (every query row of that head evaluated by the oracle)."""
    q, k, v, do = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                          cfg["dtype"], seed=cfg["seed"])
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    kw = dict(scale=cfg["scale"], causal=cfg["causal"])
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    dq, dk, dv = (t.cpu() for t in api.fa_bwd(dod, qd, kd, vd, out, lse, **kw))
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    Q, K, V, DO = (t.to(torch.float64).numpy() for t in (q, k, v, do))
    rng = np.random.default_rng(cfg["seed"])
    S, Hq = cfg["Sq"], cfg["Hq"]
    for h in (0, Hq - 1):
        rows = _sample(S, rng, 16)
        dq_r, _, _ = oracle.attn_bwd_rows(DO, Q, K, V, 0, h, rows, cfg["scale"], cfg["causal"])
        check_grad(dq[0, rows, h], dq_r, f"dQ h{h}")
    g = cfg["Hkv"] - 1
    cols = _sample(S, rng, 8)
    dk_r, dv_r = oracle.attn_bwd_cols(DO, Q, K, V, 0, g, cols, cfg["scale"], cfg["causal"])
    check_grad(dk[0, cols, g], dk_r, f"dK g{g}")
    check_grad(dv[0, cols, g], dv_r, f"dV g{g}")
