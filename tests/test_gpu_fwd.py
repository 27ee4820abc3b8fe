"""Forward parity: CUDA path vs the float64 oracle on the same seeded inputs.

Small problems (several tiles plus ragged tails) are compared element by
element; the full-size workloads (seqlen sweep at hidden 2048, GQA + local
attention) are compared on sampled query rows that the oracle evaluates one
by one, in the launch configuration the benchmark uses.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_lse, check_out, f64
from exact_attention_121_b200 import api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# (B, Sq, Sk, Hq, Hkv, D, dtype, causal, window, softcap, scale, amp)
SMALL = [
    (1, 128, 128, 2, 2, 64, "fp16", False, (-1, -1), 0.0, 1 / 8, 1.0),      # tiny forward workload
    (2, 77, 77, 4, 4, 64, "bf16", True, (-1, -1), 0.0, None, 1.0),
    (1, 130, 200, 4, 2, 128, "fp16", False, (-1, -1), 5.0, None, 1.0),
    (2, 200, 130, 8, 2, 64, "bf16", True, (-1, -1), 0.0, None, 1.0),         # Sq > Sk: empty rows
    (1, 257, 257, 2, 1, 128, "bf16", False, (32, 16), 0.0, None, 1.0),
    (1, 1, 300, 4, 4, 64, "fp16", True, (-1, -1), 0.0, None, 1.0),
    (1, 300, 1, 2, 2, 128, "bf16", False, (-1, -1), 0.0, None, 1.0),
    (1, 64, 64, 2, 2, 64, "fp16", False, (0, 0), 0.0, None, 1.0),
    (3, 190, 190, 6, 3, 128, "fp16", True, (50, 0), 10.0, None, 2.0),
    (1, 512, 512, 4, 1, 128, "bf16", True, (-1, -1), 30.0, 0.3, 2.0),
    (2, 384, 384, 2, 2, 64, "bf16", False, (-1, -1), 0.0, None, 1.0),
    # more key tiles than K/V stages (5 at head dim 64, 3 and 2 at 128), ragged
    # tails: every stage is reused and every stage-free wait runs
    (1, 300, 1317, 2, 1, 64, "bf16", False, (-1, -1), 0.0, None, 1.0),
    (1, 1100, 1100, 2, 2, 64, "fp16", True, (-1, -1), 0.0, None, 1.0),
    (1, 260, 777, 2, 2, 128, "bf16", False, (-1, -1), 0.0, None, 1.0),
    (1, 900, 900, 2, 1, 128, "bf16", True, (-1, -1), 0.0, None, 1.0),
]


def _run(case, which, seed):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, scale, amp = case
    q, k, v, _ = inputs.attention_inputs(B, Sq, Sk, Hq, Hkv, D, dt, seed=seed, amp=amp, with_dout=False)
    api.fa_set_fwd_kernel(which)
    try:
        out, lse = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=causal, window=window,
                              softcap=cap)
        torch.cuda.synchronize()
    finally:
        api.fa_set_fwd_kernel(0)
    return q, k, v, out, lse


@pytest.mark.parametrize("which", [0, 1, 2], ids=["auto", "mma", "tc"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B%dSq%dSk%dH%d-%dD%d%s%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], c[6], "c" if c[7] else "", "w" if c[8] != (-1, -1) else ""))
def test_fwd_small_full_compare(case, which):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, scale, amp = case
    q, k, v, out, lse = _run(case, which, seed=11)
    o_ref, l_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), scale or 1 / math.sqrt(D), causal, window[0],
                                   window[1], cap)
    check_out(out, o_ref, DT[dt])
    check_lse(lse, l_ref)
    assert api.fa_last_device_status() == 0


def _sample_rows(S, rng, n=24):
    rows = set([0, 1, S // 2, S - 2, S - 1]) | set(rng.integers(0, S, n).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < S))


def _check_sampled(cfg, q, k, v, out, lse, heads, batches, seed=0):
    rng = np.random.default_rng(seed)
    dt = DT[cfg["dtype"]]
    for b in batches:
        for h in heads:
            rows = _sample_rows(cfg["Sq"], rng)
            o_ref, l_ref = oracle.attn_fwd_rows(q, k, v, b, h, rows, cfg["scale"], cfg["causal"],
                                                cfg["window"][0], cfg["window"][1], cfg["softcap"])
            check_out(out[b, rows, h], o_ref, dt)
            check_lse(lse[b, h, rows], l_ref)


SWEEP = inputs.seqlen_sweep_configs()


@pytest.mark.parametrize("cfg", SWEEP, ids=lambda c: "H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"],
                                                                      "c" if c["causal"] else "n"))
def test_fwd_seqlen_sweep_sampled(cfg):
    q, k, v, _ = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                         cfg["dtype"], seed=cfg["seed"], with_dout=False)
    out, lse = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), scale=cfg["scale"], causal=cfg["causal"])
    out, lse = f64(out), f64(lse)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _check_sampled(cfg, qn, kn, vn, out, lse, heads=[0, cfg["Hq"] - 1], batches=sorted({0, cfg["B"] - 1}))
    assert np.isfinite(out).all()


@pytest.mark.parametrize("cfg", inputs.long_context_configs(),
                         ids=lambda c: "H%dD%dS%d%s" % (c["Hq"], c["D"], c["Sq"], "c" if c["causal"] else "n"))
def test_fwd_long_context_sampled(cfg):
    """32k tokens in one sequence: the LSE and O of sampled rows of the first
    and last head, the rows near the end seeing every key."""
    q, k, v, _ = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                         cfg["dtype"], seed=cfg["seed"], with_dout=False)
    out, lse = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), scale=cfg["scale"], causal=cfg["causal"])
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    out, lse = f64(out), f64(lse)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _check_sampled(cfg, qn, kn, vn, out, lse, heads=[0, cfg["Hq"] - 1], batches=[0], seed=cfg["seed"])
    assert np.isfinite(out).all()


def test_fwd_gqa_local_sampled():
    cfg = inputs.gqa_local_config()
    q, k, v, _ = inputs.attention_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                         cfg["dtype"], seed=cfg["seed"], amp=cfg["amp"], with_dout=False)
    out, lse = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), scale=cfg["scale"], causal=cfg["causal"],
                          window=cfg["window"], softcap=cfg["softcap"])
    out, lse = f64(out), f64(lse)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _check_sampled(cfg, qn, kn, vn, out, lse, heads=[0, 5, 31], batches=[0, 1])


def test_fwd_no_keys_gives_zero_and_neg_inf():
    q, k, v, _ = inputs.attention_inputs(1, 70, 1, 2, 2, 64, "bf16", seed=3, with_dout=False)
    out, lse = api.fa_fwd(q.cuda(), k.cuda()[:, :0].contiguous(), v.cuda()[:, :0].contiguous())
    torch.cuda.synchronize()
    assert (out == 0).all() and torch.isneginf(lse).all()


def test_fwd_allocates_nothing():
    q, k, v, _ = inputs.attention_inputs(2, 1024, 1024, 8, 8, 128, "bf16", seed=4, with_dout=False)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(q)
    lse = torch.empty(2, 8, 1024, device="cuda")
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.max_memory_allocated()
    api.fa_fwd(q, k, v, out=out, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before


def test_fwd_kernels_agree_bitwise_on_softmax_rows():
    """Both forward kernels satisfy the same invariant: rows of P sum to 1,
    checked through O for V = 1 (O must be exactly representable 1)."""
    q, k, _, _ = inputs.attention_inputs(2, 300, 300, 4, 4, 128, "bf16", seed=5, with_dout=False)
    v = torch.ones_like(k)
    for which in (1, 2):
        api.fa_set_fwd_kernel(which)
        out, _ = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True)
        torch.cuda.synchronize()
        api.fa_set_fwd_kernel(0)
        assert torch.allclose(out.float(), torch.ones_like(out, dtype=torch.float32), atol=8e-3)
