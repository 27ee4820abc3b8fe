"""FP8 (E4M3) forward on the tcgen05 kernel against the float64 oracle.

The scores are exact products of E4M3 values, so LSE is held to the usual
1e-4.  O goes through P quantised to E4M3 (relative rounding <= 2^-4 per
weight, zero mean): the expected relative RMS error of O from that alone is
about 2^-4 / sqrt(3) ~ 0.036, and the bound used is 0.05.  A second case
makes every P exactly representable (integer scores spanning <= 8 with
scale ln 2, so P = 2^k with |k| <= 8) and holds O to the bf16 bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_lse, check_out, f64, rel_fro
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

FP8_REL_RMS = 0.05

# (B, Sq, Sk, Hq, Hkv, causal, window, softcap, with descales)
CASES = [
    (2, 300, 300, 4, 2, True, (-1, -1), 0.0, True),
    (1, 200, 513, 4, 4, False, (-1, -1), 0.0, False),
    (2, 129, 129, 8, 1, True, (40, 0), 0.0, True),
    (1, 257, 257, 2, 2, False, (-1, -1), 20.0, True),
    (1, 1024, 1024, 4, 2, False, (64, 64), 0.0, True),
]


def _codes(t):
    return t.view(torch.uint8).numpy()


def _run(case, seed=70):
    B, Sq, Sk, Hq, Hkv, causal, window, cap, desc = case
    q, k, v, dq, dk, dv = inputs.fp8_inputs(B, Sq, Sk, Hq, Hkv, 128, seed=seed)
    if not desc:
        dq = dk = dv = None
    dev = lambda t: None if t is None else t.cuda()
    out, lse = api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), dev(dq), dev(dk), dev(dv), causal=causal, window=window,
                              softcap=cap)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    npd = lambda t: None if t is None else t.double().numpy()
    o_r, l_r = oracle.attn_fwd_fp8(_codes(q), _codes(k), _codes(v), npd(dq), npd(dk), npd(dv), None, causal,
                                   window[0], window[1], cap)
    return out, lse, o_r, l_r


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dS%dx%dH%d-%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], "c" if c[5] else "", "w" if c[6] != (-1, -1) else ""))
def test_fp8_forward_vs_oracle(case):
    out, lse, o_r, l_r = _run(case)
    check_lse(lse, l_r)
    g = f64(out)
    assert np.isfinite(g).all()
    e = rel_fro(out, o_r)
    assert e <= FP8_REL_RMS, f"O relative RMS error {e:.3e}"


def test_fp8_exact_powers_of_two_match_to_bf16():
    # q one-hot in dim 0, k[:, :, :, 0] integers in [-4, 4]: raw scores are
    # those integers; scale ln 2 and dq * dk = 1 make P = 2^(score - max),
    # exact in E4M3, so O differs from the oracle by bf16 rounding only
    B, S, H, D = 2, 384, 4, 128
    g = torch.Generator().manual_seed(71)
    q = torch.zeros((B, S, H, D))
    q[..., 0] = 1.0
    k = torch.randn((B, S, H, D), generator=g)
    k[..., 0] = torch.randint(-4, 5, (B, S, H), generator=g).float()
    v = torch.randn((B, S, H, D), generator=g)
    q8, k8, v8 = (t.to(torch.float8_e4m3fn) for t in (q, k, v))
    dq = torch.full((B, H), 2.0)
    dk = torch.full((B, H), 0.5)
    dv = torch.rand((B, H), generator=g) + 0.5
    sc = math.log(2.0)
    for causal in (False, True):
        out, lse = api.fa_fwd_fp8(q8.cuda(), k8.cuda(), v8.cuda(), dq.cuda(), dk.cuda(), dv.cuda(), scale=sc,
                                  causal=causal)
        torch.cuda.synchronize()
        o_r, l_r = oracle.attn_fwd_fp8(_codes(q8), _codes(k8), _codes(v8), dq.double().numpy(), dk.double().numpy(),
                                       dv.double().numpy(), sc, causal)
        check_out(out, o_r, torch.bfloat16)
        check_lse(lse, l_r)


def test_fp8_full_size_sampled_rows():
    cfg = inputs.fp8_config()
    q, k, v, dq, dk, dv = inputs.fp8_inputs(cfg["B"], cfg["Sq"], cfg["Sk"], cfg["Hq"], cfg["Hkv"], cfg["D"],
                                            seed=cfg["seed"], amp=cfg["amp"])
    out, lse = api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), dq.cuda(), dk.cuda(), dv.cuda())
    torch.cuda.synchronize()
    rows = np.array([0, 1, 255, 2048, 4095])
    qv, kv, vv = (oracle.e4m3_decode(_codes(t)) for t in (q, k, v))
    for b, h in ((0, 0), (3, 15)):
        f = lambda d: float(d[b, h])
        o_r, l_r = oracle.attn_fwd_rows(qv * f(dq), kv * f(dk), vv * f(dv), b, h, rows)
        check_lse(lse[b, h, rows], l_r)
        assert rel_fro(out[b, rows, h], o_r) <= FP8_REL_RMS


def test_fp8_refusals():
    q, k, v, *_ = inputs.fp8_inputs(1, 16, 16, 2, 2, 128, seed=72)
    with pytest.raises(_lib.FaError):  # the mma.sync kernel has no 8-bit path
        api.fa_set_fwd_kernel(1)
        try:
            api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda())
        finally:
            api.fa_set_fwd_kernel(0)
    q64, k64, v64, *_ = inputs.fp8_inputs(1, 16, 16, 2, 2, 64, seed=72)
    with pytest.raises(_lib.FaError):  # head dim 64 is not laid out for 8 bits
        api.fa_fwd_fp8(q64.cuda(), k64.cuda(), v64.cuda())
