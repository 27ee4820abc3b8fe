"""FP8 (E4M3) forward on the tcgen05 kernel against the float64 oracle.

The scores are exact products of E4M3 values, so LSE is held to the usual
1e-4.  O goes through P rounded to E4M3, so every element of O is held to a
bound derived from that rounding: the oracle's fp8_p_rounding_sigma gives,
per element, the scale sigma of the error that rounding the weights of its
row to the E4M3 grid leaves in O (at any running-maximum factor the scale
is at most 2 sigma), and each element must lie within 7 x 2 sigma plus half
a bf16 unit of the oracle; the root mean square of error / sigma over all
checked elements must stay below 2.5 (an error twice the E4M3 scale would
fail it).  A second case makes every P exactly representable (integer
scores spanning <= 8 with scale ln 2, so P = 2^k with |k| <= 8) and holds O
to the bf16 bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_lse, check_out, f64, ulp
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

SIGMA_K = 7.0          # elementwise bound: SIGMA_K x (2 sigma) + half a bf16 unit
RMS_RATIO_MAX = 2.5    # root mean square of error / sigma over the checked elements


def _real(q8, k8, v8, dq, dk, dv):
    """Real inputs: decoded codes times the (batch, kv-head) factors."""
    q, k, v = (oracle.e4m3_decode(_codes(t)) for t in (q8, k8, v8))
    B, Hq, Hkv = q.shape[0], q.shape[2], k.shape[2]
    G = Hq // Hkv

    def fac(d, rep):
        if d is None:
            return 1.0
        return np.repeat(d.double().numpy().reshape(B, Hkv), rep, axis=1)[:, None, :, None]

    return q * fac(dq, G), k * fac(dk, 1), v * fac(dv, 1)


def check_fp8_rows(out, lse, real, b, h, rows, ratios, **kw):
    """O of the given rows of (b, h) elementwise within the E4M3 rounding
    bound, LSE within 1e-4; appends error / sigma to `ratios`."""
    o_r, l_r, sig = oracle.fp8_p_rounding_sigma(*real, b, h, rows, **kw)
    g = f64(out[b, rows, h])
    assert np.isfinite(g).all()
    err = np.abs(g - o_r)
    half_ulp = 0.5 * ulp(o_r, torch.bfloat16)
    tol = SIGMA_K * 2.0 * sig + half_ulp + 1e-6
    bad = err > tol
    assert not bad.any(), (f"O b{b} h{h}: {int(bad.sum())} elements outside the E4M3 bound; "
                           f"worst err/tol {float((err / tol).max()):.2f}")
    check_lse(lse[b, h, rows], l_r)
    ratios.append((np.maximum(err - half_ulp, 0.0) / np.maximum(sig, 1e-12)).ravel())


def check_rms_ratio(ratios):
    r = float(np.sqrt(np.mean(np.concatenate(ratios) ** 2)))
    assert r <= RMS_RATIO_MAX, f"RMS of error / sigma {r:.2f}"
    return r

# (B, Sq, Sk, Hq, Hkv, D, causal, window, softcap, with descales)
CASES = [
    (2, 300, 300, 4, 2, 128, True, (-1, -1), 0.0, True),
    (1, 200, 513, 4, 4, 128, False, (-1, -1), 0.0, False),
    (2, 129, 129, 8, 1, 128, True, (40, 0), 0.0, True),
    (1, 257, 257, 2, 2, 128, False, (-1, -1), 20.0, True),
    (1, 1024, 1024, 4, 2, 128, False, (64, 64), 0.0, True),
    (2, 300, 300, 4, 2, 64, True, (-1, -1), 0.0, True),
    (1, 200, 513, 4, 4, 64, False, (-1, -1), 0.0, False),
    (1, 257, 257, 2, 2, 64, False, (-1, -1), 20.0, True),
    (1, 700, 700, 4, 1, 64, True, (100, 0), 0.0, True),
    # more key tiles than the 5 K/V stages of head dim 64, ragged tail
    (1, 256, 1300, 2, 2, 64, False, (-1, -1), 0.0, True),
]


def _codes(t):
    return t.view(torch.uint8).numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dS%dx%dH%d-%dD%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "c" if c[6] else "", "w" if c[7] != (-1, -1) else ""))
def test_fp8_forward_vs_oracle(case):
    B, Sq, Sk, Hq, Hkv, D, causal, window, cap, desc = case
    q, k, v, dq, dk, dv = inputs.fp8_inputs(B, Sq, Sk, Hq, Hkv, D, seed=70)
    if not desc:
        dq = dk = dv = None
    dev = lambda t: None if t is None else t.cuda()
    out, lse = api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), dev(dq), dev(dk), dev(dv), causal=causal, window=window,
                              softcap=cap)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    real = _real(q, k, v, dq, dk, dv)
    # the whole-tensor definition and the per-row one agree (LSE of every row)
    npd = lambda t: None if t is None else t.double().numpy()
    _, l_all = oracle.attn_fwd_fp8(_codes(q), _codes(k), _codes(v), npd(dq), npd(dk), npd(dv), None, causal,
                                   window[0], window[1], cap)
    check_lse(lse, l_all)
    ratios = []
    for b in range(B):
        for h in range(Hq):
            check_fp8_rows(out, lse, real, b, h, np.arange(Sq), ratios, causal=causal, window_left=window[0],
                           window_right=window[1], softcap=cap)
    check_rms_ratio(ratios)


@pytest.mark.parametrize("D", [128, 64])
def test_fp8_exact_powers_of_two_match_to_bf16(D):
    # q one-hot in dim 0, k[:, :, :, 0] integers in [-4, 4]: raw scores are
    # those integers; scale ln 2 and dq * dk = 1 make P = 2^(score - max),
    # exact in E4M3, so O differs from the oracle by bf16 rounding only
    B, S, H = 2, 384, 4
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
    assert api.fa_last_device_status() == 0
    rng = np.random.default_rng(cfg["seed"])
    real = _real(q, k, v, dq, dk, dv)
    ratios = []
    for b, h in ((0, 0), (cfg["B"] - 1, cfg["Hq"] - 1), (1, 7)):
        rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 2048, cfg["Sq"] - 1],
                                         rng.integers(0, cfg["Sq"], 24)]))
        check_fp8_rows(out, lse, real, b, h, rows, ratios, causal=cfg["causal"])
    check_rms_ratio(ratios)


def test_fp8_refusals():
    q, k, v, *_ = inputs.fp8_inputs(1, 16, 16, 2, 2, 128, seed=72)
    with pytest.raises(_lib.FaError):  # the mma.sync kernel has no 8-bit path
        api.fa_set_fwd_kernel(1)
        try:
            api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda())
        finally:
            api.fa_set_fwd_kernel(0)
    q96, k96, v96, *_ = inputs.fp8_inputs(1, 16, 16, 2, 2, 96, seed=72)
    with pytest.raises(_lib.FaError):  # head dims other than 64 and 128
        api.fa_fwd_fp8(q96.cuda(), k96.cuda(), v96.cuda())
