"""ALiBi slopes (alibi_slopes): tcgen05 forward and backward against the
float64 oracle, per-head and per-batch-row slopes, with masks, windows,
softcap, GQA, strided views and the deterministic backward."""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_grad, check_lse, check_out, f64
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# (B, Sq, Sk, Hq, Hkv, D, dtype, causal, window, softcap, per-batch slopes)
CASES = [
    (2, 300, 300, 4, 2, 64, "bf16", True, (-1, -1), 0.0, False),
    (2, 200, 333, 4, 4, 128, "fp16", False, (-1, -1), 5.0, True),
    (1, 513, 513, 8, 1, 128, "bf16", True, (100, 0), 0.0, False),
    (2, 129, 129, 2, 2, 64, "fp16", False, (32, 16), 0.0, True),
    (1, 1000, 1000, 4, 2, 128, "bf16", False, (-1, -1), 30.0, False),
]


def _ids(c):
    return "B%dS%dx%dH%d-%dD%d%s%s%s%s" % (c[0], c[1], c[2], c[3], c[4], c[5], c[6], "c" if c[7] else "",
                                          "w" if c[8] != (-1, -1) else "", "pb" if c[10] else "")


def _slopes(case):
    B, Hq = case[0], case[3]
    return inputs.alibi_slopes(Hq, B, seed=50) if case[10] else inputs.alibi_slopes(Hq)


def _run(case, det=False, seed=51):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, _ = case
    q, k, v, do = inputs.attention_inputs(B, Sq, Sk, Hq, Hkv, D, dt, seed=seed)
    m = _slopes(case)
    kw = dict(causal=causal, window=window, softcap=cap, alibi_slopes=m.cuda())
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    dq, dk, dv = api.fa_bwd(dod, qd, kd, vd, out, lse, deterministic=det, **kw)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    return (q, k, v, do, m), (out, lse, dq, dk, dv)


def _oracle_args(case, q, k, v, m):
    B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, _ = case
    return (f64(q), f64(k), f64(v), 1.0 / math.sqrt(D), causal, window[0], window[1], cap), m.double().numpy()


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_alibi_fwd_bwd_vs_oracle(case):
    (q, k, v, do, m), (out, lse, dq, dk, dv) = _run(case)
    args, mn = _oracle_args(case, q, k, v, m)
    o_r, l_r = oracle.attn_fwd(*args, alibi_slopes=mn)
    check_out(out, o_r, DT[case[6]])
    check_lse(lse, l_r)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(f64(do), *args, alibi_slopes=mn)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


def test_alibi_deterministic_backward_repeats_and_matches():
    case = CASES[0]
    _, (_, _, dq1, dk1, dv1) = _run(case, det=True)
    (q, k, v, do, m), (_, _, dq2, dk2, dv2) = _run(case, det=True)
    for a, b in ((dq1, dq2), (dk1, dk2), (dv1, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    args, mn = _oracle_args(case, q, k, v, m)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(f64(do), *args, alibi_slopes=mn)
    check_grad(dq1, dq_r, "dQ")
    check_grad(dk1, dk_r, "dK")
    check_grad(dv1, dv_r, "dV")


def test_alibi_qkvpacked_view_equals_packed_tensors():
    B, S, H, D = 2, 257, 4, 128
    g = torch.Generator().manual_seed(52)
    qkv = torch.randn((B, S, 3, H, D), generator=g).to(torch.bfloat16).cuda()
    do = torch.randn((B, S, H, D), generator=g).to(torch.bfloat16).cuda()
    m = inputs.alibi_slopes(H).cuda()
    q, k, v = (t.contiguous() for t in qkv.unbind(2))
    o1, l1 = api.fa_fwd(q, k, v, causal=True, alibi_slopes=m)
    d1 = api.fa_bwd(do, q, k, v, o1, l1, causal=True, deterministic=True, alibi_slopes=m)
    o2, l2 = api.fa_fwd_qkvpacked(qkv, causal=True, alibi_slopes=m)
    dqkv = api.fa_bwd_qkvpacked(do, qkv, o2, l2, causal=True, deterministic=True, alibi_slopes=m)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(d1, dqkv.unbind(2)):
        assert torch.equal(a, b)


def test_alibi_sampled_rows_at_long_sequence():
    # one 8k causal problem: sampled rows against the row-wise oracle
    B, S, Hq, Hkv, D = 1, 8192, 8, 2, 128
    q, k, v, _ = inputs.attention_inputs(B, S, S, Hq, Hkv, D, "bf16", seed=53, with_dout=False)
    m = inputs.alibi_slopes(Hq)
    out, lse = api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), causal=True, alibi_slopes=m.cuda())
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 4095, 6000, 8191])
    qn, kn, vn = f64(q), f64(k), f64(v)
    for h in (0, 5):
        o_r, l_r = oracle.attn_fwd_rows(qn, kn, vn, 0, h, rows, None, True, alibi_slopes=m.double().numpy())
        check_out(out[0, rows, h], o_r, torch.bfloat16)
        check_lse(lse[0, h, rows], l_r)


def test_alibi_mma_kernel_is_refused():
    q, k, v, _ = inputs.attention_inputs(1, 16, 16, 2, 2, 64, "bf16", seed=54, with_dout=False)
    api.fa_set_fwd_kernel(1)
    try:
        with pytest.raises(_lib.FaError):
            api.fa_fwd(q.cuda(), k.cuda(), v.cuda(), alibi_slopes=inputs.alibi_slopes(2).cuda())
    finally:
        api.fa_set_fwd_kernel(0)
