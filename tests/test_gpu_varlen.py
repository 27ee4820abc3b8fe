"""Packed variable-length batches (cu_seqlens): CUDA forward and backward vs
the float64 oracle, every sequence attended on its own."""

import math

import numpy as np
import pytest
import torch

import oracle
from _parity import check_grad, check_lse, check_out, f64
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# (lens_q, lens_k, Hq, Hkv, D, dtype, causal, window, softcap, amp)
CASES = [
    ([77, 200, 1, 130], [77, 200, 1, 130], 4, 2, 64, "bf16", True, (-1, -1), 0.0, 1.0),
    ([5, 300, 64], [200, 300, 1], 4, 4, 128, "fp16", False, (-1, -1), 5.0, 2.0),
    ([0, 50, 129], [10, 0, 257], 2, 1, 128, "bf16", False, (32, 16), 0.0, 1.0),
    ([1000, 3, 300], [1000, 3, 300], 4, 1, 64, "fp16", True, (100, 0), 0.0, 1.0),
    ([256, 256, 513], [128, 640, 513], 8, 2, 128, "bf16", True, (-1, -1), 5.0, 1.0),
]
# N(0,1) inputs as in the pages' workloads.  With inputs scaled by 2, a causal
# row that sees only two or three keys can miss the bf16 bound by one element
# in a million (the 16-bit rounding of two comparable probabilities does not
# cancel, and |V0 - V1| reaches ~12): a property of 16-bit P, not of packing.


def _ids(c):
    return "Lq%s-Lk%s-H%d-%dD%d%s%s" % ("_".join(map(str, c[0])), "_".join(map(str, c[1])), c[2], c[3], c[4],
                                         c[5], "c" if c[6] else "")


def _run(case, det=False, seed=31):
    lq, lk, Hq, Hkv, D, dt, causal, window, cap, amp = case
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs(lq, lk, Hq, Hkv, D, dt, seed=seed, amp=amp)
    kw = dict(causal=causal, window=window, softcap=cap)
    qd, kd, vd, dod, cqd, ckd = (t.cuda() for t in (q, k, v, do, cu_q, cu_k))
    out, lse = api.fa_fwd_varlen(qd, kd, vd, cqd, ckd, max(lq), max(lk), **kw)
    dq, dk, dv = api.fa_bwd_varlen(dod, qd, kd, vd, out, lse, cqd, ckd, max(lq), max(lk), deterministic=det, **kw)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    return (q, k, v, do, cu_q, cu_k, kw), (out, lse, dq, dk, dv)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_varlen_fwd_bwd_vs_oracle(case):
    (q, k, v, do, cu_q, cu_k, kw), (out, lse, dq, dk, dv) = _run(case)
    D = q.shape[-1]
    sc = 1.0 / math.sqrt(D)
    args = (f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(), sc, kw["causal"], kw["window"][0],
            kw["window"][1], kw["softcap"])
    o_r, l_r = oracle.attn_fwd_varlen(*args)
    check_out(out, o_r, DT[case[5]])
    check_lse(lse, l_r)
    dq_r, dk_r, dv_r = oracle.attn_bwd_varlen(f64(do), *args)
    check_grad(dq, dq_r, "dQ")
    check_grad(dk, dk_r, "dK")
    check_grad(dv, dv_r, "dV")


@pytest.mark.parametrize("case", CASES[:3], ids=_ids)
def test_varlen_deterministic_matches_and_repeats(case):
    _, (o1, l1, dq1, dk1, dv1) = _run(case, det=True)
    _, (o2, l2, dq2, dk2, dv2) = _run(case, det=True)
    for a, b in ((dq1, dq2), (dk1, dk2), (dv1, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    (q, k, v, do, cu_q, cu_k, kw), _ = _run(case)
    sc = 1.0 / math.sqrt(q.shape[-1])
    dq_r, dk_r, dv_r = oracle.attn_bwd_varlen(f64(do), f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(), sc,
                                              kw["causal"], kw["window"][0], kw["window"][1], kw["softcap"])
    check_grad(dq1, dq_r, "dQ")
    check_grad(dk1, dk_r, "dK")
    check_grad(dv1, dv_r, "dV")


def test_varlen_equals_dense_batch():
    # equal lengths: the packed call equals the dense call bit for bit
    B, S, H, D = 3, 300, 4, 128
    q, k, v, do = inputs.attention_inputs(B, S, S, H, H, D, "bf16", seed=33)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = api.fa_fwd(qd, kd, vd, causal=True)
    dq, dk, dv = api.fa_bwd(dod, qd, kd, vd, out, lse, causal=True, deterministic=True)
    cu = torch.arange(B + 1, dtype=torch.int32, device="cuda") * S
    flat = lambda t: t.reshape(B * S, H, D)
    out_v, lse_v = api.fa_fwd_varlen(flat(qd), flat(kd), flat(vd), cu, cu, S, S, causal=True)
    dq_v, dk_v, dv_v = api.fa_bwd_varlen(flat(dod), flat(qd), flat(kd), flat(vd), out_v, lse_v, cu, cu, S, S,
                                         causal=True, deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(out_v, flat(out))
    assert torch.equal(lse_v, lse.permute(1, 0, 2).reshape(H, B * S))
    for a, b in ((dq_v, dq), (dk_v, dk), (dv_v, dv)):
        assert torch.equal(a, flat(b))


def test_varlen_training_mix_forward_and_sampled_backward():
    cfg = inputs.varlen_config()
    lens = cfg["lens"]
    case = (lens, lens, cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["dtype"], cfg["causal"], cfg["window"],
            cfg["softcap"], cfg["amp"])
    (q, k, v, do, cu_q, cu_k, kw), (out, lse, dq, dk, dv) = _run(case, seed=cfg["seed"])
    sc = cfg["scale"]
    cq = cu_q.numpy()
    # forward: every sequence; backward: three sequences (gradients of a
    # sequence depend on that sequence only)
    o_r, l_r = oracle.attn_fwd_varlen(f64(q), f64(k), f64(v), cq, cq, sc, True)
    check_out(out, o_r, torch.bfloat16)
    check_lse(lse, l_r)
    for b in (0, len(lens) // 2, len(lens) - 1):
        s0, s1 = int(cq[b]), int(cq[b + 1])
        g = oracle.attn_bwd(f64(do)[None, s0:s1], f64(q)[None, s0:s1], f64(k)[None, s0:s1], f64(v)[None, s0:s1],
                            sc, True)
        check_grad(dq[s0:s1], g[0][0], "dQ")
        check_grad(dk[s0:s1], g[1][0], "dK")
        check_grad(dv[s0:s1], g[2][0], "dV")


def test_varlen_bad_offsets_are_clamped_and_reported():
    # cu_seqlens_q ends past total_q: the kernel clamps (no access leaves the
    # tensors) and records FA_ERR_INVALID_ARG in the status word
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs([64, 64], [64, 64], 2, 2, 64, "bf16", seed=34)
    bad = cu_q.clone()
    bad[-1] = 200
    qd, kd, vd, cqd, ckd = (t.cuda() for t in (q, k, v, bad, cu_k))
    api.fa_fwd_varlen(qd, kd, vd, cqd, ckd, 136, 64)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 1  # FA_ERR_INVALID_ARG
    # the status word is cleared by the read; a good call reports 0
    api.fa_fwd_varlen(qd, kd, vd, cu_q.cuda(), ckd, 64, 64)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0


def test_varlen_mma_kernel_is_refused():
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs([16], [16], 2, 2, 64, "bf16", seed=35)
    api.fa_set_fwd_kernel(1)
    try:
        with pytest.raises(_lib.FaError):
            api.fa_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cu_q.cuda(), cu_k.cuda(), 16, 16)
    finally:
        api.fa_set_fwd_kernel(0)
