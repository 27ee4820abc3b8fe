"""Tensors with arbitrary layouts (head dimension contiguous): the pages'
qkvpacked variant and a (B, H, S, D) layout, against the float64 oracle and
bit for bit against the same call on packed copies."""

import math

import pytest
import torch

import oracle
from _parity import check_grad, check_lse, check_out, f64
from exact_attention_121_b200 import api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


@pytest.mark.parametrize("B,S,H,D,dt,causal", [(2, 300, 4, 64, "bf16", True), (1, 257, 2, 128, "fp16", False),
                                               (2, 512, 8, 128, "bf16", True)])
def test_qkvpacked_vs_oracle(B, S, H, D, dt, causal):
    q, k, v, do = inputs.attention_inputs(B, S, S, H, H, D, dt, seed=51)
    qkv = torch.stack([q, k, v], dim=2).cuda()  # (B, S, 3, H, D)
    out, lse = api.fa_fwd_qkvpacked(qkv, causal=causal)
    dqkv = api.fa_bwd_qkvpacked(do.cuda(), qkv, out, lse, causal=causal)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    sc = 1.0 / math.sqrt(D)
    o_r, l_r = oracle.attn_fwd(f64(q), f64(k), f64(v), sc, causal)
    check_out(out, o_r, DT[dt])
    check_lse(lse, l_r)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(f64(do), f64(q), f64(k), f64(v), sc, causal)
    check_grad(dqkv[:, :, 0], dq_r, "dQ")
    check_grad(dqkv[:, :, 1], dk_r, "dK")
    check_grad(dqkv[:, :, 2], dv_r, "dV")


@pytest.mark.parametrize("layout", ["qkvpacked", "bhsd"])
def test_strided_equals_packed_bit_for_bit(layout):
    B, S, Hq, Hkv, D = 2, 384, 8, 2, 128
    q, k, v, do = inputs.attention_inputs(B, S, S, Hq, Hkv, D, "bf16", seed=52)
    if layout == "qkvpacked":
        # GQA: q heads and kv heads packed side by side in one tensor
        buf = torch.cat([q, k, v], dim=2).cuda()  # (B, S, Hq + 2 Hkv, D)
        qs, ks, vs = buf[:, :, :Hq], buf[:, :, Hq:Hq + Hkv], buf[:, :, Hq + Hkv:]
    else:
        qs, ks, vs = (t.cuda().transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v))
    assert not qs.is_contiguous()
    kw = dict(causal=True, window=(100, 0), softcap=20.0)
    out_s, lse_s = api.fa_fwd(qs, ks, vs, **kw)
    dq_s, dk_s, dv_s = api.fa_bwd(do.cuda(), qs, ks, vs, out_s, lse_s, deterministic=True, **kw)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    out_c, lse_c = api.fa_fwd(qc, kc, vc, **kw)
    dq_c, dk_c, dv_c = api.fa_bwd(do.cuda(), qc, kc, vc, out_c, lse_c, deterministic=True, **kw)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    assert torch.equal(out_s, out_c) and torch.equal(lse_s, lse_c)
    assert torch.equal(dq_s, dq_c) and torch.equal(dk_s, dk_c) and torch.equal(dv_s, dv_c)


def test_strided_outputs_write_only_their_view():
    # dq, dk, dv as views of one buffer with a guard head between them: the
    # guard values are untouched
    B, S, H, D = 1, 200, 2, 64
    q, k, v, do = inputs.attention_inputs(B, S, S, H, H, D, "bf16", seed=53)
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    out, lse = api.fa_fwd(qc, kc, vc, causal=True)
    buf = torch.full((B, S, 4 * H, D), 7.0, dtype=torch.bfloat16, device="cuda")
    dq, dk, dv = buf[:, :, 0:H], buf[:, :, H + 1:2 * H + 1], buf[:, :, 3 * H - 1:4 * H - 1]
    api.fa_bwd(doc, qc, kc, vc, out, lse, dq=dq, dk=dk, dv=dv, causal=True)
    ref = api.fa_bwd(doc, qc, kc, vc, out, lse, causal=True, deterministic=False)
    torch.cuda.synchronize()
    assert torch.all(buf[:, :, H] == 7.0) and torch.all(buf[:, :, 4 * H - 1] == 7.0)
    for a, b, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
        check_grad(a, f64(b), name)
