"""Run by test_gpu_debug_bounds.py in a child process: small cases of every
kernel through the bounds-checked build (libfa_debug.so), each checked for a
clean device status word and against the float64 oracle.  Prints one line
"bounds-checked build clean: N cases" on success; any failure raises."""

import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402
import torch  # noqa: E402

from exact_attention_121_b200 import _lib  # noqa: E402

_lib.LIB_PATH = os.path.join(os.path.dirname(_lib.LIB_PATH), "libfa_debug.so")

import oracle  # noqa: E402
from _parity import check_grad, check_lse, check_out, f64  # noqa: E402
from exact_attention_121_b200 import api, inputs  # noqa: E402

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}
n_cases = 0


def clean():
    torch.cuda.synchronize()
    st = api.fa_last_device_status()
    assert st == 0, f"device status {st} ({_lib.load().fa_status_string(st).decode()})"


def dense(B, Sq, Sk, Hq, Hkv, D, dt, causal, window, cap, det):
    global n_cases
    q, k, v, do = inputs.attention_inputs(B, Sq, Sk, Hq, Hkv, D, dt, seed=90)
    kw = dict(causal=causal, window=window, softcap=cap)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = api.fa_fwd(qd, kd, vd, **kw)
    dq, dk, dv = api.fa_bwd(dod, qd, kd, vd, out, lse, deterministic=det, **kw)
    clean()
    sc = 1 / math.sqrt(D)
    o_r, l_r = oracle.attn_fwd(f64(q), f64(k), f64(v), sc, causal, window[0], window[1], cap)
    check_out(out, o_r, DT[dt])
    check_lse(lse, l_r)
    g = oracle.attn_bwd(f64(do), f64(q), f64(k), f64(v), sc, causal, window[0], window[1], cap)
    for a, r, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(a, r, n)
    n_cases += 1


def varlen():
    global n_cases
    lens = [37, 130, 1, 200]
    q, k, v, do, cu_q, cu_k = inputs.varlen_inputs(lens, lens, 4, 2, 128, "bf16", seed=91)
    qd, kd, vd, dod, cq, ck = (t.cuda() for t in (q, k, v, do, cu_q, cu_k))
    out, lse = api.fa_fwd_varlen(qd, kd, vd, cq, ck, max(lens), max(lens), causal=True)
    dq, dk, dv = api.fa_bwd_varlen(dod, qd, kd, vd, out, lse, cq, ck, max(lens), max(lens), causal=True)
    clean()
    o_r, l_r = oracle.attn_fwd_varlen(f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(), None, True)
    check_out(out, o_r, torch.bfloat16)
    check_lse(lse, l_r)
    g = oracle.attn_bwd_varlen(f64(do), f64(q), f64(k), f64(v), cu_q.numpy(), cu_k.numpy(), None, True)
    for a, r, n in zip((dq, dk, dv), g, ("dQ", "dK", "dV")):
        check_grad(a, r, n)
    n_cases += 1


def qkvpacked():
    global n_cases
    B, S, H, D = 2, 150, 4, 64
    g = torch.Generator().manual_seed(92)
    qkv = torch.randn(B, S, 3, H, D, generator=g).to(torch.float16).cuda()
    do = torch.randn(B, S, H, D, generator=g).to(torch.float16).cuda()
    out, lse = api.fa_fwd_qkvpacked(qkv, causal=True)
    dqkv = api.fa_bwd_qkvpacked(do, qkv, out, lse, causal=True)
    clean()
    q, k, v = (f64(qkv[:, :, i]) for i in range(3))
    o_r, l_r = oracle.attn_fwd(q, k, v, 1 / math.sqrt(D), True)
    check_out(out, o_r, torch.float16)
    check_lse(lse, l_r)
    gr = oracle.attn_bwd(f64(do), q, k, v, 1 / math.sqrt(D), True)
    for i, n in enumerate(("dQ", "dK", "dV")):
        check_grad(dqkv[:, :, i], gr[i], n)
    n_cases += 1


def alibi():
    global n_cases
    B, S, H, D = 1, 200, 4, 128
    q, k, v, do = inputs.attention_inputs(B, S, S, H, H, D, "bf16", seed=93)
    sl = inputs.alibi_slopes(H)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out, lse = api.fa_fwd(qd, kd, vd, causal=True, alibi_slopes=sl.cuda())
    dq, dk, dv = api.fa_bwd(dod, qd, kd, vd, out, lse, causal=True, alibi_slopes=sl.cuda())
    clean()
    sc = 1 / math.sqrt(D)
    o_r, l_r = oracle.attn_fwd(f64(q), f64(k), f64(v), sc, True, alibi_slopes=sl.double().numpy())
    check_out(out, o_r, torch.bfloat16)
    check_lse(lse, l_r)
    g = oracle.attn_bwd(f64(do), f64(q), f64(k), f64(v), sc, True, alibi_slopes=sl.double().numpy())
    for a, r, n in zip((dq, dk, dv), g[:3], ("dQ", "dK", "dV")):
        check_grad(a, r, n)
    n_cases += 1


def fp8():
    global n_cases
    q, k, v, dq, dk, dv = inputs.fp8_inputs(1, 140, 140, 4, 2, 128, seed=94)
    out, lse = api.fa_fwd_fp8(q.cuda(), k.cuda(), v.cuda(), dq.cuda(), dk.cuda(), dv.cuda(), causal=True)
    clean()
    codes = lambda t: t.view(torch.uint8).numpy()
    _, l_r = oracle.attn_fwd_fp8(codes(q), codes(k), codes(v), dq.double().numpy(), dk.double().numpy(),
                                 dv.double().numpy(), None, True)
    check_lse(lse, l_r)
    n_cases += 1


def decode(page, paged, splits, Sq, Snew, rotary=False):
    global n_cases
    d = inputs.kvcache_inputs(3, 8, 2, 128, page, 400 // page + 2, 380, Sq=Sq, Snew=Snew, dtype="bf16", seed=95,
                              paged=paged, min_len=0)
    kw = {}
    if rotary:
        cos, sin = inputs.rotary_tables(800, 128)
        kw = dict(rotary_cos=cos.cuda(), rotary_sin=sin.cuda())
    cu = lambda t: None if t is None else t.cuda()
    out, lse = api.fa_fwd_kvcache(cu(d["q"]), cu(d["k_cache"]), cu(d["v_cache"]), cu(d["k_new"]), cu(d["v_new"]),
                                  cu(d["cache_seqlens"]), cu(d["block_table"]), page_size=page, causal=True,
                                  num_splits=splits, **kw)
    clean()
    if not rotary:
        bt = None if d["block_table"] is None else d["block_table"].numpy()
        o_r, l_r, _, _ = oracle.attn_with_kvcache(d["q"].float().numpy(), d["k_cache"].float().numpy(),
                                                  d["v_cache"].float().numpy(), d["k_new"].float().numpy(),
                                                  d["v_new"].float().numpy(), d["cache_seqlens"].numpy(), bt,
                                                  page, None, True)
        check_out(out, o_r, torch.bfloat16)
        check_lse(lse, l_r)
    n_cases += 1


def main():
    torch.cuda.set_device(0)
    assert _lib.load().fa_build_flags() & 1, "the bounds-checked build was not loaded"
    for det in (False, True):
        dense(1, 128, 128, 2, 2, 64, "fp16", False, (-1, -1), 0.0, det)
        dense(2, 512, 512, 16, 16, 64, "fp16", True, (-1, -1), 0.0, det)
        dense(2, 300, 200, 8, 2, 128, "bf16", True, (50, 0), 10.0, det)
        dense(1, 257, 257, 4, 1, 128, "bf16", False, (32, 16), 0.0, det)
    varlen()
    qkvpacked()
    alibi()
    fp8()
    for page, paged in ((256, True), (16, True), (48, True), (12, True), (64, False)):
        for splits in (1, 3, 0):
            decode(page, paged, splits, 1, 1)
    decode(16, True, 0, 3, 3)
    decode(256, True, 4, 1, 1, rotary=True)
    print(f"bounds-checked build clean: {n_cases} cases")


if __name__ == "__main__":
    main()
