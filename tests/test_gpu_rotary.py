"""Rotary position embedding in the kvcache call: new keys rotated into the
cache and queries rotated at cache_seqlens[b] + t, against the float64
oracle."""

import numpy as np
import pytest
import torch

import oracle
from _parity import check_lse, check_out, f64
from exact_attention_121_b200 import api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _tables(n_pos, half, base=10000.0):
    inv = base ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


CASES = [
    # B, Hq, Hkv, D, page, pages/seq, max_len, Sq, Snew, dtype, paged, rotary_dim, interleaved
    (3, 8, 2, 128, 16, 6, 90, 1, 1, "bf16", True, 128, False),
    (2, 4, 4, 64, 64, 3, 150, 2, 2, "fp16", True, 32, True),
    (3, 16, 4, 128, 64, 4, 200, 1, 1, "bf16", False, 64, False),
    (2, 6, 2, 128, 8, 40, 300, 5, 5, "fp16", True, 128, True),
]


@pytest.mark.parametrize("splits", [1, 0])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%d-%dD%d%s-r%d%s-Sq%d" % (
    c[0], c[1], c[2], c[3], "paged" if c[10] else "contig", c[11], "i" if c[12] else "h", c[7]))
def test_rotary_decode_vs_oracle(case, splits):
    B, Hq, Hkv, D, page, pps, max_len, Sq, Snew, dt, paged, rdim, inter = case
    d = inputs.kvcache_inputs(B, Hq, Hkv, D, page, pps, max_len, Sq=Sq, Snew=Snew, dtype=dt, seed=9, paged=paged,
                              min_len=0)
    cos, sin = _tables(max_len + Snew + 8, rdim // 2)
    q, kc, vc, kn, vn = (d[n].cuda() for n in ("q", "k_cache", "v_cache", "k_new", "v_new"))
    sl = d["cache_seqlens"].cuda()
    bt = d["block_table"].cuda() if d["block_table"] is not None else None
    out, lse = api.fa_fwd_kvcache(q, kc, vc, kn, vn, sl, bt, page_size=d["page_size"], causal=True,
                                  num_splits=splits, rotary_cos=torch.from_numpy(cos).cuda(),
                                  rotary_sin=torch.from_numpy(sin).cuda(), rotary_interleaved=inter)
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    bt_np = None if d["block_table"] is None else d["block_table"].numpy()
    sl_np = d["cache_seqlens"].numpy()
    o_r, l_r, kc_r, vc_r = oracle.attn_with_kvcache(
        d["q"].float().numpy(), d["k_cache"].float().numpy(), d["v_cache"].float().numpy(),
        d["k_new"].float().numpy(), d["v_new"].float().numpy(), sl_np, bt_np, d["page_size"],
        None, True, rotary_cos=cos, rotary_sin=sin, rotary_interleaved=inter)
    # values are appended as they are, rotated keys within one 16-bit rounding
    np.testing.assert_array_equal(f64(vc), vc_r)
    check_out(kc, kc_r, DT[dt], "K cache")
    check_out(out, o_r, DT[dt])
    # The cache holds 16-bit keys and the queries enter the product in the
    # 16-bit type, so the rotated q and k are rounded once to that type
    # before the attention; O and LSE are held to the oracle attending over
    # those rounded rows (the unrounded oracle moves LSE by ~1e-3 in bf16).
    rnd = lambda x: torch.from_numpy(x).to(DT[dt]).double().numpy()
    pos = sl_np[:, None] + np.arange(Sq)[None, :]
    q_rot = rnd(oracle.rotary(d["q"].float().numpy(), cos, sin, pos, inter))
    o_16, l_16, _, _ = oracle.attn_with_kvcache(q_rot, rnd(kc_r), vc_r, None, None, sl_np + Snew, bt_np,
                                                d["page_size"], None, True)
    check_out(out, o_16, DT[dt])
    check_lse(lse, l_16)


def test_rotary_position_outside_table_is_reported():
    d = inputs.kvcache_inputs(2, 4, 2, 64, 16, 4, 60, Sq=1, Snew=1, dtype="bf16", seed=10)
    cos, sin = _tables(8, 32)  # far fewer positions than the cached lengths
    q, kc, vc, kn, vn = (d[n].cuda() for n in ("q", "k_cache", "v_cache", "k_new", "v_new"))
    api.fa_fwd_kvcache(q, kc, vc, kn, vn, d["cache_seqlens"].cuda(), d["block_table"].cuda(),
                       page_size=d["page_size"], causal=True, rotary_cos=torch.from_numpy(cos).cuda(),
                       rotary_sin=torch.from_numpy(sin).cuda())
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 1  # FA_ERR_INVALID_ARG


def test_rotary_paged_decode_full_size():
    # the bench's paged-decode workload with full-width tables: every
    # sequence against the oracle on its gathered prefix plus the rotated
    # new token (rows rounded to bf16 as stored and multiplied)
    cfg = inputs.paged_decode_rotary_config()
    d = inputs.kvcache_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["page_size"], cfg["pages_per_seq"],
                              cfg["max_len"], Sq=1, Snew=1, dtype="bf16", seed=cfg["seed"])
    cos_t, sin_t = inputs.rotary_tables(cfg["max_len"] + 1, cfg["D"])
    q, kc, vc, kn, vn = (d[n].cuda() for n in ("q", "k_cache", "v_cache", "k_new", "v_new"))
    out, lse = api.fa_fwd_kvcache(q, kc, vc, kn, vn, d["cache_seqlens"].cuda(), d["block_table"].cuda(),
                                  page_size=cfg["page_size"], scale=cfg["scale"], causal=True,
                                  rotary_cos=cos_t.cuda(), rotary_sin=sin_t.cuda())
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    cos, sin = cos_t.numpy(), sin_t.numpy()
    rnd = lambda x: torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    bt = d["block_table"].numpy()
    kc_h, vc_h = d["k_cache"].float().numpy(), d["v_cache"].float().numpy()
    ps = cfg["page_size"]
    for b in range(cfg["B"]):
        L0 = int(d["cache_seqlens"][b])
        pos = np.array([[L0]])
        k_rot = oracle.rotary(d["k_new"][b:b + 1].float().numpy(), cos, sin, pos)[0]
        q_rot = rnd(oracle.rotary(d["q"][b:b + 1].float().numpy(), cos, sin, pos))
        K = np.concatenate([oracle.gather_cache(kc_h, b, L0, bt, ps), rnd(k_rot)])[None]
        V = np.concatenate([oracle.gather_cache(vc_h, b, L0, bt, ps), d["v_new"][b].float().numpy()])[None]
        o_r, l_r = oracle.attn_fwd(q_rot, K, V, cfg["scale"], True)
        check_out(out[b:b + 1], o_r, torch.bfloat16)
        check_lse(lse[b:b + 1], l_r)
        page, slot = bt[b, L0 // ps], L0 % ps
        assert torch.equal(vc[page, slot].cpu(), d["v_new"][b, 0])
        check_out(kc[page, slot], k_rot[0], torch.bfloat16, "rotated K slot")
