"""Paged KV-cache decode parity: append then attend, split-KV + combine, vs the
float64 oracle; the appended cache slots are checked bit for bit."""

import numpy as np
import pytest
import torch

import oracle
from _parity import check_lse, check_out, f64
from exact_attention_121_b200 import api, inputs

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _run_case(d, num_splits, causal=True, window=(-1, -1), softcap=0.0, scale=None):
    q, kc, vc = d["q"].cuda(), d["k_cache"].cuda(), d["v_cache"].cuda()
    kn = d["k_new"].cuda() if d["k_new"] is not None else None
    vn = d["v_new"].cuda() if d["v_new"] is not None else None
    sl = d["cache_seqlens"].cuda()
    bt = d["block_table"].cuda() if d["block_table"] is not None else None
    out, lse = api.fa_fwd_kvcache(q, kc, vc, kn, vn, sl, bt, page_size=d["page_size"], scale=scale,
                                  causal=causal, window=window, softcap=softcap, num_splits=num_splits)
    torch.cuda.synchronize()
    status = api.fa_last_device_status()
    return out, lse, kc, vc, status


def _oracle(d, causal=True, window=(-1, -1), softcap=0.0, scale=None):
    bt = None if d["block_table"] is None else d["block_table"].numpy()
    kn = None if d["k_new"] is None else d["k_new"].float().numpy()
    vn = None if d["v_new"] is None else d["v_new"].float().numpy()
    return oracle.attn_with_kvcache(d["q"].float().numpy(), d["k_cache"].float().numpy(),
                                    d["v_cache"].float().numpy(), kn, vn, d["cache_seqlens"].numpy(), bt,
                                    d["page_size"], scale, causal, window[0], window[1], softcap)


SMALL = [
    # B, Hq, Hkv, D, page, pages/seq, max_len, Sq, Snew, dtype, paged, seqlens
    (3, 8, 2, 128, 16, 6, 90, 1, 1, "bf16", True, [0, 37, 95]),
    (2, 4, 4, 64, 64, 3, 150, 2, 2, "fp16", True, None),
    (4, 32, 8, 128, 256, 3, 700, 1, 1, "bf16", True, None),
    (2, 8, 1, 64, 32, 5, 140, 3, 0, "fp16", True, [40, 159]),
    (3, 16, 4, 128, 64, 4, 200, 1, 1, "bf16", False, None),
    (2, 6, 2, 128, 8, 40, 300, 5, 5, "bf16", True, None),           # 15 packed rows per kv-head
    (1, 20, 1, 64, 16, 8, 100, 2, 1, "fp16", True, None),           # 40 packed rows: 3 row tiles
    (2, 8, 2, 128, 48, 4, 180, 3, 3, "bf16", True, [46, 142]),      # 16-row boxes; new rows cross a page
    (2, 8, 2, 64, 24, 6, 130, 2, 2, "fp16", True, [23, 100]),       # 8-row boxes; new rows cross a page
    (2, 4, 2, 128, 12, 10, 100, 1, 1, "bf16", True, None),          # 12-token pages: cp.async kernel
]


@pytest.mark.parametrize("splits", [1, 3, 8, 0])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B%dH%d-%dD%dp%d%s%s" % (
    c[0], c[1], c[2], c[3], c[4], "paged" if c[10] else "contig", "Sq%dn%d" % (c[7], c[8])))
def test_decode_small(case, splits):
    B, Hq, Hkv, D, page, pps, max_len, Sq, Snew, dt, paged, seqlens = case
    d = inputs.kvcache_inputs(B, Hq, Hkv, D, page, pps, max_len, Sq=Sq, Snew=Snew, dtype=dt, seed=7,
                              paged=paged, min_len=0, seqlens=seqlens)
    out, lse, kc, vc, status = _run_case(d, splits)
    assert status == 0
    o_r, l_r, kc_r, vc_r = _oracle(d)
    check_out(out, o_r, DT[dt])
    check_lse(lse, l_r)
    np.testing.assert_array_equal(f64(kc), kc_r)
    np.testing.assert_array_equal(f64(vc), vc_r)


@pytest.mark.parametrize("page,launches", [(16, 2), (64, 2), (256, 2), (12, 3)])
def test_decode_call_launches(page, launches):
    """With TMA-friendly pages the split kernel appends the new rows itself
    (split + combine: two kernels); other page sizes take separate append,
    split and combine kernels."""
    from exact_attention_121_b200 import _lib
    d = inputs.kvcache_inputs(2, 8, 2, 128, page, 512 // page + 1, 500, Sq=1, Snew=1, dtype="bf16", seed=12)
    out, lse, kc, vc, status = _run_case(d, 4)
    assert status == 0
    assert _lib.load().fa_last_launch_count() == launches
    o_r, l_r, kc_r, vc_r = _oracle(d)
    check_out(out, o_r, torch.bfloat16)
    check_lse(lse, l_r)
    np.testing.assert_array_equal(f64(kc), kc_r)


@pytest.mark.parametrize("kw", [dict(window=(20, 0)), dict(softcap=3.0, scale=0.2), dict(causal=False)])
def test_decode_masks_and_softcap(kw):
    d = inputs.kvcache_inputs(2, 8, 2, 128, 16, 8, 120, Sq=3, Snew=2, dtype="bf16", seed=8)
    out, lse, _, _, status = _run_case(d, 4, **kw)
    assert status == 0
    o_r, l_r, _, _ = _oracle(d, **kw)
    check_out(out, o_r, torch.bfloat16)
    check_lse(lse, l_r)


@pytest.mark.parametrize("splits", [1, 4, 16, 0])
def test_paged_decode_full_size(splits):
    cfg = inputs.paged_decode_config()
    d = inputs.kvcache_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["page_size"], cfg["pages_per_seq"],
                              cfg["max_len"], Sq=1, Snew=1, dtype="bf16", seed=cfg["seed"])
    out, lse, kc, vc, status = _run_case(d, splits, causal=True)
    assert status == 0
    # oracle on the gathered valid prefix of every sequence
    bt = d["block_table"].numpy()
    kc_h = d["k_cache"].float().numpy()
    vc_h = d["v_cache"].float().numpy()
    seqlens = d["cache_seqlens"].numpy()
    ps = cfg["page_size"]
    for b in range(cfg["B"]):
        L0 = int(seqlens[b])
        K = oracle.gather_cache(kc_h, b, L0, bt, ps)
        V = oracle.gather_cache(vc_h, b, L0, bt, ps)
        K = np.concatenate([K, d["k_new"][b].float().numpy()])[None]
        V = np.concatenate([V, d["v_new"][b].float().numpy()])[None]
        o_r, l_r = oracle.attn_fwd(d["q"][b:b + 1].float().numpy(), K, V, cfg["scale"], True)
        check_out(out[b:b + 1], o_r, torch.bfloat16)
        check_lse(lse[b:b + 1], l_r)
        # the appended token landed in its page slot, bit for bit
        pos = L0
        page, slot = bt[b, pos // ps], pos % ps
        assert torch.equal(kc[page, slot].cpu(), d["k_new"][b, 0])
        assert torch.equal(vc[page, slot].cpu(), d["v_new"][b, 0])


def test_decode_overflow_is_reported_not_faulted():
    d = inputs.kvcache_inputs(2, 4, 2, 64, 16, 2, 10, Sq=1, Snew=1, dtype="bf16", seed=9, seqlens=[5, 32])
    out, lse, _, _, status = _run_case(d, 2)
    assert status == 1  # FA_ERR_INVALID_ARG recorded on the device for sequence 1
    o_r, l_r, _, _ = _oracle(dict(d, cache_seqlens=torch.tensor([5, 0], dtype=torch.int32),
                                  k_new=d["k_new"][:1], v_new=d["v_new"][:1], q=d["q"][:1],
                                  block_table=d["block_table"][:1]))
    check_out(out[:1], o_r, torch.bfloat16)
    assert (out[1] == 0).all()


def test_decode_bad_page_id_is_reported():
    d = inputs.kvcache_inputs(1, 4, 2, 64, 16, 2, 20, Sq=1, Snew=0, dtype="bf16", seed=10, seqlens=[20])
    d["block_table"] = torch.tensor([[0, 99]], dtype=torch.int32)
    _, _, _, _, status = _run_case(d, 1)
    assert status == 1


def test_bounded_wait_times_out_and_context_survives():
    from exact_attention_121_b200 import _lib
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib = _lib.load()
    code = lib.fa_selftest_bounded_wait(flag.data_ptr(), 1, 50_000_000, torch.cuda.current_stream().cuda_stream)
    assert code == 0
    assert api.fa_last_device_status() == 4  # FA_ERR_TIMEOUT, and the status word is cleared
    assert api.fa_last_device_status() == 0
    flag.fill_(1)
    lib.fa_selftest_bounded_wait(flag.data_ptr(), 1, 50_000_000, torch.cuda.current_stream().cuda_stream)
    assert api.fa_last_device_status() == 0
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0
