"""Pins for the float64 oracle, against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a closed form, a
brute-force index rule, an invariant of the method (online softmax, GQA as
repeated KV, paging, splits) or central finite differences.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attn64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")

_NS = {"ln": math.log, "tanh": math.tanh, "atanh": math.atanh, "sqrt": math.sqrt,
       "inf": math.inf, "__builtins__": {}}


def _ev(x):
    if isinstance(x, list):
        return [_ev(e) for e in x]
    return float(eval(x, _NS))  # expressions are fixture text: numbers, ln, tanh, atanh


def _arr(x):
    return np.array(_ev(x), dtype=np.float64)


def _load():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand(shape, rng, amp=1.0):
    return amp * rng.standard_normal(shape)


# ---------------------------------------------------------------------------
# hand-derived closed forms (tests/golden/hand_examples.json)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("ex", _load()["examples"], ids=lambda e: e["name"])
def test_hand_examples_forward(ex):
    q, k, v = _arr(ex["q"]), _arr(ex["k"]), _arr(ex["v"])
    extra = {"alibi_slopes": _arr(ex["alibi_slopes"])} if "alibi_slopes" in ex else {}
    o, lse = oracle.attn_fwd(q, k, v, scale=_ev(ex["scale"]), causal=ex["causal"],
                             window_left=ex["window"][0], window_right=ex["window"][1],
                             softcap=_ev(ex["softcap"]), **extra)
    np.testing.assert_allclose(o, _arr(ex["out"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, _arr(ex["lse"]), rtol=0, atol=1e-13)


@pytest.mark.parametrize("ex", _load()["backward"], ids=lambda e: e["name"])
def test_hand_examples_backward(ex):
    q, k, v, do = _arr(ex["q"]), _arr(ex["k"]), _arr(ex["v"]), _arr(ex["dout"])
    kw = dict(scale=_ev(ex["scale"]), causal=ex["causal"], window_left=ex["window"][0],
              window_right=ex["window"][1], softcap=_ev(ex["softcap"]))
    o, _ = oracle.attn_fwd(q, k, v, **kw)
    np.testing.assert_allclose(o, _arr(ex["out"]), atol=1e-13)
    dq, dk, dv, delta = oracle.attn_bwd(do, q, k, v, **kw)
    np.testing.assert_allclose(dq, _arr(ex["dq"]), atol=1e-13)
    np.testing.assert_allclose(dk, _arr(ex["dk"]), atol=1e-13)
    np.testing.assert_allclose(dv, _arr(ex["dv"]), atol=1e-13)
    np.testing.assert_allclose(delta, _arr(ex["delta"]), atol=1e-13)


@pytest.mark.parametrize("ex", _load()["kvcache"], ids=lambda e: e["name"])
def test_hand_examples_kvcache(ex):
    o, lse, kc, vc = oracle.attn_with_kvcache(
        _arr(ex["q"]), _arr(ex["k_cache"]), _arr(ex["v_cache"]), _arr(ex["k_new"]),
        _arr(ex["v_new"]), np.array(ex["cache_seqlens"]), np.array(ex["block_table"]),
        ex["page_size"], scale=_ev(ex["scale"]), causal=ex["causal"])
    np.testing.assert_allclose(o, _arr(ex["out"]), atol=1e-13)
    np.testing.assert_allclose(lse, _arr(ex["lse"]), atol=1e-13)
    np.testing.assert_array_equal(vc, _arr(ex["v_cache_after"]))


# ---------------------------------------------------------------------------
# softmax rows, masks
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal,wl,wr,cap", [(False, -1, -1, 0.0), (True, -1, -1, 0.0),
                                              (True, 5, 0, 3.0), (False, 3, 2, 0.0)])
def test_probability_rows(causal, wl, wr, cap):
    rng = np.random.default_rng(0)
    q, k, v = _rand((2, 13, 4, 8), rng), _rand((2, 13, 2, 8), rng), _rand((2, 13, 2, 8), rng)
    _, lse, P, _ = oracle.attn_fwd(q, k, v, 0.3, causal, wl, wr, cap, return_probs=True)
    vis = attn64.visible(13, 13, causal, wl, wr)
    assert (P >= 0).all()
    assert (P[..., ~vis] == 0).all()
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    assert np.isfinite(lse).all()


def _brute_visible(Sq, Sk, causal, wl, wr):
    """Index rule written out element by element, independent of numpy masks."""
    off = Sk - Sq
    out = set()
    for i in range(Sq):
        for j in range(Sk):
            lo = -10**9 if wl < 0 else i + off - wl
            hi = 10**9 if wr < 0 else i + off + wr
            if causal:
                hi = min(hi, i + off)
            if lo <= j <= hi:
                out.add((i, j))
    return out


@pytest.mark.parametrize("Sq,Sk", [(7, 7), (3, 9), (9, 3), (1, 5)])
@pytest.mark.parametrize("causal,wl,wr", [(False, -1, -1), (True, -1, -1), (False, 2, 0),
                                          (False, 1, 3), (True, 4, 5), (False, 0, 0),
                                          (False, 100, 100)])
def test_visible_matches_brute_force(Sq, Sk, causal, wl, wr):
    m = attn64.visible(Sq, Sk, causal, wl, wr)
    got = {(i, j) for i in range(Sq) for j in range(Sk) if m[i, j]}
    assert got == _brute_visible(Sq, Sk, causal, wl, wr)


def test_window_special_cases():
    S = 11
    none = attn64.visible(S, S)
    assert none.all()
    np.testing.assert_array_equal(attn64.visible(S, S, False, -1, -1), none)
    np.testing.assert_array_equal(attn64.visible(S, S, False, S, S), none)
    np.testing.assert_array_equal(attn64.visible(S, S, True), attn64.visible(S, S, False, -1, 0))
    np.testing.assert_array_equal(attn64.visible(S, S, True), np.tril(np.ones((S, S), bool)))


# ---------------------------------------------------------------------------
# online softmax == two-pass
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("block", [16, 32, 128])
@pytest.mark.parametrize("causal,wl,wr,cap", [(False, -1, -1, 0.0), (True, -1, -1, 0.0),
                                              (True, 20, 0, 5.0), (False, 7, 9, 0.0)])
def test_online_softmax_equals_two_pass(block, causal, wl, wr, cap):
    rng = np.random.default_rng(1)
    q = _rand((2, 40, 4, 16), rng, 2.0)
    k = _rand((2, 77, 2, 16), rng, 2.0)
    v = _rand((2, 77, 2, 16), rng)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.25, causal, wl, wr, cap)
    o2, l2 = oracle.attn_fwd_online(q, k, v, 0.25, causal, wl, wr, cap, block=block)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    fin = np.isfinite(l1)
    np.testing.assert_array_equal(fin, np.isfinite(l2))
    np.testing.assert_allclose(l2[fin], l1[fin], rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# special cases with closed forms
# ---------------------------------------------------------------------------

def test_single_key():
    rng = np.random.default_rng(2)
    q, k, v = _rand((1, 5, 2, 8), rng), _rand((1, 1, 2, 8), rng), _rand((1, 1, 2, 8), rng)
    o, lse = oracle.attn_fwd(q, k, v, 0.7)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-14)
    s00 = 0.7 * np.einsum("bihd,bjhd->bhi", q, k)
    np.testing.assert_allclose(lse, s00, atol=1e-14)


def test_identical_keys_give_uniform_weights():
    rng = np.random.default_rng(3)
    n = 9
    q = _rand((1, 4, 1, 8), rng)
    k = np.repeat(_rand((1, 1, 1, 8), rng), n, axis=1)
    v = _rand((1, n, 1, 8), rng)
    o, lse = oracle.attn_fwd(q, k, v, 0.5)
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (4, 8)), atol=1e-14)
    s = 0.5 * (q[0, :, 0] @ k[0, 0, 0])
    np.testing.assert_allclose(lse[0, 0], s + math.log(n), atol=1e-13)


def test_zero_query_is_uniform():
    rng = np.random.default_rng(4)
    k, v = _rand((1, 6, 1, 4), rng), _rand((1, 6, 1, 4), rng)
    o, lse = oracle.attn_fwd(np.zeros((1, 2, 1, 4)), k, v, 1.0)
    np.testing.assert_allclose(o[0, 0, 0], v[0, :, 0].mean(0), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(6), atol=1e-14)


def test_softcap_limit_and_bound():
    rng = np.random.default_rng(5)
    q, k, v = _rand((1, 6, 2, 8), rng), _rand((1, 6, 2, 8), rng), _rand((1, 6, 2, 8), rng)
    o0, l0, _, U = oracle.attn_fwd(q, k, v, 0.5, return_probs=True)
    c = 1e4
    o1, l1 = oracle.attn_fwd(q, k, v, 0.5, softcap=c)
    # c*tanh(u/c) = u - u^3/(3c^2) + ...: scores move by at most max|u|^3/(3c^2)
    bound = np.abs(U).max() ** 3 / (3 * c * c)
    np.testing.assert_allclose(l1, l0, atol=4 * bound + 1e-14)
    assert not np.allclose(oracle.attn_fwd(q, k, v, 0.5, softcap=0.5)[0], o0, atol=1e-3)
    # capped scores stay inside [-c, c]
    _, _, P, _ = oracle.attn_fwd(q * 50, k, v, 1.0, softcap=2.0, return_probs=True)
    assert np.isfinite(P).all()


def test_fully_masked_rows():
    rng = np.random.default_rng(6)
    q, k, v = _rand((1, 5, 1, 4), rng), _rand((1, 3, 1, 4), rng), _rand((1, 3, 1, 4), rng)
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=True)   # Sq > Sk: first 2 rows see nothing
    assert np.isneginf(lse[0, 0, :2]).all() and np.isfinite(lse[0, 0, 2:]).all()
    np.testing.assert_array_equal(o[0, :2], 0.0)
    o2, l2 = oracle.attn_fwd_online(q, k, v, 1.0, causal=True, block=2)
    np.testing.assert_allclose(o2, o, atol=1e-13)


def test_gqa_requires_integer_multiple():
    with pytest.raises(ValueError):
        oracle.attn_fwd(np.zeros((1, 2, 3, 4)), np.zeros((1, 2, 2, 4)), np.zeros((1, 2, 2, 4)))


# ---------------------------------------------------------------------------
# GQA == MHA on repeated K/V (forward and backward)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("Hq,Hkv", [(4, 1), (8, 2), (6, 3)])
def test_gqa_equals_repeated_kv(Hq, Hkv):
    rng = np.random.default_rng(7)
    G = Hq // Hkv
    q, do = _rand((2, 9, Hq, 8), rng), _rand((2, 9, Hq, 8), rng)
    k, v = _rand((2, 11, Hkv, 8), rng), _rand((2, 11, Hkv, 8), rng)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    kw = dict(scale=0.4, causal=True, window_left=5, window_right=0, softcap=2.0)
    o, l = oracle.attn_fwd(q, k, v, **kw)
    o_r, l_r = oracle.attn_fwd(q, kr, vr, **kw)
    np.testing.assert_allclose(o, o_r, atol=1e-14)
    np.testing.assert_allclose(l, l_r, atol=1e-14)
    dq, dk, dv, _ = oracle.attn_bwd(do, q, k, v, **kw)
    dq_r, dk_r, dv_r, _ = oracle.attn_bwd(do, q, kr, vr, **kw)
    np.testing.assert_allclose(dq, dq_r, atol=1e-13)
    np.testing.assert_allclose(dk, dk_r.reshape(2, 11, Hkv, G, 8).sum(3), atol=1e-13)
    np.testing.assert_allclose(dv, dv_r.reshape(2, 11, Hkv, G, 8).sum(3), atol=1e-13)


# ---------------------------------------------------------------------------
# gradients: central finite differences
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("S", [3, 5])
@pytest.mark.parametrize("causal,wl,wr,cap", [(False, -1, -1, 0.0), (True, -1, -1, 0.0),
                                              (False, 1, 1, 0.0), (True, 2, 0, 1.5)])
def test_gradients_match_finite_differences(S, causal, wl, wr, cap):
    rng = np.random.default_rng(10 + S)
    q, k, v = _rand((1, S, 2, 4), rng), _rand((1, S, 1, 4), rng), _rand((1, S, 1, 4), rng)
    do = _rand((1, S, 2, 4), rng)
    kw = dict(scale=0.6, causal=causal, window_left=wl, window_right=wr, softcap=cap)

    def loss(qq, kk, vv):
        return float((oracle.attn_fwd(qq, kk, vv, **kw)[0] * do).sum())

    dq, dk, dv, _ = oracle.attn_bwd(do, q, k, v, **kw)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if x is t else t for t in (q, k, v)]
            args_m = [xm if x is t else t for t in (q, k, v)]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert err <= 1e-6, err


def test_delta_identity():
    rng = np.random.default_rng(20)
    q, k, v = _rand((2, 7, 4, 8), rng), _rand((2, 7, 2, 8), rng), _rand((2, 7, 2, 8), rng)
    do = _rand((2, 7, 4, 8), rng)
    o, _ = oracle.attn_fwd(q, k, v, 0.3, True, 3, 0, 2.0)
    _, _, _, delta = oracle.attn_bwd(do, q, k, v, 0.3, True, 3, 0, 2.0)
    np.testing.assert_allclose(delta, np.einsum("bihd,bihd->bhi", do, o), atol=1e-13)


# ---------------------------------------------------------------------------
# KV cache: paged == contiguous, append-then-attend == full attention
# ---------------------------------------------------------------------------

def _paged_setup(rng, B=3, Hq=4, Hkv=2, D=8, page=4, pps=5, Snew=2):
    num_pages = B * pps + 3
    bt = rng.permutation(num_pages)[: B * pps].reshape(B, pps)
    seqlens = np.array([0, 7, pps * page - Snew])[:B]
    kc = _rand((num_pages, page, Hkv, D), rng)
    vc = _rand((num_pages, page, Hkv, D), rng)
    kn, vn = _rand((B, Snew, Hkv, D), rng), _rand((B, Snew, Hkv, D), rng)
    q = _rand((B, Snew, Hq, D), rng)
    return q, kc, vc, kn, vn, seqlens, bt, page


@pytest.mark.parametrize("causal", [False, True])
def test_paged_equals_contiguous(causal):
    rng = np.random.default_rng(30)
    q, kc, vc, kn, vn, seqlens, bt, page = _paged_setup(rng)
    B, pps = bt.shape
    # contiguous copy of every sequence's pages
    kcc = np.stack([np.concatenate([kc[p] for p in bt[b]]) for b in range(B)])
    vcc = np.stack([np.concatenate([vc[p] for p in bt[b]]) for b in range(B)])
    o1, l1, kc1, _ = oracle.attn_with_kvcache(q, kc, vc, kn, vn, seqlens, bt, page, 0.5, causal)
    o2, l2, kc2, _ = oracle.attn_with_kvcache(q, kcc, vcc, kn, vn, seqlens, None, None, 0.5, causal)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    kcc1 = np.stack([np.concatenate([kc1[p] for p in bt[b]]) for b in range(B)])
    np.testing.assert_array_equal(kcc1, kc2)


def test_append_then_attend_equals_full_attention():
    rng = np.random.default_rng(31)
    q, kc, vc, kn, vn, seqlens, bt, page = _paged_setup(rng)
    o, l, _, _ = oracle.attn_with_kvcache(q, kc, vc, kn, vn, seqlens, bt, page, 0.5, True, 3, 0, 1.5)
    for b in range(bt.shape[0]):
        L0 = int(seqlens[b])
        Kold = np.array([kc[bt[b, t // page], t % page] for t in range(L0)]).reshape(L0, *kc.shape[2:])
        Vold = np.array([vc[bt[b, t // page], t % page] for t in range(L0)]).reshape(L0, *vc.shape[2:])
        Kfull = np.concatenate([Kold, kn[b]])
        Vfull = np.concatenate([Vold, vn[b]])
        # full self-attention over the concatenation; keep its last Snew rows
        qfull = np.concatenate([np.zeros((L0,) + q.shape[2:]), q[b]])[None]
        of, lf = oracle.attn_fwd(qfull, Kfull[None], Vfull[None], 0.5, True, 3, 0, 1.5)
        np.testing.assert_allclose(o[b], of[0, L0:], atol=1e-14)
        np.testing.assert_allclose(l[b], lf[0, :, L0:], atol=1e-14)


# ---------------------------------------------------------------------------
# splits: combine(partials) == unsplit
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L", [1, 5, 37, 64])
@pytest.mark.parametrize("n", [1, 4, 16])
def test_split_combine_equals_unsplit(L, n):
    rng = np.random.default_rng(40 + L)
    q = _rand((2, 4, 8), rng)
    K, V = _rand((L, 2, 8), rng), _rand((L, 2, 8), rng)
    ranges = oracle.split_token_ranges(L, 4, n)
    assert ranges[0][0] == 0 and ranges[-1][1] == L
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(n - 1))
    parts = [oracle.attn_partial(q, K, V, t0, t1, 0.5, True, 9, 0, 2.0) for t0, t1 in ranges]
    o, lse = oracle.combine_splits([p[0] for p in parts], [p[1] for p in parts])
    of, lf = oracle.attn_fwd(q[None], K[None], V[None], 0.5, True, 9, 0, 2.0)
    np.testing.assert_allclose(o, of[0], atol=1e-12)
    np.testing.assert_allclose(lse, lf[0], atol=1e-12)


def test_split_ranges_page_aligned_with_empty_splits():
    r = oracle.split_token_ranges(1, 256, 16)
    assert sum(t1 - t0 for t0, t1 in r) == 1
    assert sum(1 for t0, t1 in r if t1 > t0) == 1
    r = oracle.split_token_ranges(32769, 256, 16)
    assert all(t0 % 256 == 0 for t0, _ in r)
    assert r[-1][1] == 32769


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------

def _hand(name, section="examples"):
    return next(e for e in _load()[section] if e["name"] == name)


def test_planted_clamp_softcap_is_caught(monkeypatch):
    monkeypatch.setattr(attn64, "transform_scores",
                        lambda u, c: np.clip(u, -c, c) if c and c > 0 else u)
    with pytest.raises(AssertionError):
        test_hand_examples_forward(_hand("softcap_tanh"))


def test_planted_gqa_modulo_mapping_is_caught(monkeypatch):
    orig = attn64.raw_scores

    def bad_fwd(q, k, v, scale=None, causal=False, window_left=-1, window_right=-1, softcap=0.0,
                return_probs=False):
        # q-head h reads kv-head h % Hkv instead of h // G
        Hq, Hkv = q.shape[2], k.shape[2]
        idx = [h % Hkv for h in range(Hq)]
        return orig_fwd(q, k[:, :, idx], v[:, :, idx], scale, causal, window_left, window_right,
                        softcap, return_probs)

    orig_fwd = attn64.attn_fwd
    assert orig is attn64.raw_scores
    monkeypatch.setattr(oracle, "attn_fwd", bad_fwd)
    with pytest.raises(AssertionError):
        test_hand_examples_forward(_hand("gqa_head_mapping"))


def test_planted_missing_scale_is_caught(monkeypatch):
    monkeypatch.setattr(attn64, "raw_scores",
                        lambda q, k, scale, h, g: np.einsum("bid,bjd->bij", q[:, :, h, :], k[:, :, g, :]))
    with pytest.raises(AssertionError):
        test_hand_examples_forward(_hand("rectangular_noncausal"))


def test_planted_exclusive_window_is_caught(monkeypatch):
    orig = attn64.visible

    def excl(Sq, Sk, causal=False, window_left=-1, window_right=-1, key_offset=0, n_keys=None):
        wl = window_left - 1 if window_left is not None and window_left > 0 else window_left
        return orig(Sq, Sk, causal, wl, window_right, key_offset, n_keys)

    monkeypatch.setattr(attn64, "visible", excl)
    with pytest.raises(AssertionError):
        test_hand_examples_forward(_hand("window_left1"))


def test_rows_equal_full_forward():
    rng = np.random.default_rng(50)
    q, k, v = _rand((2, 37, 4, 8), rng), _rand((2, 41, 2, 8), rng), _rand((2, 41, 2, 8), rng)
    kw = dict(scale=0.3, causal=True, window_left=9, window_right=0, softcap=2.0)
    o, lse = oracle.attn_fwd(q, k, v, **kw)
    rows = np.array([0, 5, 17, 36])
    for b in range(2):
        for h in range(4):
            orow, lrow = oracle.attn_fwd_rows(q, k, v, b, h, rows, **kw)
            np.testing.assert_allclose(orow, o[b, rows, h], atol=1e-14)
            np.testing.assert_allclose(lrow, lse[b, h, rows], atol=1e-14)


@pytest.mark.parametrize("kw", [
    dict(scale=0.3, causal=True, window_left=9, window_right=0, softcap=2.0),
    dict(scale=0.4, causal=False, window_left=-1, window_right=-1, softcap=0.0),
    dict(scale=0.5, causal=False, window_left=4, window_right=6, softcap=0.0),
    dict(scale=0.2, causal=True, softcap=0.0, alibi_slopes=np.array([0.5, 0.25, 0.125, 1.0])),
], ids=["causal-window-cap", "full", "two-sided-window", "alibi"])
@pytest.mark.parametrize("Sq,Sk", [(37, 41), (41, 37), (30, 30)])
def test_sampled_gradients_equal_full_backward(kw, Sq, Sk):
    """attn_bwd_rows / attn_bwd_cols give the rows and columns of attn_bwd
    (itself pinned by finite differences), GQA group sums included; a row
    chunk smaller than Sq exercises sums that run across chunks."""
    rng = np.random.default_rng(51)
    q, k, v = _rand((2, Sq, 4, 8), rng), _rand((2, Sk, 2, 8), rng), _rand((2, Sk, 2, 8), rng)
    do = _rand((2, Sq, 4, 8), rng)
    dq, dk, dv, delta = oracle.attn_bwd(do, q, k, v, **kw)
    _, lse = oracle.attn_fwd(q, k, v, **kw)
    rows = np.array([0, 5, Sq // 2, Sq - 1])
    cols = np.array([0, 3, Sk // 2, Sk - 1])
    for b in range(2):
        for h in range(4):
            dq_r, lse_r, delta_r = oracle.attn_bwd_rows(do, q, k, v, b, h, rows, **kw)
            np.testing.assert_allclose(dq_r, dq[b, rows, h], atol=1e-12)
            np.testing.assert_allclose(lse_r, lse[b, h, rows], atol=1e-12)
            np.testing.assert_allclose(delta_r, delta[b, h, rows], atol=1e-12)
        for g in range(2):
            dk_c, dv_c = oracle.attn_bwd_cols(do, q, k, v, b, g, cols, row_chunk=7, **kw)
            np.testing.assert_allclose(dk_c, dk[b, cols, g], atol=1e-12)
            np.testing.assert_allclose(dv_c, dv[b, cols, g], atol=1e-12)


def test_sampled_gradients_match_finite_differences():
    """Direct pin of the sampled-row and sampled-column gradients: central
    differences of sum(dO * O) in one query row and one key/value row."""
    rng = np.random.default_rng(52)
    q, k, v = _rand((1, 6, 2, 4), rng), _rand((1, 7, 1, 4), rng), _rand((1, 7, 1, 4), rng)
    do = _rand((1, 6, 2, 4), rng)
    kw = dict(scale=0.7, causal=True, window_left=3, window_right=0, softcap=1.5)

    def loss(qq, kk, vv):
        return float((oracle.attn_fwd(qq, kk, vv, **kw)[0] * do).sum())

    def num_grad(x, idx):
        g = np.zeros(x.shape[-1])
        for d in range(x.shape[-1]):
            xp, xm = x.copy(), x.copy()
            xp[idx + (d,)] += 1e-6
            xm[idx + (d,)] -= 1e-6
            a = [xp if x is t else t for t in (q, k, v)]
            m = [xm if x is t else t for t in (q, k, v)]
            g[d] = (loss(*a) - loss(*m)) / 2e-6
        return g

    dq_r, _, _ = oracle.attn_bwd_rows(do, q, k, v, 0, 1, np.array([4]), **kw)
    np.testing.assert_allclose(dq_r[0], num_grad(q, (0, 4, 1)), rtol=1e-6, atol=1e-9)
    dk_c, dv_c = oracle.attn_bwd_cols(do, q, k, v, 0, 0, np.array([3]), row_chunk=2, **kw)
    np.testing.assert_allclose(dk_c[0], num_grad(k, (0, 3, 0)), rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(dv_c[0], num_grad(v, (0, 3, 0)), rtol=1e-6, atol=1e-9)


# ---------------------------------------------------------------------------
# variable-length (packed) batches
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("causal,wl,wr,cap", [(False, -1, -1, 0.0), (True, -1, -1, 0.0), (False, 3, 2, 4.0)])
def test_varlen_equal_lengths_equal_dense_batch(causal, wl, wr, cap):
    rng = np.random.default_rng(40)
    B, Sq, Sk, Hq, Hkv, D = 3, 7, 9, 4, 2, 8
    q, k, v, do = _rand((B, Sq, Hq, D), rng), _rand((B, Sk, Hkv, D), rng), _rand((B, Sk, Hkv, D), rng), \
        _rand((B, Sq, Hq, D), rng)
    cq, ck = np.arange(B + 1) * Sq, np.arange(B + 1) * Sk
    o_d, l_d = attn64.attn_fwd(q, k, v, 0.4, causal, wl, wr, cap)
    o_v, l_v = attn64.attn_fwd_varlen(q.reshape(B * Sq, Hq, D), k.reshape(B * Sk, Hkv, D), v.reshape(B * Sk, Hkv, D),
                                      cq, ck, 0.4, causal, wl, wr, cap)
    np.testing.assert_allclose(o_v, o_d.reshape(B * Sq, Hq, D), atol=1e-13)
    # LSE (B, Hq, Sq) -> (Hq, B*Sq)
    np.testing.assert_allclose(l_v, l_d.transpose(1, 0, 2).reshape(Hq, B * Sq), atol=1e-13)
    g_d = attn64.attn_bwd(do, q, k, v, 0.4, causal, wl, wr, cap)
    g_v = attn64.attn_bwd_varlen(do.reshape(B * Sq, Hq, D), q.reshape(B * Sq, Hq, D), k.reshape(B * Sk, Hkv, D),
                                 v.reshape(B * Sk, Hkv, D), cq, ck, 0.4, causal, wl, wr, cap)
    for a, b in zip(g_v, g_d[:3]):
        np.testing.assert_allclose(a, b.reshape(a.shape), atol=1e-12)


def test_varlen_sequences_do_not_see_each_other():
    # changing one sequence's tokens leaves the other sequences' outputs and
    # gradients unchanged (no attention across the packing boundary)
    rng = np.random.default_rng(41)
    cq, ck = np.array([0, 5, 5, 12]), np.array([0, 3, 9, 17])
    q, k, v, do = _rand((12, 2, 4), rng), _rand((17, 1, 4), rng), _rand((17, 1, 4), rng), _rand((12, 2, 4), rng)
    o1, l1 = attn64.attn_fwd_varlen(q, k, v, cq, ck, None, True)
    g1 = attn64.attn_bwd_varlen(do, q, k, v, cq, ck, None, True)
    k2, v2, q2 = k.copy(), v.copy(), q.copy()
    k2[9:], v2[9:], q2[5:] = 5.0, -3.0, 2.0  # sequence 2 changed
    o2, l2 = attn64.attn_fwd_varlen(q2, k2, v2, cq, ck, None, True)
    g2 = attn64.attn_bwd_varlen(do, q2, k2, v2, cq, ck, None, True)
    np.testing.assert_array_equal(o1[:5], o2[:5])
    np.testing.assert_array_equal(l1[:, :5], l2[:, :5])
    np.testing.assert_array_equal(g1[1][:9], g2[1][:9])
    np.testing.assert_array_equal(g1[2][:9], g2[2][:9])
    # sequence 1 has no queries: it contributes nothing, its keys get no gradient
    assert np.all(g1[1][3:9] == 0) and np.all(g1[2][3:9] == 0)
    # a packed sequence equals the same problem run alone
    o_s, l_s = attn64.attn_fwd(q[None, 5:12], k[None, 9:17], v[None, 9:17], None, True)
    np.testing.assert_allclose(o1[5:12], o_s[0], atol=1e-13)
    np.testing.assert_allclose(l1[:, 5:12], l_s[0], atol=1e-13)


def test_varlen_permuting_sequences_permutes_results():
    rng = np.random.default_rng(42)
    lq, lk = [4, 1, 6], [6, 3, 6]
    seqs = [(_rand((a, 2, 4), rng), _rand((b, 2, 4), rng), _rand((b, 2, 4), rng)) for a, b in zip(lq, lk)]

    def pack(order):
        qs = np.concatenate([seqs[i][0] for i in order])
        ks = np.concatenate([seqs[i][1] for i in order])
        vs = np.concatenate([seqs[i][2] for i in order])
        cq = np.concatenate([[0], np.cumsum([lq[i] for i in order])])
        ck = np.concatenate([[0], np.cumsum([lk[i] for i in order])])
        return attn64.attn_fwd_varlen(qs, ks, vs, cq, ck, None, True, 2, 0)

    o_a, l_a = pack([0, 1, 2])
    o_b, l_b = pack([2, 0, 1])
    np.testing.assert_allclose(o_b[:6], o_a[5:11], atol=1e-13)   # sequence 2
    np.testing.assert_allclose(o_b[6:10], o_a[:4], atol=1e-13)   # sequence 0
    np.testing.assert_allclose(l_b[:, 10:], l_a[:, 4:5], atol=1e-13)  # sequence 1


def test_varlen_backward_finite_differences():
    rng = np.random.default_rng(43)
    cq, ck = np.array([0, 3, 5]), np.array([0, 4, 6])
    q, k, v, do = _rand((5, 2, 3), rng), _rand((6, 1, 3), rng), _rand((6, 1, 3), rng), _rand((5, 2, 3), rng)
    dq, dk, dv = attn64.attn_bwd_varlen(do, q, k, v, cq, ck, 0.7, True, -1, -1, 3.0)

    def loss(q_, k_, v_):
        return float(np.sum(do * attn64.attn_fwd_varlen(q_, k_, v_, cq, ck, 0.7, True, -1, -1, 3.0)[0]))

    h = 1e-6
    for arr, grad, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def test_varlen_sequence_without_keys():
    rng = np.random.default_rng(44)
    cq, ck = np.array([0, 3, 7]), np.array([0, 0, 5])
    q, k, v = _rand((7, 2, 4), rng), _rand((5, 1, 4), rng), _rand((5, 1, 4), rng)
    o, l = attn64.attn_fwd_varlen(q, k, v, cq, ck)
    assert np.all(o[:3] == 0) and np.all(l[:, :3] == -np.inf)
    o_s, l_s = attn64.attn_fwd(q[None, 3:], k[None], v[None])
    np.testing.assert_allclose(o[3:], o_s[0], atol=1e-13)
    dq, dk, dv = attn64.attn_bwd_varlen(_rand((7, 2, 4), rng), q, k, v, cq, ck)
    assert np.all(dq[:3] == 0)


# ---------------------------------------------------------------------------
# rotary position embedding in the kvcache call
# ---------------------------------------------------------------------------

def _rope_tables(n_pos, half, base=10000.0):
    inv = base ** (-np.arange(half) / half)
    ang = np.arange(n_pos)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def test_rotary_two_dims_is_a_rotation_matrix():
    # D = 2, one pair: (x, y) -> (x cos t - y sin t, y cos t + x sin t)
    t = 0.7
    cos, sin = np.array([[1.0], [math.cos(t)]]), np.array([[0.0], [math.sin(t)]])
    x = np.array([[[[3.0, -2.0]]]])  # (1, 1, 1, 2)
    for inter in (False, True):
        r = attn64.rotary(x, cos, sin, np.array([[1]]), inter)
        np.testing.assert_allclose(r[0, 0, 0], [3 * math.cos(t) + 2 * math.sin(t), -2 * math.cos(t) + 3 * math.sin(t)],
                                   atol=1e-15)
        np.testing.assert_array_equal(attn64.rotary(x, cos, sin, np.array([[0]]), inter), x)  # angle 0


@pytest.mark.parametrize("inter", [False, True])
def test_rotary_keeps_norms_and_depends_on_relative_position(inter):
    rng = np.random.default_rng(45)
    D, half = 16, 6
    cos, sin = _rope_tables(64, half)
    q, k = _rand((1, 1, 1, D), rng), _rand((1, 1, 1, D), rng)
    # pairwise rotation keeps the norm
    r = attn64.rotary(q, cos, sin, np.array([[37]]), inter)
    np.testing.assert_allclose(np.linalg.norm(r), np.linalg.norm(q), rtol=1e-13)
    np.testing.assert_array_equal(r[..., 2 * half:], q[..., 2 * half:])  # dims past r untouched
    # <R(p) q, R(p') k> depends on p - p' only
    dots = [float(np.sum(attn64.rotary(q, cos, sin, np.array([[p + 5]]), inter) *
                         attn64.rotary(k, cos, sin, np.array([[p]]), inter))) for p in (0, 9, 40)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-12)


def test_rotary_interleaved_is_a_permutation_of_halves():
    rng = np.random.default_rng(46)
    D, half = 8, 4
    cos, sin = _rope_tables(10, half)
    x = _rand((1, 3, 2, D), rng)
    pos = np.array([[1, 4, 7]])
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])  # interleaved -> halves
    r_int = attn64.rotary(x, cos, sin, pos, True)
    r_half = attn64.rotary(x[..., perm], cos, sin, pos, False)
    np.testing.assert_allclose(r_int[..., perm], r_half, atol=1e-14)


def test_kvcache_rotary_matches_prerotated_inputs():
    rng = np.random.default_rng(47)
    B, Hq, Hkv, D, Snew, L = 2, 4, 2, 8, 2, 6
    cos, sin = _rope_tables(16, 3)
    kc, vc = _rand((B, 12, Hkv, D), rng), _rand((B, 12, Hkv, D), rng)
    q, kn, vn = _rand((B, Snew, Hq, D), rng), _rand((B, Snew, Hkv, D), rng), _rand((B, Snew, Hkv, D), rng)
    sl = np.array([L, 3])
    o1, l1, kc1, _ = attn64.attn_with_kvcache(q, kc, vc, kn, vn, sl, causal=True, rotary_cos=cos, rotary_sin=sin)
    pos = sl[:, None] + np.arange(Snew)[None, :]
    o2, l2, kc2, _ = attn64.attn_with_kvcache(attn64.rotary(q, cos, sin, pos), kc, vc, attn64.rotary(kn, cos, sin, pos),
                                              vn, sl, causal=True)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(kc1, kc2, atol=1e-13)
    # the appended keys are rotated, the old cache rows are not touched
    np.testing.assert_array_equal(kc1[0, :L], kc[0, :L])
    assert not np.allclose(kc1[0, L:L + Snew], kn[0])


# ---------------------------------------------------------------------------
# ALiBi (alibi_slopes): distance bias -m * |i + off - j|
# ---------------------------------------------------------------------------

def _geo(n, r):
    """sum_{d=0}^{n} r^d and sum_{d=0}^{n} d r^d in closed form (n >= 0)."""
    g0 = (1.0 - r ** (n + 1)) / (1.0 - r)
    g1 = r * (1.0 - (n + 1) * r ** n + n * r ** (n + 1)) / (1.0 - r) ** 2
    return g0, g1


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("Sq,Sk", [(9, 9), (4, 9)])
def test_alibi_geometric_weights_closed_form(causal, Sq, Sk):
    # q = 0: every raw score is 0 and the weights are r^distance with
    # r = exp(-m); with V = key index the output is a mean position
    slopes = np.array([[0.3, 1.1], [0.05, 2.0]])  # (B, Hq)
    B, H = slopes.shape
    q = np.zeros((B, Sq, H, 2))
    k = np.ones((B, Sk, H, 2))
    v = np.zeros((B, Sk, H, 2))
    v[:, :, :, 0] = np.arange(Sk)[None, :, None]
    v[:, :, :, 1] = 1.0
    o, lse = oracle.attn_fwd(q, k, v, causal=causal, alibi_slopes=slopes)
    for b in range(B):
        for h in range(H):
            r = math.exp(-slopes[b, h])
            for i in range(Sq):
                p = i + Sk - Sq
                g0l, g1l = _geo(p, r)                      # keys p, p-1, ..., 0
                if causal:
                    s0, s1 = g0l, -g1l
                else:
                    g0r, g1r = _geo(Sk - 1 - p, r)         # keys p, p+1, ..., Sk-1
                    s0, s1 = g0l + g0r - 1.0, g1r - g1l
                assert lse[b, h, i] == pytest.approx(math.log(s0), abs=1e-12)
                assert o[b, i, h, 0] == pytest.approx(p + s1 / s0, abs=1e-12)
                assert o[b, i, h, 1] == pytest.approx(1.0, abs=1e-12)


@pytest.mark.parametrize("wl", [-1, 3])
def test_alibi_causal_equals_augmented_dot_product(wl):
    # causal: -m (p - j) = m j - m p; the row constant -m p leaves P alone and
    # m j is one more dot-product term: q' = [q, 1], k' = [k, m j / scale]
    rng = np.random.default_rng(40)
    B, Sq, Sk, H, D, sc = 2, 5, 8, 3, 4, 0.7
    q, k, v = _rand((B, Sq, H, D), rng), _rand((B, Sk, H, D), rng), _rand((B, Sk, H, D), rng)
    m = np.array([0.25, 0.5, 1.5])
    o, lse = oracle.attn_fwd(q, k, v, sc, True, wl, -1, alibi_slopes=m)
    qa = np.concatenate([q, np.ones((B, Sq, H, 1))], axis=3)
    ka = np.concatenate([k, (m[None, None, :] * np.arange(Sk)[None, :, None] / sc)[..., None]
                         * np.ones((B, 1, 1, 1))], axis=3)
    va = np.concatenate([v, np.zeros((B, Sk, H, 1))], axis=3)
    oa, la = oracle.attn_fwd(qa, ka, va, sc, True, wl, -1)
    np.testing.assert_allclose(o, oa[..., :D], rtol=0, atol=1e-12)
    p = np.arange(Sq) + Sk - Sq
    np.testing.assert_allclose(lse, la - m[None, :, None] * p[None, None, :], rtol=0, atol=1e-11)


def test_alibi_is_added_after_the_softcap():
    # capped scores lie in [-c, c], so log(P_ij / P_il) differs from the bias
    # difference by at most 2c, however far apart the keys are
    rng = np.random.default_rng(41)
    B, S, H, D, c = 1, 12, 2, 8, 0.5
    q, k, v = _rand((B, S, H, D), rng, 3.0), _rand((B, S, H, D), rng, 3.0), _rand((B, S, H, D), rng)
    m = np.array([1.0, 2.5])
    _, _, P, _ = oracle.attn_fwd(q, k, v, None, False, softcap=c, return_probs=True, alibi_slopes=m)
    for h in range(H):
        for i in range(S):
            bias = -m[h] * np.abs(i - np.arange(S))
            lr = np.log(P[0, h, i]) - np.log(P[0, h, i, i])
            assert np.all(np.abs(lr - (bias - bias[i])) <= 2 * c + 1e-12)


def test_alibi_zero_slopes_and_rows():
    rng = np.random.default_rng(42)
    q, k, v = _rand((2, 6, 4, 8), rng), _rand((2, 9, 2, 8), rng), _rand((2, 9, 2, 8), rng)
    o0, l0 = oracle.attn_fwd(q, k, v, causal=True)
    o1, l1 = oracle.attn_fwd(q, k, v, causal=True, alibi_slopes=np.zeros(4))
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)
    # the row-wise form agrees with the whole-matrix form
    m = np.array([[0.1, 0.2, 0.4, 0.8], [1.0, 0.5, 0.25, 0.125]])
    o, l = oracle.attn_fwd(q, k, v, None, False, 3, 2, 1.5, alibi_slopes=m)
    for b, h in ((0, 1), (1, 3)):
        orow, lrow = oracle.attn_fwd_rows(q, k, v, b, h, np.arange(6), None, False, 3, 2, 1.5, alibi_slopes=m)
        np.testing.assert_allclose(orow, o[b, :, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lrow, l[b, h], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,cap", [(False, 0.0), (True, 1.5)])
def test_alibi_gradients_match_finite_differences(causal, cap):
    rng = np.random.default_rng(43)
    q, k, v = _rand((2, 4, 2, 3), rng), _rand((2, 5, 1, 3), rng), _rand((2, 5, 1, 3), rng)
    do = _rand((2, 4, 2, 3), rng)
    kw = dict(scale=0.6, causal=causal, softcap=cap, alibi_slopes=np.array([[0.3, 0.9], [1.7, 0.1]]))

    def loss(qq, kk, vv):
        return float((oracle.attn_fwd(qq, kk, vv, **kw)[0] * do).sum())

    dq, dk, dv, _ = oracle.attn_bwd(do, q, k, v, **kw)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if x is t else t for t in (q, k, v)]
            args_m = [xm if x is t else t for t in (q, k, v)]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
        assert err <= 1e-6, err


def test_planted_alibi_sign_is_caught(monkeypatch):
    orig = attn64.alibi_bias
    monkeypatch.setattr(attn64, "alibi_bias", lambda m, rows, Sq, Sk: -orig(m, rows, Sq, Sk))
    with pytest.raises(AssertionError):
        test_alibi_geometric_weights_closed_form(True, 9, 9)
    with pytest.raises(AssertionError):
        test_hand_examples_forward(_hand("alibi_causal_two_keys"))


def test_planted_alibi_top_left_alignment_is_caught(monkeypatch):
    orig = attn64.alibi_bias
    monkeypatch.setattr(attn64, "alibi_bias", lambda m, rows, Sq, Sk: orig(m, np.asarray(rows) - (Sk - Sq), Sq, Sk))
    with pytest.raises(AssertionError):
        test_alibi_geometric_weights_closed_form(False, 4, 9)


# ---------------------------------------------------------------------------
# FP8 E4M3 forward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("code,value", [(0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
                                        (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x46, 3.5), (0x4B, 5.5), (0x7E, 448.0),
                                        (0xB8, -1.0), (0xFE, -448.0)])
def test_e4m3_known_codes(code, value):
    # sign | exponent (bias 7) | 3-bit mantissa, worked by hand
    assert oracle.e4m3_decode(np.array([code], np.uint8))[0] == value


def test_e4m3_nan_and_negative_zero():
    v = oracle.e4m3_decode(np.array([0x7F, 0xFF, 0x80], np.uint8))
    assert np.isnan(v[0]) and np.isnan(v[1])
    assert v[2] == 0.0 and math.copysign(1.0, v[2]) < 0


def test_e4m3_decode_matches_torch_float8():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(lib))
    fin = ~np.isnan(lib)
    np.testing.assert_array_equal(mine[fin], lib[fin])


def _codes(shape, rng):
    # finite codes only (NaN codes 0x7F/0xFF excluded), magnitudes up to 8
    c = rng.integers(0, 0x58, size=shape).astype(np.uint8)
    return np.where(rng.random(shape) < 0.5, c | 0x80, c).astype(np.uint8)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_zero_queries_give_uniform_weights(causal):
    # q = 0: every visible key gets the same weight, O is the mean of the
    # visible V rows (times the V factor) and LSE = log(number visible)
    rng = np.random.default_rng(60)
    B, Sq, Sk, H, D = 2, 3, 7, 2, 4
    q8 = np.zeros((B, Sq, H, D), np.uint8)
    k8, v8 = _codes((B, Sk, H, D), rng), _codes((B, Sk, H, D), rng)
    dv = np.array([[0.5, 2.0], [3.0, 0.25]])
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, descale_v=dv, causal=causal)
    vals = oracle.e4m3_decode(v8)
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                n = i + Sk - Sq + 1 if causal else Sk
                np.testing.assert_allclose(o[b, i, h], dv[b, h] * vals[b, :n, h].mean(axis=0), rtol=0, atol=1e-12)
                assert lse[b, h, i] == pytest.approx(math.log(n), abs=1e-12)


def test_fp8_descales_act_per_batch_and_kv_head():
    # the q and k factors of (b, kv-head g) only rescale the scores of the
    # q-heads reading g: the same as a softmax scale times dq * dk for them
    rng = np.random.default_rng(61)
    B, S, Hq, Hkv, D = 2, 5, 4, 2, 8
    q8, k8, v8 = _codes((B, S, Hq, D), rng), _codes((B, S, Hkv, D), rng), _codes((B, S, Hkv, D), rng)
    dq = np.array([[0.5, 0.125], [0.25, 1.0]])
    dk = np.array([[0.25, 0.5], [0.0625, 0.75]])
    dv = np.array([[1.5, 0.5], [2.0, 0.25]])
    sc = 0.2
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, dq, dk, dv, scale=sc, causal=True)
    qv, kv, vv = oracle.e4m3_decode(q8), oracle.e4m3_decode(k8), oracle.e4m3_decode(v8)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            o1, l1 = oracle.attn_fwd(qv[b:b + 1, :, h:h + 1], kv[b:b + 1, :, g:g + 1], vv[b:b + 1, :, g:g + 1],
                                     sc * dq[b, g] * dk[b, g], True)
            np.testing.assert_allclose(o[b, :, h], dv[b, g] * o1[0, :, 0], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], l1[0, 0], rtol=0, atol=1e-12)


def test_planted_fp8_descale_by_q_head_is_caught(monkeypatch):
    orig = oracle.attn_fwd_fp8

    def bad(q8, k8, v8, descale_q=None, descale_k=None, descale_v=None, **kw):
        # q factor taken by q-head index modulo Hkv instead of its kv-head
        Hq, Hkv = q8.shape[2], k8.shape[2]
        qv = oracle.e4m3_decode(q8) * np.asarray(descale_q)[:, None, [h % Hkv for h in range(Hq)], None]
        return oracle.attn_fwd(qv, oracle.e4m3_decode(k8) * np.asarray(descale_k)[:, None, :, None],
                               oracle.e4m3_decode(v8) * np.asarray(descale_v)[:, None, :, None], kw.get("scale"),
                               kw.get("causal", False))

    monkeypatch.setattr(oracle, "attn_fwd_fp8", bad)
    with pytest.raises(AssertionError):
        test_fp8_descales_act_per_batch_and_kv_head()
    monkeypatch.setattr(oracle, "attn_fwd_fp8", orig)


# ---------------------------------------------------------------------------
# FP8: spacing of the E4M3 grid and the P-rounding error scale
# ---------------------------------------------------------------------------

def _e4m3_grid():
    """Sorted non-negative finite E4M3 values, decoded from all 128 codes
    with the sign bit clear."""
    vals = oracle.e4m3_decode(np.arange(128, dtype=np.uint8))
    return np.sort(vals[np.isfinite(vals)])


def test_e4m3_spacing_matches_the_code_table():
    grid = _e4m3_grid()
    gaps = np.diff(grid)
    np.testing.assert_array_equal(oracle.e4m3_spacing(grid[:-1]), gaps)
    assert grid[-1] == 448.0 and grid[1] == 2.0 ** -9


def _round_e4m3(x):
    """Round non-negative x to the nearest E4M3 value (ties to the even
    mantissa, i.e. the even code), by search in the decoded table."""
    grid = _e4m3_grid()
    i = np.clip(np.searchsorted(grid, x), 1, len(grid) - 1)
    lo, hi = grid[i - 1], grid[i]
    pick_hi = (x - lo > hi - x) | ((x - lo == hi - x) & (i % 2 == 0))
    return np.where(pick_hi, hi, lo)


@pytest.mark.parametrize("c", [1.0, 3.7, 200.0])
def test_fp8_sigma_bounds_e4m3_rounded_probabilities(c):
    """Quantising c * P to E4M3 (c = the factor a running maximum leaves on
    the row's largest probability, 1 <= c <= 2^8) stays within 7 x 2 sigma
    elementwise, and at c = 1 the errors have RMS ~ sigma: sigma is the
    scale of the error, not a vacuous bound."""
    rng = np.random.default_rng(60)
    B, Sq, Sk, H, D = 1, 48, 700, 2, 16
    q, k, v = _rand((B, Sq, H, D), rng), _rand((B, Sk, H, D), rng), _rand((B, Sk, H, D), rng)
    kw = dict(scale=0.25, causal=True)
    ratios = []
    for h in range(H):
        rows = np.arange(Sq)
        o, lse, sig = oracle.fp8_p_rounding_sigma(q, k, v, 0, h, rows, **kw)
        o_ref, lse_ref = oracle.attn_fwd_rows(q, k, v, 0, h, rows, **kw)
        np.testing.assert_allclose(o, o_ref, atol=1e-13)
        np.testing.assert_allclose(lse, lse_ref, atol=1e-13)
        u = 0.25 * (q[0, :, h, :] @ k[0, :, h, :].T)
        vis = oracle.visible(Sq, Sk, True)
        u = np.where(vis, u, -np.inf)
        P = np.where(vis, np.exp(u - u.max(axis=1, keepdims=True)), 0.0) * c
        R = _round_e4m3(P)
        oq = (R @ v[0, :, h, :]) / R.sum(axis=1, keepdims=True)
        err = np.abs(oq - o_ref)
        assert (err <= 14.0 * sig + 1e-12).all(), float((err / sig).max())
        ratios.append(err / sig)
    rms = float(np.sqrt(np.mean(np.concatenate(ratios) ** 2)))
    if c == 1.0:
        assert 0.5 <= rms <= 1.5, rms
    else:
        assert rms <= 2.0, rms
