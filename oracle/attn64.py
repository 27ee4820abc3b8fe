"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls this
module; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` do.  It shares no code, header, table
or constant with the CUDA path: every function here is the plain definition,
written with NumPy in float64, and it materialises the whole score matrix on
purpose.

Sources (three web pages about FlashAttention; formulas are never written out
there, so each function states the reading it implements):

* "FlashAttention 实战指南" (mhpq.cn), section on why long sequences run out of
  memory: standard scaled dot-product attention is QK^T, then softmax, then a
  product with V; the method's output is numerically the same as that standard
  attention ("exact").  -> :func:`attn_fwd` is that definition.
* same page, section on advanced parameters: ``window_size=(left, right)`` with
  (-1, -1) meaning an unbounded window; ``softcap`` bounds the logits to
  [-softcap, softcap]; K/V may have fewer heads than Q as long as the Q head
  count is an integer multiple (MQA/GQA); ``deterministic`` backward.
* same page, section on incremental decoding: ``flash_attn_with_kvcache``
  appends the new K/V into the existing cache and attends in place,
  ``cache_seqlens`` marks each sample's valid length, ``block_table`` pages the
  cache, ``num_splits`` splits the KV range.  -> :func:`attn_with_kvcache`.
* same page, advanced parameters: ``alibi_slopes`` adds an ALiBi position
  bias that lowers the scores of distant keys, instead of an explicit
  position encoding.  -> :func:`alibi_bias`.
* same page, versions: FlashAttention-3 adds an FP8 forward (and an AMD
  backend's fp8 path keeps precision while lowering bandwidth).
  -> :func:`attn_fwd_fp8`.
* same page, the three techniques: tiling, online softmax (running row max and
  running sum updated block by block), recomputation in the backward.
  -> :func:`attn_fwd_online` (used only to pin :func:`attn_fwd`).

Readings where the pages are silent:

* softcap: ``s = softcap * tanh(u / softcap)`` applied after the scale and
  before the mask; ``softcap <= 0`` switches it off.
* window: key j is visible to query i iff
  ``i+off-left <= j <= i+off+right`` (inclusive), a negative extent is
  unbounded; ``causal`` is the same as ``right = 0`` and intersects with a
  given window.  ``off = Sk - Sq`` (bottom-right alignment).
* GQA: q-head h reads kv-head ``h // (Hq // Hkv)``.
* LSE is the natural-log row log-sum-exp, layout (B, Hq, Sq).
* a row with no visible key has O = 0 and LSE = -inf.
* ``cache_seqlens`` is the length before the append; the call attends over
  ``cache_seqlens[b] + Snew`` keys and does not update ``cache_seqlens``.
* split s of a sequence with P pages covers pages
  ``ceil(s*P/n) .. ceil((s+1)*P/n) - 1``.
* rotary (kvcache call): new token t of sequence b and its query sit at
  position ``cache_seqlens[b] + t``; pairs (j, j + r/2) are rotated, or
  (2j, 2j+1) when interleaved, with r = 2 * rotary_cos.shape[1]; the cache
  holds keys already rotated.
* ALiBi: with slope m of (batch b, q-head h) the score of query i and key j
  gains ``-m * |i + off - j|`` (``off`` of the bottom-right alignment),
  added after the soft cap and before the mask; slopes are (Hq,) shared by
  the batch or (B, Hq).
* FP8 forward: q, k, v are OCP FP8 E4M3 codes; each of the three tensors
  has one float32 descale factor per (batch, kv-head) (a q-head uses the
  factor of the kv-head it reads), default 1; the real inputs are code value
  times factor, and the output is the exact attention of those real inputs.
* varlen: sequences packed along the token axis with ``cu_seqlens`` offsets
  (sequence b is tokens ``cu[b] .. cu[b+1]-1``); each sequence is attended on
  its own, with the masks and the bottom-right alignment of its own lengths;
  the LSE layout is (Hq, total_q).

Layouts follow the pages' (batch, seqlen, nheads, headdim) convention.
"""

import math

import numpy as np

# -inf arithmetic on masked entries is intended (the results are selected
# away): the functions that do it silence NumPy's warnings for their own
# duration only, leaving the caller's error state alone.
_masked_math = np.errstate(invalid="ignore", divide="ignore")

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# visibility (mask) rule
# ---------------------------------------------------------------------------

def effective_window(causal, window_left, window_right):
    """Return (left, right) extents after folding ``causal`` in.

    Negative means unbounded.  Causal attention is the window with right
    extent 0; when a window is also given the two are intersected.
    """
    left = int(window_left) if window_left is not None and window_left >= 0 else -1
    right = int(window_right) if window_right is not None and window_right >= 0 else -1
    if causal:
        right = 0 if right < 0 else min(right, 0)
    return left, right


def visible_rows(rows, Sq, Sk, causal=False, window_left=-1, window_right=-1, key_offset=0,
                 n_keys=None):
    """Boolean (len(rows), n_keys): may query ``rows[r]`` see key (key_offset + j)?

    Query i sits at absolute position ``i + Sk - Sq`` (bottom-right
    alignment).  ``key_offset`` and ``n_keys`` select a sub-range of the Sk
    keys (used for KV splits).
    """
    if n_keys is None:
        n_keys = Sk - key_offset
    rows = np.asarray(rows)
    left, right = effective_window(causal, window_left, window_right)
    qpos = rows[:, None] + (Sk - Sq)
    kpos = np.arange(key_offset, key_offset + n_keys)[None, :]
    ok = np.broadcast_to((kpos >= 0) & (kpos < Sk), (len(rows), n_keys)).copy()
    if right >= 0:
        ok &= kpos <= qpos + right
    if left >= 0:
        ok &= kpos >= qpos - left
    return ok


def visible(Sq, Sk, causal=False, window_left=-1, window_right=-1, key_offset=0, n_keys=None):
    """Boolean (Sq, n_keys) matrix for all queries; see :func:`visible_rows`."""
    return visible_rows(np.arange(Sq), Sq, Sk, causal, window_left, window_right, key_offset, n_keys)


# ---------------------------------------------------------------------------
# forward: the plain definition
# ---------------------------------------------------------------------------

def _check_heads(Hq, Hkv):
    if Hkv <= 0 or Hq % Hkv != 0:
        raise ValueError(f"Hq={Hq} must be an integer multiple of Hkv={Hkv}")
    return Hq // Hkv


def raw_scores(q, k, scale, h, g):
    """u[b, i, j] = scale * sum_d q[b,i,h,d] * k[b,j,g,d]  (float64)."""
    return scale * np.matmul(q[:, :, h, :], k[:, :, g, :].transpose(0, 2, 1))


def transform_scores(u, softcap):
    """Apply the soft cap ``softcap * tanh(u / softcap)`` (off when <= 0)."""
    if softcap is not None and softcap > 0:
        return softcap * np.tanh(u / softcap)
    return u


def head_slopes(alibi_slopes, B, h):
    """Slope of q-head h for each of the B batch rows: slopes (Hq,) are
    shared by the batch, (B, Hq) are per batch row."""
    m = np.asarray(alibi_slopes, np.float64)
    return np.full(B, m[h]) if m.ndim == 1 else m[:, h].copy()


def alibi_bias(slope, rows, Sq, Sk):
    """Bias ``-slope * |i + Sk - Sq - j|`` of query rows ``rows`` against keys
    0..Sk-1 (distance at the bottom-right aligned positions)."""
    qpos = np.asarray(rows)[:, None] + (Sk - Sq)
    return -float(slope) * np.abs(qpos - np.arange(Sk)[None, :]).astype(np.float64)


@_masked_math
def attn_fwd(q, k, v, scale=None, causal=False, window_left=-1, window_right=-1,
             softcap=0.0, return_probs=False, alibi_slopes=None):
    """Exact attention O = softmax(transform(scale * Q K^T) [+ ALiBi] + mask) V.

    q: (B, Sq, Hq, D); k, v: (B, Sk, Hkv, D), any float dtype (upcast to f64).
    ``alibi_slopes`` (Hq,) or (B, Hq) adds :func:`alibi_bias`.
    Returns O (B, Sq, Hq, D) f64 and LSE (B, Hq, Sq) f64 (natural log).
    With ``return_probs`` also returns P (B, Hq, Sq, Sk) and the raw
    scores u (B, Hq, Sq, Sk).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = _check_heads(Hq, Hkv)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    vis = visible(Sq, Sk, causal, window_left, window_right)
    out = np.zeros((B, Sq, Hq, D))
    lse = np.full((B, Hq, Sq), NEG_INF)
    P_all = np.zeros((B, Hq, Sq, Sk)) if return_probs else None
    U_all = np.zeros((B, Hq, Sq, Sk)) if return_probs else None
    for h in range(Hq):
        g = h // G
        u = raw_scores(q, k, scale, h, g)              # (B, Sq, Sk)
        s = transform_scores(u, softcap)
        if alibi_slopes is not None:
            ms = head_slopes(alibi_slopes, B, h)
            s = s + np.stack([alibi_bias(ms[b], np.arange(Sq), Sq, Sk) for b in range(B)])
        s = np.where(vis[None], s, NEG_INF)
        any_vis = vis.any(axis=1)                       # (Sq,)
        m = np.where(any_vis[None], s.max(axis=2), 0.0)  # row max over visible keys
        e = np.where(vis[None], np.exp(s - m[:, :, None]), 0.0)
        l = e.sum(axis=2)
        row_lse = np.where(any_vis[None], m + np.log(np.where(l > 0, l, 1.0)), NEG_INF)
        P = np.where(vis[None], np.exp(s - row_lse[:, :, None]), 0.0)
        out[:, :, h, :] = np.matmul(P, v[:, :, g, :])
        lse[:, h, :] = row_lse
        if return_probs:
            P_all[:, h] = P
            U_all[:, h] = u
    if return_probs:
        return out, lse, P_all, U_all
    return out, lse


@_masked_math
def attn_fwd_rows(q, k, v, b, h, rows, scale=None, causal=False, window_left=-1, window_right=-1,
                  softcap=0.0, alibi_slopes=None):
    """O and LSE of selected query rows of one (batch b, q-head h).

    Each row is the plain definition on its own: its scores against every
    key, the visibility rule at its absolute position, a softmax over the
    visible keys and the weighted sum of V.  Returns O (len(rows), D) and LSE
    (len(rows),).  Used to check outputs of problems too large to evaluate
    whole.
    """
    q = np.asarray(q)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = _check_heads(Hq, Hkv)
    g = h // G
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    rows = np.asarray(rows)
    Kg = np.asarray(k[b, :, g, :], np.float64)
    Vg = np.asarray(v[b, :, g, :], np.float64)
    u = scale * (np.asarray(q[b, rows, h, :], np.float64) @ Kg.T)   # (R, Sk)
    s = transform_scores(u, softcap)
    if alibi_slopes is not None:
        s = s + alibi_bias(head_slopes(alibi_slopes, B, h)[b], rows, Sq, Sk)
    vis = visible_rows(rows, Sq, Sk, causal, window_left, window_right)
    s = np.where(vis, s, NEG_INF)
    anyv = vis.any(axis=1)
    m = np.where(anyv, s.max(axis=1), 0.0)
    e = np.where(vis, np.exp(s - m[:, None]), 0.0)
    l = e.sum(axis=1)
    lse = np.where(anyv, m + np.log(np.where(anyv, l, 1.0)), NEG_INF)
    o = np.where(anyv[:, None], (e @ Vg) / np.where(anyv, l, 1.0)[:, None], 0.0)
    return o, lse


# ---------------------------------------------------------------------------
# forward: the tiled online-softmax algorithm (pins attn_fwd, never the GPU)
# ---------------------------------------------------------------------------

@_masked_math
def attn_fwd_online(q, k, v, scale=None, causal=False, window_left=-1, window_right=-1,
                    softcap=0.0, block=16):
    """Same result as :func:`attn_fwd`, reached block by block.

    Follows the page's description of the online softmax: walk the keys in
    blocks, keep a running row maximum m and running sum l, and rescale the
    partial output by exp(m_old - m_new) whenever the maximum grows.  The full
    score matrix of a row is never formed.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = _check_heads(Hq, Hkv)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((B, Sq, Hq, D))
    lse = np.full((B, Hq, Sq), NEG_INF)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            m = np.full(Sq, NEG_INF)
            l = np.zeros(Sq)
            acc = np.zeros((Sq, D))
            for j0 in range(0, Sk, block):
                j1 = min(Sk, j0 + block)
                vis = visible(Sq, Sk, causal, window_left, window_right, key_offset=j0, n_keys=j1 - j0)
                u = scale * (q[b, :, h, :] @ k[b, j0:j1, g, :].T)
                s = np.where(vis, transform_scores(u, softcap), NEG_INF)
                m_blk = s.max(axis=1)
                m_new = np.maximum(m, m_blk)
                safe = np.isfinite(m_new)
                alpha = np.where(safe & np.isfinite(m), np.exp(np.where(safe, m - m_new, 0.0)), 0.0)
                p = np.where(vis & safe[:, None], np.exp(s - np.where(safe, m_new, 0.0)[:, None]), 0.0)
                l = alpha * l + p.sum(axis=1)
                acc = alpha[:, None] * acc + p @ v[b, j0:j1, g, :]
                m = m_new
            has = l > 0
            out[b, :, h, :] = np.where(has[:, None], acc / np.where(has, l, 1.0)[:, None], 0.0)
            lse[b, h, :] = np.where(has, m + np.log(np.where(has, l, 1.0)), NEG_INF)
    return out, lse


# ---------------------------------------------------------------------------
# backward: chain rule on the materialised tensors
# ---------------------------------------------------------------------------

@_masked_math
def attn_bwd(dout, q, k, v, scale=None, causal=False, window_left=-1, window_right=-1,
             softcap=0.0, alibi_slopes=None):
    """Gradients of L = sum(dout * O) with respect to q, k, v.

    Steps (per q-head h reading kv-head g):
      dV_g += P^T dO ; dP = dO V^T ; Delta_i = sum_j P_ij dP_ij ;
      dS = P * (dP - Delta) ; dU = dS * (1 - tanh^2(u/softcap)) when capped ;
      dQ = scale * dU K ; dK_g += scale * dU^T Q.
    The ALiBi bias is a constant of the inputs: it changes P, not the chain.
    Returns dq, dk, dv (f64, shapes of q, k, v) and Delta (B, Hq, Sq).
    """
    dout = np.asarray(dout, np.float64)
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = _check_heads(Hq, Hkv)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    delta = np.zeros((B, Hq, Sq))
    for h in range(Hq):
        g = h // G
        # forward of this head alone (same definition as attn_fwd)
        sl_h = None if alibi_slopes is None else head_slopes(alibi_slopes, B, h)[:, None]
        _, _, P, U = attn_fwd(q[:, :, h:h + 1], k[:, :, g:g + 1], v[:, :, g:g + 1], scale, causal,
                              window_left, window_right, softcap, return_probs=True, alibi_slopes=sl_h)
        Ph, Uh = P[:, 0], U[:, 0]                       # (B, Sq, Sk)
        del P, U
        dO = dout[:, :, h, :]                           # (B, Sq, D)
        dv[:, :, g, :] += np.matmul(Ph.transpose(0, 2, 1), dO)
        dP = np.matmul(dO, v[:, :, g, :].transpose(0, 2, 1))
        dl = (Ph * dP).sum(axis=2)                      # Delta
        dS = Ph * (dP - dl[:, :, None])
        del dP
        if softcap is not None and softcap > 0:
            t = np.tanh(Uh / softcap)
            dS = dS * (1.0 - t * t)
        dq[:, :, h, :] = scale * np.matmul(dS, k[:, :, g, :])
        dk[:, :, g, :] += scale * np.matmul(dS.transpose(0, 2, 1), q[:, :, h, :])
        delta[:, h, :] = dl
    return dq, dk, dv, delta


@_masked_math
def _bwd_row_terms(dout, q, k, v, b, h, rows, scale, causal, window_left, window_right, softcap,
                   alibi_slopes):
    """Per-row backward quantities of query ``rows`` of (batch b, q-head h),
    each row on its own with the definitions of :func:`attn_bwd`: the raw
    scores u against every key, P, dP = dO V^T, Delta = sum_j P dP and
    dU = P (dP - Delta) [* (1 - tanh^2(u/softcap))].  Returns (P, dU, LSE,
    Delta) with P and dU of shape (len(rows), Sk)."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    g = h // _check_heads(Hq, Hkv)
    rows = np.asarray(rows)
    Kg = np.asarray(k[b, :, g, :], np.float64)
    Vg = np.asarray(v[b, :, g, :], np.float64)
    u = scale * (np.asarray(q[b, rows, h, :], np.float64) @ Kg.T)      # (R, Sk)
    s = transform_scores(u, softcap)
    if alibi_slopes is not None:
        s = s + alibi_bias(head_slopes(alibi_slopes, B, h)[b], rows, Sq, Sk)
    vis = visible_rows(rows, Sq, Sk, causal, window_left, window_right)
    s = np.where(vis, s, NEG_INF)
    anyv = vis.any(axis=1)
    m = np.where(anyv, s.max(axis=1), 0.0)
    l = np.where(vis, np.exp(s - m[:, None]), 0.0).sum(axis=1)
    lse = np.where(anyv, m + np.log(np.where(anyv, l, 1.0)), NEG_INF)
    P = np.where(vis, np.exp(s - np.where(anyv, lse, 0.0)[:, None]), 0.0)
    dP = np.asarray(dout[b, rows, h, :], np.float64) @ Vg.T             # (R, Sk)
    delta = (P * dP).sum(axis=1)
    dU = P * (dP - delta[:, None])
    if softcap is not None and softcap > 0:
        t = np.tanh(u / softcap)
        dU = dU * (1.0 - t * t)
    return P, dU, lse, delta


def attn_bwd_rows(dout, q, k, v, b, h, rows, scale=None, causal=False, window_left=-1, window_right=-1,
                  softcap=0.0, alibi_slopes=None):
    """dQ of selected query rows of one (batch b, q-head h).

    dQ_i = scale * sum_j dU_ij K_j, with dU of the row from the chain rule of
    :func:`attn_bwd` (each row needs only its own scores).  Returns dq
    (len(rows), D), LSE and Delta (len(rows),).  Used to check gradients of
    problems too large to evaluate whole.
    """
    q = np.asarray(q)
    D = q.shape[3]
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    g = h // _check_heads(q.shape[2], k.shape[2])
    _, dU, lse, delta = _bwd_row_terms(dout, q, k, v, b, h, rows, scale, causal, window_left, window_right,
                                       softcap, alibi_slopes)
    dq = scale * (dU @ np.asarray(k[b, :, g, :], np.float64))
    return dq, lse, delta


def attn_bwd_cols(dout, q, k, v, b, g, cols, scale=None, causal=False, window_left=-1, window_right=-1,
                  softcap=0.0, alibi_slopes=None, row_chunk=1024):
    """dK and dV of selected key rows ``cols`` of one (batch b, kv-head g).

    dV_j = sum_{h in g} sum_i P_ij dO_i and dK_j = scale * sum_{h in g}
    sum_i dU_ij Q_i: the sums of :func:`attn_bwd` over every query row i of
    every q-head of the group.  A column needs the row statistics (LSE,
    Delta) of every query, so all rows are evaluated with the per-row
    definitions, ``row_chunk`` rows at a time to bound memory (the rows are
    independent; only the sums over i run across chunks).  Returns dk, dv
    (len(cols), D).
    """
    q = np.asarray(q)
    B, Sq, Hq, D = q.shape
    G = _check_heads(Hq, k.shape[2])
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    cols = np.asarray(cols)
    dk = np.zeros((len(cols), D))
    dv = np.zeros((len(cols), D))
    for h in range(g * G, (g + 1) * G):
        for r0 in range(0, Sq, row_chunk):
            rows = np.arange(r0, min(Sq, r0 + row_chunk))
            P, dU, _, _ = _bwd_row_terms(dout, q, k, v, b, h, rows, scale, causal, window_left, window_right,
                                         softcap, alibi_slopes)
            dv += P[:, cols].T @ np.asarray(dout[b, rows, h, :], np.float64)
            dk += scale * (dU[:, cols].T @ np.asarray(q[b, rows, h, :], np.float64))
    return dk, dv


# ---------------------------------------------------------------------------
# incremental decoding with a (paged) KV cache
# ---------------------------------------------------------------------------

def cache_slot(b, pos, block_table, page_size):
    """(page, slot) that holds token ``pos`` of sequence ``b``.

    Without a block table the cache is contiguous per sequence and the
    "page" is the sequence index itself.
    """
    if block_table is None:
        return b, pos
    return int(block_table[b, pos // page_size]), pos % page_size


def kvcache_append(k_cache, v_cache, k_new, v_new, cache_seqlens, block_table=None,
                   page_size=None):
    """Write k_new/v_new (B, Snew, Hkv, D) at positions cache_seqlens[b] + t.

    Returns new (k_cache, v_cache) arrays; the inputs are not modified.  The
    caches are (num_pages, page_size, Hkv, D) with a block table, else
    (B, max_seqlen, Hkv, D).
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    if k_new is None:
        return kc, vc
    B, Snew = k_new.shape[0], k_new.shape[1]
    for b in range(B):
        for t in range(Snew):
            page, slot = cache_slot(b, int(cache_seqlens[b]) + t, block_table, page_size)
            kc[page, slot] = k_new[b, t]
            vc[page, slot] = v_new[b, t]
    return kc, vc


def gather_cache(cache, b, L, block_table=None, page_size=None):
    """Contiguous (L, Hkv, D) view of the first L tokens of sequence b."""
    rows = [cache[cache_slot(b, pos, block_table, page_size)] for pos in range(L)]
    if not rows:
        return np.zeros((0,) + cache.shape[2:], dtype=np.float64)
    return np.stack(rows).astype(np.float64)


def rotary(x, cos, sin, positions, interleaved=False):
    """Rotary position embedding of the rows of ``x`` (..., R, H, D) at
    ``positions`` (..., R): the first ``r = 2 * cos.shape[1]`` dims of each
    head are rotated pairwise by angle theta[pos, j] with cos/sin[pos, j]
    given; non-interleaved pairs are (j, j + r/2), interleaved (2j, 2j+1).
    Dims past r are unchanged."""
    x = np.array(x, np.float64, copy=True)
    c = np.asarray(cos, np.float64)[np.asarray(positions)][..., None, :]  # (..., R, 1, r/2)
    s = np.asarray(sin, np.float64)[np.asarray(positions)][..., None, :]
    half = c.shape[-1]
    if interleaved:
        a, b = x[..., 0:2 * half:2].copy(), x[..., 1:2 * half:2].copy()
        x[..., 0:2 * half:2] = a * c - b * s
        x[..., 1:2 * half:2] = b * c + a * s
    else:
        a, b = x[..., :half].copy(), x[..., half:2 * half].copy()
        x[..., :half] = a * c - b * s
        x[..., half:2 * half] = b * c + a * s
    return x


@_masked_math
def attn_with_kvcache(q, k_cache, v_cache, k_new=None, v_new=None, cache_seqlens=None,
                      block_table=None, page_size=None, scale=None, causal=False,
                      window_left=-1, window_right=-1, softcap=0.0, rotary_cos=None, rotary_sin=None,
                      rotary_interleaved=False):
    """Append then attend: q (B, Sq, Hq, D) against each sequence's cache.

    Sequence b attends over L_b = cache_seqlens[b] + Snew keys (Snew = 0 when
    no new K/V is given), with the bottom-right alignment of
    :func:`visible`.  With rotary tables, new key row t of sequence b and
    query row i are first rotated (:func:`rotary`) at positions
    cache_seqlens[b] + t and cache_seqlens[b] + i (the queries are the new
    tokens'); the cache already holds rotated keys.  Returns O
    (B, Sq, Hq, D), LSE (B, Hq, Sq) and the updated caches.
    """
    q = np.asarray(q, np.float64)
    B, Sq, Hq, D = q.shape
    Snew = 0 if k_new is None else k_new.shape[1]
    if rotary_cos is not None:
        base = np.asarray(cache_seqlens, np.int64)[:, None]
        q = rotary(q, rotary_cos, rotary_sin, base + np.arange(Sq)[None, :], rotary_interleaved)
        if Snew:
            k_new = rotary(k_new, rotary_cos, rotary_sin, base + np.arange(Snew)[None, :], rotary_interleaved)
    kc, vc = kvcache_append(k_cache, v_cache, k_new, v_new, cache_seqlens, block_table, page_size)
    out = np.zeros((B, Sq, Hq, D))
    lse = np.full((B, Hq, Sq), NEG_INF)
    for b in range(B):
        L = int(cache_seqlens[b]) + Snew
        Kb = gather_cache(kc, b, L, block_table, page_size)[None]
        Vb = gather_cache(vc, b, L, block_table, page_size)[None]
        o, s = attn_fwd(q[b:b + 1], Kb, Vb, scale, causal, window_left, window_right, softcap)
        out[b] = o[0]
        lse[b] = s[0]
    return out, lse, kc, vc


# ---------------------------------------------------------------------------
# KV splits and their combination
# ---------------------------------------------------------------------------

def split_token_ranges(L, unit, num_splits):
    """Token range [t0, t1) of each of ``num_splits`` splits of L keys.

    The keys are grouped in units of ``unit`` tokens (the cache page); split
    s takes units ceil(s*P/n) .. ceil((s+1)*P/n) - 1 with P = ceil(L/unit).
    Splits may be empty.
    """
    P = -(-L // unit)
    out = []
    for s in range(num_splits):
        u0 = -(-(s * P) // num_splits)
        u1 = -(-((s + 1) * P) // num_splits)
        out.append((min(L, u0 * unit), min(L, u1 * unit)))
    return out


@_masked_math
def attn_partial(q, K, V, t0, t1, scale, causal=False, window_left=-1, window_right=-1,
                 softcap=0.0):
    """Attention of q (Sq, Hq, D) over keys [t0, t1) of K, V (L, Hkv, D).

    Masks use absolute positions in the full length L.  Returns the
    split-normalised partial output (Sq, Hq, D) and its LSE (Hq, Sq); an
    empty or fully masked split gives O = 0, LSE = -inf.
    """
    Sq, Hq, D = q.shape
    L, Hkv = K.shape[0], K.shape[1]
    G = _check_heads(Hq, Hkv)
    o = np.zeros((Sq, Hq, D))
    lse = np.full((Hq, Sq), NEG_INF)
    if t1 <= t0:
        return o, lse
    vis = visible(Sq, L, causal, window_left, window_right, key_offset=t0, n_keys=t1 - t0)
    for h in range(Hq):
        g = h // G
        u = scale * (q[:, h, :] @ K[t0:t1, g, :].T)
        s = np.where(vis, transform_scores(u, softcap), NEG_INF)
        anyv = vis.any(axis=1)
        m = np.where(anyv, s.max(axis=1), 0.0)
        e = np.where(vis, np.exp(s - m[:, None]), 0.0)
        l = e.sum(axis=1)
        o[:, h, :] = np.where(anyv[:, None], (e @ V[t0:t1, g, :]) / np.where(anyv, l, 1.0)[:, None], 0.0)
        lse[h] = np.where(anyv, m + np.log(np.where(anyv, l, 1.0)), NEG_INF)
    return o, lse


@_masked_math
def combine_splits(o_parts, lse_parts):
    """Merge split results: LSE = ln sum_s e^{LSE_s}; O = sum_s e^{LSE_s-LSE} O_s.

    o_parts (n, Sq, Hq, D); lse_parts (n, Hq, Sq).  All-empty rows give
    O = 0, LSE = -inf.
    """
    o_parts = np.asarray(o_parts, np.float64)
    lse_parts = np.asarray(lse_parts, np.float64)
    m = lse_parts.max(axis=0)                               # (Hq, Sq)
    finite = np.isfinite(m)
    w = np.where(finite[None], np.exp(lse_parts - np.where(finite, m, 0.0)[None]), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(finite, np.where(finite, m, 0.0) + np.log(np.where(finite, tot, 1.0)), NEG_INF)
    wn = np.where(finite[None], w / np.where(finite, tot, 1.0)[None], 0.0)  # (n, Hq, Sq)
    o = np.einsum("nhi,nihd->ihd", wn, o_parts)
    return o, lse


# ---------------------------------------------------------------------------
# variable-length (packed) batches
# ---------------------------------------------------------------------------

@_masked_math
def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale=None, causal=False, window_left=-1,
                    window_right=-1, softcap=0.0):
    """Packed batch: q (total_q, Hq, D), k/v (total_k, Hkv, D).  Every
    sequence b is the dense problem on its own token slices.  Returns O
    (total_q, Hq, D) and LSE (Hq, total_q)."""
    cq, ck = np.asarray(cu_seqlens_q), np.asarray(cu_seqlens_k)
    Hq = q.shape[1]
    out = np.zeros(q.shape, dtype=np.float64)
    lse = np.full((Hq, q.shape[0]), NEG_INF)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 == q0 or k1 == k0:
            continue  # no queries, or no keys: rows stay O = 0, LSE = -inf
        o_b, l_b = attn_fwd(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale, causal, window_left,
                            window_right, softcap)
        out[q0:q1] = o_b[0]
        lse[:, q0:q1] = l_b[0]
    return out, lse


@_masked_math
def attn_bwd_varlen(dout, q, k, v, cu_seqlens_q, cu_seqlens_k, scale=None, causal=False, window_left=-1,
                    window_right=-1, softcap=0.0):
    """Gradients of sum(dout * O) for a packed batch; each sequence is the
    dense backward on its own slices.  Returns dq, dk, dv in the packed
    layouts."""
    cq, ck = np.asarray(cu_seqlens_q), np.asarray(cu_seqlens_k)
    dq = np.zeros(q.shape, dtype=np.float64)
    dk = np.zeros(k.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = int(cq[b]), int(cq[b + 1]), int(ck[b]), int(ck[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        g = attn_bwd(dout[None, q0:q1], q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale, causal,
                     window_left, window_right, softcap)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = g[0][0], g[1][0], g[2][0]
    return dq, dk, dv


# ---------------------------------------------------------------------------
# FP8 (E4M3) forward
# ---------------------------------------------------------------------------

@_masked_math
def e4m3_decode(codes):
    """Float64 values of OCP FP8 E4M3 codes (uint8): sign in bit 7, a 4-bit
    exponent (bits 6..3, bias 7) and a 3-bit mantissa; exponent 0 holds the
    subnormals m * 2^-9; S.1111.111 is NaN and there is no infinity, so the
    largest finite magnitude is 1.75 * 2^8 = 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


@_masked_math
def attn_fwd_fp8(q8, k8, v8, descale_q=None, descale_k=None, descale_v=None, scale=None, causal=False,
                 window_left=-1, window_right=-1, softcap=0.0):
    """FP8 forward: q8 (B, Sq, Hq, D), k8/v8 (B, Sk, Hkv, D) E4M3 codes; the
    descales are (B, Hkv) float arrays or None (factor 1).  Returns O and
    LSE of :func:`attn_fwd` on the real inputs code * factor."""
    q = e4m3_decode(q8)
    k = e4m3_decode(k8)
    v = e4m3_decode(v8)
    B, Hq, Hkv = q.shape[0], q.shape[2], k.shape[2]
    G = _check_heads(Hq, Hkv)

    def fac(d, heads_per_factor, H):
        if d is None:
            return np.ones((B, 1, H, 1))
        d = np.asarray(d, np.float64).reshape(B, Hkv)
        return np.repeat(d, heads_per_factor, axis=1)[:, None, :, None]

    return attn_fwd(q * fac(descale_q, G, Hq), k * fac(descale_k, 1, Hkv), v * fac(descale_v, 1, Hkv), scale,
                    causal, window_left, window_right, softcap)


def e4m3_spacing(x):
    """Distance between adjacent E4M3 values around non-negative x (the OCP
    format of :func:`e4m3_decode`): 2^(e-3) for a normal value with exponent
    e (x >= 2^-6), 2^-9 in the subnormal range."""
    x = np.asarray(x, np.float64)
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -6)))
    return np.where(x >= 2.0 ** -6, np.exp2(e - 3.0), 2.0 ** -9)


@_masked_math
def fp8_p_rounding_sigma(q, k, v, b, h, rows, scale=None, causal=False, window_left=-1, window_right=-1,
                         softcap=0.0):
    """Scale of the output error that rounding the probabilities to E4M3
    introduces, per element of selected query rows of (batch b, q-head h).

    q, k, v are the real inputs (decoded codes times their factors).  An
    FP8 forward that forms O = sum_j R(P_j) v_j / sum_j R(P_j), with R the
    round-to-nearest onto E4M3 and P_j = c e^{s_j - max s} for some factor c,
    is off by sum_j (R(P_j) - P_j)(v_j - O) / sum_j R(P_j).  Each rounding
    error lies within half the E4M3 spacing u_j at P_j; taking the errors as
    independent and uniform (variance u_j^2 / 12) gives
        sigma_id = sqrt(sum_j u_j^2 / 12 (v_jd - O_id)^2) / sum_j P_j,
    evaluated here with c = 1 (the row's largest P equal to 1).  A factor
    c >= 1 never more than doubles u_j / c (normal values keep a relative
    spacing within [2^-4, 2^-3]; the fixed subnormal spacing only shrinks
    relative to c P_j), so 2 sigma bounds the scale for every c >= 1.
    Returns O (R, D), LSE (R,) and sigma (R, D).
    """
    q = np.asarray(q, np.float64)
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    g = h // _check_heads(Hq, Hkv)
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(D)
    rows = np.asarray(rows)
    Kg = np.asarray(k[b, :, g, :], np.float64)
    Vg = np.asarray(v[b, :, g, :], np.float64)
    s = transform_scores(scale * (q[b, rows, h, :] @ Kg.T), softcap)
    vis = visible_rows(rows, Sq, Sk, causal, window_left, window_right)
    s = np.where(vis, s, NEG_INF)
    anyv = vis.any(axis=1)
    m = np.where(anyv, s.max(axis=1), 0.0)
    P = np.where(vis, np.exp(s - m[:, None]), 0.0)                      # largest P of a row = 1
    l = np.where(anyv, P.sum(axis=1), 1.0)
    o = np.where(anyv[:, None], (P @ Vg) / l[:, None], 0.0)
    lse = np.where(anyv, m + np.log(l), NEG_INF)
    var = np.where(vis, e4m3_spacing(P) ** 2 / 12.0, 0.0)                # (R, Sk)
    sigma = np.zeros_like(o)
    for r in range(len(rows)):                                          # one row at a time: (Sk, D) terms
        sigma[r] = np.sqrt(var[r] @ (Vg - o[r]) ** 2) / l[r]
    return o, lse, sigma
