"""Thin PyTorch-facing binding of libfa.so with the C entry points' names.

PyTorch supplies device memory and the current CUDA stream; every step of the
computation runs in the library's kernels.  Tensors are (batch, seqlen,
nheads, headdim), contiguous, fp16 or bf16, on one CUDA device.  There is no
CPU or fallback path: if libfa.so is missing, the import of ``_lib`` fails.
"""

import ctypes

import torch

from . import _lib

_DT = {torch.float16: _lib.FA_FP16, torch.bfloat16: _lib.FA_BF16}


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check_tensor(t, name, dtype=None, device=None, strided=False):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if strided:
        if t.dim() != 4 or t.stride(3) != 1:
            raise ValueError(f"{name} must be (B, S, H, D) with a contiguous last dimension")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _window(window):
    wl, wr = (-1, -1) if window is None else window
    return int(wl), int(wr)


def fa_status_string(code):
    return _lib.load().fa_status_string(int(code)).decode()


def fa_set_fwd_kernel(which):
    """0 = automatic (tcgen05 where it applies), 1 = force the mma.sync kernel."""
    _lib.load().fa_set_fwd_kernel(int(which))


def fa_last_launch_count():
    return int(_lib.load().fa_last_launch_count())


def _stride_array(tensors):
    """(batch, token, head) element strides of (B, S, H, D) tensors, as int64."""
    vals = [int(x) for t in tensors for x in t.stride()[:3]]
    return (ctypes.c_longlong * len(vals))(*vals)


def _alibi(slopes, B, Hq, device):
    """(pointer, batch stride) of ALiBi slopes: float32 (Hq,) or (B, Hq)."""
    if slopes.dtype != torch.float32 or slopes.device != device:
        raise ValueError("alibi_slopes must be a float32 tensor on the device of q")
    if slopes.dim() == 1 and slopes.shape == (Hq,) and slopes.is_contiguous():
        return _ptr(slopes), 0
    if slopes.dim() == 2 and slopes.shape == (B, Hq) and slopes.stride(1) == 1:
        return _ptr(slopes), slopes.stride(0)
    raise ValueError(f"alibi_slopes must be ({Hq},) or ({B}, {Hq}) with contiguous heads")


def fa_fwd(q, k, v, out=None, lse=None, scale=None, causal=False, window=(-1, -1), softcap=0.0,
           stream=None, alibi_slopes=None):
    """Forward attention; returns (out, lse).  lse is fp32 (B, Hq, Sq).

    q, k, v (and out) may be views with any strides as long as the head
    dimension is contiguous (e.g. slices of a packed qkv tensor); those go
    through fa_fwd_strided.  ``alibi_slopes`` (float32 (Hq,) or (B, Hq))
    adds the ALiBi bias through fa_fwd_alibi."""
    lib = _lib.load()
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check_tensor(t, n, dt, q.device, strided=True)
    if out is None:
        out = torch.empty(q.shape, dtype=dt, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _check_tensor(lse, "lse", torch.float32, q.device)
    wl, wr = _window(window)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv, D, _DT[dt], float(scale or 0.0),
            int(bool(causal)), wl, wr, float(softcap or 0.0))
    packed = all(t.is_contiguous() for t in (q, k, v, out))
    if alibi_slopes is not None:
        ap, ab = _alibi(alibi_slopes, B, Hq, q.device)
        code = lib.fa_fwd_alibi(*args, None if packed else _stride_array((q, k, v, out)), ap, ab, _stream(stream))
        _lib.check(code, "fa_fwd_alibi")
    elif packed:
        code = lib.fa_fwd(*args, _stream(stream))
        _lib.check(code, "fa_fwd")
    else:
        code = lib.fa_fwd_strided(*args, _stride_array((q, k, v, out)), _stream(stream))
        _lib.check(code, "fa_fwd_strided")
    return out, lse


def fa_fwd_fp8(q, k, v, descale_q=None, descale_k=None, descale_v=None, out=None, lse=None, scale=None,
               causal=False, window=(-1, -1), softcap=0.0, stream=None):
    """FP8 forward: q, k, v torch.float8_e4m3fn (B, S, H, D), head dim 64 or 128;
    descales float32 (B, Hkv) or None.  Returns (out bf16, lse fp32)."""
    lib = _lib.load()
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_tensor(t, n, torch.float8_e4m3fn, q.device)
    for t, n in ((descale_q, "descale_q"), (descale_k, "descale_k"), (descale_v, "descale_v")):
        _check_tensor(t, n, torch.float32, q.device)
        if t is not None and t.shape != (B, Hkv):
            raise ValueError(f"{n} must be ({B}, {Hkv})")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    _check_tensor(out, "out", torch.bfloat16, q.device)
    _check_tensor(lse, "lse", torch.float32, q.device)
    wl, wr = _window(window)
    code = lib.fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Sq, Sk, Hq, Hkv, D,
                          _ptr(descale_q), _ptr(descale_k), _ptr(descale_v), float(scale or 0.0),
                          int(bool(causal)), wl, wr, float(softcap or 0.0), _stream(stream))
    _lib.check(code, "fa_fwd_fp8")
    return out, lse


def fa_bwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, deterministic=False):
    return int(_lib.load().fa_bwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, int(bool(deterministic))))


def fa_bwd(dout, q, k, v, out, lse, dq=None, dk=None, dv=None, scale=None, causal=False,
           window=(-1, -1), softcap=0.0, deterministic=False, workspace=None, stream=None, alibi_slopes=None):
    """Backward attention; returns (dq, dk, dv).  ``alibi_slopes`` as in
    :func:`fa_fwd` (the same slopes the forward used)."""
    lib = _lib.load()
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    dt = q.dtype
    for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _check_tensor(t, n, dt, q.device, strided=True)
    _check_tensor(lse, "lse", torch.float32, q.device)
    dq = torch.empty(q.shape, dtype=dt, device=q.device) if dq is None else dq
    dk = torch.empty(k.shape, dtype=dt, device=q.device) if dk is None else dk
    dv = torch.empty(v.shape, dtype=dt, device=q.device) if dv is None else dv
    need = fa_bwd_workspace_size(B, Sq, Sk, Hq, Hkv, D, deterministic)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    wl, wr = _window(window)
    args = (_ptr(dout), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, Sq, Sk,
            Hq, Hkv, D, _DT[dt], float(scale or 0.0), int(bool(causal)), wl, wr, float(softcap or 0.0),
            int(bool(deterministic)), _ptr(workspace), workspace.numel())
    tensors = (dout, q, k, v, out, dq, dk, dv)
    packed = all(t.is_contiguous() for t in tensors)
    if alibi_slopes is not None:
        ap, ab = _alibi(alibi_slopes, B, Hq, q.device)
        code = lib.fa_bwd_alibi(*args, None if packed else _stride_array(tensors), ap, ab, _stream(stream))
        _lib.check(code, "fa_bwd_alibi")
    elif packed:
        code = lib.fa_bwd(*args, _stream(stream))
        _lib.check(code, "fa_bwd")
    else:
        code = lib.fa_bwd_strided(*args, _stride_array(tensors), _stream(stream))
        _lib.check(code, "fa_bwd_strided")
    return dq, dk, dv


def fa_fwd_qkvpacked(qkv, **kw):
    """Forward attention on a packed (B, S, 3, H, D) tensor; returns (out, lse)."""
    q, k, v = qkv.unbind(2)
    return fa_fwd(q, k, v, **kw)


def fa_bwd_qkvpacked(dout, qkv, out, lse, dqkv=None, **kw):
    """Backward of :func:`fa_fwd_qkvpacked`; returns dqkv (B, S, 3, H, D)."""
    q, k, v = qkv.unbind(2)
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    dq, dk, dv = dqkv.unbind(2)
    fa_bwd(dout, q, k, v, out, lse, dq=dq, dk=dk, dv=dv, **kw)
    return dqkv


def _cu(t, name, device):
    if t.dtype != torch.int32 or t.dim() != 1:
        raise ValueError(f"{name} must be a 1-D int32 tensor")
    _check_tensor(t, name, torch.int32, device)


def fa_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, out=None, lse=None,
                  scale=None, causal=False, window=(-1, -1), softcap=0.0, stream=None):
    """Forward attention on a packed batch: q (total_q, Hq, D), k/v (total_k,
    Hkv, D), cu_seqlens_* (B+1) int32 device offsets.  Returns (out, lse), lse
    fp32 (Hq, total_q)."""
    lib = _lib.load()
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    dt = q.dtype
    if dt not in _DT:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out")):
        _check_tensor(t, n, dt, q.device)
    _cu(cu_seqlens_q, "cu_seqlens_q", q.device)
    _cu(cu_seqlens_k, "cu_seqlens_k", q.device)
    if cu_seqlens_k.numel() != B + 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k differ in length")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((Hq, total_q), dtype=torch.float32, device=q.device)
    _check_tensor(lse, "lse", torch.float32, q.device)
    wl, wr = _window(window)
    code = lib.fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                             _ptr(cu_seqlens_k), B, int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, Hq,
                             Hkv, D, _DT[dt], float(scale or 0.0), int(bool(causal)), wl, wr,
                             float(softcap or 0.0), _stream(stream))
    _lib.check(code, "fa_fwd_varlen")
    return out, lse


def fa_bwd_varlen_workspace_size(B, max_seqlen_q, total_q, Hq, D, deterministic=False):
    return int(_lib.load().fa_bwd_varlen_workspace_size(B, max_seqlen_q, total_q, Hq, D, int(bool(deterministic))))


def fa_bwd_varlen(dout, q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, dq=None,
                  dk=None, dv=None, scale=None, causal=False, window=(-1, -1), softcap=0.0, deterministic=False,
                  workspace=None, stream=None):
    """Backward of :func:`fa_fwd_varlen`; returns (dq, dk, dv)."""
    lib = _lib.load()
    total_q, Hq, D = q.shape
    total_k, Hkv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    dt = q.dtype
    for t, n in ((dout, "dout"), (q, "q"), (k, "k"), (v, "v"), (out, "out"), (dq, "dq"), (dk, "dk"),
                 (dv, "dv")):
        _check_tensor(t, n, dt, q.device)
    _check_tensor(lse, "lse", torch.float32, q.device)
    _cu(cu_seqlens_q, "cu_seqlens_q", q.device)
    _cu(cu_seqlens_k, "cu_seqlens_k", q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = fa_bwd_varlen_workspace_size(B, max_seqlen_q, total_q, Hq, D, deterministic)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    wl, wr = _window(window)
    code = lib.fa_bwd_varlen(_ptr(dout), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dq), _ptr(dk),
                             _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, int(max_seqlen_q),
                             int(max_seqlen_k), total_q, total_k, Hq, Hkv, D, _DT[dt], float(scale or 0.0),
                             int(bool(causal)), wl, wr, float(softcap or 0.0), int(bool(deterministic)),
                             _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(code, "fa_bwd_varlen")
    return dq, dk, dv


def fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits):
    return int(_lib.load().fa_kvcache_workspace_size(B, Sq, Hq, D, int(num_splits)))


def fa_kvcache_rotary_workspace_size(B, Sq, Hq, D, num_splits):
    return int(_lib.load().fa_kvcache_rotary_workspace_size(B, Sq, Hq, D, num_splits))


def fa_fwd_kvcache(q, k_cache, v_cache, k_new=None, v_new=None, cache_seqlens=None, block_table=None,
                   page_size=256, out=None, lse=None, scale=None, causal=False, window=(-1, -1),
                   softcap=0.0, num_splits=0, workspace=None, stream=None, return_lse=True, rotary_cos=None,
                   rotary_sin=None, rotary_interleaved=False):
    """Append k_new/v_new into the cache (in place), then attend; returns (out, lse).

    Paged when ``block_table`` (B, max_pages_per_seq) int32 is given: caches
    are (num_pages, page_size, Hkv, D).  Otherwise caches are
    (B, max_seqlen, Hkv, D).  ``cache_seqlens`` (B,) int32 is the length
    before the append and is not modified.  ``rotary_cos``/``rotary_sin``
    (seqlen_ro, rotary_dim/2) float32 tables rotate the new keys and the
    queries at positions cache_seqlens[b] + t (fa_fwd_kvcache_rotary).
    """
    lib = _lib.load()
    B, Sq, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    dt = q.dtype
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (k_new, "k_new"),
                 (v_new, "v_new"), (out, "out")):
        _check_tensor(t, n, dt, q.device)
    _check_tensor(cache_seqlens, "cache_seqlens", torch.int32, q.device)
    _check_tensor(block_table, "block_table", torch.int32, q.device)
    Snew = 0 if k_new is None else k_new.shape[1]
    if block_table is not None:
        max_pages_per_seq = block_table.shape[1]
        cap = k_cache.shape[0]
        page_size = k_cache.shape[1]
    else:
        max_pages_per_seq = 0
        cap = k_cache.shape[1]
    out = torch.empty_like(q) if out is None else out
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    wl, wr = _window(window)
    head = (_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_new), _ptr(v_new), _ptr(cache_seqlens), _ptr(block_table),
            int(page_size), int(max_pages_per_seq), int(cap), _ptr(out), _ptr(lse), B, Sq, Snew, Hq, Hkv, D, _DT[dt],
            float(scale or 0.0), int(bool(causal)), wl, wr, float(softcap or 0.0))
    if rotary_cos is None:
        need = fa_kvcache_workspace_size(B, Sq, Hq, D, num_splits)
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        code = lib.fa_fwd_kvcache(*head, int(num_splits), _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream))
        _lib.check(code, "fa_fwd_kvcache")
        return out, lse
    for t, n in ((rotary_cos, "rotary_cos"), (rotary_sin, "rotary_sin")):
        _check_tensor(t, n, torch.float32, q.device)
    if rotary_cos.shape != rotary_sin.shape or rotary_cos.dim() != 2:
        raise ValueError("rotary_cos and rotary_sin must be (seqlen_ro, rotary_dim/2) float32")
    need = int(lib.fa_kvcache_rotary_workspace_size(B, Sq, Hq, D, num_splits))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    code = lib.fa_fwd_kvcache_rotary(*head, _ptr(rotary_cos), _ptr(rotary_sin), 2 * rotary_cos.shape[1],
                                     rotary_cos.shape[0], int(bool(rotary_interleaved)), int(num_splits),
                                     _ptr(workspace), workspace.numel(), _stream(stream))
    _lib.check(code, "fa_fwd_kvcache_rotary")
    return out, lse


def fa_last_device_status(stream=None):
    """Wait for the stream; return and clear the device status word (an int)."""
    return int(_lib.load().fa_last_device_status(_stream(stream)))
