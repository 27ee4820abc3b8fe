"""Seeded synthetic inputs shared by the tests, the bench and the oracle legs.

This module only draws random numbers and builds index tables; it holds none
of the attention arithmetic.  Everything is drawn on the CPU with a
``torch.Generator`` so that the GPU RNG is never involved: the same host
tensor is copied to the device for the kernels and upcast to float64 for the
oracle.

Workload recipes follow the pages' benchmark setting (FP16/BF16, head dim 64
and 128, hidden size 2048, sequence length 512 to 16k) and the paged-decode
example; the draw order is fixed: Q, K, V, then dO.
"""

import math

import torch

DTYPES = {"fp16": torch.float16, "bf16": torch.bfloat16}


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def randn(shape, gen, dtype, amp=1.0):
    """i.i.d. N(0, amp^2) drawn in fp32 then rounded to ``dtype``."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if amp != 1.0:
        x.mul_(amp)
    return x.to(dtype)


def attention_inputs(B, Sq, Sk, Hq, Hkv, D, dtype="bf16", seed=0, amp=1.0, with_dout=True,
                     pin=False):
    """(q, k, v, dout) host tensors in (batch, seqlen, nheads, headdim) layout."""
    dt = DTYPES[dtype] if isinstance(dtype, str) else dtype
    g = _gen(seed)
    q = randn((B, Sq, Hq, D), g, dt, amp)
    k = randn((B, Sk, Hkv, D), g, dt, amp)
    v = randn((B, Sk, Hkv, D), g, dt, amp)
    dout = randn((B, Sq, Hq, D), g, dt, amp) if with_dout else None
    if pin:
        q, k, v = q.pin_memory(), k.pin_memory(), v.pin_memory()
        dout = dout.pin_memory() if dout is not None else None
    return q, k, v, dout


def alibi_slopes(Hq, B=None, seed=None):
    """ALiBi slopes, float32: the geometric sequence 2^(-8 (h+1) / Hq) of
    the ALiBi paper shared by the batch (shape (Hq,)), or with ``B`` and
    ``seed`` seeded draws U(0, 1) per (batch row, head) (shape (B, Hq))."""
    if B is None:
        return torch.tensor([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=torch.float32)
    return torch.rand((B, Hq), generator=_gen(seed), dtype=torch.float32)


def rotary_tables(n_pos, rotary_dim, base=10000.0):
    """Float32 (n_pos, rotary_dim/2) cos/sin tables of the usual rotary
    frequencies base^(-2j/rotary_dim) at positions 0..n_pos-1 (inputs of the
    kvcache call, like the caches; no draws)."""
    half = rotary_dim // 2
    inv = base ** (-torch.arange(half, dtype=torch.float64) / half)
    ang = torch.arange(n_pos, dtype=torch.float64)[:, None] * inv[None, :]
    return torch.cos(ang).float(), torch.sin(ang).float()


def kvcache_inputs(B, Hq, Hkv, D, page_size, pages_per_seq, max_len, Sq=1, Snew=1,
                   dtype="bf16", seed=5, num_pages=None, paged=True, min_len=1,
                   seqlens=None):
    """Paged (or contiguous) KV-cache decode inputs.

    Draw order: cache_seqlens ~ U{min_len..max_len}, the block-table
    permutation, q, k_new, v_new, k_cache, v_cache.  With ``paged`` the pool
    holds ``num_pages`` (default B * pages_per_seq) pages of shape
    (page_size, Hkv, D) and the block table is a random permutation of the
    physical pages reshaped to (B, pages_per_seq); otherwise the cache is
    (B, pages_per_seq * page_size, Hkv, D) and the block table is None.
    """
    dt = DTYPES[dtype] if isinstance(dtype, str) else dtype
    g = _gen(seed)
    if seqlens is None:
        seqlens = torch.randint(min_len, max_len + 1, (B,), generator=g, dtype=torch.int32)
    else:
        seqlens = torch.as_tensor(seqlens, dtype=torch.int32)
    if num_pages is None:
        num_pages = B * pages_per_seq
    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    block_table = perm[: B * pages_per_seq].reshape(B, pages_per_seq).contiguous() if paged else None
    q = randn((B, Sq, Hq, D), g, dt)
    k_new = randn((B, Snew, Hkv, D), g, dt) if Snew > 0 else None
    v_new = randn((B, Snew, Hkv, D), g, dt) if Snew > 0 else None
    if paged:
        cache_shape = (num_pages, page_size, Hkv, D)
    else:
        cache_shape = (B, pages_per_seq * page_size, Hkv, D)
    k_cache = randn(cache_shape, g, dt)
    v_cache = randn(cache_shape, g, dt)
    return dict(q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                cache_seqlens=seqlens, block_table=block_table, page_size=page_size,
                pages_per_seq=pages_per_seq)


# ---------------------------------------------------------------------------
# the five workloads (names describe what they are)
# ---------------------------------------------------------------------------

def tiny_fwd_config():
    """B=1, Hq=Hkv=2, S=128, D=64, fp16, non-causal, scale 1/8, seed 1."""
    return dict(B=1, Sq=128, Sk=128, Hq=2, Hkv=2, D=64, dtype="fp16", causal=False,
                window=(-1, -1), softcap=0.0, scale=1.0 / 8.0, seed=1, amp=1.0)


def fwd_bwd_512_config():
    """B=2, S=512, Hq=Hkv=16, D=64, fp16, causal, seed 2."""
    return dict(B=2, Sq=512, Sk=512, Hq=16, Hkv=16, D=64, dtype="fp16", causal=True,
                window=(-1, -1), softcap=0.0, scale=1.0 / 8.0, seed=2, amp=1.0)


def seqlen_sweep_configs():
    """Hidden 2048: (H=32, D=64) and (H=16, D=128), S in 512..16k, B=16384/S."""
    out = []
    idx = 0
    for H, D in ((32, 64), (16, 128)):
        for S in (512, 1024, 2048, 4096, 8192, 16384):
            for causal in (False, True):
                out.append(dict(B=16384 // S, Sq=S, Sk=S, Hq=H, Hkv=H, D=D, dtype="bf16",
                                causal=causal, window=(-1, -1), softcap=0.0,
                                scale=1.0 / math.sqrt(D), seed=300 + idx, amp=1.0))
                idx += 1
    return out


def long_context_configs():
    """One 32k-token sequence at hidden 2048: (H=16, D=128) causal and
    (H=32, D=64) non-causal, twice the longest sweep point."""
    return [dict(B=1, Sq=32768, Sk=32768, Hq=H, Hkv=H, D=D, dtype="bf16", causal=causal,
                 window=(-1, -1), softcap=0.0, scale=1.0 / math.sqrt(D), seed=seed, amp=1.0)
            for H, D, causal, seed in ((16, 128, True, 401), (32, 64, False, 402))]


def gqa_local_config():
    """B=2, S=4096, Hq=32, Hkv=8, D=128, bf16, causal, window (1024,0), softcap 30, x2."""
    return dict(B=2, Sq=4096, Sk=4096, Hq=32, Hkv=8, D=128, dtype="bf16", causal=True,
                window=(1024, 0), softcap=30.0, scale=1.0 / math.sqrt(128), seed=4, amp=2.0)


def paged_decode_config():
    """B=8, Hq=32, Hkv=8, D=128, bf16, Sq=Snew=1, lengths U[1,32768], page 256."""
    return dict(B=8, Hq=32, Hkv=8, D=128, dtype="bf16", page_size=256, pages_per_seq=129,
                max_len=32768, Sq=1, Snew=1, causal=True, seed=5,
                scale=1.0 / math.sqrt(128))


def varlen_lengths(B, min_len, max_len, seed):
    """B sequence lengths drawn U{min_len..max_len} (a packed batch's mix)."""
    g = _gen(seed)
    return torch.randint(min_len, max_len + 1, (B,), generator=g).tolist()


def varlen_inputs(lens_q, lens_k, Hq, Hkv, D, dtype="bf16", seed=0, amp=1.0):
    """Packed (q, k, v, dout) host tensors (total, nheads, headdim) and the
    (B+1) int32 cu_seqlens offsets of the query and key sequences."""
    dt = DTYPES[dtype] if isinstance(dtype, str) else dtype
    g = _gen(seed)
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    q = randn((tq, Hq, D), g, dt, amp)
    k = randn((tk, Hkv, D), g, dt, amp)
    v = randn((tk, Hkv, D), g, dt, amp)
    dout = randn((tq, Hq, D), g, dt, amp)
    cu_q = torch.tensor([0] + list(torch.tensor(lens_q).cumsum(0).tolist()), dtype=torch.int32)
    cu_k = torch.tensor([0] + list(torch.tensor(lens_k).cumsum(0).tolist()), dtype=torch.int32)
    return q, k, v, dout, cu_q, cu_k


def varlen_config():
    """Packed training batch at hidden 2048 (Hq=Hkv=16, D=128, bf16, causal):
    32 sequences with lengths U{64..1024} (seed 6), as a document-packing mix."""
    lens = varlen_lengths(32, 64, 1024, seed=6)
    return dict(lens=lens, Hq=16, Hkv=16, D=128, dtype="bf16", causal=True, window=(-1, -1), softcap=0.0,
                scale=1.0 / math.sqrt(128), seed=7, amp=1.0)


def alibi_config():
    """ALiBi at hidden 2048: B=4, S=4096, Hq=Hkv=16, D=128, bf16, causal, the
    geometric slopes of :func:`alibi_slopes`; the shape of the seqlen-sweep
    point H16 D128 S4096 causal (seed 8)."""
    return dict(B=4, Sq=4096, Sk=4096, Hq=16, Hkv=16, D=128, dtype="bf16", causal=True, window=(-1, -1),
                softcap=0.0, scale=1.0 / math.sqrt(128), seed=8, amp=1.0, alibi=True)


def paged_decode_rotary_config():
    """The paged-decode workload with rotary tables over the full head dim
    (halves pairing, base 10000, positions up to 32768 + 1)."""
    cfg = paged_decode_config()
    cfg["rotary"] = True
    return cfg


def fp8_inputs(B, Sq, Sk, Hq, Hkv, D, seed=0, amp=1.0):
    """E4M3 q, k, v (torch.float8_e4m3fn, rounded from N(0, amp^2) draws in
    the order q, k, v) and float32 (B, Hkv) descale factors U(0.5, 2) for q,
    k, v, drawn after them."""
    g = _gen(seed)
    q = (amp * torch.randn((B, Sq, Hq, D), generator=g)).to(torch.float8_e4m3fn)
    k = (amp * torch.randn((B, Sk, Hkv, D), generator=g)).to(torch.float8_e4m3fn)
    v = (amp * torch.randn((B, Sk, Hkv, D), generator=g)).to(torch.float8_e4m3fn)
    d = [0.5 + 1.5 * torch.rand((B, Hkv), generator=g) for _ in range(3)]
    return q, k, v, d[0], d[1], d[2]


def fp8_config():
    """FP8 forward at hidden 2048: B=4, S=4096, Hq=Hkv=16, D=128, non-causal,
    N(0,1) inputs rounded to E4M3 with U(0.5, 2) descales (seed 9)."""
    return dict(B=4, Sq=4096, Sk=4096, Hq=16, Hkv=16, D=128, causal=False, window=(-1, -1), softcap=0.0,
                scale=1.0 / math.sqrt(128), seed=9, amp=1.0)
