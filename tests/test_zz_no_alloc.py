"""fa_fwd_kvcache_noalloc, the decode entry point for callers that cannot
allocate device memory (a plugin inside a runtime that owns all device
memory, a serving loop with a fixed footprint): its split-KV partials live in
a fixed device array inside libfa.so instead of a caller workspace.

Checked through the C ABI against fa_fwd_kvcache (the workspace entry point)
on calls in a row with different inputs and split counts (explicit, one, and
the automatic choice), since the array keeps the previous call's contents.
"Allocates nothing" is checked twice: PyTorch's allocator counter and the
driver's free-memory figure (cudaMemGetInfo) are unchanged across a call.
The first call on the device is the set-up call: it looks up the array's
address, and with CUDA's lazy module loading (the default) that is when the
driver loads this part of the library's device image, array included; the
memory figures are compared on the calls after it.
Collected last so that a stop-at-first-failure run has already run every
other test; it also passes alone.
"""

import ctypes
import gc

import pytest
import torch

from _parity import check_lse, check_out, f64
from exact_attention_121_b200 import _lib, api, inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 * 1024 * 1024
DT = {torch.float16: _lib.FA_FP16, torch.bfloat16: _lib.FA_BF16}


def _device_case(seed, dtype="bf16"):
    d = inputs.kvcache_inputs(4, 32, 8, 128, 64, 6, 380, Sq=1, Snew=1, dtype=dtype, seed=seed)
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def _noalloc(lib, d, num_splits, out, lse):
    q = d["q"]
    B, Sq, Hq, D = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.fa_fwd_kvcache_noalloc(
        q.data_ptr(), d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["k_new"].data_ptr(),
        d["v_new"].data_ptr(), d["cache_seqlens"].data_ptr(), d["block_table"].data_ptr(), d["page_size"],
        d["block_table"].shape[1], d["k_cache"].shape[0], out.data_ptr(), lse.data_ptr(), B, Sq,
        d["k_new"].shape[1], Hq, d["k_cache"].shape[2], D, DT[q.dtype], 0.0, 1, -1, -1, 0.0, num_splits,
        ctypes.c_void_p(stream))


def _reference(d, num_splits):
    return api.fa_fwd_kvcache(d["q"], d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["cache_seqlens"],
                              d["block_table"], page_size=d["page_size"], causal=True, num_splits=num_splits)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = _lib.load()
    # set-up call (array address lookup, device image of the entry point)
    d0 = _device_case(30)
    assert _noalloc(lib, d0, 4, torch.empty_like(d0["q"]), torch.empty(4, 32, 1, device="cuda")) == _lib.FA_OK
    torch.cuda.synchronize()
    for seed, splits in ((31, 4), (32, 7), (34, 0), (35, 1)):
        d = _device_case(seed)
        ref_out, ref_lse = _reference(d, splits)
        out = torch.empty_like(d["q"])
        lse = torch.empty_like(ref_lse)
        torch.cuda.synchronize()
        # tensors that earlier tests left in reference cycles must not be
        # freed inside the measured call
        gc.collect()
        gc.disable()
        try:
            before = torch.cuda.memory_allocated()
            free_before = torch.cuda.mem_get_info()[0]
            code = _noalloc(lib, d, splits, out, lse)
            torch.cuda.synchronize()
            free_after = torch.cuda.mem_get_info()[0]
            after = torch.cuda.memory_allocated()
        finally:
            gc.enable()
        assert code == _lib.FA_OK, api.fa_status_string(code)
        assert api.fa_last_device_status() == 0
        assert after == before
        assert free_after == free_before, (free_before, free_after)
        check_out(out, f64(ref_out), torch.bfloat16)
        check_lse(lse, f64(ref_lse))


def test_noalloc_refuses_requests_beyond_the_array():
    lib = _lib.load()
    d = _device_case(33)
    out = torch.empty_like(d["q"])
    lse = torch.empty(4, 32, 1, device="cuda")
    # 64 splits x 4 x 32 x 1 rows of 128 fp32 partials = 4 MiB + 32 KiB: fits
    assert _noalloc(lib, d, 64, out, lse) == _lib.FA_OK
    # 16,384 rows x 516 bytes > 8 MiB: refused before any launch
    big = dict(d, q=torch.zeros(4, 2, 32, 128, dtype=torch.bfloat16, device="cuda"),
               k_new=torch.zeros(4, 2, 8, 128, dtype=torch.bfloat16, device="cuda"),
               v_new=torch.zeros(4, 2, 8, 128, dtype=torch.bfloat16, device="cuda"))
    out2 = torch.empty_like(big["q"])
    lse2 = torch.empty(4, 32, 2, device="cuda")
    assert _noalloc(lib, big, 64, out2, lse2) == _lib.FA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0


def test_noalloc_automatic_splits_fit_the_array():
    """A shape whose automatic split count would need more partial rows than
    the array holds (16 sequences x 32 heads x 16 queries) runs with the
    largest count that fits instead of being refused."""
    lib = _lib.load()
    d = inputs.kvcache_inputs(16, 32, 8, 128, 64, 4, 200, Sq=16, Snew=16, dtype="bf16", seed=36)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ref_out, ref_lse = _reference(d, 0)
    out = torch.empty_like(d["q"])
    lse = torch.empty_like(ref_lse)
    assert _noalloc(lib, d, 0, out, lse) == _lib.FA_OK
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == 0
    check_out(out, f64(ref_out), torch.bfloat16)
    check_lse(lse, f64(ref_lse))


def test_noalloc_matches_the_oracle():
    """O, LSE and the appended cache rows of the allocation-free call against
    the float64 oracle (append, then attend), at an explicit and at the
    automatic split count, for fp16 and bf16."""
    import oracle
    import numpy as np

    lib = _lib.load()
    for seed, splits, dtype in ((37, 3, "bf16"), (38, 0, "fp16")):
        host = inputs.kvcache_inputs(4, 32, 8, 128, 64, 6, 380, Sq=1, Snew=1, dtype=dtype, seed=seed)
        d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in host.items()}
        out = torch.empty_like(d["q"])
        lse = torch.empty(4, 32, 1, device="cuda")
        assert _noalloc(lib, d, splits, out, lse) == _lib.FA_OK
        torch.cuda.synchronize()
        assert api.fa_last_device_status() == 0
        o_ref, l_ref, kc_ref, vc_ref = oracle.attn_with_kvcache(
            host["q"].double().numpy(), host["k_cache"].double().numpy(), host["v_cache"].double().numpy(),
            host["k_new"].double().numpy(), host["v_new"].double().numpy(), host["cache_seqlens"].numpy(),
            host["block_table"].numpy(), host["page_size"], causal=True)
        check_out(out, o_ref, host["q"].dtype)
        check_lse(lse, l_ref)
        # the appended rows are exact copies of k_new / v_new
        assert np.array_equal(d["k_cache"].double().cpu().numpy(), kc_ref)
        assert np.array_equal(d["v_cache"].double().cpu().numpy(), vc_ref)
