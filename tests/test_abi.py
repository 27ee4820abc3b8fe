"""The C ABI without a GPU: libfa.so loads, exports every symbol include/fa.h
declares with the declared arity, and rejects bad arguments on the host
before touching CUDA.  Workspace sizes are linear in the sequence length."""

import ctypes
import os
import re

import pytest

from exact_attention_121_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def _declarations():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for m in re.finditer(r"^\s*(?:const\s+char\s*\*|fa_status|size_t|void|int)\s+(fa_\w+)\s*\(([^)]*)\)\s*;",
                         text, flags=re.M):
        args = m.group(2).strip()
        n = 0 if args in ("", "void") else len(args.split(","))
        decls[m.group(1)] = n
    return decls


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_entry_points():
    d = _declarations()
    for name in ("fa_fwd", "fa_bwd", "fa_fwd_kvcache", "fa_bwd_workspace_size",
                 "fa_kvcache_workspace_size", "fa_status_string", "fa_last_device_status"):
        assert name in d


def test_every_declared_symbol_is_exported_with_its_arity(lib):
    d = _declarations()
    assert set(d) == set(_lib.SIGNATURES), set(d) ^ set(_lib.SIGNATURES)
    for name, nargs in d.items():
        assert hasattr(lib, name), name
        assert len(_lib.SIGNATURES[name][1]) == nargs, name


def _ctype_of(param):
    """ctypes class a C parameter declaration binds to: pointers (and the
    stream handle) as c_void_p, float as c_float, size_t as c_size_t, int
    and the enums as c_int."""
    decl = param.strip()
    if "*" in decl or decl.startswith("fa_stream_t"):
        return ctypes.c_void_p
    words = decl.replace("const ", "").split()
    base = " ".join(words[:-1])
    return {"float": ctypes.c_float, "size_t": ctypes.c_size_t, "int": ctypes.c_int, "fa_dtype": ctypes.c_int,
            "fa_status": ctypes.c_int, "long long": ctypes.c_longlong}[base]


def test_every_binding_matches_the_declared_parameter_types():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    seen = 0
    for m in re.finditer(r"^\s*(?:const\s+char\s*\*|fa_status|size_t|void|int)\s+(fa_\w+)\s*\(([^)]*)\)\s*;",
                         text, flags=re.M):
        args = m.group(2).strip()
        params = [] if args in ("", "void") else args.split(",")
        want = [_ctype_of(a) for a in params]
        got = _lib.SIGNATURES[m.group(1)][1]
        assert got == want, (m.group(1), [t.__name__ for t in got], [t.__name__ for t in want])
        seen += 1
    assert seen == len(_lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.fa_status_string(0) == b"FA_OK"
    assert lib.fa_status_string(4) == b"FA_ERR_TIMEOUT"
    assert lib.fa_status_string(5) == b"FA_ERR_BOUNDS"
    assert lib.fa_status_string(99) == b"FA_ERR_UNKNOWN"


def _fwd(lib, ptr=0x1000, B=1, Sq=8, Sk=8, Hq=2, Hkv=2, D=64, dt=1, scale=0.0, softcap=0.0):
    p = ctypes.c_void_p(ptr)
    return lib.fa_fwd(p, p, p, p, p, B, Sq, Sk, Hq, Hkv, D, dt, scale, 0, -1, -1, softcap, None)


def test_host_validation_rejects_before_launch(lib):
    assert _fwd(lib, Hq=3, Hkv=2) == _lib.FA_ERR_INVALID_ARG      # GQA needs Hq % Hkv == 0
    assert _fwd(lib, D=96) == _lib.FA_ERR_UNSUPPORTED
    assert _fwd(lib, dt=7) == _lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, ptr=0x1008) == _lib.FA_ERR_INVALID_ARG       # not 16-byte aligned
    assert _fwd(lib, ptr=0) == _lib.FA_ERR_INVALID_ARG            # null pointers
    assert _fwd(lib, scale=float("nan")) == _lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=-1) == _lib.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=0) == _lib.FA_OK                            # empty batch: no-op
    assert _fwd(lib, Sq=0) == _lib.FA_OK


def test_bwd_rejects_short_workspace(lib):
    p = ctypes.c_void_p(0x1000)
    need = lib.fa_bwd_workspace_size(1, 64, 64, 2, 2, 64, 0)
    assert need > 0
    code = lib.fa_bwd(p, p, p, p, p, p, p, p, p, 1, 64, 64, 2, 2, 64, 1, 0.0, 0, -1, -1, 0.0, 0,
                      ctypes.c_void_p(0x10000), need - 1, None)
    assert code == _lib.FA_ERR_INVALID_ARG


def test_kvcache_rejects_bad_split_count_and_pages(lib):
    p = ctypes.c_void_p(0x1000)
    args = [p, p, p, p, p, p, p, 256, 4, 8, p, p, 2, 1, 1, 8, 2, 128, 1, 0.0, 1, -1, -1, 0.0]
    assert lib.fa_fwd_kvcache(*args, _lib.FA_MAX_SPLITS + 1, p, 0, None) == _lib.FA_ERR_INVALID_ARG
    bad = list(args)
    bad[7] = 0  # page_size
    assert lib.fa_fwd_kvcache(*bad, 1, p, 0, None) == _lib.FA_ERR_INVALID_ARG
    gqa = list(args)
    gqa[15] = 3  # Hkv does not divide Hq=8
    assert lib.fa_fwd_kvcache(*gqa, 1, p, 0, None) == _lib.FA_ERR_INVALID_ARG


@pytest.mark.parametrize("det", [0, 1])
def test_bwd_workspace_is_linear_in_seqlen(lib, det):
    sizes = [lib.fa_bwd_workspace_size(2, S, S, 16, 16, 128, det) for S in (1024, 2048, 4096, 8192)]
    for a, b in zip(sizes, sizes[1:]):
        assert abs(b / a - 2.0) < 0.01
    # the attention matrix would be B*H*S*S*2 bytes: the workspace is far below it
    assert sizes[-1] < 2 * 16 * 8192 * 8192 * 2 / 20


def test_kvcache_workspace(lib):
    assert lib.fa_kvcache_workspace_size(8, 1, 32, 128, 1) == 0
    r256 = lambda x: (x + 255) // 256 * 256
    rows = 8 * 1 * 32
    for n in (2, 4, 16, 64):
        # partial outputs and partial LSEs of every split
        want = r256(n * rows * 128 * 4) + r256(n * rows * 4)
        assert lib.fa_kvcache_workspace_size(8, 1, 32, 128, n) == want
    assert lib.fa_kvcache_workspace_size(8, 1, 32, 128, 0) == lib.fa_kvcache_workspace_size(8, 1, 32, 128, 64)


def test_selftest_rejects_null_flag(lib):
    assert lib.fa_selftest_bounded_wait(None, 1, 1000, None) == _lib.FA_ERR_INVALID_ARG


def test_strided_and_varlen_host_validation(lib):
    p = ctypes.c_void_p(0x1000)
    good = [16, 8, 8] * 4  # (batch, token, head) element strides of q, k, v, out
    arr = lambda vals: (ctypes.c_longlong * len(vals))(*vals)
    fwd = lambda st: lib.fa_fwd_strided(p, p, p, p, p, 1, 8, 8, 1, 1, 64, 1, 0.0, 0, -1, -1, 0.0, st, None)
    bad = list(good)
    bad[1] = 12  # token stride not a multiple of 8 elements
    assert fwd(arr(bad)) == _lib.FA_ERR_INVALID_ARG
    bad = list(good)
    bad[5] = -8
    assert fwd(arr(bad)) == _lib.FA_ERR_INVALID_ARG
    assert fwd(None) == _lib.FA_ERR_INVALID_ARG
    bst = arr([8] * 23 + [4])
    assert lib.fa_bwd_strided(p, p, p, p, p, p, p, p, p, 1, 8, 8, 1, 1, 64, 1, 0.0, 0, -1, -1, 0.0, 0,
                              ctypes.c_void_p(0x10000), 1 << 20, bst, None) == _lib.FA_ERR_INVALID_ARG
    # packed batches: missing offsets, negative sizes, empty batch
    vfwd = lambda cu, B=2, tq=16: lib.fa_fwd_varlen(p, p, p, p, p, cu, cu, B, 8, 8, tq, 16, 2, 2, 64, 1, 0.0, 0,
                                                    -1, -1, 0.0, None)
    assert vfwd(None) == _lib.FA_ERR_INVALID_ARG
    assert vfwd(p, tq=-1) == _lib.FA_ERR_INVALID_ARG
    assert vfwd(ctypes.c_void_p(0x1002)) == _lib.FA_ERR_INVALID_ARG  # offsets not 4-byte aligned
    assert vfwd(p, B=0) == _lib.FA_OK
    # the packed workspace is linear in the token count
    w = [lib.fa_bwd_varlen_workspace_size(8, 1024, T, 16, 128, 0) for T in (4096, 8192)]
    assert abs(w[1] / w[0] - 2.0) < 0.01


def test_alibi_host_validation(lib):
    p = ctypes.c_void_p(0x1000)
    fwd = lambda a, bs, Hq=4, B=1: lib.fa_fwd_alibi(p, p, p, p, p, B, 8, 8, Hq, 2, 64, 1, 0.0, 0, -1, -1, 0.0,
                                                    None, a, bs, None)
    assert fwd(None, 0) == _lib.FA_ERR_INVALID_ARG               # slopes are required
    assert fwd(ctypes.c_void_p(0x1002), 0) == _lib.FA_ERR_INVALID_ARG  # not 4-byte aligned
    assert fwd(p, 2) == _lib.FA_ERR_INVALID_ARG                  # batch stride between 0 and Hq
    assert fwd(p, -4) == _lib.FA_ERR_INVALID_ARG
    assert fwd(p, 0, B=0) == _lib.FA_OK                          # empty batch: nothing to do
    assert fwd(p, 4, B=0) == _lib.FA_OK
    bwd = lambda a, bs: lib.fa_bwd_alibi(p, p, p, p, p, p, p, p, p, 1, 8, 8, 4, 2, 64, 1, 0.0, 0, -1, -1, 0.0, 0,
                                         ctypes.c_void_p(0x10000), 1 << 20, None, a, bs, None)
    assert bwd(None, 0) == _lib.FA_ERR_INVALID_ARG
    assert bwd(p, 3) == _lib.FA_ERR_INVALID_ARG


def test_fp8_host_validation(lib):
    p = ctypes.c_void_p(0x1000)
    fwd = lambda D=128, B=1, Sk=8, d=None: lib.fa_fwd_fp8(p, p, p, p, p, B, 8, Sk, 2, 2, D, d, None, None, 0.0, 0,
                                                          -1, -1, 0.0, None)
    assert fwd(D=96) == _lib.FA_ERR_UNSUPPORTED                   # head dims 64 and 128 only
    assert fwd(d=ctypes.c_void_p(0x1002)) == _lib.FA_ERR_INVALID_ARG  # descale not 4-byte aligned
    assert fwd(B=0) == _lib.FA_OK                                 # nothing to do
    assert fwd(Sk=0) == _lib.FA_ERR_UNSUPPORTED
    assert fwd(Sk=-1) == _lib.FA_ERR_INVALID_ARG


def test_kvcache_rotary_host_validation(lib):
    p = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x100000)  # 256-byte aligned
    # B=2 Sq=Snew=1 Hq=8 Hkv=2 D=128 bf16, paged (page 256, 4 pages/seq, 8 pages), causal, one split
    head = [p, p, p, p, p, p, p, 256, 4, 8, p, p, 2, 1, 1, 8, 2, 128, 1, 0.0, 1, -1, -1, 0.0]

    def call(cos=p, sin=p, dim=128, seqlen_ro=100, w=ws, nbytes=1 << 20):
        return lib.fa_fwd_kvcache_rotary(*head, cos, sin, dim, seqlen_ro, 0, 1, w, nbytes, None)

    bad = _lib.FA_ERR_INVALID_ARG
    assert call(cos=None) == bad and call(sin=None) == bad       # tables required
    assert call(dim=0) == bad and call(dim=127) == bad            # even and positive
    assert call(dim=256) == bad                                   # at most the head dim
    assert call(seqlen_ro=0) == bad                               # at least one position
    assert call(cos=ctypes.c_void_p(0x1002)) == bad               # 4-byte aligned tables
    assert call(w=None) == bad                                    # the rotated q copy needs room
    assert call(w=ctypes.c_void_p(0x100010)) == bad               # 256-byte aligned workspace
    assert call(nbytes=16) == bad
    # workspace: the 16-bit q copy rounded to 256 bytes, then the split partials
    r256 = lambda n: (n + 255) // 256 * 256
    for splits in (1, 4, 0):
        assert lib.fa_kvcache_rotary_workspace_size(2, 1, 8, 128, splits) == \
            r256(2 * 1 * 8 * 128 * 2) + lib.fa_kvcache_workspace_size(2, 1, 8, 128, splits)


def test_library_proper_is_not_the_bounds_checked_build(lib):
    assert lib.fa_build_flags() == 0
