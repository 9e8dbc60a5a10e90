"""C ABI checks that need no GPU: the library builds, loads, exports every function declared in
include/attn.h, and rejects bad arguments on the host before anything is launched.

Pointers passed here are fake addresses (never dereferenced: every call below returns from its
host-side argument checks).
"""
import ctypes
import os
import re

import pytest

from exact_attention_139_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")
HEADERS = [HEADER, os.path.join(ROOT, "include", "attn_diag.h")]

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA, TIMEOUT = range(7)
A = 0x10000  # 256-byte aligned fake device address
B_ = 0x20000
C_ = 0x30000
D_ = 0x40000


def header_functions():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    path = build.build()
    L = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.attn_fwd.argtypes = [vp] * 5 + [i] * 7 + [f, i, vp]
    L.attn_decode_ex.argtypes = [vp] * 5 + [i] * 8 + [f, i, i, vp, sz, i, vp]
    L.attn_decode.argtypes = [vp] * 5 + [i] * 8 + [f, i, i, vp, sz, vp]
    L.attn_combine.argtypes = [vp] * 4 + [i] * 5 + [vp]
    L.attn_fwd_typed.argtypes = [vp] * 5 + [i] * 7 + [f, i, i, vp]
    L.attn_decode_typed.argtypes = [vp] * 5 + [i] * 8 + [f, i, i, vp, sz, i, i, vp]
    L.attn_combine_typed.argtypes = [vp] * 4 + [i] * 6 + [vp]
    L.attn_decode_workspace_size.argtypes = [i] * 7
    L.attn_decode_workspace_size.restype = sz
    L.attn_status_string.argtypes = [i]
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
    return L


def test_header_declares_expected_entry_points():
    names = header_functions()
    for required in ("attn_fwd", "attn_decode", "attn_combine", "attn_decode_workspace_size",
                     "attn_status_string"):
        assert required in names


def test_library_exports_every_header_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings(lib):
    seen = set()
    for code in range(7):
        s = lib.attn_status_string(code).decode()
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 7
    assert lib.attn_status_string(99).decode() == "unknown status"
    assert lib.attn_abi_version() == 10300


def fwd(lib, q=A, k=B_, v=C_, o=D_, lse=None, B=1, Hq=2, Hkv=1, Lq=128, Lk=128, d=128, dv=128, scale=0.1,
        causal=1):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, scale, causal, None)


def test_fwd_argument_checks(lib):
    assert fwd(lib, q=None) == INVALID
    assert fwd(lib, o=None) == INVALID
    assert fwd(lib, B=0) == INVALID
    assert fwd(lib, Lk=0) == INVALID
    assert fwd(lib, Hq=3, Hkv=2) == INVALID
    assert fwd(lib, Lq=256, Lk=128, causal=1) == INVALID
    assert fwd(lib, scale=0.0) == INVALID
    assert fwd(lib, scale=float("nan")) == INVALID
    assert fwd(lib, scale=float("inf")) == INVALID
    assert fwd(lib, scale=-1.0) == INVALID
    assert fwd(lib, d=96, dv=96) == UNSUPPORTED
    assert fwd(lib, d=128, dv=64) == UNSUPPORTED
    assert fwd(lib, q=A + 8) == MISALIGNED
    assert fwd(lib, o=D_ + 2) == MISALIGNED
    assert fwd(lib, lse=A + 2) == MISALIGNED


def dec(lib, q=A, k=B_, v=B_, o=D_, lse=None, B=2, Hq=16, Hkv=1, Lq=2, Lk=1000, d=576, dv=512, ldv=576,
        scale=0.04, causal=1, splits=4, ws=0x100000, ws_bytes=1 << 30, impl=0):
    return lib.attn_decode_ex(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, splits, ws,
                              ws_bytes, impl, None)


def test_decode_argument_checks(lib):
    assert dec(lib, q=None) == INVALID
    assert dec(lib, Hq=15, Hkv=2) == INVALID
    assert dec(lib, ldv=256) == INVALID           # ldv < dv
    assert dec(lib, splits=-1) == INVALID
    assert dec(lib, splits=257) == INVALID
    assert dec(lib, impl=7) == INVALID
    assert dec(lib, Lq=3, Lk=2) == INVALID         # causal with Lq > Lk
    assert dec(lib, d=100, dv=96, ldv=100) == MISALIGNED  # 200-byte rows are not 16-byte multiples
    assert dec(lib, Hq=64, Lq=2) == UNSUPPORTED    # 128 rows per kv head
    assert dec(lib, d=640, dv=512, ldv=640) == UNSUPPORTED
    assert dec(lib, v=C_, ldv=512, impl=2) == UNSUPPORTED  # tensor-core kernel needs latent KV
    assert dec(lib, ws=None) == WORKSPACE
    assert dec(lib, ws_bytes=1024) == WORKSPACE
    assert dec(lib, ws=0x100010) == WORKSPACE      # not 256-byte aligned
    assert dec(lib, k=B_ + 4, v=B_ + 4) == MISALIGNED


def test_combine_argument_checks(lib):
    f = lambda **kw: lib.attn_combine(kw.get("op", A), kw.get("lp", B_), kw.get("o", C_), kw.get("lse", None),
                                      kw.get("B", 1), kw.get("Hq", 2), kw.get("Lq", 3), kw.get("dv", 64),
                                      kw.get("S", 4), None)
    assert f(op=None) == INVALID
    assert f(o=None) == INVALID
    assert f(S=0) == INVALID
    assert f(dv=62) == MISALIGNED
    assert f(op=A + 4) == MISALIGNED


def test_workspace_size_formula(lib):
    def ref(B, Hq, Lq, dv, s):
        a = lambda x: (x + 255) // 256 * 256
        rows = B * Hq * Lq
        return a(s * rows * dv * 4) + a(s * rows * 4)
    for args in [(32, 16, 1, 2, 65536, 512, 9), (1, 1, 1, 1, 1, 8, 1), (4, 8, 2, 1, 5000, 128, 37)]:
        B, Hq, Hkv, Lq, Lk, dv, s = args
        assert lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, s) == ref(B, Hq, Lq, dv, s)
    assert lib.attn_decode_workspace_size(0, 1, 1, 1, 1, 8, 1) == 0
    assert lib.attn_decode_workspace_size(1, 3, 2, 1, 1, 8, 1) == 0
    assert lib.attn_decode_workspace_size(1, 1, 1, 1, 1, 8, 300) == 0


def test_selftest_limit_checked(lib):
    assert lib.attn_selftest_wait_timeout(0, None) == INVALID
    assert lib.attn_selftest_wait_timeout(2_000_000, None) == INVALID


def test_binding_has_c_names():
    from exact_attention_139_b200 import attn
    for name in ("attn_fwd", "attn_decode", "attn_combine", "attn_decode_workspace_size", "attn_status_string",
                 "attn_check_device"):
        assert callable(getattr(attn, name))


BF16, F16 = 0, 1


@pytest.mark.parametrize("dtype", [BF16, F16])
def test_typed_entry_points_check_like_untyped(lib, dtype):
    """The *_typed entry points apply the same host checks for both element types."""
    def fwd_t(**kw):
        a = dict(q=A, k=B_, v=C_, o=D_, lse=None, B=1, Hq=2, Hkv=1, Lq=128, Lk=128, d=128, dv=128,
                 scale=0.1, causal=1)
        a.update(kw)
        return lib.attn_fwd_typed(*a.values(), dtype, None)

    def dec_t(**kw):
        a = dict(q=A, k=B_, v=B_, o=D_, lse=None, B=2, Hq=16, Hkv=1, Lq=2, Lk=1000, d=576, dv=512,
                 ldv=576, scale=0.04, causal=1, splits=4, ws=0x100000, ws_bytes=1 << 30, impl=0)
        a.update(kw)
        return lib.attn_decode_typed(*a.values(), dtype, None)

    assert fwd_t(q=None) == INVALID
    assert fwd_t(Hq=3, Hkv=2) == INVALID
    assert fwd_t(d=96, dv=96) == UNSUPPORTED
    assert fwd_t(q=A + 8) == MISALIGNED
    assert dec_t(ldv=256) == INVALID
    assert dec_t(Hq=64) == UNSUPPORTED
    assert dec_t(ws=None) == WORKSPACE
    assert dec_t(k=B_ + 4, v=B_ + 4) == MISALIGNED
    assert lib.attn_combine_typed(A, B_, C_, None, 1, 2, 3, 62, 4, dtype, None) == MISALIGNED
    assert lib.attn_combine_typed(None, B_, C_, None, 1, 2, 3, 64, 4, dtype, None) == INVALID


@pytest.mark.parametrize("bad", [-1, 2, 7])
def test_typed_entry_points_reject_unknown_dtype(lib, bad):
    # arguments otherwise valid: only the element type is wrong, so nothing reaches a launch
    assert lib.attn_fwd_typed(A, B_, C_, D_, None, 1, 2, 1, 128, 128, 128, 128, 0.1, 1, bad, None) == INVALID
    assert lib.attn_decode_typed(A, B_, B_, D_, None, 2, 16, 1, 2, 1000, 576, 512, 576, 0.04, 1, 4,
                                 0x100000, 1 << 30, 0, bad, None) == INVALID
    assert lib.attn_combine_typed(A, B_, C_, None, 1, 2, 3, 64, 4, bad, None) == INVALID


def test_default_workspace_covers_default_splits(lib):
    """num_splits = 0 sizes the workspace for whichever split count attn_decode will choose."""
    lib.attn_decode_default_splits.argtypes = [ctypes.c_int] * 8
    for B, Hq, Hkv, Lq, Lk, d, dv, lat in [(16, 32, 8, 1, 32768, 128, 128, 0), (32, 16, 1, 2, 65536, 576, 512, 1),
                                           (2, 8, 2, 1, 777, 128, 128, 0), (4, 16, 2, 2, 5000, 256, 256, 0),
                                           (8, 16, 1, 1, 9000, 128, 128, 1), (3, 4, 1, 2, 3000, 576, 512, 0)]:
        s = lib.attn_decode_default_splits(B, Hq, Hkv, Lq, Lk, d, dv, lat)
        assert 1 <= s <= 256
        assert lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, 0) >= \
            lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, s)


def test_sparse_argument_checks(lib):
    """Every call below fails a host check: nothing is launched with the fake addresses."""
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.attn_fwd_sparse_typed.argtypes = [vp] * 5 + [i] * 7 + [f, i, vp, vp, i, i, vp]

    def sp(**kw):
        a = dict(q=A, k=B_, v=C_, o=D_, lse=None, B=1, Hq=2, Hkv=1, Lq=256, Lk=256, d=128, dv=128,
                 scale=0.1, causal=1, idx=0x50000, cnt=0x60000, max_blocks=2, dtype=0)
        a.update(kw)
        return lib.attn_fwd_sparse_typed(*a.values(), None)

    assert sp(idx=None) == INVALID
    assert sp(cnt=None) == INVALID
    assert sp(max_blocks=0) == INVALID
    assert sp(dtype=3) == INVALID
    assert sp(Hq=3, Hkv=2) == INVALID
    assert sp(idx=0x50002) == MISALIGNED
    assert sp(cnt=0x60001) == MISALIGNED
    assert sp(d=96, dv=96) == UNSUPPORTED
    assert sp(q=A + 8) == MISALIGNED


def _balanced_pieces(units, Lk, slots):
    """Partials per kv head under the balanced schedule documented in attn.h / decode.cuh: runs of
    W = ceil(units * Lk / slots) keys rounded up to 64 (None when W > Lk: equal chunks instead)."""
    w = -(-units * Lk // slots)
    w = -(-w // 64) * 64
    if w > Lk:
        return None
    return max(((u + 1) * Lk - 1) // w - (u * Lk) // w + 1 for u in range(units))


def test_decode_plan_balanced_schedule(lib):
    """Without a GPU the library assumes 148 SMs; the latent kernel runs one CTA per SM, the dense
    d = 128 kernel two."""
    lib.attn_decode_default_splits.argtypes = [ctypes.c_int] * 8
    mla = lib.attn_decode_default_splits(32, 16, 1, 2, 65536, 576, 512, 1)
    assert mla == _balanced_pieces(32, 65536, 148)
    gqa = lib.attn_decode_default_splits(16, 32, 8, 1, 32768, 128, 128, 0)
    assert gqa == _balanced_pieces(128, 32768, 296)
    odd = lib.attn_decode_default_splits(3, 16, 1, 2, 4097, 576, 512, 1)
    assert odd == _balanced_pieces(3, 4097, 148)
    # many short kv heads: a run would span more than two heads, so equal chunks are used
    assert _balanced_pieces(64 * 8, 100, 296) is None
    s = lib.attn_decode_default_splits(64, 32, 8, 1, 100, 128, 128, 0)
    assert 1 <= s <= 256
    for (B, Hq, Hkv, Lq, Lk, d, dv), pieces in [((32, 16, 1, 2, 65536, 576, 512), mla),
                                                 ((16, 32, 8, 1, 32768, 128, 128), gqa),
                                                 ((3, 16, 1, 2, 4097, 576, 512), odd)]:
        assert lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, 0) >= \
            lib.attn_decode_workspace_size(B, Hq, Hkv, Lq, Lk, dv, pieces)


def _header_param_counts():
    text = re.sub(r"/\*.*?\*/", "", "".join(open(h).read() for h in HEADERS), flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(attn_\w+)\s*\(([^)]*)\)\s*;", text):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_argtypes_match_header():
    """Every function the Python binding declares has as many ctypes arguments as the C header."""
    from exact_attention_139_b200 import attn
    counts = _header_param_counts()
    checked = 0
    for name, n in counts.items():
        fn = getattr(attn.lib(), name)
        if getattr(fn, "argtypes", None) is not None:
            assert len(fn.argtypes) == n, f"{name}: header {n} parameters, binding {len(fn.argtypes)}"
            checked += 1
    assert checked >= 10


def test_binding_checks_shapes_against_q():
    """The C calls receive only pointers and q's sizes, so the binding rejects a k, v or output
    whose shape disagrees (their tensor maps would otherwise reach past the end of the tensor)."""
    import torch
    from exact_attention_139_b200 import attn
    q = torch.empty(2, 8, 300, 128, dtype=torch.bfloat16)
    k = torch.empty(2, 2, 500, 128, dtype=torch.bfloat16)
    v = torch.empty(2, 2, 500, 128, dtype=torch.bfloat16)
    assert attn._qkv_dims(q, k, v) == (2, 8, 300, 128, 2, 500, 128)
    assert attn._qkv_dims(q, k, k) == (2, 8, 300, 128, 2, 500, 128)  # latent: v is k
    for bad_k in (torch.empty(1, 2, 500, 128), torch.empty(2, 2, 500, 64), torch.empty(2, 2, 500)):
        with pytest.raises(ValueError):
            attn._qkv_dims(q, bad_k, v)
    for bad_v in (torch.empty(2, 2, 499, 128), torch.empty(2, 1, 500, 128), torch.empty(1, 2, 500, 128)):
        with pytest.raises(ValueError):
            attn._qkv_dims(q, k, bad_v)
    with pytest.raises(ValueError):
        attn._shape(torch.empty(2, 8, 300), "lse", (2, 8, 301))
    attn._same_device("x", q, None, k)
    with pytest.raises(ValueError):
        attn._same_device("x", q, torch.empty(1, device="meta"))


def test_host_path_checks_inputs_before_device_work():
    """attn_fwd_host validates shapes and reused buffers before it touches a device."""
    import torch
    from exact_attention_139_b200 import attn
    q = torch.empty(1, 4, 256, 128, dtype=torch.bfloat16)
    k = torch.empty(1, 2, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd_host(q, k, torch.empty(1, 2, 128, 128, dtype=torch.bfloat16), causal=True)
    with pytest.raises(ValueError):
        attn.attn_fwd_host(q, k, k.float(), causal=True)
    with pytest.raises(ValueError):
        attn.attn_fwd_host(torch.empty(1, 3, 256, 128, dtype=torch.bfloat16), k, k, causal=True)
    stale = {"key": ((1, 4, 128, 128), tuple(k.shape), tuple(k.shape), torch.bfloat16)}
    with pytest.raises(ValueError, match="another shape"):
        attn.attn_fwd_host(q, k, k, causal=True, bufs=stale)


def test_host_entry_point_argument_checks(lib):
    """attn_fwd_host rejects bad arguments before touching a device (fake addresses)."""
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd_host.argtypes = [vp] * 5 + [i] * 7 + [f, i, i, vp, sz, i, vp]
    lib.attn_fwd_host_scratch_size.argtypes = [i] * 7
    lib.attn_fwd_host_scratch_size.restype = sz
    need = lib.attn_fwd_host_scratch_size(1, 32, 8, 8192, 8192, 128, 128)
    # q, k, v, o in 16-bit elements plus fp32 LSE, each 256-byte aligned
    assert need == 2 * (2 * 32 * 8192 * 128 + 2 * 8 * 8192 * 128) + 32 * 8192 * 4
    assert lib.attn_fwd_host_scratch_size(1, 3, 2, 10, 10, 64, 64) == 0

    def host(**kw):
        a = dict(q=A, k=B_, v=C_, o=D_, lse=None, B=1, Hq=2, Hkv=1, Lq=128, Lk=128, d=128, dv=128, scale=0.1,
                 causal=1, dtype=0, scratch=0x100000, scratch_bytes=1 << 30, pieces=0)
        a.update(kw)
        return lib.attn_fwd_host(*a.values(), None)

    assert host(q=None) == INVALID
    assert host(dtype=5) == INVALID
    assert host(pieces=-1) == INVALID
    assert host(pieces=65) == INVALID
    assert host(scratch=None) == WORKSPACE
    assert host(scratch_bytes=1000) == WORKSPACE
    assert host(scratch=0x100010) == WORKSPACE
    assert host(d=96, dv=96) == UNSUPPORTED
    assert host(Hq=3, Hkv=2) == INVALID
