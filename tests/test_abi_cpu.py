"""Host-side checks of the C ABI that need no GPU.

The library must load on a machine without a GPU driver, export every function
that include/la.h declares, and reject bad arguments on the host (before any
CUDA call) with the documented status codes.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

import linear_attention_diffusion_b200 as la  # noqa: E402

FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced: every call below fails validation first


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(la_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("la_state_reduce", "la_apply", "la_block_causal_step", "la_state_reset",
                     "la_workspace_bytes", "la_status_string", "la_attention"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(la.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert hasattr(la, name), f"binding lacks {name}"


def test_shape_struct_matches_header_layout():
    # int B, N, H, D, io_dtype, rope, T, Hh, W, t_offset (10 ints = 40 bytes),
    # then double rope_base at 40 and float eps at 48; sizeof = 56.
    assert ctypes.sizeof(la.LaShape) == 56
    assert la.LaShape.rope_base.offset == 40
    assert la.LaShape.eps.offset == 48


def test_status_strings():
    for code in range(5):
        assert la.la_status_string(code).startswith("LA_")
    assert "unknown" in la.la_status_string(99)


def test_workspace_bytes_is_shape_only_and_rejects_bad_shapes():
    s = la.make_shape(1, 16384, 70)
    n = la.la_workspace_bytes(s)
    assert n > 0 and n % 256 == 0
    assert la.la_workspace_bytes(la.make_shape(1, 16384, 70)) == n
    # constant-size state: the state part does not grow with N
    assert la.la_workspace_bytes(la.make_shape(1, 10 ** 6, 70)) < 64 * 70 * 1056 * 4 + 2 * 70 * 1056 * 4 + 4096
    assert la.la_workspace_bytes(la.make_shape(1, 16, 70, D=64)) == 0
    assert la.la_workspace_bytes(la.make_shape(1, 10, 2, rope=True, T=2, Hh=2, W=2)) == 0
    assert la.la_workspace_bytes(la.make_shape(-1, 10, 2)) == 0
    assert la.la_workspace_bytes(la.make_shape(1, 10, 2, eps=float("nan"))) == 0
    assert la.la_workspace_bytes(la.make_shape(0, 0, 0)) > 0  # empty is valid


def _call(fn, *args):
    return getattr(la._lib, fn)(*args)


def test_host_validation_statuses():
    s = la.make_shape(2, 256, 3)
    ws_n = la.la_workspace_bytes(s)
    ref = ctypes.byref
    st = _call("la_state_reduce", ref(s), FAKE, FAKE, FAKE + (1 << 20), FAKE + (2 << 20), FAKE + (3 << 20), ws_n - 16, None)
    assert st == la.LA_ERR_WORKSPACE
    assert "workspace" in la.la_last_error()
    st = _call("la_state_reduce", ref(s), None, FAKE, FAKE, FAKE, FAKE, ws_n, None)
    assert st == la.LA_ERR_INVALID_ARG and "K" in la.la_last_error()
    st = _call("la_state_reduce", ref(s), FAKE + 8, FAKE, FAKE, FAKE, FAKE, ws_n, None)
    assert st == la.LA_ERR_INVALID_ARG and "aligned" in la.la_last_error()
    st = _call("la_state_reduce", ref(s), FAKE, FAKE, FAKE, FAKE, None, ws_n, None)
    assert st == la.LA_ERR_WORKSPACE
    s64 = la.make_shape(2, 256, 3, D=64)
    assert _call("la_apply", ref(s64), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_UNSUPPORTED
    bad_io = la.make_shape(2, 256, 3)
    bad_io.io_dtype = 7
    assert _call("la_apply", ref(bad_io), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_INVALID_ARG
    neg_eps = la.make_shape(2, 256, 3, eps=-1.0)
    assert _call("la_apply", ref(neg_eps), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_INVALID_ARG
    # O aliasing Q
    assert _call("la_apply", ref(s), FAKE, FAKE + (1 << 30), FAKE + (2 << 30), FAKE + 64,
                 None) == la.LA_ERR_INVALID_ARG
    assert "overlap" in la.la_last_error()
    # bad update flag, RoPE grid mismatch, bad base
    assert _call("la_block_causal_step", ref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 3, FAKE,
                 ws_n, None) == la.LA_ERR_INVALID_ARG
    r = la.make_shape(1, 24, 2, rope=True, T=2, Hh=3, W=5)
    assert _call("la_apply", ref(r), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_INVALID_ARG
    r = la.make_shape(1, 30, 2, rope=True, T=2, Hh=3, W=5, rope_base=1.0)
    assert _call("la_apply", ref(r), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_INVALID_ARG
    r = la.make_shape(1, 30, 2, rope=True, T=2, Hh=3, W=5, t_offset=-1)
    assert _call("la_apply", ref(r), FAKE, FAKE, FAKE, FAKE, None) == la.LA_ERR_INVALID_ARG
    assert _call("la_state_reset", None, FAKE, 1, 1, 32, None) == la.LA_ERR_INVALID_ARG
    assert _call("la_state_reset", FAKE, FAKE, 1, 1, 16, None) == la.LA_ERR_UNSUPPORTED
    assert _call("la_state_reset", FAKE, FAKE, -1, 1, 32, None) == la.LA_ERR_INVALID_ARG
    assert _call("la_attention", None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20,
                 None) == la.LA_ERR_INVALID_ARG


def test_empty_problems_need_no_pointers():
    # B*H == 0: nothing to do, nothing launched, no pointer needed.
    s = la.make_shape(0, 128, 4)
    assert _call("la_apply", ctypes.byref(s), None, None, None, None, None) == la.LA_OK
    n = la.la_workspace_bytes(s)
    assert _call("la_state_reduce", ctypes.byref(s), None, None, None, None, FAKE, n,
                 None) == la.LA_OK
    assert _call("la_state_reset", None, None, 0, 3, 32, None) == la.LA_OK


def test_binding_raises_with_detail():
    s = la.make_shape(1, 8, 1, D=16)
    with pytest.raises(la.LaError, match="only 32"):
        la._check(_call("la_apply", ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, None), "la_apply")


def test_wait_selftest_rejects_limits_out_of_range():
    import linear_attention_diffusion_b200 as la
    for bad in (0, 10_000_001):  # refused on the host, before any launch
        with pytest.raises(la.LaError):
            la.la_wait_selftest(bad, stream=0)


def test_qkv_state_host_checks():
    ref = ctypes.byref
    s = la.make_shape(2, 300, 6)
    C = 192
    n = la.la_qkv_workspace_bytes(s, C)
    assert n > 0 and n % 256 == 0 and la.la_qkv_workspace_bytes(s, C) == n
    assert la.la_qkv_workspace_bytes(s, 100) == 0          # C not a multiple of 8
    assert la.la_qkv_workspace_bytes(s, 0) == 0
    assert la.la_qkv_workspace_bytes(la.make_shape(2, 300, 6, io_dtype="f32"), C) == 0
    assert la.la_qkv_workspace_bytes(la.make_shape(2, 300, 6, D=64), C) == 0
    big = 1 << 32
    X, W, Q, S, z, ws = (FAKE + i * big for i in range(6))
    args = lambda **kw: [kw.get(k, v) for k, v in
                         (("X", X), ("W", W), ("b", None), ("Q", Q), ("S", S), ("z", z),
                          ("ws", ws), ("n", n))]
    call = lambda shape=s, c=C, **kw: _call("la_qkv_state", ref(shape), c, *args(**kw), None)
    assert call(c=100) == la.LA_ERR_UNSUPPORTED
    assert call(shape=la.make_shape(2, 300, 6, io_dtype="f32")) == la.LA_ERR_UNSUPPORTED
    assert call(X=None) == la.LA_ERR_INVALID_ARG and "X" in la.la_last_error()
    assert call(W=FAKE + 8) == la.LA_ERR_INVALID_ARG and "aligned" in la.la_last_error()
    assert call(ws=None) == la.LA_ERR_WORKSPACE
    assert call(n=n - 256) == la.LA_ERR_WORKSPACE
    assert call(Q=X + 64) == la.LA_ERR_INVALID_ARG and "overlap" in la.la_last_error()
    assert call(z=S + 16) == la.LA_ERR_INVALID_ARG and "overlap" in la.la_last_error()
    r = la.make_shape(1, 24, 2, rope=True, T=2, Hh=3, W=5)  # N != T*Hh*W
    assert call(shape=r) == la.LA_ERR_INVALID_ARG
    # nothing to do: no pointer needed
    assert _call("la_qkv_state", ref(la.make_shape(0, 300, 6)), C, None, None, None, None, None,
                 None, None, 0, None) == la.LA_OK


def test_qkv_state_wrapper_checks_shapes():
    import torch
    X = torch.zeros((1, 4, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        la.qkv_state(X, torch.zeros((95, 64), dtype=torch.bfloat16))   # rows not 3*H*32
    with pytest.raises(ValueError):
        la.qkv_state(X, torch.zeros((96, 32), dtype=torch.bfloat16))   # C mismatch
    with pytest.raises(ValueError):
        la.qkv_state(X, torch.zeros((96, 64), dtype=torch.bfloat16),
                     torch.zeros((95,), dtype=torch.bfloat16))


def test_causal_workspace_bytes():
    # bf16, with or without RoPE: room for every 128-token chunk's state (4224
    # bytes a head), never less than the ordinary workspace
    s = la.make_shape(1, 16384, 70)
    n = la.la_causal_workspace_bytes(s)
    assert n >= la.la_workspace_bytes(s)
    assert n >= 70 * (16384 // 128) * 4224
    assert la.la_causal_workspace_bytes(la.make_shape(2, 300, 5)) >= 2 * 5 * 3 * 4224
    r = la.make_shape(1, 16384, 70, rope=True, T=16, Hh=32, W=32)
    assert la.la_causal_workspace_bytes(r) == n
    # float32 I/O uses the ordinary workspace
    f = la.make_shape(1, 300, 3, io_dtype="f32")
    assert la.la_causal_workspace_bytes(f) == la.la_workspace_bytes(f)
    assert la.la_causal_workspace_bytes(la.make_shape(1, 16, 70, D=64)) == 0


def test_causal_attention_refuses_a_short_workspace():
    s = la.make_shape(1, 16384, 4)
    short = la.la_workspace_bytes(s)  # enough for la_attention, not for the chunk states
    assert short < la.la_causal_workspace_bytes(s)
    st = la._lib.la_causal_attention(ctypes.byref(s), FAKE, FAKE, FAKE, None, None, FAKE + (1 << 30),
                                     0, FAKE + (2 << 30), short, None)
    assert st == la.LA_ERR_WORKSPACE
    assert "la_causal_workspace_bytes" in la.la_last_error()
