"""ReLU linear attention on B200 (sm_100a): a thin ctypes binding of ``libla_b200.so``.

The functions below carry the names of the C ABI in ``include/la.h`` and only
marshal arguments (tensor pointers, sizes, the stream) into it; every step of
the computation runs in the library's CUDA kernels. There is no CPU path:
importing this package fails if the library has not been built
(``python linear_attention_diffusion_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libla_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python linear_attention_diffusion_b200/build.py`"
        " (this package has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)

LA_OK = 0
LA_ERR_INVALID_ARG = 1
LA_ERR_UNSUPPORTED = 2
LA_ERR_WORKSPACE = 3
LA_ERR_CUDA = 4
LA_IO_BF16 = 0
LA_IO_F32 = 1
HEAD_DIM = 32


class LaShape(ctypes.Structure):
    """Mirror of ``la_shape`` in include/la.h."""

    _fields_ = [
        ("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
        ("io_dtype", ctypes.c_int), ("rope", ctypes.c_int),
        ("T", ctypes.c_int), ("Hh", ctypes.c_int), ("W", ctypes.c_int),
        ("t_offset", ctypes.c_int), ("rope_base", ctypes.c_double), ("eps", ctypes.c_float),
    ]


class LaConvShape(ctypes.Structure):
    """Mirror of ``la_conv_shape`` in include/la.h."""

    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hh", ctypes.c_int), ("W", ctypes.c_int),
        ("C", ctypes.c_int), ("io_dtype", ctypes.c_int),
    ]


class LaError(RuntimeError):
    def __init__(self, status: int, func: str):
        self.status = status
        detail = la_last_error()
        super().__init__(f"{func}: {la_status_string(status)}" + (f" -- {detail}" if detail else ""))


_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i = ctypes.c_int
_shape_p = ctypes.POINTER(LaShape)

_lib.la_workspace_bytes.argtypes = [_shape_p]
_lib.la_workspace_bytes.restype = _sz
_lib.la_causal_workspace_bytes.argtypes = [_shape_p]
_lib.la_causal_workspace_bytes.restype = _sz
_lib.la_state_reduce.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.la_state_reduce.restype = _i
_lib.la_state_reduce_static.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp]
_lib.la_state_reduce_static.restype = _i
_lib.la_apply.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp]
_lib.la_apply.restype = _i
_lib.la_attention.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_lib.la_attention.restype = _i
_lib.la_block_causal_step.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]
_lib.la_block_causal_step.restype = _i
_lib.la_attention_backward.argtypes = [_shape_p] + [_vp] * 11 + [_vp, _sz, _vp]
_lib.la_attention_backward.restype = _i
_lib.la_causal_attention.argtypes = [_shape_p, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _sz, _vp]
_lib.la_causal_attention.restype = _i
_lib.la_temporal_conv.argtypes = [ctypes.POINTER(LaConvShape), _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.la_temporal_conv.restype = _i
_lib.la_qkv_workspace_bytes.argtypes = [_shape_p, _i]
_lib.la_qkv_workspace_bytes.restype = _sz
_lib.la_qkv_state.argtypes = [_shape_p, _i] + [_vp] * 7 + [_sz, _vp]
_lib.la_qkv_state.restype = _i
_lib.la_state_reset.argtypes = [_vp, _vp, _i, _i, _i, _vp]
_lib.la_state_reset.restype = _i
_lib.la_status_string.argtypes = [_i]
_lib.la_status_string.restype = ctypes.c_char_p
_lib.la_last_error.argtypes = []
_lib.la_last_error.restype = ctypes.c_char_p
_lib.la_attention_launches.argtypes = [_shape_p]
_lib.la_attention_launches.restype = _i
_lib.la_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), _i]
_lib.la_wait_selftest.argtypes = [ctypes.c_uint, _vp]
_lib.la_wait_selftest.restype = _i
_lib.la_device_error.restype = _i


def make_shape(B: int, N: int, H: int, D: int = HEAD_DIM, io_dtype: str = "bf16",
               rope: bool = False, T: int = 0, Hh: int = 0, W: int = 0,
               t_offset: int = 0, rope_base: float = 10000.0, eps: float = 1e-6) -> LaShape:
    io = {"bf16": LA_IO_BF16, "f32": LA_IO_F32, "float32": LA_IO_F32}[io_dtype]
    return LaShape(int(B), int(N), int(H), int(D), io, int(bool(rope)), int(T), int(Hh),
                   int(W), int(t_offset), float(rope_base), float(eps))


def _ptr(x) -> Optional[int]:
    """Device address of a tensor (or an int address); None for NULL."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("tensor arguments must live on a CUDA device")
    if not x.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return x.data_ptr()


def _nbytes(x) -> int:
    return 0 if x is None else x.numel() * x.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, func: str) -> None:
    if status != LA_OK:
        raise LaError(status, func)


def la_workspace_bytes(shape: LaShape) -> int:
    return int(_lib.la_workspace_bytes(ctypes.byref(shape)))


def la_causal_workspace_bytes(shape: LaShape) -> int:
    return int(_lib.la_causal_workspace_bytes(ctypes.byref(shape)))


def la_state_reduce(shape: LaShape, K, V, S, z, ws, stream=None) -> None:
    _check(_lib.la_state_reduce(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(S), _ptr(z),
                                _ptr(ws), _nbytes(ws), _stream(stream)), "la_state_reduce")


def la_state_reduce_static(shape: LaShape, K, V, S, z, stream=None) -> None:
    """la_state_reduce without a workspace: the scratch is the library's own
    fixed device array (for callers that cannot allocate; see include/la.h)."""
    _check(_lib.la_state_reduce_static(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(S), _ptr(z),
                                       _stream(stream)), "la_state_reduce_static")


def la_apply(shape: LaShape, Q, S, z, O, stream=None) -> None:
    _check(_lib.la_apply(ctypes.byref(shape), _ptr(Q), _ptr(S), _ptr(z), _ptr(O),
                         _stream(stream)), "la_apply")


def la_attention(shape: LaShape, Q, K, V, S, z, O, ws, stream=None) -> None:
    _check(_lib.la_attention(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(S), _ptr(z),
                             _ptr(O), _ptr(ws), _nbytes(ws), _stream(stream)), "la_attention")


def la_block_causal_step(shape: LaShape, Q, K, V, S_carry, z_carry, O, update: int, ws,
                         stream=None) -> None:
    _check(_lib.la_block_causal_step(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V),
                                     _ptr(S_carry), _ptr(z_carry), _ptr(O), int(update),
                                     _ptr(ws), _nbytes(ws), _stream(stream)),
           "la_block_causal_step")


def la_attention_backward(shape: LaShape, Q, K, V, S, z, dO, dQ, dK, dV, dS, dz, ws,
                          stream=None) -> None:
    """Gradients of la_attention; S and z None makes the call reduce the state again."""
    _check(_lib.la_attention_backward(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(S),
                                      _ptr(z), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dS),
                                      _ptr(dz), _ptr(ws), _nbytes(ws), _stream(stream)),
           "la_attention_backward")


def la_causal_attention(shape: LaShape, Q, K, V, S_carry, z_carry, O, update: int, ws,
                        stream=None) -> None:
    """Token-causal attention; the carry (S_carry, z_carry) may be None when update = 0."""
    _check(_lib.la_causal_attention(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(V),
                                    _ptr(S_carry), _ptr(z_carry), _ptr(O), int(update),
                                    _ptr(ws), _nbytes(ws), _stream(stream)),
           "la_causal_attention")


def make_conv_shape(B: int, T: int, Hh: int, W: int, C: int, io_dtype: str = "bf16") -> LaConvShape:
    return LaConvShape(int(B), int(T), int(Hh), int(W), int(C),
                       LA_IO_BF16 if io_dtype == "bf16" else LA_IO_F32)


def la_temporal_conv(shape: LaConvShape, x, w, bias, f_in, f_out, y, stream=None) -> None:
    """Temporal depth-wise conv with shortcut and conv cache (see include/la.h)."""
    _check(_lib.la_temporal_conv(ctypes.byref(shape), _ptr(x), _ptr(w), _ptr(bias), _ptr(f_in),
                                 _ptr(f_out), _ptr(y), _stream(stream)), "la_temporal_conv")


def la_qkv_workspace_bytes(shape: LaShape, C: int) -> int:
    return int(_lib.la_qkv_workspace_bytes(ctypes.byref(shape), int(C)))


def la_qkv_state(shape: LaShape, C: int, X, W, bias, Q, S, z, ws, stream=None) -> None:
    """QKV projection fused with the state reduce (see include/la.h)."""
    _check(_lib.la_qkv_state(ctypes.byref(shape), int(C), _ptr(X), _ptr(W), _ptr(bias), _ptr(Q),
                             _ptr(S), _ptr(z), _ptr(ws), _nbytes(ws), _stream(stream)),
           "la_qkv_state")


def la_state_reset(S, z, B: int, H: int, D: int = HEAD_DIM, stream=None) -> None:
    _check(_lib.la_state_reset(_ptr(S), _ptr(z), int(B), int(H), int(D), _stream(stream)),
           "la_state_reset")


def la_attention_launches(shape: LaShape) -> int:
    """Kernel launches of la_attention / la_block_causal_step (update 0, 1)."""
    return int(_lib.la_attention_launches(ctypes.byref(shape)))


def la_status_string(status: int) -> str:
    return _lib.la_status_string(int(status)).decode()


def la_last_error() -> str:
    return _lib.la_last_error().decode()


def la_wait_selftest(limit_us: int, stream=None) -> None:
    """Launch a warp whose wait nothing satisfies; it gives up after limit_us
    and raises the device error word (see la_device_error)."""
    _check(_lib.la_wait_selftest(int(limit_us), _stream(stream)), "la_wait_selftest")


def la_device_error(reset: bool = False) -> int:
    """The device error word of the current device (0: no kernel gave up a wait)."""
    code = ctypes.c_uint(0)
    _check(_lib.la_device_error(ctypes.byref(code), int(bool(reset))), "la_device_error")
    return int(code.value)


# ---------------------------------------------------------------------------
# Convenience wrappers that allocate outputs with torch (device memory only).

def shape_for(Q, eps: float = 1e-6, rope_grid=None, t_offset: int = 0,
              rope_base: float = 10000.0) -> LaShape:
    """la_shape for a [B, N, H, D] tensor; ``rope_grid`` = (T, Hh, W) turns on RoPE."""
    import torch
    B, N, H, D = Q.shape
    io = "bf16" if Q.dtype == torch.bfloat16 else "f32"
    if rope_grid is None:
        return make_shape(B, N, H, D, io, False, eps=eps)
    T, Hh, W = rope_grid
    return make_shape(B, N, H, D, io, True, T, Hh, W, t_offset, rope_base, eps)


def workspace(shape: LaShape, device="cuda", causal: bool = False):
    """A zero-filled workspace of la_workspace_bytes(shape) bytes
    (la_causal_workspace_bytes(shape) with causal=True)."""
    import torch
    n = la_causal_workspace_bytes(shape) if causal else la_workspace_bytes(shape)
    if n == 0:
        raise LaError(LA_ERR_INVALID_ARG, "la_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def attention(Q, K, V, eps: float = 1e-6, rope_grid=None, t_offset: int = 0,
              rope_base: float = 10000.0, stream=None):
    """O, S, z of non-causal ReLU linear attention for [B, N, H, 32] CUDA tensors."""
    import torch
    shape = shape_for(Q, eps, rope_grid, t_offset, rope_base)
    B, N, H, D = Q.shape
    S = torch.empty((B, H, D, D), dtype=torch.float32, device=Q.device)
    z = torch.empty((B, H, D), dtype=torch.float32, device=Q.device)
    O = torch.empty_like(Q)
    la_attention(shape, Q, K, V, S, z, O, workspace(shape, Q.device), stream)
    return O, S, z


def attention_backward(Q, K, V, dO, S=None, z=None, eps: float = 1e-6, rope_grid=None,
                       t_offset: int = 0, rope_base: float = 10000.0, stream=None):
    """dQ, dK, dV, dS, dz of non-causal ReLU linear attention for [B, N, H, 32] CUDA tensors."""
    import torch
    shape = shape_for(Q, eps, rope_grid, t_offset, rope_base)
    B, N, H, D = Q.shape
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dS = torch.empty((B, H, D, D), dtype=torch.float32, device=Q.device)
    dz = torch.empty((B, H, D), dtype=torch.float32, device=Q.device)
    la_attention_backward(shape, Q, K, V, S, z, dO, dQ, dK, dV, dS, dz,
                          workspace(shape, Q.device), stream)
    return dQ, dK, dV, dS, dz


def causal_attention(Q, K, V, S_carry=None, z_carry=None, update: int = 0, eps: float = 1e-6,
                     rope_grid=None, t_offset: int = 0, rope_base: float = 10000.0, stream=None):
    """O of token-causal ReLU linear attention for [B, N, H, 32] CUDA tensors."""
    shape = shape_for(Q, eps, rope_grid, t_offset, rope_base)
    import torch
    O = torch.empty_like(Q)
    la_causal_attention(shape, Q, K, V, S_carry, z_carry, O, update,
                        workspace(shape, Q.device, causal=True), stream)
    return O


def temporal_conv(x, w, bias=None, f_in=None, want_cache: bool = False, stream=None):
    """y (and the next conv cache when ``want_cache``) for x [B, T, Hh, W, C] CUDA tensors."""
    import torch
    B, T, Hh, W, C = x.shape
    shape = make_conv_shape(B, T, Hh, W, C, "bf16" if x.dtype == torch.bfloat16 else "f32")
    y = torch.empty_like(x)
    f_out = torch.empty((B, Hh, W, C), dtype=x.dtype, device=x.device) if want_cache else None
    la_temporal_conv(shape, x, w, bias, f_in, f_out, y, stream)
    return (y, f_out) if want_cache else y


def qkv_state(X, W, bias=None, rope_grid=None, t_offset: int = 0, rope_base: float = 10000.0,
              stream=None):
    """Q [B, N, H, 32], S, z of the fused QKV projection + state reduce for
    X [B, N, C] and W [3 H 32, C] bf16 CUDA tensors."""
    import torch
    B, N, C = X.shape
    if W.dim() != 2 or W.shape[1] != C or W.shape[0] % (3 * HEAD_DIM) != 0:
        raise ValueError(f"W must be [3*H*{HEAD_DIM}, C={C}], got {tuple(W.shape)}")
    H = W.shape[0] // (3 * HEAD_DIM)
    if bias is not None and tuple(bias.shape) != (W.shape[0],):
        raise ValueError(f"bias must be [{W.shape[0]}], got {tuple(bias.shape)}")
    if rope_grid is None:
        shape = make_shape(B, N, H, HEAD_DIM, "bf16", False)
    else:
        T, Hh, Wd = rope_grid
        shape = make_shape(B, N, H, HEAD_DIM, "bf16", True, T, Hh, Wd, t_offset, rope_base)
    Q = torch.empty((B, N, H, HEAD_DIM), dtype=torch.bfloat16, device=X.device)
    S = torch.empty((B, H, HEAD_DIM, HEAD_DIM), dtype=torch.float32, device=X.device)
    z = torch.empty((B, H, HEAD_DIM), dtype=torch.float32, device=X.device)
    n = la_qkv_workspace_bytes(shape, C)
    if n == 0:
        raise LaError(LA_ERR_INVALID_ARG, "la_qkv_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=X.device)
    la_qkv_state(shape, C, X, W, bias, Q, S, z, ws, stream)
    return Q, S, z
