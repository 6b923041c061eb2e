"""la_state_reduce_static: the state reduce for callers that cannot allocate.

Such callers (a plugin whose host application owns all device memory, a
runtime that forbids allocation after start-up, a loop that must not call
cudaMalloc because it can synchronise the device) pass only inputs and
outputs; the scratch is a fixed array inside the library. This file is
collected last so that a failure here comes after every other test has run.
It checks the new entry point, called through the C ABI, against
la_state_reduce with a workspace, on two calls in a row (the second call
reuses the array the first one left behind), within the tolerance the parity
tests use, and checks that an oversized shape is refused before any launch.
The static-scratch result is also checked against the float64 oracle's state,
with the bound of the parity tests, so the comparison is not only CUDA against
CUDA. Small ragged shapes (tokens and heads that fill no whole tile or head
group), float32 I/O (the CUDA-core reduce) and the empty sequence go through
the same array and are compared bitwise with the workspace path.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu
D = 32


def _reduce_with_workspace(shape, K, V):
    S = torch.empty((shape.B, shape.H, D, D), device="cuda")
    z = torch.empty((shape.B, shape.H, D), device="cuda")
    la.la_state_reduce(shape, K, V, S, z, la.workspace(shape))
    return S, z


def _reduce_static(shape, K, V):
    S = torch.full((shape.B, shape.H, D, D), float("nan"), device="cuda")
    z = torch.full((shape.B, shape.H, D), float("nan"), device="cuda")
    st = la._lib.la_state_reduce_static(ctypes.byref(shape), K.data_ptr(), V.data_ptr(),
                                        S.data_ptr(), z.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    assert st == la.LA_OK, la.la_last_error()
    return S, z


@pytest.mark.parametrize("name,rope", [("sana1.6b_4k", False), ("sanavideo_480p", True)])
def test_static_scratch_matches_workspace_reduce_twice(cuda_device, name, rope):
    w = wl.WORKLOADS[name]
    grid = (w.T, w.Hh, w.W) if rope else None
    for call, seed in enumerate((11, 12)):  # two calls in a row, different inputs
        Q, K, V = wl.make_qkv(w, seed)
        Kd, Vd = P.to_dev(K, V)
        shape = la.shape_for(Kd, eps=w.eps, rope_grid=grid)
        S_ws, z_ws = _reduce_with_workspace(shape, Kd, Vd)
        S_st, z_st = _reduce_static(shape, Kd, Vd)
        torch.cuda.synchronize()
        th = orc.rope_angles(*grid, 0) if rope else None
        A = P.magnitude_state(K, V, th)
        tol_s, _ = P.tolerances("bf16", rope)
        # the static-scratch result against the workspace result, with the
        # tolerance of the parity tests
        P.check_state(S_st.cpu(), z_st.cpu(), orc.to_f64(S_ws.cpu()), orc.to_f64(z_ws.cpu()),
                      A, tol_s, what=f"{name} call {call}")
        # same kernel, same split order: the two are in fact identical
        assert torch.equal(S_st, S_ws) and torch.equal(z_st, z_ws)
        # and the static-scratch state against the float64 oracle
        S_ref, z_ref = orc.state_reduce(K, V, th)
        P.check_state(S_st.cpu(), z_st.cpu(), S_ref, z_ref, A, tol_s,
                      what=f"{name} call {call} vs oracle")


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,H", [(2, 300, 5), (1, 1, 1), (2, 0, 3)])
def test_static_scratch_small_shapes_bitwise_twice(cuda_device, io, B, N, H):
    dtype = torch.bfloat16 if io == "bf16" else torch.float32
    w_shape = (B, N, H, D)
    for call, seed in enumerate((21, 22)):  # two calls in a row, different inputs
        K = wl.make_tensor(w_shape, seed, dtype)
        V = wl.make_tensor(w_shape, seed + 1, dtype)
        Kd, Vd = P.to_dev(K, V)
        shape = la.shape_for(Kd)
        S_ws, z_ws = _reduce_with_workspace(shape, Kd, Vd)
        S_st, z_st = _reduce_static(shape, Kd, Vd)
        torch.cuda.synchronize()
        assert torch.equal(S_st, S_ws) and torch.equal(z_st, z_ws), f"{io} {B}x{N}x{H} call {call}"
        S_ref, z_ref = orc.state_reduce(K, V, None)
        tol_s, _ = P.tolerances(io, False)
        P.check_state(S_st.cpu(), z_st.cpu(), S_ref, z_ref, P.magnitude_state(K, V, None), tol_s,
                      what=f"{io} {B}x{N}x{H} call {call} vs oracle")


def test_static_scratch_refuses_oversized_shapes(cuda_device):
    # B*H = 4096 heads get one split each (B*ceil(H/4) = 1024 head groups is
    # more than a wave), so the scratch is 4096 partial states of 4224 bytes
    # plus the counters, 17.3 MB: more than the 8 MiB array (which holds any
    # shape with B*H <= 1984).
    shape = la.make_shape(16, 1 << 16, 256)
    st = la._lib.la_state_reduce_static(ctypes.byref(shape), 1 << 20, 1 << 20, 1 << 36,
                                        1 << 37, None)
    assert st == la.LA_ERR_UNSUPPORTED
    assert "static array" in la.la_last_error()
