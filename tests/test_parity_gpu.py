"""GPU parity of the non-causal path (la_state_reduce, la_apply, la_attention)
against the float64 oracle, element by element, on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu

D = 32


def _case(B, N, H, seed, io="bf16", grid=None, t_offset=0, outliers=False, eps=1e-6):
    w = wl.Workload("case", B=B, N=N, H=H, outlier_frac=0.01 if outliers else 0.0,
                    outlier_scale=20.0)
    Q, K, V = wl.make_qkv(w, seed)
    if io == "f32":
        Q, K, V = (x.float() for x in (Q, K, V))
    th = None if grid is None else orc.rope_angles(*grid, t_offset)
    return Q, K, V, th, eps


def _full_check(Q, K, V, th, eps, io, grid=None, t_offset=0, what=""):
    O, S, z = P.gpu_attention(Q, K, V, eps, grid, t_offset)
    S_ref, z_ref = orc.state_reduce(K, V, th)
    A = P.magnitude_state(K, V, th)
    tol_s, tol_o = P.tolerances(io, th is not None)
    P.check_state(S, z, S_ref, z_ref, A, tol_s, what)
    O_ref = orc.apply(Q, S_ref, z_ref, eps, th)
    P.check_output(O, O_ref, io, tol_o, Q, th, A, z_ref, eps, what=what)
    return O, S, z


SMALL = [
    # B, N, H, grid (T, Hh, W) or None, t_offset
    (2, 1000, 5, None, 0),          # ragged tokens (1000 = 7*128 + 104) and heads (5 = 4 + 1)
    (1, 1000, 5, (5, 10, 20), 3),   # RoPE with a frame offset
    (3, 130, 9, None, 0),
    (1, 1, 1, None, 0),             # one token, one head
    (1, 129, 70, (1, 3, 43), 0),    # one frame, 70 heads
    (2, 4096, 7, (4, 32, 32), 11),  # several splits per head
    (1, 512, 5, (1, 2, 256), 7),    # RoPE table too large for shared memory: per-token angles
]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}{'rope' if c[3] else ''}")
def test_small_shapes(cuda_device, io, case):
    B, N, H, grid, t0 = case
    Q, K, V, th, eps = _case(B, N, H, 1234 + N + H, io, grid, t0)
    _full_check(Q, K, V, th, eps, io, grid, t0, what=f"{io} {case}")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_outliers_and_eps(cuda_device, io):
    Q, K, V, th, _ = _case(1, 3000, 6, 77, io, outliers=True)
    _full_check(Q, K, V, th, 1e-6, io, what="outliers")
    # a large eps makes the denominator guard matter
    _full_check(Q, K, V, th, 500.0, io, what="eps=500")


@pytest.mark.parametrize("name", ["sana0.6b_512px", "sana1.6b_1024px", "sana1.6b_4k",
                                  "sanavideo_480p"])
def test_workload_full_size(cuda_device, name):
    """Every element of every output at the workload's full size."""
    w = wl.WORKLOADS[name]
    Q, K, V = wl.make_qkv(w, 0)
    grid = (w.T, w.Hh, w.W) if w.rope else None
    th = orc.rope_angles(*grid, 0, w.rope_base) if w.rope else None
    _full_check(Q, K, V, th, w.eps, "bf16", grid, 0, what=name)


def test_split_calls_match_fused_call_and_are_deterministic(cuda_device):
    w = wl.WORKLOADS["sana1.6b_4k"]
    Q, K, V = P.to_dev(*wl.make_qkv(w, 5))
    shape = la.shape_for(Q, eps=w.eps)
    ws = la.workspace(shape)
    S = torch.empty((1, w.H, D, D), device="cuda")
    z = torch.empty((1, w.H, D), device="cuda")
    O = torch.empty_like(Q)
    la.la_state_reduce(shape, K, V, S, z, ws)
    la.la_apply(shape, Q, S, z, O)
    O1, S1, z1 = la.attention(Q, K, V, eps=w.eps)
    torch.cuda.synchronize()
    assert torch.equal(S, S1) and torch.equal(z, z1) and torch.equal(O, O1)
    for _ in range(10):
        O2, S2, z2 = la.attention(Q, K, V, eps=w.eps)
        torch.cuda.synchronize()
        assert torch.equal(S2, S1) and torch.equal(z2, z1) and torch.equal(O2, O1)


def test_degenerate_rows_are_exact_zero(cuda_device):
    Q, K, V, th, eps = _case(1, 300, 3, 9)
    Q[0, 100:140] = -Q[0, 100:140].abs()
    Q[0, 7, 1] = 0.0
    O, _, _ = P.gpu_attention(Q, K, V, eps)
    assert torch.all(O[0, 100:140] == 0)
    assert torch.all(O[0, 7, 1] == 0)


def test_empty_sequence_gives_zero_state(cuda_device):
    shape = la.make_shape(2, 0, 3)
    S = torch.full((2, 3, D, D), 7.0, device="cuda")
    z = torch.full((2, 3, D), 7.0, device="cuda")
    ws = la.workspace(shape)
    la.la_state_reduce(shape, None, None, S, z, ws)
    la.la_apply(shape, None, S, z, None)
    torch.cuda.synchronize()
    assert torch.all(S == 0) and torch.all(z == 0)


def test_stream_argument_is_honoured(cuda_device):
    Q, K, V, th, eps = _case(1, 2048, 4, 21)
    Qd, Kd, Vd = P.to_dev(Q, K, V)
    s = torch.cuda.Stream()
    shape = la.shape_for(Qd, eps=eps)
    ws = la.workspace(shape)
    S = torch.empty((1, 4, D, D), device="cuda")
    z = torch.empty((1, 4, D), device="cuda")
    O = torch.empty_like(Qd)
    torch.cuda.synchronize()
    la.la_attention(shape, Qd, Kd, Vd, S, z, O, ws, stream=s)
    s.synchronize()
    O_ref, S_ref, z_ref = P.gpu_attention(Q, K, V, eps)
    assert torch.equal(O.cpu(), O_ref) and torch.equal(S.cpu(), S_ref)


def test_single_launch_layer_and_two_kernel_fallback(cuda_device):
    """la_attention runs a small layer as one cooperative launch when one wave of
    CTAs covers it, else as reduce + apply; both match the oracle and each
    other bit for bit."""
    assert la.la_attention_launches(la.make_shape(4, 1024, 70)) == 1
    assert la.la_attention_launches(la.make_shape(1, 16384, 70)) == 1   # 144 CTAs: one wave
    assert la.la_attention_launches(la.make_shape(4, 1024, 70, io_dtype="f32")) == 2
    # 80 batch elements x 2 head groups = 160 CTAs > one wave: two kernels
    shape = la.make_shape(80, 200, 8)
    assert la.la_attention_launches(shape) == 2
    Q, K, V, th, eps = _case(80, 200, 8, 99)
    _full_check(Q, K, V, th, eps, "bf16", what="two-kernel fallback")


@pytest.mark.parametrize("name", ["sana1.6b_1024px", "sana1.6b_4k"])
def test_fused_and_two_kernel_paths_are_bitwise_equal(cuda_device, name):
    w = wl.WORKLOADS[name]
    Q, K, V = P.to_dev(*wl.make_qkv(w, 17))
    shape = la.shape_for(Q, eps=w.eps)
    assert la.la_attention_launches(shape) == 1
    O1, S1, z1 = la.attention(Q, K, V, eps=w.eps)          # single launch
    S2 = torch.empty_like(S1)
    z2 = torch.empty_like(z1)
    O2 = torch.empty_like(O1)
    la.la_state_reduce(shape, K, V, S2, z2, la.workspace(shape))
    la.la_apply(shape, Q, S2, z2, O2)                       # two kernels
    torch.cuda.synchronize()
    assert torch.equal(S1, S2) and torch.equal(z1, z2) and torch.equal(O1, O2)
