"""GPU parity of la_attention_backward against the float64 oracle's backward,
element by element, on seeded inputs (bound derived in tests/parity.py)."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu


def _inputs(w, seed, io):
    Q, K, V = wl.make_qkv(w, seed)
    dO = wl.make_tensor(tuple(Q.shape), seed + 3)
    if io == "f32":
        Q, K, V, dO = (x.float() for x in (Q, K, V, dO))
    return Q, K, V, dO


def _gpu_backward(Q, K, V, dO, S, z, eps, grid, t0):
    Qd, Kd, Vd, gd = P.to_dev(Q, K, V, dO)
    Sd = None if S is None else torch.from_numpy(np.ascontiguousarray(S)).float().cuda()
    zd = None if z is None else torch.from_numpy(np.ascontiguousarray(z)).float().cuda()
    out = la.attention_backward(Qd, Kd, Vd, gd, Sd, zd, eps=eps, rope_grid=grid, t_offset=t0)
    torch.cuda.synchronize()
    assert la.la_device_error() == 0
    return [x.cpu() for x in out]


def _check(Q, K, V, dO, eps, io, grid=None, t0=0, heads=None, what=""):
    """Run the GPU on the whole tensors; compare every element of the heads in
    ``heads`` (all when None) with the oracle."""
    th = None if grid is None else orc.rope_angles(*grid, t0)
    S, z = orc.state_reduce(K, V, th)
    got = _gpu_backward(Q, K, V, dO, S, z, eps, grid, t0)
    if heads is not None:
        Q, K, V, dO = (x[:, :, heads] for x in (Q, K, V, dO))
        S, z = S[:, heads], z[:, heads]
        got = [g[:, :, heads] for g in got[:3]] + [g[:, heads] for g in got[3:]]
    ref = orc.backward(Q, K, V, dO, eps, th)
    mags = P.backward_magnitudes(Q, K, V, dO, eps, th, S, z)
    P.check_backward(got, ref, mags, io, Q, K, what)
    return got


SMALL = [
    # B, N, H, grid (T, Hh, W) or None, t_offset
    (2, 1000, 5, None, 0),          # ragged tokens (1000 = 15*64 + 40) and heads
    (1, 1000, 5, (5, 10, 20), 3),   # RoPE with a frame offset
    (3, 130, 9, None, 0),
    (1, 1, 1, None, 0),             # one token, one head
    (2, 4096, 7, (4, 32, 32), 11),  # several splits per head
    (1, 512, 5, (1, 2, 256), 7),    # a long axis: large angles
    # 37 head groups: 8 tiles per CTA on both sides, so every stage, TMEM
    # buffer and barrier of the tensor-core kernels goes through several phases
    (1, 4096, 148, None, 0),
    (1, 4096, 148, (4, 32, 32), 5),
]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}{'rope' if c[3] else ''}")
def test_backward_small_shapes(cuda_device, io, case):
    B, N, H, grid, t0 = case
    w = wl.Workload("case", B=B, N=N, H=H)
    Q, K, V, dO = _inputs(w, 4321 + N + H, io)
    _check(Q, K, V, dO, 1e-6, io, grid, t0, what=f"{io} {case}")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_backward_outliers_and_eps(cuda_device, io):
    w = wl.Workload("case", B=1, N=3000, H=6, outlier_frac=0.01, outlier_scale=20.0)
    Q, K, V, dO = _inputs(w, 99, io)
    _check(Q, K, V, dO, 1e-6, io, what="outliers")
    _check(Q, K, V, dO, 500.0, io, what="eps=500")


@pytest.mark.parametrize("name,heads", [
    ("sana1.6b_1024px", None),
    ("sana1.6b_4k", [0, 23, 46, 69]),
    ("sanavideo_480p", [0, 35, 69]),
])
def test_backward_workload_full_size(cuda_device, name, heads):
    """Full-size launch; every element of the checked heads (heads are
    independent problems, so a sample of them is exact)."""
    w = wl.WORKLOADS[name]
    Q, K, V, dO = _inputs(w, 0, "bf16")
    grid = (w.T, w.Hh, w.W) if w.rope else None
    _check(Q, K, V, dO, w.eps, "bf16", grid, 0, heads=heads, what=name)


def test_backward_zero_rows_and_keys(cuda_device):
    """Rows with ReLU(q) = 0 and keys with ReLU(k) = 0 get exactly zero gradient."""
    w = wl.Workload("case", B=2, N=700, H=3)
    Q, K, V, dO = _inputs(w, 7, "bf16")
    Q[:, :50] = -Q[:, :50].abs()
    K[:, 600:] = -K[:, 600:].abs()
    dQ, dK, dV, dS, dz = _check(Q, K, V, dO, 1e-3, "bf16", what="zero rows")
    assert (dQ[:, :50] == 0).all() and (dK[:, 600:] == 0).all()
    assert (dV[:, 600:] == 0).all()  # phi(k) = 0 there


def test_backward_recomputed_state_and_determinism(cuda_device):
    """S, z = NULL (state reduced again) is bitwise equal to passing the
    forward's state, and repeated calls are bitwise equal."""
    w = wl.Workload("case", B=2, N=3 * 16 * 40, H=9)
    Qc, Kc, Vc, gc = _inputs(w, 11, "bf16")
    Q, K, V, dO = P.to_dev(Qc, Kc, Vc, gc)
    grid = (3, 16, 40)
    _, S, z = la.attention(Q, K, V, eps=1e-6, rope_grid=grid, t_offset=2)
    a = la.attention_backward(Q, K, V, dO, S, z, eps=1e-6, rope_grid=grid, t_offset=2)
    b = la.attention_backward(Q, K, V, dO, S, z, eps=1e-6, rope_grid=grid, t_offset=2)
    c = la.attention_backward(Q, K, V, dO, None, None, eps=1e-6, rope_grid=grid, t_offset=2)
    torch.cuda.synchronize()
    for x, y, u in zip(a, b, c):
        assert torch.equal(x, y) and torch.equal(x, u)


def test_backward_empty_sequence(cuda_device):
    Q = torch.empty((2, 0, 3, 32), dtype=torch.bfloat16, device="cuda")
    S = torch.randn((2, 3, 32, 32), device="cuda")
    z = torch.rand((2, 3, 32), device="cuda")
    shape = la.shape_for(Q)
    dS = torch.full((2, 3, 32, 32), float("nan"), device="cuda")
    dz = torch.full((2, 3, 32), float("nan"), device="cuda")
    la.la_attention_backward(shape, Q, Q, Q, S, z, Q, Q.clone(), Q.clone(), Q.clone(), dS, dz,
                             la.workspace(shape))
    torch.cuda.synchronize()
    assert (dS == 0).all() and (dz == 0).all()


def test_backward_rejects_overlapping_outputs(cuda_device):
    w = wl.Workload("case", B=1, N=256, H=2)
    Q, K, V, dO = P.to_dev(*_inputs(w, 3, "bf16"))
    shape = la.shape_for(Q)
    dQ = torch.empty_like(Q)
    dS = torch.empty((1, 2, 32, 32), device="cuda")
    dz = torch.empty((1, 2, 32), device="cuda")
    with pytest.raises(la.LaError):
        la.la_attention_backward(shape, Q, K, V, None, None, dO, dQ, dQ, torch.empty_like(V),
                                 dS, dz, la.workspace(shape))
