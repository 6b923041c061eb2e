"""GPU parity of la_causal_attention (token-causal linear attention with a
carried state) against the float64 oracle, element by element."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu
D = 32


def _tol(io, rope):
    """Relative error per term: float32 arithmetic on exact operands (1e-4);
    bf16 with RoPE: the split states come from the tensor-core reduce, whose
    rotated key features are rounded to bf16 (2^-8); bf16 without RoPE: the
    tensor-core kernel rounds the masked weights P and the running state R to
    bf16 for its second MMA (2^-9 each, so 2^-7 with a factor 2 to spare)."""
    if io != "bf16":
        return 1e-4
    return 2.0 ** -8 if rope else 2.0 ** -7


def _inputs(B, N, H, seed, io):
    Q, K, V = wl.make_qkv(wl.Workload("case", B=B, N=N, H=H), seed)
    if io == "f32":
        Q, K, V = (x.float() for x in (Q, K, V))
    return Q, K, V


def _gpu(Q, K, V, S0=None, z0=None, update=0, grid=None, t0=0, eps=1e-6):
    Qd, Kd, Vd = P.to_dev(Q, K, V)
    Sd = None if S0 is None else torch.from_numpy(np.ascontiguousarray(S0)).float().cuda()
    zd = None if z0 is None else torch.from_numpy(np.ascontiguousarray(z0)).float().cuda()
    O = la.causal_attention(Qd, Kd, Vd, Sd, zd, update, eps=eps, rope_grid=grid, t_offset=t0)
    torch.cuda.synchronize()
    assert la.la_device_error() == 0
    return O.cpu(), (None if Sd is None else Sd.cpu()), (None if zd is None else zd.cpu())


SMALL = [
    # B, N, H, grid or None, t_offset
    (2, 1000, 5, None, 0),          # ragged chunks, splits and heads
    (1, 1000, 5, (5, 10, 20), 3),   # RoPE with a frame offset
    (3, 130, 9, None, 0),
    (1, 1, 1, None, 0),
    (2, 4096, 7, (4, 32, 32), 11),  # several splits per head
    (1, 4096, 148, None, 0),        # many head groups
    (1, 2048, 3, (32, 8, 8), 5),    # a 128-token chunk spans two frames
    (2, 600, 2, (4, 150, 1), 0),    # W = 1: a chunk steps 128 rows at once
]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}{'rope' if c[3] else ''}")
def test_causal_small_shapes(cuda_device, io, case):
    B, N, H, grid, t0 = case
    Q, K, V = _inputs(B, N, H, 900 + N + H, io)
    th = None if grid is None else orc.rope_angles(*grid, t0)
    O, _, _ = _gpu(Q, K, V, grid=grid, t0=t0)
    ref, _, _ = orc.causal_attention(Q, K, V, 1e-6, th)
    P.check_causal(O, ref, P.causal_magnitude(Q, K, V, 1e-6, th), io, _tol(io, th is not None),
                   what=f"{io} {case}")


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_causal_carry_update_and_streaming(cuda_device, io):
    """A carried state is added to every token's prefix; update = 1 leaves the
    final state in the carry, so two calls equal one call on the whole."""
    B, H, T1, T2, Hh, W = 2, 5, 3, 2, 8, 12
    Q, K, V = _inputs(B, (T1 + T2) * Hh * W, H, 31, io)
    n1 = T1 * Hh * W
    th = orc.rope_angles(T1 + T2, Hh, W, 0)
    ref, S_end, z_end = orc.causal_attention(Q, K, V, 1e-6, th)
    # first part from a zero carry, second part from the first's final state
    S0 = np.zeros((B, H, D, D))
    z0 = np.zeros((B, H, D))
    O1, S1, z1 = _gpu(Q[:, :n1], K[:, :n1], V[:, :n1], S0, z0, 1, (T1, Hh, W), 0)
    O2, S2, z2 = _gpu(Q[:, n1:], K[:, n1:], V[:, n1:], S1.double().numpy(), z1.double().numpy(),
                      1, (T2, Hh, W), T1)
    tol = _tol(io, True)
    M = P.causal_magnitude(Q, K, V, 1e-6, th)
    P.check_causal(torch.cat([O1, O2], dim=1), ref, M, io, tol, what=f"{io} streamed")
    A = P.magnitude_state(K, V, th)
    P.check_state(S2, z2, S_end, z_end, A, tol, what=f"{io} carry after both parts")
    # a non-zero carry read but not updated (update = 0)
    Sc = np.abs(np.random.default_rng(5).standard_normal((B, H, D, D)))
    zc = np.abs(np.random.default_rng(6).standard_normal((B, H, D))) * 10
    O3, S3, z3 = _gpu(Q[:, :n1], K[:, :n1], V[:, :n1], Sc, zc, 0, (T1, Hh, W), 0)
    ref3, _, _ = orc.causal_attention(Q[:, :n1], K[:, :n1], V[:, :n1], 1e-6, th[:n1],
                                      Sc.astype(np.float32), zc.astype(np.float32))
    M3 = P.causal_magnitude(Q[:, :n1], K[:, :n1], V[:, :n1], 1e-6, th[:n1],
                            Sc.astype(np.float32), zc.astype(np.float32))
    P.check_causal(O3, ref3, M3, io, tol, what=f"{io} carry, update 0")
    assert torch.equal(S3, torch.from_numpy(Sc).float())
    assert torch.equal(z3, torch.from_numpy(zc).float())


@pytest.mark.parametrize("name,heads", [("sana1.6b_4k", [0, 35, 69]),
                                        ("sanavideo_480p", [0, 69])])
def test_causal_workload_full_size(cuda_device, name, heads):
    """Full-size launch; every element of the sampled heads (independent problems)."""
    w = wl.WORKLOADS[name]
    Q, K, V = wl.make_qkv(w, 0)
    grid = (w.T, w.Hh, w.W) if w.rope else None
    th = orc.rope_angles(*grid, 0) if w.rope else None
    O, _, _ = _gpu(Q, K, V, grid=grid, eps=w.eps)
    Qh, Kh, Vh = (x[:, :, heads] for x in (Q, K, V))
    ref, _, _ = orc.causal_attention(Qh, Kh, Vh, w.eps, th)
    M = P.causal_magnitude(Qh, Kh, Vh, w.eps, th)
    P.check_causal(O[:, :, heads], ref, M, "bf16", _tol("bf16", w.rope), what=name)


def test_causal_deterministic_and_empty(cuda_device):
    Q, K, V = P.to_dev(*_inputs(1, 3000, 6, 8, "bf16"))
    a = la.causal_attention(Q, K, V)
    b = la.causal_attention(Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    # an empty sequence leaves the carry as it was, bit for bit
    E = torch.empty((2, 0, 3, D), dtype=torch.bfloat16, device="cuda")
    S = torch.randn((2, 3, D, D), device="cuda")
    z = torch.rand((2, 3, D), device="cuda")
    S_before, z_before = S.clone(), z.clone()
    la.causal_attention(E, E, E, S, z, 1)
    torch.cuda.synchronize()
    assert torch.equal(S, S_before) and torch.equal(z, z_before)
