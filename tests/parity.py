"""Helpers of the GPU parity tests: run the CUDA path, compute the oracle, and
compare them element by element with tolerances stated here.

Tolerances.

* Spec bar for O: |gpu - ref| <= 2e-3 + 2e-2 |ref| for bf16 output and
  |gpu - ref| <= 1e-4 + 1e-4 |ref| for float32 output.
* A tighter bar derived from the arithmetic, checked as well. With
  A = sum_n |phi(k_n)|^T |v_n| (the magnitude of every term of S):
    S:  |S_gpu - S_ref| <= tol_s * A
    z:  |z_gpu - z_ref| <= 1e-5 * z_ref          (a sum of non-negative terms)
    O:  |O_gpu - O_ref| <= out_round * |O_ref| + tol_o * (|phi(q)| A) / den
  where den = ReLU(q).z + eps. out_round is the output rounding (2^-8 for
  bf16, 1e-6 for float32). tol_s / tol_o are the relative errors of the
  operands the kernels feed their contractions: 2e-5 when they are exact (bf16
  inputs without RoPE) or float32, 2^-8 / 2^-7 when a rotated feature or the
  state is rounded to bf16 for the tensor cores.
"""
from __future__ import annotations

import numpy as np
import torch

import linear_attention_diffusion_b200 as la
import oracle as orc

NS_BF16 = (2e-2, 2e-3)   # (rtol, atol)
NS_F32 = (1e-4, 1e-4)


def theta_for(w_rope, T, Hh, W, t_offset=0, base=10000.0):
    return orc.rope_angles(T, Hh, W, t_offset, base) if w_rope else None


def to_dev(*xs, dtype=None):
    out = []
    for x in xs:
        x = x if dtype is None else x.to(dtype)
        out.append(x.contiguous().cuda())
    return out


def gpu_attention(Q, K, V, eps, rope_grid=None, t_offset=0):
    """Run la_attention on device copies of CPU tensors; return CPU O, S, z."""
    Qd, Kd, Vd = to_dev(Q, K, V)
    O, S, z = la.attention(Qd, Kd, Vd, eps=eps, rope_grid=rope_grid, t_offset=t_offset)
    torch.cuda.synchronize()
    assert la.la_device_error() == 0, "a kernel gave up a bounded wait"
    return O.cpu(), S.cpu(), z.cpu()


def magnitude_state(K, V, theta):
    kf = orc.to_f64(K)
    vf = orc.to_f64(V)
    phik = np.abs(orc.feature_map(kf, theta))
    return np.matmul(phik.transpose(0, 2, 3, 1), np.abs(vf).transpose(0, 2, 1, 3))


def check_state(S_gpu, z_gpu, S_ref, z_ref, A, tol_s, what=""):
    S_gpu = orc.to_f64(S_gpu)
    z_gpu = orc.to_f64(z_gpu)
    err = np.abs(S_gpu - S_ref)
    bound = tol_s * A + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what} S: {bad.sum()} of {bad.size} outside tol; worst ratio "
                           f"{float((err / bound).max()):.3g}")
    zerr = np.abs(z_gpu - z_ref)
    zb = 1e-5 * np.abs(z_ref) + 1e-30
    assert not (zerr > zb).any(), f"{what} z: worst ratio {float((zerr / zb).max()):.3g}"


def check_output(O_gpu, O_ref, io, tol_o, Q=None, theta=None, A=None, z_ref=None, eps=None,
                 rows=None, what=""):
    """Spec tolerance always; the derived bound when Q, A, z_ref are given."""
    O_gpu = orc.to_f64(O_gpu)
    rtol, atol = NS_BF16 if io == "bf16" else NS_F32
    err = np.abs(O_gpu - O_ref)
    assert np.isfinite(O_gpu).all(), f"{what}: non-finite output"
    ns = atol + rtol * np.abs(O_ref)
    assert not (err > ns).any(), (f"{what}: {(err > ns).sum()} elements outside the "
                                  f"north-star tolerance; max err {err.max():.3g}")
    if Q is None:
        return
    qf = orc.to_f64(Q)
    th = theta
    if rows is not None:
        qf = qf[:, rows]
        th = None if theta is None else theta[rows]
    phq = np.abs(orc.feature_map(qf, th))
    num_abs = np.matmul(phq.transpose(0, 2, 1, 3), A).transpose(0, 2, 1, 3)
    den = np.einsum("bnhd,bhd->bnh", orc.relu(qf), z_ref) + eps
    out_round = 2.0 ** -8 if io == "bf16" else 1e-6
    bound = out_round * np.abs(O_ref) + tol_o * num_abs / den[..., None] + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements outside the derived bound; worst "
                           f"ratio {float((err / bound).max()):.3g}")


def tolerances(io, rope):
    """(tol_s, tol_o) of the current kernels for this I/O type and feature map."""
    if io == "bf16" and rope:
        return 2.0 ** -8, 2.0 ** -7
    if io == "bf16":
        return 2e-5, 2.0 ** -7
    return 2e-5, 2e-5


# ---------------------------------------------------------------------------
# Backward pass.
#
# The GPU is given the oracle's (S, z) rounded to float32, so the comparison
# isolates the backward kernels. Their arithmetic is sums of products whose
# magnitudes are written out below with absolute values (M_*); each gradient
# must satisfy
#     |g_gpu - g_ref| <= out_round * |g_ref| + tol_b * M
# with out_round the output rounding (2^-8 for bf16 gradients, 1e-6 for
# float32, 0 for dS/dz which are float32 sums). tol_b:
#   float32 I/O (CUDA cores, float32 throughout): 1e-4; the longest float32
#     running sum is a few thousand terms per thread, well inside it.
#   bf16 I/O (tensor cores): 2^-7. The MMA operands dnum = dO/den, S, dS and
#     the rotated phi(q), phi(k) are rounded to bf16 (2^-9 each), so every
#     product carries at most 2^-8 relative error; 2^-7 leaves a factor 2 for
#     the float32 accumulation and for errors carried from dS into dK, dV.
# Elements whose ReLU input is <= 0 must be exactly zero in dQ and dK.

TOL_B = {"f32": 1e-4, "bf16": 2.0 ** -7}


def _pair_sum(x):
    """|R^T y|_d <= |y_d| + |y_{d xor 1}| for a rotation R of the pairs (2i, 2i+1)."""
    y = x.copy()
    y[..., 0::2] += x[..., 1::2]
    y[..., 1::2] += x[..., 0::2]
    return y


def backward_magnitudes(Q, K, V, dO, eps, theta, S, z):
    """Magnitudes M of every term of each gradient (float64, same shapes)."""
    qf, kf, vf, gf = (orc.to_f64(x) for x in (Q, K, V, dO))
    qp, kp = orc.relu(qf), orc.relu(kf)
    phq = np.abs(orc.feature_map(qf, theta))
    phk = np.abs(orc.feature_map(kf, theta))
    den = np.einsum("bnhd,bhd->bnh", qp, z) + eps
    adnum = np.abs(gf) / den[..., None]
    heads = lambda x: x.transpose(0, 2, 1, 3)
    aS = np.abs(S)
    Mt = heads(np.matmul(heads(adnum), aS.transpose(0, 1, 3, 2)))          # |S| |dnum|
    rot = _pair_sum if theta is not None else (lambda x: x)
    Mu = rot(Mt)                                                            # >= |R^T t|
    # dden = -(phi(q) . t) / den = -(ReLU(q) . R^T t) / den; this bounds the
    # terms of either form (|phi(q)_d| <= ReLU(q)_d + ReLU(q)_{d xor 1})
    Mdden = np.einsum("bnhd,bnhd->bnh", qp, Mu) / den
    M_dS = np.matmul(heads(phq).transpose(0, 1, 3, 2), heads(adnum))
    M_dz = np.einsum("bnh,bnhd->bhd", Mdden, qp)
    M_dQ = Mu + Mdden[..., None] * z[:, None]
    M_dK = rot(heads(np.matmul(heads(np.abs(vf)), M_dS.transpose(0, 1, 3, 2)))) + M_dz[:, None]
    M_dV = heads(np.matmul(heads(phk), M_dS))
    return M_dQ, M_dK, M_dV, M_dS, M_dz


def check_backward(got, ref, mags, io, Q, K, what=""):
    """got/ref/mags: (dQ, dK, dV, dS, dz). Element by element, with the bound above."""
    names = ("dQ", "dK", "dV", "dS", "dz")
    out_round = 2.0 ** -8 if io == "bf16" else 1e-6
    for i, (name, g, r, m) in enumerate(zip(names, got, ref, mags)):
        g = orc.to_f64(g)
        assert g.shape == r.shape, f"{what} {name}: shape {g.shape} != {r.shape}"
        assert np.isfinite(g).all(), f"{what} {name}: non-finite values"
        rr = out_round if i < 3 else 0.0
        err = np.abs(g - r)
        bound = rr * np.abs(r) + TOL_B[io] * m + 1e-30
        bad = err > bound
        assert not bad.any(), (f"{what} {name}: {bad.sum()} of {bad.size} outside the derived "
                               f"bound; worst ratio {float((err / bound).max()):.3g}")
    for name, g, x in (("dQ", got[0], Q), ("dK", got[1], K)):
        masked = orc.to_f64(x) <= 0
        assert (orc.to_f64(g)[masked] == 0).all(), f"{what} {name}: non-zero where the input <= 0"


# ---------------------------------------------------------------------------
# Token-causal attention.
#
# With M_i = |phi(q_i)| (|S0| + sum_{j<=i} |phi(k_j)|^T |v_j|) / den_i (every
# term of the numerator in absolute value):
#     |O_gpu - O_ref| <= out_round * |O_ref| + tol_c * M_i
# tol_c = 1e-4 for float32 arithmetic on exact operands; 2^-8 when the split
# partial states come from the tensor-core reduce with RoPE (the rotated key
# feature is rounded to bf16 there, 2^-9 per term).


def causal_magnitude(Q, K, V, eps, theta, S0=None, z0=None):
    """M_i above, by the same token-order recurrence as the oracle."""
    qf, kf, vf = orc.to_f64(Q), orc.to_f64(K), orc.to_f64(V)
    B, N, H, D_ = qf.shape
    phq = np.abs(orc.feature_map(qf, theta))
    phk = np.abs(orc.feature_map(kf, theta))
    qp, kp = orc.relu(qf), orc.relu(kf)
    A = np.zeros((B, H, D_, D_)) if S0 is None else np.abs(np.asarray(S0, np.float64))
    z = np.zeros((B, H, D_)) if z0 is None else np.asarray(z0, np.float64)
    av = np.abs(vf)
    M = np.empty((B, N, H, D_))
    for n in range(N):
        A = A + phk[:, n, :, :, None] * av[:, n, :, None, :]
        z = z + kp[:, n]
        den = np.einsum("bhd,bhd->bh", qp[:, n], z) + eps
        M[:, n] = np.einsum("bhd,bhde->bhe", phq[:, n], A) / den[..., None]
    return M


def check_causal(O_gpu, O_ref, M, io, tol, what=""):
    O_gpu = orc.to_f64(O_gpu)
    assert np.isfinite(O_gpu).all(), f"{what}: non-finite output"
    rtol, atol = NS_BF16 if io == "bf16" else NS_F32
    err = np.abs(O_gpu - O_ref)
    ns = atol + rtol * np.abs(O_ref)
    assert not (err > ns).any(), (f"{what}: {(err > ns).sum()} elements outside the "
                                  f"north-star tolerance; max err {err.max():.3g}")
    out_round = 2.0 ** -8 if io == "bf16" else 1e-6
    bound = out_round * np.abs(O_ref) + tol * M + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements outside the derived bound; worst "
                           f"ratio {float((err / bound).max()):.3g}")
