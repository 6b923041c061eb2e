"""GPU parity of la_qkv_state (QKV projection fused with the state reduce)
against the float64 oracle, element by element.

Bounds, derived from the arithmetic. Every projected feature is
y = x . w + b, summed in float32 on the tensor cores and rounded once to bf16;
the oracle rounds the exact value. With M_y = |x| . |w| + |b| (the magnitude
of the terms), the float32 sum y' is within tau = 2e-6 M_y of y (the products
of bf16 values are exact in float32; a float32 SGEMM of these inputs measured
at most 2e-7 M_y off on a B200, and the tensor-core sum matched cuBLAS's bf16
GEMM bit for bit). So the two roundings agree unless y lies within tau of a
rounding midpoint ("near"); there bf16(y') is within tau plus one bf16 step of
the oracle's value (for tiny y, tau spans many steps):
    E_y = tau + sp(|y| + tau) if near else 0,   |q_gpu - q_ref| <= E_q
(bit-exact elsewhere).
The state is summed from the rounded features, so the flips above carry into
it; with A = sum_n |phi(k_n)|^T |v_n|:
    |S_gpu - S_ref| <= sum_n rot(E_k)^T (|v| + E_v) + |phi(k)|^T E_v + tol_s A
    |z_gpu - z_ref| <= sum_n E_k + 1e-5 z_ref
rot = sum over the RoPE pair (|R e|_d <= e_d + e_(d xor 1)), identity without
RoPE. tol_s = 2e-5 without RoPE (exact bf16 MMA operands, float32
accumulation); 2^-8 with RoPE (the rotated key feature is rounded to bf16 for
the tensor cores, 2^-9 a term). Also checked: the spec bar
(rtol 2e-2, atol 2e-3) on Q, bitwise determinism, and N = 0.
"""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl

import linear_attention_diffusion_b200 as la

pytestmark = pytest.mark.gpu
D = 32
TAU = 2e-6


def _step_and_near(y, mag):
    """The oracle's rounding r of y, and the bound E on |bf16(y') - r| for a
    float32 sum y' within TAU*mag of y: 0 unless y is within TAU*mag of the
    rounding midpoint on its side."""
    r = orc.bf16_round(y)
    m, e = np.frexp(np.abs(r))
    sp = np.ldexp(1.0, e - 8)                     # bf16 spacing above |r|
    sp_low = np.where(m == 0.5, sp / 2, sp)       # below a power of two it halves
    away = np.abs(y) >= np.abs(r)
    dist = np.where(away, sp / 2, sp_low / 2) - np.abs(y - r)
    tau = TAU * mag
    near = (dist <= tau) | (r == 0)
    _, e2 = np.frexp(np.abs(y) + tau)
    return r, np.where(near, tau + np.ldexp(1.0, e2 - 8), 0.0)


def _project(X, W, b, rows):
    """Exact y and term magnitudes of the features `rows` of every token."""
    x = orc.to_f64(X)
    w = orc.to_f64(W)[rows]
    y = np.matmul(x, w.T)
    mag = np.matmul(np.abs(x), np.abs(w).T)
    if b is not None:
        bb = orc.to_f64(b)[rows]
        y = y + bb
        mag = mag + np.abs(bb)
    return y, mag


def _pair_sum(e):
    out = e.copy()
    out[..., 0::2] += e[..., 1::2]
    out[..., 1::2] += e[..., 0::2]
    return out


def _check_q(Q_gpu, q_ref, E_q, what):
    g = orc.to_f64(Q_gpu)
    assert np.isfinite(g).all(), what
    err = np.abs(g - q_ref)
    ns = 2e-3 + 2e-2 * np.abs(q_ref)
    assert not (err > ns).any(), f"{what} Q: {(err > ns).sum()} outside the north-star bar"
    bad = err > E_q
    assert not bad.any(), (f"{what} Q: {bad.sum()} of {bad.size} differ from the oracle's "
                           f"rounding away from a midpoint; max err {err.max():.3g}")


def _check_state(S_gpu, z_gpu, k, v, Ek, Ev, theta, rope, what, heads=None):
    """k, v: the oracle's rounded features [B, N, h, 32]; Ek, Ev: their flip bounds."""
    S_ref, z_ref = orc.state_reduce(k, v, theta)
    phik = np.abs(orc.feature_map(k, theta))
    av = np.abs(v)
    rot = _pair_sum if rope else (lambda e: e)
    hd = lambda x: x.transpose(0, 2, 3, 1)          # [B, h, 32, N]
    hn = lambda x: x.transpose(0, 2, 1, 3)          # [B, h, N, 32]
    A = np.matmul(hd(phik), hn(av))
    flip = np.matmul(hd(rot(Ek)), hn(av + Ev)) + np.matmul(hd(phik), hn(Ev))
    tol_s = 2.0 ** -8 if rope else 2e-5
    Sg = orc.to_f64(S_gpu)
    zg = orc.to_f64(z_gpu)
    if heads is not None:
        Sg, zg = Sg[:, heads], zg[:, heads]
    err = np.abs(Sg - S_ref)
    bound = flip + tol_s * A + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what} S: {bad.sum()} of {bad.size} outside the bound; worst "
                           f"ratio {float((err / bound).max()):.3g}")
    zerr = np.abs(zg - z_ref)
    zb = Ek.sum(axis=1) + 1e-5 * z_ref + 1e-30
    assert not (zerr > zb).any(), f"{what} z: worst ratio {float((zerr / zb).max()):.3g}"


def _inputs(B, N, H, C, seed, with_bias=True):
    w = wl.Workload("case", B=B, N=N, H=H)
    X, W, b = wl.make_projection(w, C, seed)
    return X, W, (b if with_bias else None)


def _run(X, W, b, rope_grid=None, t_offset=0):
    dev = torch.device("cuda:0")
    Q, S, z = la.qkv_state(X.to(dev), W.to(dev), None if b is None else b.to(dev),
                           rope_grid=rope_grid, t_offset=t_offset)
    torch.cuda.synchronize()
    assert la.la_device_error() == 0, "a kernel gave up a bounded wait"
    return Q.cpu(), S.cpu(), z.cpu()


CASES = [
    # B, N, H, C, bias, rope grid (T, Hh, W), t_offset
    (2, 300, 6, 192, True, None, 0),        # ragged tokens, head group and query tile
    (4, 4000, 7, 136, True, None, 0),       # runs of 2 tiles; C not a multiple of 64
    (1, 105, 5, 160, False, (3, 5, 7), 2),  # RoPE with an offset, no bias
    (1, 6240, 24, 96, True, (4, 30, 52), 20),  # RoPE, runs of 2 tiles
    (1, 200, 70, 2240, True, None, 0),      # Sana-1.6B widths, two token tiles
    (3, 1, 1, 8, True, None, 0),            # one token, one head, one channel group
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:4])))
def test_qkv_state_matches_oracle(cuda_device, case):
    B, N, H, C, with_bias, grid, t_off = case
    X, W, b = _inputs(B, N, H, C, seed=11 + N, with_bias=with_bias)
    Q, S, z = _run(X, W, b, grid, t_off)
    theta = orc.rope_angles(*grid, t_off) if grid is not None else None
    q_o, S_o, z_o = orc.qkv_state(X, W, b, H, theta)
    hd = H * D
    y, mag = _project(X, W, b, np.arange(3 * hd))
    r, E = _step_and_near(y, mag)
    assert np.array_equal(r[..., :hd].reshape(B, N, H, D), q_o)  # the test's view of the oracle
    _check_q(Q, q_o, E[..., :hd].reshape(B, N, H, D), str(case))
    k = r[..., hd:2 * hd].reshape(B, N, H, D)
    v = r[..., 2 * hd:].reshape(B, N, H, D)
    Ek = E[..., hd:2 * hd].reshape(B, N, H, D)
    Ev = E[..., 2 * hd:].reshape(B, N, H, D)
    assert np.allclose(orc.state_reduce(k, v, theta)[0], S_o, rtol=0, atol=0)
    _check_state(S, z, k, v, Ek, Ev, theta, grid is not None, str(case))


def test_qkv_state_full_size_sampled(cuda_device):
    """The bench's workload and launch (Sana-1.6B 1024px layer, C = 2240): Q at
    sampled tokens, S and z of sampled heads over every token."""
    w = wl.WORKLOADS["sana1.6b_1024px"]
    C = wl.hidden_width(w)
    X, W, b = wl.make_projection(w, C, seed=30)
    Q, S, z = _run(X, W, b)
    hd = w.H * D
    rng = np.random.default_rng(5)
    toks = np.sort(rng.choice(w.N, size=48, replace=False))
    toks[-1] = w.N - 1
    Xs = X[:, toks]
    y, mag = _project(Xs, W, b, np.arange(hd))
    r, E = _step_and_near(y, mag)
    q_o, _, _ = orc.qkv_state(Xs[:, :4], W, b, w.H)  # the oracle itself, on a few tokens
    assert np.array_equal(r[:, :4].reshape(w.B, 4, w.H, D), q_o)
    _check_q(Q[:, toks], r.reshape(w.B, len(toks), w.H, D), E.reshape(w.B, len(toks), w.H, D),
             "1024px sampled tokens")
    heads = [0, 33, 69]
    k_o, v_o = orc.key_value_heads(X, W, b, w.H, heads)
    rows_k = np.concatenate([np.arange(hd + D * h, hd + D * h + D) for h in heads])
    yk, mk = _project(X, W, b, rows_k)
    yv, mv = _project(X, W, b, rows_k + hd)
    rk, Ek = _step_and_near(yk, mk)
    rv, Ev = _step_and_near(yv, mv)
    shp = (w.B, w.N, len(heads), D)
    assert np.array_equal(rk.reshape(shp), k_o) and np.array_equal(rv.reshape(shp), v_o)
    _check_state(S, z, k_o, v_o, Ek.reshape(shp), Ev.reshape(shp), None, False,
                 "1024px sampled heads", heads=heads)


def test_qkv_state_is_deterministic(cuda_device):
    X, W, b = _inputs(2, 2500, 10, 320, seed=4)
    first = _run(X, W, b)
    second = _run(X, W, b)
    for a, c in zip(first, second):
        assert torch.equal(a, c)


def test_qkv_state_empty_sequence(cuda_device):
    dev = torch.device("cuda:0")
    B, H, C = 2, 3, 64
    shape = la.make_shape(B, 0, H)
    X = torch.empty((B, 0, C), dtype=torch.bfloat16, device=dev)
    W = wl.make_tensor((3 * H * D, C), 1).to(dev)
    Q = torch.empty((B, 0, H, D), dtype=torch.bfloat16, device=dev)
    S = torch.full((B, H, D, D), 7.0, device=dev)
    z = torch.full((B, H, D), 7.0, device=dev)
    la.la_qkv_state(shape, C, X, W, None, Q, S, z, None)
    torch.cuda.synchronize()
    assert (S == 0).all() and (z == 0).all()


def test_qkv_state_video_rope_full_size_sampled(cuda_device):
    """SANA-Video 480p grid (21 x 30 x 52 tokens, 3D RoPE on the keys, C = 2240):
    Q at sampled tokens, S and z of sampled heads over every token."""
    w = wl.WORKLOADS["sanavideo_480p"]
    C = wl.hidden_width(w)
    X, W, b = wl.make_projection(w, C, seed=31)
    Q, S, z = _run(X, W, b, rope_grid=(w.T, w.Hh, w.W))
    hd = w.H * D
    rng = np.random.default_rng(6)
    toks = np.sort(rng.choice(w.N, size=32, replace=False))
    toks[-1] = w.N - 1
    y, mag = _project(X[:, toks], W, b, np.arange(hd))
    r, E = _step_and_near(y, mag)
    _check_q(Q[:, toks], r.reshape(w.B, len(toks), w.H, D), E.reshape(w.B, len(toks), w.H, D),
             "480p sampled tokens")
    heads = [1, 38, 69]
    theta = orc.rope_angles(w.T, w.Hh, w.W, 0)
    k_o, v_o = orc.key_value_heads(X, W, b, w.H, heads)
    rows_k = np.concatenate([np.arange(hd + D * h, hd + D * h + D) for h in heads])
    yk, mk = _project(X, W, b, rows_k)
    yv, mv = _project(X, W, b, rows_k + hd)
    rk, Ek = _step_and_near(yk, mk)
    rv, Ev = _step_and_near(yv, mv)
    shp = (w.B, w.N, len(heads), D)
    assert np.array_equal(rk.reshape(shp), k_o) and np.array_equal(rv.reshape(shp), v_o)
    _check_state(S, z, k_o, v_o, Ek.reshape(shp), Ev.reshape(shp), theta, True,
                 "480p sampled heads", heads=heads)
