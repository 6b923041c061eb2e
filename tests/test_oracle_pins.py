"""Pins of the float64 oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: a hand-worked
example, a closed form, an invariant, or an independent formulation (complex
multiplication for RoPE, the block-masked quadratic form for the carry).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
D = 32


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _qkv(B, N, H, seed, Nk=None):
    Nk = N if Nk is None else Nk
    return (_rand((B, N, H, D), seed), _rand((B, Nk, H, D), seed + 1),
            _rand((B, Nk, H, D), seed + 2))


def _vec(spec):
    x = np.zeros(D)
    for k, val in spec.items():
        x[int(k)] = val
    return x


# --------------------------------------------------------------------------
# Hand-worked examples (tests/golden)


def test_worked_example_relu_attention():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_relu.json")))
    Q = _vec(g["q"]).reshape(1, 1, 1, D)
    K = np.stack([_vec(s) for s in g["k"]]).reshape(1, 2, 1, D)
    V = np.stack([_vec(s) for s in g["v"]]).reshape(1, 2, 1, D)
    want = _vec(g["expected_o"])
    for out in (orc.attention(Q, K, V, g["eps"]),
                orc.attention_bruteforce(Q, K, V, g["eps"])):
        np.testing.assert_allclose(out[0, 0, 0], want, rtol=1e-15, atol=1e-15)


def test_rope_convention_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "rope_convention.json")))
    T, Hh, W, t0 = (g["grid"][k] for k in ("T", "Hh", "W", "t_offset"))
    theta = orc.rope_angles(T, Hh, W, t0)
    N = T * Hh * W
    for case in g["cases"]:
        t, h, w = case["token"]
        n = (t * Hh + h) * W + w
        d = case["dim"]
        ang = eval(case["angle"], {"__builtins__": {}}, {})  # arithmetic only
        for which, want in ((d, (math.cos(ang), math.sin(ang))),
                            (d + 1, (-math.sin(ang), math.cos(ang)))):
            x = np.zeros((1, N, 1, D))
            x[0, n, 0, which] = 1.0
            y = orc.rope_rotate(x, theta)[0, n, 0]
            np.testing.assert_allclose(y[d:d + 2], want, rtol=0, atol=1e-14,
                                       err_msg=case["note"])
            others = np.delete(y, [d, d + 1])
            assert np.all(others == 0.0), case["note"]


# --------------------------------------------------------------------------
# RoPE against an independent formulation and its invariants


def test_rope_equals_complex_multiplication():
    theta = orc.rope_angles(3, 4, 5, t_offset=7)
    x = _rand((2, 60, 3, D), 11)
    y = orc.rope_rotate(x, theta)
    zc = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * theta)[None, :, None, :]
    np.testing.assert_allclose(y[..., 0::2], zc.real, atol=1e-13)
    np.testing.assert_allclose(y[..., 1::2], zc.imag, atol=1e-13)


def test_rope_zero_positions_is_identity_and_norm_preserving():
    x = _rand((1, 1, 2, D), 3)
    th0 = orc.rope_angles(1, 1, 1, t_offset=0)
    np.testing.assert_array_equal(orc.feature_map(x, th0), orc.relu(x))
    th = orc.rope_angles(4, 3, 5, t_offset=2)
    x = _rand((1, 60, 2, D), 4)
    np.testing.assert_allclose(np.linalg.norm(orc.feature_map(x, th), axis=-1),
                               np.linalg.norm(orc.relu(x), axis=-1), rtol=1e-13)


@pytest.mark.parametrize("axis", ["t", "h", "w"])
def test_rope_relative_shift_invariance(axis):
    # phi(q_i).phi(k_j) depends only on p_i - p_j, so shifting every query and
    # key position along one axis by the same amount leaves O unchanged.
    T, Hh, W = 2, 3, 4
    N = T * Hh * W
    Q, K, V = _qkv(1, N, 2, 21)
    t, h, w = orc.rope_positions(T, Hh, W, 0)
    pos = {"t": t, "h": h, "w": w}

    def angles(shift):
        p = dict(pos)
        p[axis] = p[axis] + shift
        cols = []
        for ax, _f, width in orc.ROPE_SEGMENTS:
            for k in range(width // 2):
                cols.append(p[ax] * 10000.0 ** (-2.0 * k / width))
        return np.stack(cols, 1)

    np.testing.assert_allclose(angles(0), orc.rope_angles(T, Hh, W, 0), rtol=0, atol=0)
    th0, th9 = angles(0), angles(9)
    o0 = orc.attention_bruteforce(Q, K, V, 1e-6, th0, th0)
    o9 = orc.attention_bruteforce(Q, K, V, 1e-6, th9, th9)
    np.testing.assert_allclose(o9, o0, rtol=1e-10, atol=1e-12)
    # ...whereas shifting the queries alone changes it (the shift is not a no-op)
    o_q = orc.attention_bruteforce(Q, K, V, 1e-6, th9, th0)
    assert np.max(np.abs(o_q - o0)) > 1e-3


def test_block_t_offset_is_global_frame_index():
    th_a = orc.rope_angles(4, 2, 3, t_offset=0)
    th_b = orc.rope_angles(2, 2, 3, t_offset=2)
    np.testing.assert_array_equal(th_a[12:], th_b)


# --------------------------------------------------------------------------
# The quadratic form: closed forms and invariants


def test_one_hot_keys_give_group_means():
    # With one-hot keys and a one-hot query, ReLU(q).ReLU(k_j) is 1 for keys in
    # the query's group and 0 elsewhere, so O is the mean of that group's values.
    rng = np.random.default_rng(5)
    N = 40
    groups = rng.integers(0, D, N)
    K = np.zeros((1, N, 1, D))
    K[0, np.arange(N), 0, groups] = 1.0
    V = _rand((1, N, 1, D), 6)
    for a in np.unique(groups)[:5]:
        Q = np.zeros((1, 1, 1, D))
        Q[0, 0, 0, a] = 1.0
        want = V[0, groups == a, 0].mean(axis=0)
        for out in (orc.attention_bruteforce(Q, K, V, 0.0), orc.attention(Q, K, V, 0.0)):
            np.testing.assert_allclose(out[0, 0, 0], want, rtol=1e-13, atol=1e-14)


def test_single_key_closed_form():
    Q, K, V = _qkv(1, 3, 1, 8, Nk=1)
    Q, K = np.abs(Q), np.abs(K)
    eps = 0.25
    w = (Q[0, :, 0] @ K[0, 0, 0])
    want = w[:, None] * V[0, 0, 0][None, :] / (w[:, None] + eps)
    np.testing.assert_allclose(orc.attention(Q, K, V, eps)[0, :, 0], want, rtol=1e-13)


@pytest.mark.parametrize("rope", [False, True])
def test_factorised_equals_bruteforce(rope):
    T, Hh, W = 3, 4, 5
    N = T * Hh * W
    Q, K, V = _qkv(2, N, 3, 31)
    th = orc.rope_angles(T, Hh, W, 4) if rope else None
    fact = orc.attention(Q, K, V, 1e-6, th)
    brute = orc.attention_bruteforce(Q, K, V, 1e-6, th, th)
    np.testing.assert_allclose(fact, brute, rtol=1e-12, atol=1e-14)


def test_constant_values_closed_form():
    # v_j = c for every j gives O_i = c * x_i / (x_i + eps), x_i = ReLU(q_i).z.
    B, N, H = 1, 50, 2
    Q, K, _ = _qkv(B, N, H, 41)
    Q = Q * 1e-6  # make eps matter
    c = _rand((D,), 42)
    V = np.broadcast_to(c, (B, N, H, D)).copy()
    eps = 1e-6
    z = orc.relu(K).sum(axis=1)
    x = np.einsum("bnhd,bhd->bnh", orc.relu(Q), z)
    want = c[None, None, None, :] * (x / (x + eps))[..., None]
    np.testing.assert_allclose(orc.attention(Q, K, V, eps), want, rtol=1e-12)
    np.testing.assert_allclose(orc.attention_bruteforce(Q, K, V, eps), want, rtol=1e-12)


def test_convex_bound_and_degenerate_rows():
    Q, K, V = _qkv(1, 64, 2, 51)
    Q[0, :8] = -np.abs(Q[0, :8])  # ReLU(q) = 0 rows
    O = orc.attention(Q, K, V, 1e-6)
    assert np.all(O[0, :8] == 0.0)
    vmax = np.abs(V).max(axis=(1, 3))  # per (b, h)
    assert np.all(np.abs(O).max(axis=(1, 3)) <= vmax + 1e-12)


def test_key_permutation_linearity_and_scale():
    Q, K, V = _qkv(1, 40, 2, 61)
    O = orc.attention(Q, K, V, 0.0)
    perm = np.random.default_rng(1).permutation(40)
    np.testing.assert_allclose(orc.attention(Q, K[:, perm], V[:, perm], 0.0), O, rtol=1e-12, atol=1e-14)
    V2 = _rand(V.shape, 62)
    np.testing.assert_allclose(orc.attention(Q, K, 2 * V - 3 * V2, 0.0),
                               2 * O - 3 * orc.attention(Q, K, V2, 0.0), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(orc.attention(3.5 * Q, 0.25 * K, V, 0.0), O, rtol=1e-12, atol=1e-14)
    # an all-negative key is cut by ReLU and changes nothing
    Kx = np.concatenate([K, -np.abs(_rand((1, 1, 2, D), 63))], axis=1)
    Vx = np.concatenate([V, _rand((1, 1, 2, D), 64)], axis=1)
    np.testing.assert_allclose(orc.attention(Q, Kx, Vx, 0.0), O, rtol=1e-12, atol=1e-14)


def test_state_additivity():
    T, Hh, W = 4, 3, 5
    N = T * Hh * W
    _, K, V = _qkv(1, N, 2, 71)
    th = orc.rope_angles(T, Hh, W, 0)
    S, z = orc.state_reduce(K, V, th)
    S1, z1 = orc.state_reduce(K[:, :17], V[:, :17], th[:17])
    S2, z2 = orc.state_reduce(K[:, 17:], V[:, 17:], th[17:])
    np.testing.assert_allclose(S, S1 + S2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, z1 + z2, rtol=1e-13)
    assert S.shape == (1, 2, D, D) and z.shape == (1, 2, D)
    # constant-size state: D x D plus D, whatever N is
    Sb, zb = orc.state_reduce(K[:, :3], V[:, :3], th[:3])
    assert Sb.shape == S.shape and zb.shape == z.shape


def test_denominator_is_unrotated():
    # Rotating the keys changes S but not z; rotating the queries changes the
    # numerator only.
    T, Hh, W = 2, 2, 3
    N = T * Hh * W
    Q, K, V = _qkv(1, N, 1, 81)
    th = orc.rope_angles(T, Hh, W, 1)
    _, z_plain = orc.state_reduce(K, V)
    _, z_rope = orc.state_reduce(K, V, th)
    np.testing.assert_array_equal(z_plain, z_rope)
    # the denominator of the brute force equals the plain ReLU one
    ones = np.ones_like(V)
    S_r, z_r = orc.state_reduce(K, ones, th)
    x = np.einsum("bnhd,bhd->bnh", orc.relu(Q), z_r)
    assert np.all(x > 0)


# --------------------------------------------------------------------------
# Block-causal state carry


def _blocks(M, steps, T, Hh, W, H, seed, rope=True):
    N = T * Hh * W
    blocks = []
    for m in range(M):
        th = orc.rope_angles(T, Hh, W, m * T) if rope else None
        passes = []
        for s in range(steps):
            passes.append(_qkv(1, N, H, seed + 1000 * m + 10 * s) + (th,))
        _, Ku, Vu = _qkv(1, N, H, seed + 1000 * m + 10 * steps)
        blocks.append({"passes": passes, "update": (Ku, Vu, th)})
    return blocks


@pytest.mark.parametrize("rope", [False, True])
def test_block_carry_equals_block_masked_quadratic(rope):
    M, steps, T, Hh, W, H = 3, 2, 2, 2, 3, 2
    eps = 1e-6
    blocks = _blocks(M, steps, T, Hh, W, H, 100, rope)
    want = orc.block_causal_bruteforce(blocks, eps)
    S = np.zeros((1, H, D, D))
    z = np.zeros((1, H, D))
    for m, blk in enumerate(blocks):
        for s, (Q, K, V, th) in enumerate(blk["passes"]):
            O, S2, z2 = orc.block_causal_step(Q, K, V, S, z, 0, eps, th)
            np.testing.assert_array_equal(S2, S)
            np.testing.assert_allclose(O, want[m][s], rtol=1e-11, atol=1e-13)
        Ku, Vu, th = blk["update"]
        none, S, z = orc.block_causal_step(None, Ku, Vu, S, z, 2, eps, th)
        assert none is None
    # the final carry is the state of all update passes together
    Kall = np.concatenate([b["update"][0] for b in blocks], axis=1)
    Vall = np.concatenate([b["update"][1] for b in blocks], axis=1)
    thall = None if not rope else np.concatenate([b["update"][2] for b in blocks], 0)
    S_all, z_all = orc.state_reduce(Kall, Vall, thall)
    np.testing.assert_allclose(S, S_all, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, z_all, rtol=1e-13)


def test_single_block_is_noncausal_and_update1_matches():
    Q, K, V = _qkv(1, 30, 2, 130)
    S0 = np.zeros((1, 2, D, D))
    z0 = np.zeros((1, 2, D))
    O0, _, _ = orc.block_causal_step(Q, K, V, S0, z0, 0, 1e-6)
    np.testing.assert_allclose(O0, orc.attention(Q, K, V, 1e-6), rtol=1e-13)
    O1, S1, z1 = orc.block_causal_step(Q, K, V, S0, z0, 1, 1e-6)
    np.testing.assert_array_equal(O1, O0)
    S_own, z_own = orc.state_reduce(K, V)
    np.testing.assert_array_equal(S1, S_own)
    np.testing.assert_array_equal(z1, z_own)


# --------------------------------------------------------------------------
# Backward pass: pinned to central finite differences of the quadratic form


def _fd_grad(f, X, h=1e-6):
    g = np.zeros_like(X)
    it = np.nditer(X, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        Xp = X.copy()
        Xm = X.copy()
        Xp[idx] += h
        Xm[idx] -= h
        g[idx] = (f(Xp) - f(Xm)) / (2 * h)
    return g


def _away_from_kinks(X, margin=0.05):
    # keep every entry at least `margin` away from 0 so ReLU is smooth there
    return np.where(np.abs(X) < margin, np.sign(X + 1e-12) * margin, X)


@pytest.mark.parametrize("rope", [False, True])
def test_backward_matches_finite_differences_of_the_quadratic_form(rope):
    T, Hh, W = 2, 2, 3
    N, H = T * Hh * W, 2
    Q, K, V = (_away_from_kinks(x) for x in _qkv(1, N, H, 300))
    G = _rand(V.shape, 304)          # dL/dO for L = sum(O * G)
    eps = 0.1
    th = orc.rope_angles(T, Hh, W, 3) if rope else None

    def loss_q(Qx):
        return float((orc.attention_bruteforce(Qx, K, V, eps, th, th) * G).sum())

    def loss_k(Kx):
        return float((orc.attention_bruteforce(Q, Kx, V, eps, th, th) * G).sum())

    def loss_v(Vx):
        return float((orc.attention_bruteforce(Q, K, Vx, eps, th, th) * G).sum())

    dQ, dK, dV, _, _ = orc.backward(Q, K, V, G, eps, th)
    np.testing.assert_allclose(dQ, _fd_grad(loss_q, Q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dK, _fd_grad(loss_k, K), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dV, _fd_grad(loss_v, V), rtol=1e-6, atol=1e-8)


def test_backward_state_gradients_are_the_chain_rule_through_S_and_z():
    # dS and dz: perturbing S (or z) directly in the apply changes the loss by
    # <dS, dS_pert> (resp. <dz, dz_pert>) to first order.
    Q, K, V = _qkv(1, 20, 2, 310)
    G = _rand(V.shape, 311)
    eps = 0.05
    S, z = orc.state_reduce(K, V)
    _, _, _, dS, dz = orc.backward(Q, K, V, G, eps)
    P = _rand(S.shape, 312)
    h = 1e-6
    lp = (orc.apply(Q, S + h * P, z, eps) * G).sum()
    lm = (orc.apply(Q, S - h * P, z, eps) * G).sum()
    np.testing.assert_allclose((lp - lm) / (2 * h), (dS * P).sum(), rtol=1e-6)
    Pz = np.abs(_rand(z.shape, 313))
    lp = (orc.apply(Q, S, z + h * Pz, eps) * G).sum()
    lm = (orc.apply(Q, S, z - h * Pz, eps) * G).sum()
    np.testing.assert_allclose((lp - lm) / (2 * h), (dz * Pz).sum(), rtol=1e-6)


def test_backward_negative_inputs_get_zero_gradient():
    Q, K, V = _qkv(1, 16, 1, 320)
    Q[0, :4] = -np.abs(Q[0, :4])
    K[0, :4] = -np.abs(K[0, :4])
    dQ, dK, dV, _, _ = orc.backward(Q, K, V, _rand(V.shape, 321), 1e-3)
    assert np.all(dQ[0, :4] == 0) and np.all(dK[0, :4] == 0)
    assert np.all(dV[0, :4] == 0)  # an all-negative key carries no value


# --------------------------------------------------------------------------
# Token-causal attention (a query sees the keys up to and including its own
# token)


@pytest.mark.parametrize("rope", [False, True])
def test_causal_recurrence_equals_masked_quadratic_form(rope):
    T, Hh, W = 2, 3, 5
    N = T * Hh * W
    Q, K, V = _qkv(2, N, 3, 71)
    th = orc.rope_angles(T, Hh, W, 2) if rope else None
    O, S, z = orc.causal_attention(Q, K, V, 1e-6, th)
    np.testing.assert_allclose(O, orc.causal_bruteforce(Q, K, V, 1e-6, th), rtol=1e-12,
                               atol=1e-14)
    # the final state is the whole sequence's state
    S_ref, z_ref = orc.state_reduce(K, V, th)
    np.testing.assert_allclose(S, S_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z, z_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("rope", [False, True])
def test_causal_last_token_is_noncausal_and_first_token_closed_form(rope):
    T, Hh, W = 3, 2, 4
    N = T * Hh * W
    Q, K, V = _qkv(1, N, 2, 73)
    th = orc.rope_angles(T, Hh, W, 0) if rope else None
    O, _, _ = orc.causal_attention(Q, K, V, 1e-6, th)
    full = orc.attention(Q, K, V, 1e-6, th)
    np.testing.assert_allclose(O[:, -1], full[:, -1], rtol=1e-12, atol=1e-14)
    # token 0 sees only itself
    qp, kp = np.maximum(Q[:, 0], 0), np.maximum(K[:, 0], 0)
    phq = qp if th is None else orc.rope_rotate(qp[:, None], th[:1])[:, 0]
    phk = kp if th is None else orc.rope_rotate(kp[:, None], th[:1])[:, 0]
    w = (phq * phk).sum(-1)
    den = (qp * kp).sum(-1) + 1e-6
    np.testing.assert_allclose(O[:, 0], (w / den)[..., None] * V[:, 0], rtol=1e-12, atol=1e-14)


def test_causal_prefix_and_carry_compose():
    # causality: the first m outputs do not depend on later tokens; streaming:
    # running the second part from the first part's final state continues the
    # sequence exactly
    Q, K, V = _qkv(2, 40, 3, 75)
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    Q2[:, 25:] += 5.0
    K2[:, 25:] *= -2.0
    V2[:, 25:] = 7.0
    a, _, _ = orc.causal_attention(Q, K, V, 1e-6)
    b, _, _ = orc.causal_attention(Q2, K2, V2, 1e-6)
    np.testing.assert_array_equal(a[:, :25], b[:, :25])
    first, S1, z1 = orc.causal_attention(Q[:, :17], K[:, :17], V[:, :17], 1e-6)
    rest, S2, z2 = orc.causal_attention(Q[:, 17:], K[:, 17:], V[:, 17:], 1e-6, None, S1, z1)
    np.testing.assert_allclose(np.concatenate([first, rest], axis=1), a, rtol=1e-12, atol=1e-14)
    _, S_all, z_all = orc.causal_attention(Q, K, V, 1e-6)
    np.testing.assert_allclose(S2, S_all, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(z2, z_all, rtol=1e-12, atol=1e-12)


def test_causal_is_block_causal_with_one_token_blocks():
    # the block-causal mode with blocks of one token, each applied once with
    # update = 1, is token-causal attention
    T, Hh, W = 4, 1, 1
    Q, K, V = _qkv(1, T, 2, 77)
    th = orc.rope_angles(T, Hh, W, 0)
    O, _, _ = orc.causal_attention(Q, K, V, 1e-6, th)
    S = np.zeros((1, 2, D, D))
    z = np.zeros((1, 2, D))
    for t in range(T):
        o, S, z = orc.block_causal_step(Q[:, t:t + 1], K[:, t:t + 1], V[:, t:t + 1], S, z, 1,
                                        1e-6, th[t:t + 1])
        np.testing.assert_allclose(o[:, 0], O[:, t], rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------
# Temporal depth-wise convolution with the block-causal conv cache


def _conv_inputs(B, T, Hh, W, C, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, Hh, W, C)), rng.standard_normal((C, 3)),
            rng.standard_normal(C))


def test_temporal_conv_is_a_zero_padded_correlation_plus_shortcut():
    from scipy.ndimage import correlate1d
    x, w, b = _conv_inputs(2, 7, 3, 4, 5, 81)
    y, f = orc.temporal_conv(x, w, b)
    ref = np.empty_like(x)
    for c in range(x.shape[-1]):
        ref[..., c] = correlate1d(x[..., c], w[c], axis=1, mode="constant", cval=0.0)
    np.testing.assert_allclose(y, x + b + ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(f, x[:, -1])


def test_temporal_conv_impulse_response_fixes_tap_order():
    # a single non-zero frame t0: frame t0 - 1 sees it as its next frame (tap
    # 2), frame t0 + 1 as its previous frame (tap 0)
    B, T, Hh, W, C = 1, 6, 1, 1, 3
    x = np.zeros((B, T, Hh, W, C))
    x[0, 3, 0, 0] = [1.0, 2.0, -1.0]
    w = np.array([[0.5, 0.25, 0.125], [1.0, 2.0, 3.0], [-1.0, 0.0, 1.0]])
    y, _ = orc.temporal_conv(x, w)
    v = x[0, 3, 0, 0]
    np.testing.assert_allclose(y[0, 2, 0, 0], w[:, 2] * v)
    np.testing.assert_allclose(y[0, 3, 0, 0], v + w[:, 1] * v)
    np.testing.assert_allclose(y[0, 4, 0, 0], w[:, 0] * v)
    assert not y[0, [0, 1, 5]].any()


def test_temporal_conv_cache_carries_the_previous_block():
    # block 2 run with block 1's cache equals block 2 alone plus the previous
    # frame's contribution at its first frame; the cache is the last frame
    x, w, b = _conv_inputs(2, 9, 2, 3, 4, 83)
    x1, x2 = x[:, :5], x[:, 5:]
    y1, f1 = orc.temporal_conv(x1, w, b)
    y2, f2 = orc.temporal_conv(x2, w, b, f1)
    alone, _ = orc.temporal_conv(x2, w, b)
    np.testing.assert_array_equal(f1, x[:, 4])
    np.testing.assert_array_equal(f2, x[:, 8])
    np.testing.assert_allclose(y2[:, 1:], alone[:, 1:], rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(y2[:, 0], alone[:, 0] + w[:, 0] * x[:, 4], rtol=1e-13, atol=1e-13)
    # and block 1's last frame does not see block 2 (block-causal), unlike a
    # whole-clip convolution
    whole, _ = orc.temporal_conv(x, w, b)
    np.testing.assert_allclose(y1[:, 4] + w[:, 2] * x[:, 5], whole[:, 4], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(y2, whole[:, 5:], rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------
# QKV projection fused with the state reduce


def test_bf16_round_ties_to_even_and_matches_torch():
    """bf16 keeps 8 significant bits: 257 lies halfway between 256 and 258 and
    goes to the even 256; 259 goes to 260; 1 + 3 * 2^-8 goes to 1 + 2^-6. On
    float32-representable values the rounding equals torch's own conversion."""
    import torch
    got = orc.bf16_round(np.array([257.0, 259.0, 1 + 3 * 2.0 ** -8, -257.0, 0.0, 1 + 2.0 ** -8]))
    assert got.tolist() == [256.0, 260.0, 1 + 2.0 ** -6, -256.0, 0.0, 1.0]
    x = np.random.default_rng(5).standard_normal(20000).astype(np.float32).astype(np.float64)
    x *= np.exp2(np.random.default_rng(6).integers(-20, 20, x.shape))
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(orc.bf16_round(x), ref)


def _qkv_bruteforce(X, W, bias, H, theta):
    """Pure-Python loops over tokens, heads, dims and input channels."""
    B, N, C = X.shape
    hd = H * D
    S = np.zeros((B, H, D, D))
    z = np.zeros((B, H, D))
    Q = np.zeros((B, N, H, D))
    for b in range(B):
        for n in range(N):
            row = [sum(X[b, n, c] * W[j, c] for c in range(C)) + (bias[j] if bias is not None else 0.0)
                   for j in range(3 * hd)]
            row = [float(orc.bf16_round(np.array(v))) for v in row]
            for h in range(H):
                q = row[h * D:(h + 1) * D]
                k = row[hd + h * D:hd + (h + 1) * D]
                v = row[2 * hd + h * D:2 * hd + (h + 1) * D]
                kp = [max(t, 0.0) for t in k]
                phi = list(kp)
                if theta is not None:
                    for i in range(D // 2):
                        c, s = math.cos(theta[n, i]), math.sin(theta[n, i])
                        phi[2 * i] = kp[2 * i] * c - kp[2 * i + 1] * s
                        phi[2 * i + 1] = kp[2 * i] * s + kp[2 * i + 1] * c
                Q[b, n, h] = q
                for d in range(D):
                    z[b, h, d] += kp[d]
                    for e in range(D):
                        S[b, h, d, e] += phi[d] * v[e]
    return Q, S, z


@pytest.mark.parametrize("rope", [False, True])
def test_qkv_state_equals_loops_over_the_projection(rope):
    """Small integers keep every product and sum exact in float64, and some
    projected values need rounding (|y| > 256), so the loops and the oracle
    must agree exactly: row blocks (q, k, v), head slices, bias, rounding,
    ReLU and the state's orientation S[d][e] = sum phi(k)_d v_e."""
    rng = np.random.default_rng(17)
    B, N, C, H = 2, 3, 16, 2
    X = rng.integers(-12, 13, (B, N, C)).astype(np.float64)
    W = rng.integers(-9, 10, (3 * H * D, C)).astype(np.float64)
    bias = rng.integers(-3, 4, 3 * H * D).astype(np.float64)
    theta = orc.rope_angles(1, 1, N, 2) if rope else None
    Q, S, z = orc.qkv_state(X, W, bias, H, theta)
    Qr, Sr, zr = _qkv_bruteforce(X, W, bias, H, theta)
    Y = X @ W.T + bias
    assert ((np.abs(Y) > 256) & (Y % 2 != 0)).sum() > 10  # the rounding step is exercised
    assert np.array_equal(Q, Qr) and np.array_equal(z, zr)
    assert np.allclose(S, Sr, rtol=1e-12, atol=1e-9)
    if not rope:
        assert np.array_equal(S, Sr)


def test_qkv_state_with_selection_weights_is_the_state_reduce_of_the_inputs():
    """W that copies input channels into the key and value slots (a 0/1
    selection matrix) gives k, v = the selected inputs, so the fused state is
    the plain state reduce of those inputs (bf16 inputs round to themselves)."""
    rng = np.random.default_rng(3)
    B, N, H = 1, 50, 3
    C = 2 * H * D
    X = orc.bf16_round(rng.standard_normal((B, N, C)))
    W = np.zeros((3 * H * D, C))
    W[H * D:, :] = np.eye(C)
    Q, S, z = orc.qkv_state(X, W, None, H)
    K = X[..., :H * D].reshape(B, N, H, D)
    V = X[..., H * D:].reshape(B, N, H, D)
    S2, z2 = orc.state_reduce(K, V)
    assert np.array_equal(S, S2) and np.array_equal(z, z2)
    assert (Q == 0).all()


def test_key_value_heads_matches_the_full_projection():
    rng = np.random.default_rng(9)
    B, N, C, H = 1, 40, 24, 5
    X = orc.bf16_round(rng.standard_normal((B, N, C)))
    W = orc.bf16_round(rng.standard_normal((3 * H * D, C)) / np.sqrt(C))
    b = rng.standard_normal(3 * H * D) * 0.1
    _, k, v = orc.qkv_projection(X, W, b, H)
    k2, v2 = orc.key_value_heads(X, W, b, H, [1, 4])
    assert np.array_equal(k2, k[:, :, [1, 4]]) and np.array_equal(v2, v[:, :, [1, 4]])
