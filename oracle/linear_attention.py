"""Float64 oracle of ReLU linear attention, its 3D-RoPE variant and the
block-causal constant-memory state carry.

Test infrastructure: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code with
the CUDA library.

Sources (page title, then section):

[SANA]  "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
        Transformers", section "模型架构", item 2 (Linear DiT): every softmax
        self-attention is replaced by ReLU linear attention, and the shared
        terms sum_j ReLU(K_j)^T V_j and sum_j ReLU(K_j)^T are computed once and
        reused by every query.
[SV21]  "SANA-Video: Efficient Video Generation with Block Linear Diffusion
        Transformer", section 2.1: with the sum of phi(K_j)^T V_j computed in
        advance, each token costs O(D^2) instead of O(N D).
[SV22]  same page, section 2.2: RoPE is applied after ReLU, and the
        denominator leaves RoPE out, because a rotated denominator can come
        close to zero.
[SV23]  same page, section 2.3: the state S_j = phi(K_j)^T V_j and the key sum
        are accumulated over earlier blocks, in D x D plus D x 1 memory.
[SV4]   same page, section 4: the KV cache starts empty, each block runs its
        denoising steps against it, and after the last step the block's own
        state is folded in once.
[SVS2]  same page, "Stage 2": 3D RoPE over time, height and width.
[SI]    "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
        Transformers", section "Infra": the linear attention has a fused
        forward and backward (the backward pass below is its gradient).
[MJ]    SANA-Video article (mjgaz.cn), section "设计细节": later blocks integrate
        earlier blocks' features through the linear state, earlier blocks never
        see later ones, and each block sums the accumulated KV with its own.
[SV23t] SANA-Video section 2.3 read at token granularity (the pages' sum over
        j up to i - 1 with j indexing tokens): query i sees keys j <= i. The
        query's own token is included, as the block mode includes the block's
        own state; a token-level block of one token gives exactly this.

The pages lose the formulas of sections 2.1 and 2.3 in extraction. The
readings taken here:

* O_i = (phi(q_i) S) / (ReLU(q_i) . z + eps), with S = sum_j phi(k_j)^T v_j and
  z = sum_j ReLU(k_j); no 1/sqrt(D) scale; eps is added to the denominator.
* phi(x) = ReLU(x) without RoPE, and phi(x) = R(p) ReLU(x) with RoPE; z and
  the query in the denominator stay unrotated [SV22].
* 3D RoPE layout: dims [0,8) rotate with the frame index t, [8,20) with the
  row h, [20,32) with the column w. Pairs are interleaved, (2i, 2i+1). Pair k
  of a segment of width d uses theta = p * base^(-2k/d); base = 10000. The
  rotation maps (x0, x1) to (x0 cos - x1 sin, x0 sin + x1 cos). Tokens are in
  raster order n = (t*Hh + h)*W + w; t is the global frame index. This layout
  is not fixed by the pages (parity of the layout itself is pinned to this
  written convention, and by RoPE's relative-shift invariance).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

HEAD_DIM = 32
# (axis, first dim, number of dims) of the three RoPE segments.
ROPE_SEGMENTS = (("t", 0, 8), ("h", 8, 12), ("w", 20, 12))


def to_f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a torch tensor of any float type."""
    if hasattr(x, "detach"):  # torch tensor; bf16 -> f32 is exact
        x = x.detach().to("cpu")
        if str(x.dtype) != "torch.float64":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def relu(x: np.ndarray) -> np.ndarray:
    """The kernel function of linear attention [SANA]."""
    return np.maximum(x, 0.0)


def rope_positions(T: int, Hh: int, W: int, t_offset: int = 0):
    """(t, h, w) of each token of a T x Hh x W grid in raster order.

    t is global: the block's first frame has index ``t_offset``.
    """
    n = np.arange(T * Hh * W, dtype=np.int64)
    w = n % W
    h = (n // W) % Hh
    t = n // (W * Hh) + int(t_offset)
    return t, h, w


def rope_angles(T: int, Hh: int, W: int, t_offset: int = 0,
                base: float = 10000.0) -> np.ndarray:
    """Rotation angle of every (token, pair): array [N, D/2] in float64 [SVS2]."""
    t, h, w = rope_positions(T, Hh, W, t_offset)
    pos = {"t": t, "h": h, "w": w}
    cols = []
    for axis, _first, width in ROPE_SEGMENTS:
        for k in range(width // 2):
            inv_freq = float(base) ** (-2.0 * k / width)
            cols.append(pos[axis].astype(np.float64) * inv_freq)
    return np.stack(cols, axis=1)


def rope_rotate(x: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Rotate the pairs (2i, 2i+1) of x [B, N, H, D] by theta [N, D/2]."""
    c = np.cos(theta)[:, None, :]
    s = np.sin(theta)[:, None, :]
    even = x[..., 0::2]
    odd = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


def feature_map(x: np.ndarray, theta: Optional[np.ndarray] = None) -> np.ndarray:
    """phi(x): ReLU, then RoPE when ``theta`` is given (RoPE after ReLU) [SV22]."""
    xp = relu(x)
    return xp if theta is None else rope_rotate(xp, theta)


def state_reduce(K, V, theta: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """S[b,h] = sum_n phi(k_n)^T v_n  (D x D) and z[b,h] = sum_n ReLU(k_n)  (D).

    K, V: [B, N, H, D]. Returns S [B, H, D, D] and z [B, H, D] in float64.
    The key sum z is unrotated: it only enters the denominator [SANA, SV21, SV22].
    """
    K = to_f64(K)
    V = to_f64(V)
    kp = relu(K)
    phik = kp if theta is None else rope_rotate(kp, theta)
    # [B, H, D, N] @ [B, H, N, E] -> [B, H, D, E]
    S = np.matmul(phik.transpose(0, 2, 3, 1), V.transpose(0, 2, 1, 3))
    z = kp.sum(axis=1)
    return S, z


def apply(Q, S: np.ndarray, z: np.ndarray, eps: float,
          theta: Optional[np.ndarray] = None) -> np.ndarray:
    """O_i = phi(q_i) S / (ReLU(q_i) . z + eps), for Q [B, N, H, D].

    The numerator uses the rotated feature map, the denominator the unrotated
    ReLU [SV21, SV22]. Returns O [B, N, H, D] in float64.
    """
    Q = to_f64(Q)
    qp = relu(Q)
    phiq = qp if theta is None else rope_rotate(qp, theta)
    num = np.matmul(phiq.transpose(0, 2, 1, 3), S)  # [B, H, N, E]
    den = np.matmul(qp.transpose(0, 2, 1, 3), z[..., None])[..., 0] + float(eps)  # [B, H, N]
    out = num / den[..., None]
    return out.transpose(0, 2, 1, 3)


def apply_rows(Q, S: np.ndarray, z: np.ndarray, eps: float,
               theta: Optional[np.ndarray], rows: Sequence[int]) -> np.ndarray:
    """``apply`` restricted to the tokens ``rows`` (for sampled checks at full size)."""
    rows = np.asarray(rows, dtype=np.int64)
    Qr = to_f64(Q)[:, rows]
    return apply(Qr, S, z, eps, None if theta is None else theta[rows])


def attention(Q, K, V, eps: float, theta: Optional[np.ndarray] = None) -> np.ndarray:
    """Non-causal ReLU linear attention in the factorised (linear-time) form."""
    S, z = state_reduce(K, V, theta)
    return apply(Q, S, z, eps, theta)


def attention_bruteforce(Q, K, V, eps: float, theta_q: Optional[np.ndarray] = None,
                         theta_k: Optional[np.ndarray] = None) -> np.ndarray:
    """The quadratic form, one query-key pair at a time:

        O_i = sum_j (phi(q_i) . phi(k_j)) v_j / (sum_j ReLU(q_i) . ReLU(k_j) + eps)

    Queries and keys may have different lengths and positions. Tiny inputs only.
    """
    Q = to_f64(Q)
    K = to_f64(K)
    V = to_f64(V)
    qp, kp = relu(Q), relu(K)
    phq = qp if theta_q is None else rope_rotate(qp, theta_q)
    phk = kp if theta_k is None else rope_rotate(kp, theta_k)
    weights = np.einsum("bihd,bjhd->bhij", phq, phk)
    den = np.einsum("bihd,bjhd->bhij", qp, kp).sum(axis=-1) + float(eps)
    num = np.einsum("bhij,bjhe->bhie", weights, V)
    return (num / den[..., None]).transpose(0, 2, 1, 3)


def block_causal_step(Q, K, V, S_carry: np.ndarray, z_carry: np.ndarray,
                      update: int, eps: float, theta: Optional[np.ndarray] = None):
    """One call of the block-causal mode [SV23, SV4, MJ].

    The block's own state (S_own, z_own) is reduced from (K, V).
    update = 0: O = apply(Q, S_carry + S_own, z_carry + z_own); carry unchanged.
    update = 1: the same O, then the carry becomes carry + own.
    update = 2: no output; the carry becomes carry + own.
    Returns (O or None, S_carry', z_carry').
    """
    S_own, z_own = state_reduce(K, V, theta)
    S_carry = np.asarray(S_carry, dtype=np.float64)
    z_carry = np.asarray(z_carry, dtype=np.float64)
    out = None
    if update in (0, 1):
        out = apply(Q, S_carry + S_own, z_carry + z_own, eps, theta)
    if update in (1, 2):
        S_carry = S_carry + S_own
        z_carry = z_carry + z_own
    return out, S_carry, z_carry


def block_causal_bruteforce(blocks: List[dict], eps: float) -> List[List[np.ndarray]]:
    """Block-masked quadratic attention, one pass at a time.

    ``blocks[m]`` is ``{"passes": [(Q, K, V, theta), ...], "update": (K, V, theta)}``.
    A query of block m, pass s attends to the keys of that same pass (global
    attention inside the block) and to the update-pass keys of every block
    before m; it never sees a later block [MJ, SV4]. Returns, per block, the
    outputs of its passes.
    """
    outs: List[List[np.ndarray]] = []
    past_k, past_v, past_th = [], [], []
    for blk in blocks:
        res = []
        for (Q, K, V, th) in blk["passes"]:
            keys = past_k + [to_f64(K)]
            vals = past_v + [to_f64(V)]
            ths = past_th + [th]
            Kc = np.concatenate(keys, axis=1)
            Vc = np.concatenate(vals, axis=1)
            thc = None if th is None else np.concatenate(ths, axis=0)
            res.append(attention_bruteforce(Q, Kc, Vc, eps, th, thc))
        outs.append(res)
        Ku, Vu, thu = blk["update"]
        past_k.append(to_f64(Ku))
        past_v.append(to_f64(Vu))
        past_th.append(thu)
    return outs


def rope_unrotate(x: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """The inverse (transpose) of rope_rotate: rotate the pairs by -theta."""
    return rope_rotate(x, -theta)


def backward(Q, K, V, dO, eps: float, theta: Optional[np.ndarray] = None):
    """Gradient of the non-causal layer O = attention(Q, K, V) [SI], by hand.

    With den_i = ReLU(q_i).z + eps, num_i = phi(q_i) S, O_i = num_i / den_i:
      dnum_i = dO_i / den_i,  dden_i = -(dO_i . O_i) / den_i
      dS = sum_i phi(q_i)^T dnum_i,   dz = sum_i dden_i ReLU(q_i)
      dq_i = [R_i^T (dnum_i S^T) + dden_i z] * [q_i > 0]
      dk_j = [R_j^T (dS v_j) + dz] * [k_j > 0],   dv_j = phi(k_j) dS
    (R = the RoPE rotation, identity without RoPE; the ReLU derivative is 0 at
    0.) Returns dQ, dK, dV [B, N, H, D] and dS [B, H, D, D], dz [B, H, D].
    """
    Q, K, V, dO = to_f64(Q), to_f64(K), to_f64(V), to_f64(dO)
    qp, kp = relu(Q), relu(K)
    phq = qp if theta is None else rope_rotate(qp, theta)
    phk = kp if theta is None else rope_rotate(kp, theta)

    def heads(x):  # [B, N, H, D] -> [B, H, N, D], for batched matmuls
        return x.transpose(0, 2, 1, 3)

    def tokens(x):  # [B, H, N, D] -> [B, N, H, D]
        return x.transpose(0, 2, 1, 3)

    S = np.matmul(heads(phk).transpose(0, 1, 3, 2), heads(V))            # [B,H,D,E]
    z = kp.sum(axis=1)                                                    # [B,H,D]
    den = np.einsum("bnhd,bhd->bnh", qp, z) + float(eps)                  # [B,N,H]
    O = tokens(np.matmul(heads(phq), S)) / den[..., None]
    dnum = dO / den[..., None]
    dden = -np.einsum("bnhe,bnhe->bnh", dO, O) / den
    dS = np.matmul(heads(phq).transpose(0, 1, 3, 2), heads(dnum))         # sum_n phq^T dnum
    dz = np.einsum("bnh,bnhd->bhd", dden, qp)
    dphq = tokens(np.matmul(heads(dnum), S.transpose(0, 1, 3, 2)))        # dnum S^T
    dqp = (dphq if theta is None else rope_unrotate(dphq, theta)) + dden[..., None] * z[:, None]
    dQ = dqp * (Q > 0)
    dphk = tokens(np.matmul(heads(V), dS.transpose(0, 1, 3, 2)))          # (dS v^T)^T
    dkp = (dphk if theta is None else rope_unrotate(dphk, theta)) + dz[:, None]
    dK = dkp * (K > 0)
    dV = tokens(np.matmul(heads(phk), dS))                                # phk dS
    return dQ, dK, dV, dS, dz


def causal_attention(Q, K, V, eps: float, theta: Optional[np.ndarray] = None,
                     S0: Optional[np.ndarray] = None, z0: Optional[np.ndarray] = None):
    """Token-causal ReLU linear attention [SV23t], by its recurrence.

    With the state carried in (S0, z0) (zero when None):
      S_i = S0 + sum_{j<=i} phi(k_j)^T v_j,   z_i = z0 + sum_{j<=i} ReLU(k_j),
      O_i = phi(q_i) S_i / (ReLU(q_i) . z_i + eps).
    The state is advanced one token at a time, in token order. Returns O
    [B, N, H, D] and the final state (S_N, z_N).
    """
    Q, K, V = to_f64(Q), to_f64(K), to_f64(V)
    B, N, H, D = Q.shape
    qp, kp = relu(Q), relu(K)
    phq = qp if theta is None else rope_rotate(qp, theta)
    phk = kp if theta is None else rope_rotate(kp, theta)
    S = np.zeros((B, H, D, D)) if S0 is None else np.array(S0, dtype=np.float64)
    z = np.zeros((B, H, D)) if z0 is None else np.array(z0, dtype=np.float64)
    O = np.empty((B, N, H, D))
    for n in range(N):
        S = S + phk[:, n, :, :, None] * V[:, n, :, None, :]
        z = z + kp[:, n]
        num = np.einsum("bhd,bhde->bhe", phq[:, n], S)
        den = np.einsum("bhd,bhd->bh", qp[:, n], z) + float(eps)
        O[:, n] = num / den[..., None]
    return O, S, z


def causal_bruteforce(Q, K, V, eps: float, theta: Optional[np.ndarray] = None) -> np.ndarray:
    """The causal quadratic form: O_i = sum_{j<=i} (phi(q_i) . phi(k_j)) v_j /
    (sum_{j<=i} ReLU(q_i) . ReLU(k_j) + eps). Tiny inputs only."""
    Q, K, V = to_f64(Q), to_f64(K), to_f64(V)
    N = Q.shape[1]
    qp, kp = relu(Q), relu(K)
    phq = qp if theta is None else rope_rotate(qp, theta)
    phk = kp if theta is None else rope_rotate(kp, theta)
    seen = np.tril(np.ones((N, N)))                          # [i, j]: j <= i
    weights = np.einsum("bihd,bjhd->bhij", phq, phk) * seen
    den = (np.einsum("bihd,bjhd->bhij", qp, kp) * seen).sum(axis=-1) + float(eps)
    num = np.einsum("bhij,bjhe->bhie", weights, V)
    return (num / den[..., None]).transpose(0, 2, 1, 3)
