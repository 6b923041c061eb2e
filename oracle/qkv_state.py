"""Float64 oracle of the QKV projection fused with the state reduce.

Test infrastructure: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code
with the CUDA library.

Sources (page title, then section):

[SIq]  "Sana: Efficient High-Resolution Image Synthesis with Linear Diffusion
       Transformers", section "Infra": for deployment the QKV projection is a
       hand-written GEMM whose kernel also forms ReLU(K)^T V, so the keys and
       values need not be written out and read back.
[SANA] same page, section "模型架构", item 2: the shared sums
       sum_j ReLU(K_j)^T V_j and sum_j ReLU(K_j) are formed once per layer.
[SV22] "SANA-Video: Efficient Video Generation with Block Linear Diffusion
       Transformer", section 2.2: RoPE after ReLU in the numerator only.

Readings (the pages give the fusion, not its formula):

* The projection is one linear map of the token features x_n (width C) to
  the concatenated query, key and value features: [q_n, k_n, v_n] =
  W x_n + b, W of shape [3 H 32, C] (rows: all query features, then all key
  features, then all value features; inside each, head h owns rows
  [32 h, 32 h + 32)), b optional.
* Each of q, k, v is rounded to bfloat16, as the unfused projection would
  store it; the state is then that of the rounded keys and values, so the
  fused result equals the unfused one (projection, then state reduce) up to
  the order of the sums. The pages' deployment kernel quantised the GEMM to
  8 bits while keeping the attention itself in full precision; here the
  GEMM stays in bfloat16, the precision of every other step.
* Only the queries leave the fused operation; the state (S, z) is that of
  ``linear_attention.state_reduce`` over the rounded keys and values.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .linear_attention import HEAD_DIM, state_reduce, to_f64


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits,
    ties to even), returned as float64. Written from the format's definition:
    x = m 2^e with 0.5 <= |m| < 1, and m keeps 8 bits. Values stay in the
    normal range here (no subnormal or overflow handling)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def qkv_projection(X, W, b=None, H: Optional[int] = None):
    """q, k, v of every token, each [B, N, H, 32], rounded to bfloat16.

    X [B, N, C]; W [3 H 32, C]; b [3 H 32] or None. [SIq]"""
    X = to_f64(X)
    W = to_f64(W)
    three_hd, C = W.shape
    if H is None:
        H = three_hd // (3 * HEAD_DIM)
    assert three_hd == 3 * H * HEAD_DIM and X.shape[-1] == C
    Y = np.matmul(X, W.T)
    if b is not None:
        Y = Y + to_f64(b)
    Y = bf16_round(Y)
    B, N = X.shape[:2]
    hd = H * HEAD_DIM
    q = Y[..., :hd].reshape(B, N, H, HEAD_DIM)
    k = Y[..., hd:2 * hd].reshape(B, N, H, HEAD_DIM)
    v = Y[..., 2 * hd:].reshape(B, N, H, HEAD_DIM)
    return q, k, v


def qkv_state(X, W, b=None, H: Optional[int] = None,
              theta: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(Q, S, z): the projected queries (bfloat16 values) and the state of the
    projected keys and values, S [B, H, 32, 32] and z [B, H, 32]. [SIq, SANA]"""
    q, k, v = qkv_projection(X, W, b, H)
    S, z = state_reduce(k, v, theta)
    return q, S, z


def key_value_heads(X, W, b, H: int, heads) -> Tuple[np.ndarray, np.ndarray]:
    """k, v of the listed heads only ([B, N, len(heads), 32] each), for
    checking a sample of heads of a large projection."""
    X = to_f64(X)
    W = to_f64(W)
    hd = H * HEAD_DIM
    rows_k = np.concatenate([np.arange(hd + 32 * h, hd + 32 * h + 32) for h in heads])
    rows_v = rows_k + hd
    B, N = X.shape[:2]
    out = []
    for rows in (rows_k, rows_v):
        Y = np.matmul(X, W[rows].T)
        if b is not None:
            Y = Y + to_f64(b)[rows]
        out.append(bf16_round(Y).reshape(B, N, len(heads), HEAD_DIM))
    return out[0], out[1]
