"""Float64 oracle of the temporal depth-wise convolution of SANA-Video's
spatial-temporal Mix-FFN and its block-causal conv cache.

Test infrastructure: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code
with the CUDA library.

Sources (page title, then section):

[SVS2]  "SANA-Video: Efficient Video Generation with Block Linear Diffusion
        Transformer", "Stage 2": a 1D temporal convolution is added to the
        Mix-FFN through a shortcut (the new layers start from zero weights).
[SV4c]  same page, section 4: the KV cache has three parts, the accumulated
        state, the accumulated key sum, and the conv cache f, which is the
        last frame of the temporal convolution.
[MJc]   SANA-Video article (mjgaz.cn), the Spatial-Temporal Mix-FFN paragraph:
        the MLP alternates 1x3x3 spatial and 3x1x1 temporal filters.

Readings (the pages give no formula):

* The temporal filter is depth-wise (one 3-tap filter per channel, as the
  Mix-FFN's spatial convolution is depth-wise) and enters through a
  shortcut: y = x + b + conv(x), with
      conv(x)[t] = w[c, 0] x[t - 1] + w[c, 1] x[t] + w[c, 2] x[t + 1].
* Non-causal (a whole clip): zero padding at both ends of the time axis.
* Block-causal (section 4 loop): frame 0 of a block sees the previous
  block's last frame, kept in the conv cache f (zero for the first block);
  the block's last frame sees zero, since later blocks are never seen. After
  the block, f becomes the block's own last frame (of the update pass).

Layout: x [B, T, Hh, W, C], channels last (the DiT's tokens [B, N, C] with
N = T * Hh * W in raster order); w [C, 3]; b [C]; f [B, Hh, W, C].
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        if str(x.dtype) != "torch.float64":
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def temporal_conv(x, w, b=None, f=None) -> Tuple[np.ndarray, np.ndarray]:
    """y = x + b + conv(x) over the time axis, and the next conv cache.

    x [B, T, Hh, W, C]; w [C, 3]; b [C] or None; f [B, Hh, W, C] or None (the
    previous block's last frame; None = zero, as for a clip or a first
    block). The frame after the last one is zero. Returns y [B, T, Hh, W, C]
    and f' = x[:, T - 1] (the cache for the next block).
    """
    x = _f64(x)
    w = _f64(w)
    B, T, Hh, W, C = x.shape
    prev = np.zeros((B, 1, Hh, W, C)) if f is None else _f64(f)[:, None]
    padded = np.concatenate([prev, x, np.zeros((B, 1, Hh, W, C))], axis=1)  # frames -1..T
    y = x + w[:, 0] * padded[:, :-2] + w[:, 1] * padded[:, 1:-1] + w[:, 2] * padded[:, 2:]
    if b is not None:
        y = y + _f64(b)
    return y, x[:, -1].copy()
