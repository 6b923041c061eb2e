"""GPU parity of la_temporal_conv (temporal depth-wise conv with shortcut and
the block-causal conv cache) against the float64 oracle, element by element.

Bound: y is a float32 sum of four products and x, rounded once, so
|y_gpu - y_ref| <= out_round |y_ref| + 1e-6 (|x| + |b| + sum_k |w_k| |x_{t+k-1}|),
out_round = 2^-8 for bf16 output (round to nearest even), 1e-6 for float32.
The conv cache is a copy: bit-exact."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl

import linear_attention_diffusion_b200 as la

pytestmark = pytest.mark.gpu


def _inputs(B, T, Hh, W, C, seed, io):
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    x = wl.make_tensor((B, T, Hh, W, C), seed, dt)
    w = wl.make_tensor((C, 3), seed + 1, torch.float32)
    b = wl.make_tensor((C,), seed + 2, torch.float32)
    f = wl.make_tensor((B, Hh, W, C), seed + 3, dt)
    return x, w, b, f


def _check(y_gpu, y_ref, x, w, b, f, io, what):
    xa = np.abs(orc.to_f64(x))
    fa = np.zeros_like(xa[:, 0]) if f is None else np.abs(orc.to_f64(f))
    wa = np.abs(orc.to_f64(w))
    padded = np.concatenate([fa[:, None], xa, np.zeros_like(xa[:, :1])], axis=1)
    mag = xa + (0 if b is None else np.abs(orc.to_f64(b)))
    for k in range(3):
        mag = mag + wa[:, k] * padded[:, k:k + xa.shape[1]]
    y = orc.to_f64(y_gpu)
    assert np.isfinite(y).all(), what
    out_round = 2.0 ** -8 if io == "bf16" else 1e-6
    err = np.abs(y - y_ref)
    bound = out_round * np.abs(y_ref) + 1e-6 * mag + 1e-30
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside the bound; worst ratio "
                           f"{float((err / bound).max()):.3g}")


CASES = [
    # B, T, Hh, W, C
    (1, 5, 3, 4, 8),
    (2, 7, 5, 9, 40),          # 2 * 45 * 5 columns: several CTAs, a ragged last one
    (1, 20, 30, 52, 64),       # the LongSANA latent grid, 64 channels
    (3, 1, 2, 3, 16),          # a one-frame block: the frame sees the cache and zero
    (1, 11, 7, 13, 2048),      # more frames than slots in flight
]


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
@pytest.mark.parametrize("cached", [False, True])
def test_temporal_conv_matches_oracle(cuda_device, io, case, cached):
    B, T, Hh, W, C = case
    x, w, b, f = _inputs(B, T, Hh, W, C, 100 + C + T, io)
    fin = f if cached else None
    y_ref, f_ref = orc.temporal_conv(x, w, b, fin)
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    fd = fin.cuda() if cached else None
    y, f_out = la.temporal_conv(xd, wd, bd, fd, want_cache=True)
    torch.cuda.synchronize()
    assert la.la_device_error() == 0
    _check(y.cpu(), y_ref, x, w, b, fin, io, f"{io} {case} cached={cached}")
    assert torch.equal(f_out.cpu(), x[:, -1])  # the cache is the last frame, bit for bit


def test_temporal_conv_in_place_and_blocks_chain(cuda_device):
    """y written over x, the cache updated in place, and two blocks through
    the cache equal the clip convolution cut at the block boundary."""
    B, T, Hh, W, C = 2, 9, 6, 10, 48
    x, w, b, _ = _inputs(B, T, Hh, W, C, 7, "bf16")
    wd, bd = w.cuda(), b.cuda()
    shape1 = la.make_conv_shape(B, 4, Hh, W, C)
    shape2 = la.make_conv_shape(B, 5, Hh, W, C)
    x1, x2 = x[:, :4].contiguous().cuda(), x[:, 4:].contiguous().cuda()
    cache = torch.zeros((B, Hh, W, C), dtype=torch.bfloat16, device="cuda")
    la.la_temporal_conv(shape1, x1, wd, bd, cache, cache, x1)   # in place, cache in place
    la.la_temporal_conv(shape2, x2, wd, bd, cache, cache, x2)
    torch.cuda.synchronize()
    y_ref1, f1 = orc.temporal_conv(x[:, :4], w, b, None)
    y_ref2, f2 = orc.temporal_conv(x[:, 4:], w, b, f1)
    _check(x1.cpu(), y_ref1, x[:, :4], w, b, None, "bf16", "block 1 in place")
    _check(x2.cpu(), y_ref2, x[:, 4:], w, b, torch.from_numpy(f1).to(torch.bfloat16), "bf16",
           "block 2 in place")
    assert torch.equal(cache.cpu(), x[:, -1])


def test_temporal_conv_empty_clip_and_no_bias(cuda_device):
    B, Hh, W, C = 1, 3, 5, 16
    f = wl.make_tensor((B, Hh, W, C), 3).cuda()
    out = torch.full_like(f, float("nan"))
    empty = torch.empty((B, 0, Hh, W, C), dtype=torch.bfloat16, device="cuda")
    w = wl.make_tensor((C, 3), 4, torch.float32).cuda()
    la.la_temporal_conv(la.make_conv_shape(B, 0, Hh, W, C), empty, w, None, f, out, empty)
    torch.cuda.synchronize()
    assert torch.equal(out, f)
    x = wl.make_tensor((B, 3, Hh, W, C), 5)
    y = la.temporal_conv(x.cuda(), w)
    torch.cuda.synchronize()
    y_ref, _ = orc.temporal_conv(x, w.cpu(), None, None)
    _check(y.cpu(), y_ref, x, w.cpu(), None, None, "bf16", "no bias")


def test_temporal_conv_rejects_bad_arguments(cuda_device):
    x = torch.zeros((1, 2, 2, 2, 12), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((12, 3), device="cuda")
    with pytest.raises(la.LaError):   # C not a multiple of 8
        la.temporal_conv(x, w)
    x = torch.zeros((1, 2, 2, 2, 16), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, 3), device="cuda")
    shape = la.make_conv_shape(1, 2, 2, 2, 16)
    with pytest.raises(la.LaError):   # y overlapping x without being x
        la.la_temporal_conv(shape, x, w, None, None, None, x.view(-1)[8:].view(-1)[:128].data_ptr())
