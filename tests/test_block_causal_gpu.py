"""GPU parity of the block-causal mode (la_block_causal_step, la_state_reset)
against the float64 oracle, pass by pass, with the carry checked after every
update."""
import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu
D = 32


class Runner:
    """Drives the GPU carry and the oracle carry side by side."""

    def __init__(self, w, io, rope):
        self.w, self.io, self.rope = w, io, rope
        self.S = torch.full((w.B, w.H, D, D), 3.0, device="cuda")  # garbage: reset must clear
        self.z = torch.full((w.B, w.H, D), 3.0, device="cuda")
        la.la_state_reset(self.S, self.z, w.B, w.H)
        self.S_ref = np.zeros((w.B, w.H, D, D))
        self.z_ref = np.zeros((w.B, w.H, D))
        self.A = np.zeros((w.B, w.H, D, D))  # magnitude of every term in the carry
        self.tol_s, self.tol_o = P.tolerances(io, rope)

    def inputs(self, m, s):
        Q, K, V = wl.make_qkv(self.w, 0, block=m, step=s)
        if self.io == "f32":
            Q, K, V = Q.float(), K.float(), V.float()
        th = orc.rope_angles(self.w.T, self.w.Hh, self.w.W, m * self.w.T) if self.rope else None
        return Q, K, V, th

    def step(self, m, s, update, check=True):
        w = self.w
        Q, K, V, th = self.inputs(m, s)
        shape = la.make_shape(w.B, w.N, w.H, D, self.io, self.rope, w.T, w.Hh, w.W, m * w.T,
                              w.rope_base, w.eps)
        ws = la.workspace(shape)
        Qd, Kd, Vd = P.to_dev(Q, K, V)
        O = torch.empty_like(Qd) if update != 2 else None
        S_before = self.S.clone()
        la.la_block_causal_step(shape, Qd if update != 2 else None, Kd, Vd, self.S, self.z, O,
                                update, ws)
        torch.cuda.synchronize()
        if update == 0:
            assert torch.equal(self.S, S_before), "update=0 must leave the carry alone"
        A_own = P.magnitude_state(K, V, th)
        O_ref, S_new, z_new = orc.block_causal_step(Q, K, V, self.S_ref, self.z_ref, update,
                                                    w.eps, th)
        if update != 2 and check:
            _, z_own = orc.state_reduce(K, V, th)
            P.check_output(O.cpu(), O_ref, self.io, self.tol_o, Q, th, self.A + A_own,
                           self.z_ref + z_own, w.eps, what=f"block {m} pass {s} update {update}")
        if update >= 1:
            self.A = self.A + A_own
            self.S_ref, self.z_ref = S_new, z_new
            if check:
                P.check_state(self.S.cpu(), self.z.cpu(), self.S_ref, self.z_ref, self.A,
                              self.tol_s, what=f"carry after block {m}")


@pytest.mark.parametrize("io", ["bf16", "f32"])
@pytest.mark.parametrize("rope", [False, True])
def test_block_causal_small(cuda_device, io, rope):
    w = wl.Workload("small_causal", B=2, N=3 * 5 * 20, H=5, rope=rope, T=3, Hh=5, W=20, M=3,
                    steps=2, block_causal=True)
    r = Runner(w, io, rope)
    for m in range(w.M):
        for s in range(w.steps):
            r.step(m, s, 0)
        r.step(m, w.steps, 2 if m % 2 == 0 else 1)


def test_block_causal_matches_block_masked_quadratic(cuda_device):
    """The GPU outputs of a tiny 3-block video equal the block-masked quadratic form."""
    T, Hh, W, H, M, steps = 2, 3, 4, 3, 3, 2
    w = wl.Workload("tiny_causal", B=1, N=T * Hh * W, H=H, rope=True, T=T, Hh=Hh, W=W, M=M,
                    steps=steps, block_causal=True)
    blocks, gpu_out = [], []
    S = torch.zeros((1, H, D, D), device="cuda")
    z = torch.zeros((1, H, D), device="cuda")
    for m in range(M):
        th = orc.rope_angles(T, Hh, W, m * T)
        shape = la.make_shape(1, w.N, H, D, "bf16", True, T, Hh, W, m * T, 10000.0, w.eps)
        ws = la.workspace(shape)
        passes, outs = [], []
        for s in range(steps):
            Q, K, V = wl.make_qkv(w, 0, block=m, step=s)
            passes.append((Q, K, V, th))
            Qd, Kd, Vd = P.to_dev(Q, K, V)
            O = torch.empty_like(Qd)
            la.la_block_causal_step(shape, Qd, Kd, Vd, S, z, O, 0, ws)
            outs.append(O.cpu())
        _, Ku, Vu = wl.make_qkv(w, 0, block=m, step=steps)
        la.la_block_causal_step(shape, None, *P.to_dev(Ku, Vu), S, z, None, 2, ws)
        blocks.append({"passes": passes, "update": (Ku, Vu, th)})
        gpu_out.append(outs)
    torch.cuda.synchronize()
    want = orc.block_causal_bruteforce(blocks, w.eps)
    for m in range(M):
        for s in range(steps):
            P.check_output(gpu_out[m][s], want[m][s], "bf16", 0, what=f"block {m} pass {s}")


def test_longsana_full_size(cuda_device):
    """LongSANA at full size: 12 blocks of 20x30x52 tokens, 70 heads, RoPE.

    Every block's update pass runs (update = 1, apply + fold-in), so the carry
    follows the full 12-block video; the carry is checked after every block.
    The four denoising passes (update = 0, which never touch the carry, as the
    test asserts) are run and checked in full for the first and last blocks.
    """
    w = wl.WORKLOADS["longsana_block_causal"]
    r = Runner(w, "bf16", True)
    for m in range(w.M):
        full = m in (0, w.M - 1)
        if full:
            for s in range(w.steps):
                r.step(m, s, 0)
        r.step(m, w.steps, 1, check=True)


def test_carry_is_deterministic_and_reset(cuda_device):
    w = wl.Workload("det", B=1, N=2 * 16 * 16, H=8, rope=True, T=2, Hh=16, W=16)
    Q, K, V = P.to_dev(*wl.make_qkv(w, 3))
    shape = la.make_shape(1, w.N, w.H, D, "bf16", True, 2, 16, 16, 4, 10000.0, 1e-6)
    ws = la.workspace(shape)
    results = []
    for _ in range(5):
        S = torch.zeros((1, w.H, D, D), device="cuda")
        z = torch.zeros((1, w.H, D), device="cuda")
        O = torch.empty_like(Q)
        for _blk in range(3):
            la.la_block_causal_step(shape, Q, K, V, S, z, O, 1, ws)
        torch.cuda.synchronize()
        results.append((S.clone(), z.clone(), O.clone()))
    for S, z, O in results[1:]:
        assert torch.equal(S, results[0][0]) and torch.equal(z, results[0][1])
        assert torch.equal(O, results[0][2])
    la.la_state_reset(S, z, 1, w.H)
    torch.cuda.synchronize()
    assert torch.all(S == 0) and torch.all(z == 0)
