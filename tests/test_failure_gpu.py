"""Failure detection on the device without a GPU fault: a bounded wait that
nothing satisfies gives up after its limit, raises the device error word that
the host reads, and leaves the context usable."""
import time

import pytest
import torch

import oracle as orc
from tests import parity as P

la = P.la
pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_reports_and_context_survives(cuda_device):
    la.la_device_error(reset=True)
    assert la.la_device_error() == 0
    t0 = time.perf_counter()
    la.la_wait_selftest(20000)  # 20 ms
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert 0.015 <= elapsed < 5.0, elapsed          # it waited about its limit, then returned
    assert la.la_device_error(reset=True) & 1       # bit 0: a wait gave up
    assert la.la_device_error() == 0                # and the word is clear again
    # the context still runs the library's kernels correctly
    Q, K, V = (torch.randn((2, 300, 5, 32)).to(torch.bfloat16) for _ in range(3))
    O, S, z = P.gpu_attention(Q, K, V, 1e-6)
    S_ref, z_ref = orc.state_reduce(K, V)
    A = P.magnitude_state(K, V, None)
    P.check_state(S, z, S_ref, z_ref, A, 2e-5, "after the self-test")
    P.check_output(O, orc.apply(Q, S_ref, z_ref, 1e-6), "bf16", 2.0 ** -7, Q, None, A, z_ref,
                   1e-6, what="after the self-test")
