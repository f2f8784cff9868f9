"""Failure detection on the GPU without a fault: a bounded wait that nothing satisfies.

With TQ_TEST_WITHHOLD_COPIES=1 the decode kernels' producer warp issues no
copies, so every compute warp's wait for a ring slot runs out (about a second),
sets TQ_DERR_TIMEOUT in the device error word and returns. The context stays
usable: the same call without the flag then matches the oracle.
"""

import numpy as np
import pytest
import torch

from quantized_paged_kv_pack_b200 import tq

from helpers import DecodeProblem

pytestmark = pytest.mark.gpu

U4 = ((4,), (128,), 0)
M35 = ((4, 3), (64, 64), 3)


@pytest.mark.parametrize("H", [8, 2])  # the block kernel (8 KV heads per slot) and the per-head kernel
def test_expired_wait_sets_timeout_and_context_survives(monkeypatch, H):
    prob = DecodeProblem([300, 40], H, 4, U4, (M35[0], M35[1], 13), window=8, block_size=16, seed=60 + H)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("TQ_TEST_WITHHOLD_COPIES", "1")
    prob.run(d_err=err)
    torch.cuda.synchronize()
    assert err.item() & tq.TQ_DERR_TIMEOUT
    monkeypatch.delenv("TQ_TEST_WITHHOLD_COPIES")
    err.zero_()
    out = prob.run(d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    for b in range(prob.B):
        for hq in (0, prob.Hq - 1):
            assert np.abs(got[b, hq] - prob.oracle(b, hq)).max() <= 2e-3


def test_expired_wait_raises_in_checked_mode(monkeypatch):
    prob = DecodeProblem([200], 8, 2, U4, U4, window=0, block_size=16, seed=71)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("TQ_TEST_WITHHOLD_COPIES", "1")
    monkeypatch.setenv("TQ_CHECKED", "1")
    with pytest.raises(tq.TQTimeoutError):
        prob.run(d_err=err)
