"""The decode entry point that allocates nothing, against the regular one (GPU).

tq_decode_paged_static serves callers that cannot call cudaMalloc (another
runtime owns the device memory, or the path may not take cudaMalloc's
implicit synchronization): its split-K scratch is a fixed array inside the
library. Two calls in a row must match tq_decode_paged on the same cache.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import pytest
import torch

from quantized_paged_kv_pack_b200 import tq

from helpers import DecodeProblem

pytestmark = pytest.mark.gpu

ATOL = 2e-3  # the decode tolerance used by the other GPU tests
M35 = ((4, 3), (64, 64), 3)


def test_static_workspace_decode_matches_regular_entry_point():
    prob = DecodeProblem([3000, 17, 0, 800], 2, 4, M35, (M35[0], M35[1], 7), window=16, block_size=16, seed=31)
    ref = prob.run()
    torch.cuda.synchronize()
    assert ref.abs().max().item() > 0.5
    for _ in range(2):  # the array keeps the previous call's contents; results must not depend on them
        out = tq.decode_paged_static(prob.kc, prob.vc, prob.q, prob.k_pages, prob.v_pages, prob.bs,
                                     prob.block_tables, prob.seq_lens, prob.max_seq_len, prob.k_win, prob.v_win,
                                     prob.window, prob.scale)
        torch.cuda.synchronize()
        assert (out - ref).abs().max().item() <= ATOL


def test_static_workspace_rejects_calls_beyond_its_size():
    prob = DecodeProblem([40], 1, 2, M35, M35, window=0, block_size=16, seed=32)
    need = tq.decode_workspace_bytes(4096, 16, 8, 1 << 20, 16)
    assert need > tq.STATIC_WORKSPACE_BYTES
    q = torch.zeros(4096, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(4096, 1, dtype=torch.int32, device="cuda")
    sl = torch.zeros(4096, dtype=torch.int32, device="cuda")
    kc8 = tq.Codec(8, (4,), (128,), None, 0)
    vc8 = tq.Codec(8, (4,), (128,), None, 1)
    kp, vp = tq.page_pool(kc8, 1, 16), tq.page_pool(vc8, 1, 16)
    with pytest.raises(ValueError, match="static workspace"):
        tq.decode_paged_static(kc8, vc8, q, kp, vp, 16, bt, sl, 1 << 20, None, None, 0, 0.1)
    del prob
