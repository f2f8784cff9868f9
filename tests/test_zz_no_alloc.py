"""The decode entry point that allocates nothing, against the regular one (GPU).

tq_decode_paged_static serves callers that cannot call cudaMalloc (another
runtime owns the device memory, or the path may not take cudaMalloc's
implicit synchronization): its split-K scratch is a fixed array inside the
library that every call shares and that keeps the last call's contents.

Before the calls that are checked, a larger, different problem runs through
the same array, so every record the checked calls read holds another call's
data unless they rewrite it. Two calls in a row must then give exactly what
tq_decode_paged gives on the same cache: both run the same kernels over the
same items, and each output depends only on its own records.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""

import pytest
import torch

from quantized_paged_kv_pack_b200 import tq

from helpers import DecodeProblem

pytestmark = pytest.mark.gpu

M35 = ((4, 3), (64, 64), 3)


def _static(p):
    return tq.decode_paged_static(p.kc, p.vc, p.q, p.k_pages, p.v_pages, p.bs, p.block_tables, p.seq_lens,
                                  p.max_seq_len, p.k_win if p.window else None, p.v_win if p.window else None,
                                  p.window, p.scale)


def test_static_workspace_decode_matches_regular_entry_point():
    # more sequences, longer histories, a wider window, other formats and seeds
    filler = DecodeProblem([9000, 4100, 12000, 3300, 700, 1500, 8191, 64], 2, 4, ((4,), (128,), 5),
                           ((3,), (128,), 6), window=40, block_size=16, seed=77)
    prob = DecodeProblem([3000, 17, 0, 800], 2, 4, M35, (M35[0], M35[1], 7), window=16, block_size=16, seed=31)
    assert tq.decode_workspace_bytes(filler.B, filler.Hq, filler.H, filler.max_seq_len, 16) > \
        tq.decode_workspace_bytes(prob.B, prob.Hq, prob.H, prob.max_seq_len, 16)
    filler_out = _static(filler)
    torch.cuda.synchronize()
    assert torch.equal(filler_out, filler.run())
    ref = prob.run()
    torch.cuda.synchronize()
    assert ref.abs().max().item() > 0.5
    for call in range(2):
        out = _static(prob)
        torch.cuda.synchronize()
        diff = (out - ref).abs().max().item()
        assert torch.equal(out, ref), f"call {call}: static decode differs from tq_decode_paged by {diff}"


def test_static_workspace_rejects_calls_beyond_its_size():
    limit = tq.static_workspace_bytes()
    need = tq.decode_workspace_bytes(4096, 16, 8, 1 << 20, 16)
    assert need > limit
    q = torch.zeros(4096, 16, 128, dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros(4096, 1, dtype=torch.int32, device="cuda")
    sl = torch.zeros(4096, dtype=torch.int32, device="cuda")
    kc8 = tq.Codec(8, (4,), (128,), None, 0)
    vc8 = tq.Codec(8, (4,), (128,), None, 1)
    kp, vp = tq.page_pool(kc8, 1, 16), tq.page_pool(vc8, 1, 16)
    with pytest.raises(ValueError, match="static workspace"):
        tq.decode_paged_static(kc8, vc8, q, kp, vp, 16, bt, sl, 1 << 20, None, None, 0, 0.1)
