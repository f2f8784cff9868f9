"""tq_window_append: window eviction with append, checked against tq_pack_kv and the oracle.

Each call appends one token per sequence: the token leaving the recent window
is packed into the pages and the new token takes its ring slot. After every
call the dense buffer must hold exactly the expected tokens, the pages must
hold the rows tq_pack_kv writes for the evicted tokens, and decode over the
result must match the fp64 oracle.
"""

import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq

from helpers import D, codec_pair, slice_format

pytestmark = pytest.mark.gpu

M35 = ((4, 3), (64, 64), 3)
U3 = ((3,), (128,), 14)


def expected_dense(L, sinks, window):
    """Token index held by each dense slot after L tokens (-1: empty)."""
    slots = [-1] * (sinks + window)
    for t in range(L):
        if t < sinks:
            slots[t] = t
        elif window:
            slots[sinks + (t - sinks) % window] = t
    return slots


@pytest.mark.parametrize("H,sinks,window", [(8, 0, 8), (8, 4, 8), (2, 3, 5), (8, 2, 0)])
def test_window_append_matches_pack_and_oracle(H, sinks, window):
    B, G, bs = 3, 4, 16
    steps = [70, 45, 20]  # tokens appended per sequence (ragged: sub-batches run first)
    kc, kf = codec_pair(H, *M35)
    vc, vf = codec_pair(H, *U3)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(90 + H + sinks + window)
    rng = np.random.default_rng(window)
    T = max(steps)
    hist_k = (torch.randn(B, T, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
    hist_v = (torch.randn(B, T, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
    max_blocks = -(-T // bs) + 1
    num_blocks = B * max_blocks + 3
    order = rng.permutation(num_blocks)
    bt = torch.as_tensor(order[:B * max_blocks].reshape(B, max_blocks).astype(np.int32), device="cuda")
    kp, vp = tq.page_pool(kc, num_blocks, bs), tq.page_pool(vc, num_blocks, bs)
    dense = sinks + window
    kw = torch.zeros(B, H, max(dense, 1), D, dtype=torch.bfloat16, device="cuda")[:, :, :dense].contiguous()
    vw = torch.zeros_like(kw)
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for step in range(T):
        b1 = sum(1 for n in steps if n > step)  # sequences 0 .. b1-1 still append (steps is descending)
        L = lens[:b1]
        t = int(step)
        tq.window_append(kc, vc, hist_k[:b1, t].contiguous(), hist_v[:b1, t].contiguous(),
                         kw[:b1] if dense else None, vw[:b1] if dense else None, window, sinks, L,
                         bt[:b1].contiguous(), kp, vp, bs, d_err=err)
        lens[:b1] += 1
    torch.cuda.synchronize()
    assert err.item() == 0
    lens_h = lens.cpu().numpy()
    assert list(lens_h) == steps

    # 1. dense buffers hold exactly the expected tokens
    for b in range(B):
        exp = expected_dense(int(lens_h[b]), sinks, window)
        for j, tok in enumerate(exp):
            if tok >= 0:
                assert torch.equal(kw[b, :, j], hist_k[b, tok]) and torch.equal(vw[b, :, j], hist_v[b, tok])

    # 2. pages hold what tq_pack_kv writes for the evicted (packed) tokens
    kp2, vp2 = tq.page_pool(kc, num_blocks, bs), tq.page_pool(vc, num_blocks, bs)
    bt_h = bt.cpu().numpy()
    for b in range(B):
        L = int(lens_h[b])
        dense_idx, s0, P = O.boundary_dense_tokens(L, sinks, window)
        if P == 0:
            continue
        pos = np.arange(P)
        slots = torch.as_tensor(bt_h[b, pos // bs].astype(np.int64) * bs + pos % bs, device="cuda")
        tq.pack_kv(kc, vc, hist_k[b, s0:s0 + P].contiguous(), hist_v[b, s0:s0 + P].contiguous(), slots, kp2, vp2, bs)
        for pool, ref, c in ((kp, kp2, kc), (vp, vp2, vc)):
            ib = c.row_bytes - 2
            for p in range(P):
                blk, off = int(bt_h[b, p // bs]), p % bs
                row = pool[blk, :, off * ib:(off + 1) * ib]
                assert torch.equal(row, ref[blk, :, off * ib:(off + 1) * ib])
                nrm = pool[blk, :, bs * ib + 2 * off:bs * ib + 2 * off + 2]
                assert torch.equal(nrm, ref[blk, :, bs * ib + 2 * off:bs * ib + 2 * off + 2])

    # 3. decode over the result matches the oracle
    q = (torch.randn(B, H * G, D, generator=gen, device="cuda")).to(torch.bfloat16)
    maxL = int(lens_h.max())
    out = tq.decode_paged(kc, vc, q, kp, vp, bs, bt, lens, maxL, kw if dense else None, vw if dense else None,
                          dense, 1 / math.sqrt(D), d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    for b in range(B):
        for hq in rng.choice(H * G, 3, replace=False):
            h = hq // G
            L = int(lens_h[b])
            ref = O.decode_attention(q[b:b + 1, hq:hq + 1].float().cpu().numpy().astype(np.float64),
                                     kp[:, h:h + 1].cpu().numpy(), vp[:, h:h + 1].cpu().numpy(), bt_h[b:b + 1], [L],
                                     kw[b:b + 1, h:h + 1].float().cpu().numpy() if dense else None,
                                     vw[b:b + 1, h:h + 1].float().cpu().numpy() if dense else None, dense,
                                     1 / math.sqrt(D), slice_format(kf, h), slice_format(vf, h), bs)[0, 0]
            assert np.abs(got[b, hq] - ref).max() <= 2e-3
            assert np.abs(ref).max() > 0.3


def test_window_append_block_table_overflow_sets_error():
    H, bs = 2, 16
    kc, _ = codec_pair(H, *M35)
    vc, _ = codec_pair(H, *U3)
    kp, vp = tq.page_pool(kc, 4, bs), tq.page_pool(vc, 4, bs)
    kw = torch.zeros(1, H, 4, D, dtype=torch.bfloat16, device="cuda")
    vw = torch.zeros_like(kw)
    bt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")  # room for 16 packed tokens only
    lens = torch.full((1,), 4 + 16, dtype=torch.int32, device="cuda")  # evicts packed position 16
    new = torch.zeros(1, H, D, dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.window_append(kc, vc, new, new, kw, vw, 4, 0, lens, bt, kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() & tq.TQ_DERR_BLOCK
