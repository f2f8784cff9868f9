"""tq_window_append_decode: the append and the decode of one step in fewer launches.

Its results must be those of tq_window_append followed by tq_decode_paged (window
sinks + window, the same seq_lens) from the same state: the pages and the dense
buffers byte for byte, and the attention output element for element.
"""

import math

import numpy as np
import pytest
import torch

from quantized_paged_kv_pack_b200 import tq

from helpers import D, codec_pair

pytestmark = pytest.mark.gpu

U4 = ((4,), (128,), 0)
U2 = ((2,), (128,), 2)
M35 = ((4, 3), (64, 64), 3)
M25 = ((4, 2), (32, 96), 4)
Q25 = ((3, 2), (64, 64), 5)


def _state(H, G, kspec, vspec, lens, sinks, window, bs, seed, kqjl=False, kgw=False, vgw=False):
    """Codecs, pages packed with random tokens for every packed position the step can touch, dense
    buffers of random tokens, queries and the new tokens."""
    kc, _ = codec_pair(H, *kspec, qjl=kqjl, groupwise=kgw)
    vc, _ = codec_pair(H, *vspec, groupwise=vgw)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    rng = np.random.default_rng(seed)
    B, dense = len(lens), sinks + window
    # positions 0 .. L - min(dense, L) are packed after the step (the evicted token included)
    need = [max(L - min(dense, L), 0) + 1 for L in lens]
    max_blocks = max(-(-n // bs) for n in need) + 1
    num_blocks = B * max_blocks + 2
    order = rng.permutation(num_blocks)
    bt_np = order[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    kp, vp = tq.page_pool(kc, num_blocks, bs), tq.page_pool(vc, num_blocks, bs)
    for b, n in enumerate(need):
        t = np.arange(n)
        slots = torch.as_tensor(bt_np[b, t // bs].astype(np.int64) * bs + t % bs, device="cuda")
        k = (torch.randn(n, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
        v = (torch.randn(n, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
        tq.pack_kv(kc, vc, k, v, slots, kp, vp, bs)
    kw = (torch.randn(B, H, max(dense, 1), D, generator=gen, device="cuda")).to(torch.bfloat16)[:, :, :dense]
    vw = (torch.randn(B, H, max(dense, 1), D, generator=gen, device="cuda")).to(torch.bfloat16)[:, :, :dense]
    kw, vw = kw.contiguous(), vw.contiguous()
    q = torch.randn(B, H * G, D, generator=gen, device="cuda").to(torch.bfloat16)
    k_new = (torch.randn(B, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
    v_new = (torch.randn(B, H, D, generator=gen, device="cuda") * 2).to(torch.bfloat16)
    bt = torch.as_tensor(bt_np, device="cuda")
    sl = torch.as_tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    return kc, vc, kp, vp, kw, vw, q, k_new, v_new, bt, sl


@pytest.mark.parametrize("H,G,kspec,vspec,mode,bs", [
    (8, 8, M35, M35, "", 16),      # paired kernel
    (8, 4, U4, U4, "", 32),        # paired kernel, 32-token blocks
    (8, 4, Q25, M35, "qjl", 16),   # QJL keys
    (8, 4, M35, M35, "gw", 16),    # group-wise K and V
    (8, 4, Q25, M35, "recipe", 16),  # recipe-row keys
    (2, 4, M25, U4, "", 16),       # per-head kernel
    (8, 4, M25, U2, "", 16),       # no tensor-core decode: the two calls as they are
])
@pytest.mark.parametrize("sinks,window", [(0, 8), (4, 8), (3, 0)])
def test_fused_step_equals_append_then_decode(H, G, kspec, vspec, mode, bs, sinks, window):
    lens = [0, 1, 2, sinks + window - 1 if sinks + window > 1 else 3, sinks + window, sinks + window + 5, 700, 5000]
    kqjl = mode in ("qjl", "recipe")
    kgw = mode in ("gw", "recipe")
    vgw = mode in ("gw", "recipe")
    state = _state(H, G, kspec, vspec, lens, sinks, window, bs, 7 + H + G + sinks + window + bs,
                   kqjl=kqjl, kgw=kgw, vgw=vgw)
    kc, vc, kp, vp, kw, vw, q, k_new, v_new, bt, sl = state
    maxL = max(lens)
    dense = sinks + window
    scale = 1 / math.sqrt(D)
    ws = tq.alloc_workspace(len(lens), q.shape[1], H, maxL, bs)

    kp2, vp2, kw2, vw2 = kp.clone(), vp.clone(), kw.clone(), vw.clone()
    err_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.window_append(kc, vc, k_new, v_new, kw if dense else None, vw if dense else None, window, sinks, sl, bt,
                     kp, vp, bs, d_err=err_a)
    out_a = tq.decode_paged(kc, vc, q, kp, vp, bs, bt, sl, maxL, kw if dense else None, vw if dense else None,
                            dense, scale, workspace=ws, d_err=err_a).clone()

    err_b = torch.zeros(1, dtype=torch.int32, device="cuda")
    out_b = tq.window_append_decode(kc, vc, k_new, v_new, kw2 if dense else None, vw2 if dense else None, window,
                                    sinks, q, kp2, vp2, bs, bt, sl, maxL, scale, workspace=ws, d_err=err_b)
    torch.cuda.synchronize()
    assert err_a.item() == 0 and err_b.item() == 0
    assert torch.equal(kp, kp2) and torch.equal(vp, vp2)
    assert torch.equal(kw, kw2) and torch.equal(vw, vw2)
    assert torch.equal(out_a, out_b), (out_a - out_b).abs().max().item()
    assert out_a.abs().max().item() > 0.1


def test_fused_step_argument_errors():
    kc, vc, kp, vp, kw, vw, q, k_new, v_new, bt, sl = _state(8, 4, U4, U4, [40, 50], 0, 8, 16, 3)
    with pytest.raises(ValueError):  # dense buffers of the wrong length
        tq.window_append_decode(kc, vc, k_new, v_new, kw[:, :, :4].contiguous(), vw[:, :, :4].contiguous(), 8, 0,
                                q, kp, vp, 16, bt, sl, 50, 0.1)
    with pytest.raises(ValueError):  # k_new of the wrong shape
        tq.window_append_decode(kc, vc, k_new[:1], v_new, kw, vw, 8, 0, q, kp, vp, 16, bt, sl, 50, 0.1)
