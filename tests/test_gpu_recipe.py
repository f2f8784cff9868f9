"""GPU parity of the recipe row as printed (group-wise rotation with a QJL stage per group):
pack rows and decode against the oracle (through the C ABI)."""

import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq

from helpers import D, DecodeProblem, check_recipe_rows, codec_pair, random_kv, slice_format

pytestmark = pytest.mark.gpu



@pytest.mark.parametrize("kfmt", [((4, 3), (64, 64)), ((3, 2), (64, 64)), ((4, 2), (32, 96)), ((3, 2), (16, 112))])
@pytest.mark.parametrize("T,H,bs", [(37, 2, 16), (300, 8, 32)])
def test_recipe_pack_matches_oracle(kfmt, T, H, bs):
    kc, kf = codec_pair(H, *kfmt, 51, qjl=True, groupwise=True)
    vc, vf = codec_pair(H, (4, 3), (64, 64), 52, groupwise=True)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T + 3 * H)
    k, v = random_kv(T, H, gen)
    nb = -(-T // bs) + 2
    slots = np.random.default_rng(T).permutation(nb * bs)[:T].astype(np.int64)
    kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
    assert kc.row_bytes == O.row_bytes(kf)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    x = k.float().cpu().numpy().astype(np.float64)
    rows = np.stack([O.read_rows(kp.cpu().numpy(), slots // bs, h, slots % bs, kf, bs) for h in range(H)], 1)
    assert check_recipe_rows(rows, x, kf, range(H)) > 0.9 * T * H


@pytest.mark.parametrize("H,G,bs", [(2, 4, 16), (8, 8, 32)])
def test_recipe_decode_matches_oracle(H, G, bs):
    """Recipe-row keys (general kernel) with group-wise values, against the oracle on the same
    GPU-written pages."""
    lens = [1, 17, 300, 2100]
    prob = DecodeProblem(lens, H, G, ((4, 3), (64, 64), 61), ((4, 3), (64, 64), 62), window=8, block_size=bs,
                         seed=H + G, kqjl=True, kgw=True, vgw=True)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = prob.run(d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    worst = 0.0
    for b in range(prob.B):
        for hq in range(prob.Hq):
            ref = prob.oracle(b, hq)
            worst = max(worst, float(np.abs(got[b, hq] - ref).max()))
            assert np.abs(ref).max() > 0.3
    assert worst <= 2e-3, worst


@pytest.mark.parametrize("H,G,bs", [(8, 4, 16), (8, 8, 32), (2, 16, 16), (3, 2, 48)])
def test_recipe_decode_tensor_core_matches_oracle_and_general(monkeypatch, H, G, bs):
    """Recipe-row keys in the tensor-core formats (3/2-bit 64/64 groups, each with its QJL signs and
    residual norm; group-wise 4/3-bit values): TQ_DECODE_KERNEL=tensor fails unless the tensor-core
    kernel runs it. Paired, block and per-head layouts against the general kernel and the oracle."""
    lens = [1, 17, 300, 2100, 5000]
    prob = DecodeProblem(lens, H, G, ((3, 2), (64, 64), 63), ((4, 3), (64, 64), 64), window=8, block_size=bs,
                         seed=40 + H + G, kqjl=True, kgw=True, vgw=True)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    monkeypatch.setenv("TQ_DECODE_KERNEL", "tensor")
    fast = prob.run(d_err=err).clone()
    monkeypatch.setenv("TQ_DECODE_PAIR", "0")
    block = prob.run(d_err=err).clone()
    monkeypatch.delenv("TQ_DECODE_PAIR")
    monkeypatch.setenv("TQ_DECODE_KERNEL", "general")
    general = prob.run(d_err=err).clone()
    torch.cuda.synchronize()
    assert err.item() == 0
    assert (fast - general).abs().max().item() <= 2e-3
    assert (block - general).abs().max().item() <= 2e-3
    got = fast.cpu().numpy()
    rng = np.random.default_rng(H * G)
    worst = 0.0
    for b in range(prob.B):
        for hq in rng.choice(prob.Hq, min(prob.Hq, 6), replace=False):
            ref = prob.oracle(b, int(hq))
            worst = max(worst, float(np.abs(got[b, hq] - ref).max()))
            assert np.abs(ref).max() > 0.3
    assert worst <= 2e-3, worst


def test_recipe_window_append_rows_equal_pack(monkeypatch):
    """tq_window_append packs an evicted token through the general kernel's per-vector routine: the
    row it writes for the recipe format equals the row that kernel writes for that token."""
    monkeypatch.setenv("TQ_PACK_KERNEL", "general")
    H, bs, W = 2, 16, 4
    kc, kf = codec_pair(H, (4, 3), (64, 64), 71, qjl=True, groupwise=True)
    vc, vf = codec_pair(H, (4, 3), (64, 64), 72, groupwise=True)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    k, v = random_kv(W + 1, H, gen)
    # the window holds tokens 0..W-1 (ring slots t % W); appending token W evicts token 0 to packed slot 0
    kw = k[:W].transpose(0, 1).unsqueeze(0).contiguous()
    vw = v[:W].transpose(0, 1).unsqueeze(0).contiguous()
    bt = torch.zeros(1, 2, dtype=torch.int32, device="cuda")
    bt[0, 0] = 1
    sl = torch.tensor([W], dtype=torch.int32, device="cuda")
    kp, vp = tq.page_pool(kc, 3, bs), tq.page_pool(vc, 3, bs)
    tq.window_append(kc, vc, k[W:W + 1].view(1, H, D), v[W:W + 1].view(1, H, D), kw, vw, W, 0, sl, bt, kp, vp, bs)
    kq, vq = tq.page_pool(kc, 3, bs), tq.page_pool(vc, 3, bs)
    tq.pack_kv(kc, vc, k[:1].contiguous(), v[:1].contiguous(), torch.tensor([bs], device="cuda"), kq, vq, bs)
    torch.cuda.synchronize()
    for a, b, f in ((kp, kq, kf), (vp, vq, vf)):
        ra = np.stack([O.read_rows(a.cpu().numpy(), [1], h, [0], f, bs) for h in range(H)])
        rb = np.stack([O.read_rows(b.cpu().numpy(), [1], h, [0], f, bs) for h in range(H)])
        assert np.array_equal(ra, rb)
