"""GPU parity of group-wise rotation with per-group norms (reading R17) against the oracle."""

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq

from helpers import D, DecodeProblem, codec_pair, random_kv, slice_format

pytestmark = pytest.mark.gpu

BOUNDARY_REL = 1e-5
MAX_FLIP_FRACTION = 1e-4


@pytest.mark.parametrize("kfmt,vfmt", [(((4, 2), (32, 96)), ((4, 3), (64, 64))),
                                       (((3, 2), (16, 112)), ((2, 4), (80, 48)))])
@pytest.mark.parametrize("T,H,bs", [(41, 2, 16), (260, 8, 32)])
def test_groupwise_pack_matches_oracle(kfmt, vfmt, T, H, bs):
    kc, kf = codec_pair(H, *kfmt, 51, groupwise=True)
    vc, vf = codec_pair(H, *vfmt, 52, groupwise=True)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T * 3 + H)
    k, v = random_kv(T, H, gen)
    nb = -(-T // bs) + 2
    slots = np.random.default_rng(T).permutation(nb * bs)[:T].astype(np.int64)
    kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    flips = total = 0
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        x = src.float().cpu().numpy().astype(np.float64)
        g = pages.cpu().numpy()
        for h in range(H):
            f1 = slice_format(f, h)
            rows = O.read_rows(g, slots // bs, h, slots % bs, f1, bs)
            idx, n16, u = O.quantize(x[:, h], f1, 0)
            gidx, gn16 = O.decode_rows(rows, f1)
            assert np.array_equal(gn16.astype(np.float16).view(np.uint16), n16.astype(np.float16).view(np.uint16)), \
                "group norms differ"
            bad = gidx != idx
            if bad.any():
                margin = O.boundary_margin(u, f1)
                assert np.all(margin[bad] <= BOUNDARY_REL), "index mismatch away from a codebook boundary"
            flips += int(bad.sum())
            total += idx.size
    assert flips <= max(1, MAX_FLIP_FRACTION * total)


@pytest.mark.parametrize("H,G,kgw,vgw", [(2, 4, True, True), (8, 8, True, False), (8, 2, False, True),
                                         (2, 16, False, True)])
def test_groupwise_decode_matches_oracle(H, G, kgw, vgw):
    """Decode (general kernel) and its combine (the per-group inverse rotation) against the oracle; 16
    query heads per KV head take the combine's 8 head groups twice."""
    lens = [1, 33, 400, 1900]
    prob = DecodeProblem(lens, H, G, ((4, 2), (32, 96), 61), ((4, 3), (64, 64), 62), window=16, block_size=16,
                         seed=70 + H, kgw=kgw, vgw=vgw)
    out = prob.run()
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    rng = np.random.default_rng(G)
    for b in range(prob.B):
        for hq in rng.choice(prob.Hq, 4, replace=False):
            ref = prob.oracle(b, int(hq))
            assert np.abs(got[b, hq] - ref).max() <= 2e-3
            assert np.abs(ref).max() > 0.3


@pytest.mark.parametrize("H,G,bs", [(8, 8, 16), (8, 4, 32), (2, 16, 16), (3, 2, 48)])
def test_groupwise_decode_tensor_core_matches_oracle_and_general(monkeypatch, H, G, bs):
    """Group-wise K and V (4-bit 64 + 3-bit 64) on the tensor-core kernel: per-group score chains and
    per-group value weights, against the oracle and the general kernel."""
    lens = [3, 16 * 2 + 9, 640, 2300]
    prob = DecodeProblem(lens, H, G, ((4, 3), (64, 64), 63), ((4, 3), (64, 64), 64), window=10, block_size=bs,
                         seed=90 + H * G, kgw=True, vgw=True)
    monkeypatch.setenv("TQ_DECODE_KERNEL", "tensor")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fast = prob.run(d_err=err).clone()
    torch.cuda.synchronize()
    assert err.item() == 0
    monkeypatch.setenv("TQ_DECODE_KERNEL", "general")
    slow = prob.run().clone()
    torch.cuda.synchronize()
    assert (fast - slow).abs().max().item() <= 1e-3
    got = fast.cpu().numpy()
    rng = np.random.default_rng(H + G)
    for b in range(prob.B):
        for hq in rng.choice(prob.Hq, 3, replace=False):
            ref = prob.oracle(b, int(hq))
            assert np.abs(got[b, hq] - ref).max() <= 2e-3
            assert np.abs(ref).max() > 0.3


def test_groupwise_format_without_tensor_core_instantiation_runs_general(monkeypatch):
    """Group-wise K 4-bit 32 + 2-bit 96 with a plain 4-bit V: no tensor-core instantiation (and the two 4-bit
    codebooks, for dimensions 32 and 128, could not share one table), so forcing the tensor-core path fails
    and the default call runs the general kernel."""
    prob = DecodeProblem([100, 900], 8, 4, ((4, 2), (32, 96), 65), ((4,), (128,), 66), window=4, block_size=16,
                         seed=99, kgw=True)
    monkeypatch.setenv("TQ_DECODE_KERNEL", "tensor")
    with pytest.raises(tq.UnsupportedFormatError):
        prob.run()
    monkeypatch.delenv("TQ_DECODE_KERNEL")
    out = prob.run().cpu().numpy()
    ref = prob.oracle(1, 5)
    assert np.abs(out[1, 5] - ref).max() <= 2e-3
