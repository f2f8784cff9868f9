"""GPU parity of the QJL residual stage: pack rows and decode scores against the oracle."""

import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq

from helpers import D, DecodeProblem, check_qjl_rows, codec_pair, random_kv, slice_format

pytestmark = pytest.mark.gpu

BOUNDARY_REL = 1e-5


@pytest.mark.parametrize("kfmt", [((3,), (128,)), ((3, 2), (64, 64)), ((2,), (128,)), ((4, 3), (64, 64))])
@pytest.mark.parametrize("T,H,bs", [(37, 2, 16), (300, 8, 32)])
def test_qjl_pack_matches_oracle(kfmt, T, H, bs):
    kc, kf = codec_pair(H, *kfmt, 31, qjl=True)
    vc, vf = codec_pair(H, (3,), (128,), 32, qjl=True)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T + H)
    k, v = random_kv(T, H, gen)
    nb = -(-T // bs) + 2
    rng = np.random.default_rng(T)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        x = src.float().cpu().numpy().astype(np.float64)
        rows = np.stack([O.read_rows(pages.cpu().numpy(), slots // bs, h, slots % bs, f, bs) for h in range(H)], 1)
        assert check_qjl_rows(rows, x, f, range(H)) > 0.9 * T * H


@pytest.mark.parametrize("H,G,kfmt,vfmt", [(2, 4, ((3,), (128,)), ((3,), (128,))),
                                           (8, 8, ((3, 2), (64, 64)), ((4, 3), (64, 64)))])
def test_qjl_decode_matches_oracle(H, G, kfmt, vfmt):
    """Decode with QJL keys (general kernel) against the oracle on the same GPU-written pages."""
    lens = [1, 17, 300, 2100]
    prob = DecodeProblem(lens, H, G, (kfmt[0], kfmt[1], 41), (vfmt[0], vfmt[1], 42), window=8, block_size=16,
                         seed=H, kqjl=True)
    out = prob.run()
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    rng = np.random.default_rng(G)
    worst = 0.0
    for b in range(prob.B):
        for hq in rng.choice(prob.Hq, 4, replace=False):
            ref = prob.oracle(b, int(hq))
            worst = max(worst, float(np.abs(got[b, hq] - ref).max()))
            assert np.abs(ref).max() > 0.3
    assert worst <= 2e-3, worst


def test_qjl_value_codec_is_rejected_by_decode():
    prob = DecodeProblem([40], 2, 2, ((3,), (128,), 1), ((3,), (128,), 2), window=0, block_size=16, seed=3,
                         vqjl=True)
    with pytest.raises(tq.UnsupportedFormatError):
        prob.run()


@pytest.mark.parametrize("H,G,kfmt,vfmt,bs", [
    (8, 4, ((3, 2), (64, 64)), ((4, 3), (64, 64)), 16),   # block kernel, 4 query heads per item, 1 tile per block
    (8, 8, ((4, 3), (64, 64)), ((4,), (128,)), 32),       # block kernel, 8 query heads, 2 tiles per block
    (8, 16, ((3, 2), (64, 64)), ((4,), (128,)), 64),      # block kernel, any multiple of 16, 2 head groups
    (2, 4, ((3, 2), (64, 64)), ((4,), (128,)), 16),       # per-head kernel, whole-sub-page copies
    (3, 8, ((4, 3), (64, 64)), ((4, 3), (64, 64)), 48),   # per-head kernel, split copies
])
def test_qjl_decode_tensor_core_matches_oracle_and_general(monkeypatch, H, G, kfmt, vfmt, bs):
    """QJL keys on the tensor-core kernel: the sign k-steps against the oracle and the general kernel."""
    lens = [5, 16 * 3 + 7, 700, 2500]
    prob = DecodeProblem(lens, H, G, (kfmt[0], kfmt[1], 43), (vfmt[0], vfmt[1], 44), window=12, block_size=bs,
                         seed=5 * H + G, kqjl=True)
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
    rng = np.random.default_rng(H * G)
    for b in range(prob.B):
        for hq in rng.choice(prob.Hq, 3, replace=False):
            ref = prob.oracle(b, int(hq))
            assert np.abs(got[b, hq] - ref).max() <= 2e-3
            assert np.abs(ref).max() > 0.3
