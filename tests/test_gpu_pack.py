"""GPU parity of tq_pack_kv against the oracle (through the C ABI)."""

import math
import os

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq
from quantized_paged_kv_pack_b200 import workloads as W

from helpers import D, check_qjl_rows, check_recipe_rows, codec_pair, random_kv, slice_format, workload_codecs

pytestmark = pytest.mark.gpu

BOUNDARY_REL = 1e-5       # near-boundary exemption for index mismatches
MAX_FLIP_FRACTION = 1e-4  # exempt mismatches allowed, as a fraction of coordinates

FORMATS = [((4,), (128,)), ((3,), (128,)), ((2,), (128,)), ((4, 3), (64, 64)), ((4, 2), (32, 96)),
           ((3, 2), (16, 112)), ((2, 4), (112, 16))]


def rows_of(pages, slots, bs, fmt, H):
    """Logical rows [n][H][row_bytes] of the given slots, read by the oracle's address formula."""
    slots = np.asarray(slots, dtype=np.int64)
    return np.stack([O.read_rows(pages, slots // bs, h, slots % bs, fmt, bs) for h in range(H)], axis=1)


def compare_rows(gpu_rows, k_cpu, fmt, heads):
    """Compare GPU rows [N][H][row] with the oracle's quantization of k_cpu [N][H][d].

    Norms must be bit-identical; indices identical except near a boundary.
    Returns (number of exempt index flips, number of coordinates).
    """
    flips = total = 0
    for h in heads:
        f1 = slice_format(fmt, h)
        idx, n16, u = O.quantize(k_cpu[:, h], f1, 0)
        gidx, gn16 = O.decode_rows(gpu_rows[:, h], f1)
        assert np.array_equal(gn16.astype(np.float16).view(np.uint16), n16.astype(np.float16).view(np.uint16)), \
            "fp16 norms differ"
        bad = gidx != idx
        if bad.any():
            margin = O.boundary_margin(u, f1)
            assert np.all(margin[bad] <= BOUNDARY_REL), "index mismatch away from a codebook boundary"
            assert np.all(np.abs(gidx[bad] - idx[bad]) == 1)
        flips += int(bad.sum())
        total += idx.size
    return flips, total


@pytest.mark.parametrize("kfmt", FORMATS)
@pytest.mark.parametrize("T,H,bs", [(1, 1, 16), (37, 2, 16), (300, 8, 32), (129, 3, 5)])
def test_pack_matches_oracle(kfmt, T, H, bs):
    vfmt = FORMATS[(FORMATS.index(kfmt) + 3) % len(FORMATS)]
    kc, kf = codec_pair(H, *kfmt, 11)
    vc, vf = codec_pair(H, *vfmt, 22)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(T * 131 + H)
    k, v = random_kv(T, H, gen)
    nb = -(-T // bs) + 3
    rng = np.random.default_rng(T)
    slots = rng.permutation(nb * bs)[:T].astype(np.int64)
    slots[::7] = -1  # padding tokens
    kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    kcpu = k.float().cpu().numpy().astype(np.float64)
    vcpu = v.float().cpu().numpy().astype(np.float64)
    live = slots >= 0
    ref_kp, ref_vp = O.pack_kv(kcpu, vcpu, slots, kf, vf, nb, bs)
    gk, gv = kp.cpu().numpy(), vp.cpu().numpy()
    s = slots[live]
    for g, ref, src, f in ((gk, ref_kp, kcpu, kf), (gv, ref_vp, vcpu, vf)):
        rows = rows_of(g, s, bs, f, H)
        compare_rows(rows, src[live], f, range(H))
        # bytes of slots nobody wrote stay zero, as in the oracle's pool
        written = np.zeros(nb * bs, bool)
        written[s] = True
        free = np.nonzero(~written)[0]
        assert not rows_of(g, free, bs, f, H).any()
        # where no index sits near a boundary the whole row is byte-identical
        if len(s):
            same = (rows == rows_of(ref, s, bs, f, H)).all(axis=-1)
            assert same.mean() > 0.99
            assert (rows[..., -2:] != 0).any(axis=-1).mean() > 0.99  # norms were written


def test_pack_reconstruction_mse_within_two_percent():
    H, T = 8, 2048
    kc, kf = codec_pair(H, (4, 3), (64, 64), 5)
    vc, vf = codec_pair(H, (4, 2), (32, 96), 6)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    k, v = random_kv(T, H, gen)
    kp, vp = tq.page_pool(kc, T // 16, 16), tq.page_pool(vc, T // 16, 16)
    tq.pack_kv(kc, vc, k, v, torch.arange(T, device="cuda"), kp, vp, 16)
    torch.cuda.synchronize()
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        x = src.float().cpu().numpy().astype(np.float64)
        g = rows_of(pages.cpu().numpy(), np.arange(T), 16, f, H)
        mse_gpu = mse_ref = 0.0
        for h in range(H):
            f1 = slice_format(f, h)
            gi, gn = O.decode_rows(g[:, h], f1)
            ri, rn, _ = O.quantize(x[:, h], f1, 0)
            mse_gpu += ((O.dequantize_rows(gi, gn, f1, 0) - x[:, h]) ** 2).sum()
            mse_ref += ((O.dequantize_rows(ri, rn, f1, 0) - x[:, h]) ** 2).sum()
        assert abs(mse_gpu / mse_ref - 1) <= 0.02


def test_pack_edge_values():
    H = 2
    kc, kf = codec_pair(H, (4,), (128,), 0)
    vc, vf = codec_pair(H, (3,), (128,), 1)
    T = 6
    k = torch.zeros(T, H, D, dtype=torch.bfloat16, device="cuda")
    k[1] = 1e-30           # norm underflows fp16
    k[2, :, 0] = 70000.0   # norm overflows fp16 -> inf
    k[3] = 3.0e-3
    k[4, :, 5] = -2.5      # one-hot
    k[5] = torch.linspace(-300, 300, D, device="cuda").to(torch.bfloat16)
    v = k.flip(0).contiguous()
    kp, vp = tq.page_pool(kc, 1, 8), tq.page_pool(vc, 1, 8)
    tq.pack_kv(kc, vc, k, v, torch.arange(T, device="cuda"), kp, vp, 8)
    torch.cuda.synchronize()
    rk, rv = O.pack_kv(k.float().cpu().numpy(), v.float().cpu().numpy(), np.arange(T), kf, vf, 1, 8)
    assert np.array_equal(kp.cpu().numpy(), rk)
    assert np.array_equal(vp.cpu().numpy(), rv)


def test_pack_empty_and_all_padding():
    kc, _ = codec_pair(2, (4,), (128,), 0)
    vc, _ = codec_pair(2, (4,), (128,), 1)
    kp, vp = tq.page_pool(kc, 2, 16), tq.page_pool(vc, 2, 16)
    e = torch.empty(0, 2, D, dtype=torch.bfloat16, device="cuda")
    tq.pack_kv(kc, vc, e, e, torch.empty(0, dtype=torch.int64, device="cuda"), kp, vp, 16)
    k = torch.randn(5, 2, D, device="cuda").to(torch.bfloat16)
    tq.pack_kv(kc, vc, k, k, torch.full((5,), -1, dtype=torch.int64, device="cuda"), kp, vp, 16)
    torch.cuda.synchronize()
    assert not kp.any() and not vp.any()


def test_pack_slot_outside_pool_sets_error_and_skips(monkeypatch):
    kc, _ = codec_pair(1, (4,), (128,), 0)
    vc, _ = codec_pair(1, (4,), (128,), 1)
    kp, vp = tq.page_pool(kc, 2, 4), tq.page_pool(vc, 2, 4)
    k = torch.randn(3, 1, D, device="cuda").to(torch.bfloat16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, k, torch.tensor([0, 8, 5], device="cuda"), kp, vp, 4, d_err=err)
    torch.cuda.synchronize()
    assert err.item() & tq.TQ_DERR_SLOT
    f = O.Format(D, 1, (4,), (128,), None, 0)
    rows = rows_of(kp.cpu().numpy(), np.arange(8), 4, f, 1)
    assert rows[0].any() and rows[5].any()
    assert not rows[[1, 2, 3, 4, 6, 7]].any()
    monkeypatch.setenv("TQ_CHECKED", "1")
    err.zero_()
    with pytest.raises(IndexError):
        tq.pack_kv(kc, vc, k, k, torch.tensor([0, 8, 5], device="cuda"), kp, vp, 4, d_err=err)


def test_pack_argument_errors():
    kc, _ = codec_pair(2, (4,), (128,), 0)
    vc1, _ = codec_pair(1, (4,), (128,), 1)
    kp = tq.page_pool(kc, 2, 4)
    k = torch.randn(3, 2, D, device="cuda").to(torch.bfloat16)
    with pytest.raises(ValueError):
        tq.pack_kv(kc, vc1, k, k, torch.arange(3, device="cuda"), kp, tq.page_pool(vc1, 2, 4), 4)
    with pytest.raises(ValueError):
        tq.pack_kv(kc, kc, k.float(), k, torch.arange(3, device="cuda"), kp, kp, 4)
    with pytest.raises(ValueError):  # pool shaped for another block size
        tq.pack_kv(kc, kc, k, k, torch.arange(3, device="cuda"), kp, kp, 8)


def test_pack_workload_sample_full_size():
    """The full pack workload in the benchmark's launch, checked on sampled rows."""
    w = W.WORKLOADS["pack_llama8b_4bit"]
    kc, vc, kf, vf = workload_codecs(w)
    k, v, slots, layout = W.pack_batch(w, device="cuda")
    kp, vp = tq.page_pool(kc, layout.num_blocks, w.block_size), tq.page_pool(vc, layout.num_blocks, w.block_size)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, w.block_size, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    rng = np.random.default_rng(3)
    pick = np.sort(rng.choice(len(slots), 4096, replace=False))
    s = slots[pick]
    flips = total = 0
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        sub = pages[torch.as_tensor(s // w.block_size, device="cuda")].cpu().numpy()  # the touched sub-pages
        rows = np.stack([O.read_rows(sub, np.arange(len(s)), h, s % w.block_size, f, w.block_size)
                         for h in range(w.num_kv_heads)], axis=1)
        x = src[torch.as_tensor(pick, device="cuda")].float().cpu().numpy().astype(np.float64)
        a, b = compare_rows(rows, x, f, range(w.num_kv_heads))
        flips, total = flips + a, total + b
    assert flips <= MAX_FLIP_FRACTION * total


def test_pack_edge_values_uniform_4bit_fast_path():
    """Zero, tiny, huge and one-hot vectors through the tensor-core pack (uniform 4-bit K and V)."""
    H = 2
    kc, kf = codec_pair(H, (4,), (128,), 3)
    vc, vf = codec_pair(H, (4,), (128,), 4)
    T = 20
    k = torch.zeros(T, H, D, dtype=torch.bfloat16, device="cuda")
    k[1] = 1e-30
    k[2, :, 0] = 70000.0
    k[3] = 3.0e-3
    k[4, :, 5] = -2.5
    k[5] = torch.linspace(-300, 300, D, device="cuda").to(torch.bfloat16)
    k[6:] = torch.randn(T - 6, H, D, device="cuda").to(torch.bfloat16) * 7
    v = k.flip(0).contiguous()
    slots = torch.tensor([5, 0, 17, 3, -1, 8, 9, 10, 11, 12, 13, 14, 15, 16, 1, 2, 4, 6, 7, 18], device="cuda")
    kp, vp = tq.page_pool(kc, 3, 8), tq.page_pool(vc, 3, 8)
    tq.pack_kv(kc, vc, k, v, slots, kp, vp, 8)
    torch.cuda.synchronize()
    rk, rv = O.pack_kv(k.float().cpu().numpy(), v.float().cpu().numpy(), slots.cpu().numpy(), kf, vf, 3, 8)
    assert np.array_equal(kp.cpu().numpy(), rk)
    assert np.array_equal(vp.cpu().numpy(), rv)


@pytest.mark.parametrize("kspec,vspec,bs,mode", [(((4,), (128,)), ((4,), (128,)), 16, ""),
                                                  (((4, 3), (64, 64)), ((4, 3), (64, 64)), 16, ""),
                                                  (((4, 2), (32, 96)), ((3,), (128,)), 32, ""),
                                                  (((2,), (128,)), ((4, 3), (64, 64)), 48, ""),
                                                  (((4, 3), (64, 64)), ((4, 2), (32, 96)), 16, "gw"),
                                                  (((4, 2), (32, 96)), ((4, 3), (64, 64)), 40, "gw"),
                                                  (((3, 2), (64, 64)), ((4, 3), (64, 64)), 16, "qjl"),
                                                  (((3,), (128,)), ((2,), (128,)), 24, "qjl"),
                                                  (((3, 2), (64, 64)), ((4, 3), (64, 64)), 16, "recipe"),
                                                  (((4, 3), (64, 64)), ((3, 2), (64, 64)), 32, "recipe")])
def test_fast_and_general_pack_kernels_agree(monkeypatch, kspec, vspec, bs, mode):
    """The tensor-core packs (uniform 4-bit, the plain 2/3/4-bit mixes, the group-wise 4/3 and 4/2
    formats, QJL formats and recipe rows) against the general kernel and the oracle on the same
    tokens."""
    H, T = 4, 700
    qjl, gw = mode in ("qjl", "recipe"), mode in ("gw", "recipe")
    kc, kf = codec_pair(H, *kspec, 8, qjl=qjl, groupwise=gw)
    vc, vf = codec_pair(H, *vspec, 9, qjl=qjl, groupwise=gw)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(5)
    k, v = random_kv(T, H, gen)
    nb = -(-T // bs) + 2
    slots = torch.as_tensor(np.random.default_rng(1).permutation(nb * bs)[:T], device="cuda")
    out = []
    for kernel in ("fast", "general"):
        if kernel == "general":
            monkeypatch.setenv("TQ_PACK_KERNEL", "general")
        kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
        tq.pack_kv(kc, vc, k, v, slots, kp, vp, bs)
        torch.cuda.synchronize()
        out.append((kp.cpu().numpy(), vp.cpu().numpy()))
    s = slots.cpu().numpy()
    for i, (src, f) in enumerate(((k, kf), (v, vf))):
        x = src.float().cpu().numpy().astype(np.float64)
        for pages in (out[0][i], out[1][i]):
            if mode == "qjl":
                assert check_qjl_rows(rows_of(pages, s, bs, f, H), x, f, range(H)) > 0.99 * T * H
            elif mode == "recipe":
                assert check_recipe_rows(rows_of(pages, s, bs, f, H), x, f, range(H)) > 0.99 * T * H
            else:
                compare_rows(rows_of(pages, s, bs, f, H), x, f, range(H))
        same = (out[0][i] == out[1][i]).mean()
        assert same > 0.999


@pytest.mark.parametrize("kspec,vspec,mode", [(((4,), (128,)), ((4,), (128,)), ""),
                                              (((4, 3), (64, 64)), ((4, 2), (32, 96)), ""),
                                              (((4, 3), (64, 64)), ((4, 2), (32, 96)), "gw"),
                                              (((3, 2), (64, 64)), ((3,), (128,)), "qjl"),
                                              (((3, 2), (64, 64)), ((4, 3), (64, 64)), "recipe")])
def test_pack_tokens_not_finite(monkeypatch, kspec, vspec, mode):
    """Tokens holding inf, NaN or values near the bf16 limit (norms far beyond fp16) pack without
    an error flag in the tensor-core kernels and the general one, and leave the rows of the other
    tokens as the oracle has them."""
    H, T, bs = 4, 200, 16
    qjl, gw = mode in ("qjl", "recipe"), mode in ("gw", "recipe")
    kc, kf = codec_pair(H, *kspec, 13, qjl=qjl, groupwise=gw)
    vc, vf = codec_pair(H, *vspec, 14, qjl=qjl, groupwise=gw)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    k, v = random_kv(T, H, gen)
    k[3, 1, 5] = float("inf")
    k[10, 0, :] = float("nan")
    k[11, 2, 64:] = -float("inf")
    v[20, 2, 7] = -float("inf")
    v[21, 3, 100] = float("nan")
    k[33, 3, 0] = 3.0e38
    v[50, 1, :] = 2.0e38
    bad_tokens = {3, 10, 11, 20, 21, 33, 50}
    nb = -(-T // bs) + 1
    slots = torch.as_tensor(np.random.default_rng(3).permutation(nb * bs)[:T], device="cuda")
    for kernel in ("fast", "general"):
        if kernel == "general":
            monkeypatch.setenv("TQ_PACK_KERNEL", "general")
        kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        tq.pack_kv(kc, vc, k, v, slots, kp, vp, bs, d_err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        good = np.array([t for t in range(T) if t not in bad_tokens])
        s = slots.cpu().numpy()[good]
        for pages, src, f in ((kp, k, kf), (vp, v, vf)):
            x = src[torch.as_tensor(good, device="cuda")].float().cpu().numpy().astype(np.float64)
            rows = rows_of(pages.cpu().numpy(), s, bs, f, H)
            if mode == "qjl":
                assert check_qjl_rows(rows, x, f, range(H)) > 0.99 * len(good) * H
            elif mode == "recipe":
                assert check_recipe_rows(rows, x, f, range(H)) > 0.99 * len(good) * H
            else:
                flips, total = compare_rows(rows, x, f, range(H))
                assert flips <= max(1, MAX_FLIP_FRACTION * total)


def test_pack_workload_whole_sequence_and_mse_full_size():
    """The full pack workload in the benchmark's launch (262144 tokens, one call): every row of one
    whole 8192-token sequence (all 8 KV heads, K and V) against the oracle, and the reconstruction
    MSE of those GPU rows within 2 % of the oracle's own rows (the uniform 4-bit tensor-core pack)."""
    w = W.WORKLOADS["pack_llama8b_4bit"]
    kc, vc, kf, vf = workload_codecs(w)
    k, v, slots, layout = W.pack_batch(w, device="cuda")
    kp, vp = tq.page_pool(kc, layout.num_blocks, w.block_size), tq.page_pool(vc, layout.num_blocks, w.block_size)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, w.block_size, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    seq_len = int(layout.seq_lens[0])
    b = 5  # a sequence in the middle of the batch
    pick = np.arange(b * seq_len, (b + 1) * seq_len)
    s = slots[pick]
    flips = total = 0
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        sub = pages[torch.as_tensor(s // w.block_size, device="cuda")].cpu().numpy()
        rows = np.stack([O.read_rows(sub, np.arange(len(s)), h, s % w.block_size, f, w.block_size)
                         for h in range(w.num_kv_heads)], axis=1)
        x = src[torch.as_tensor(pick, device="cuda")].float().cpu().numpy().astype(np.float64)
        a, c = compare_rows(rows, x, f, range(w.num_kv_heads))
        flips, total = flips + a, total + c
        mse_gpu = mse_ref = 0.0
        for h in range(w.num_kv_heads):
            f1 = slice_format(f, h)
            gi, gn = O.decode_rows(rows[:, h], f1)
            ri, rn, _ = O.quantize(x[:, h], f1, 0)
            mse_gpu += ((O.dequantize_rows(gi, gn, f1, 0) - x[:, h]) ** 2).sum()
            mse_ref += ((O.dequantize_rows(ri, rn, f1, 0) - x[:, h]) ** 2).sum()
        assert abs(mse_gpu / mse_ref - 1) <= 0.02
    assert flips <= MAX_FLIP_FRACTION * total


@pytest.mark.parametrize("name", ["pack_llama70b_3p5bit", "pack_llama8b_2p5bit", "pack_llama8b_3p5bit_qjl",
                                  "pack_llama8b_3p5bit_groupwise", "pack_llama8b_3p5bit_recipe"])
def test_pack_workloads_full_size_one_sequence(name):
    """Each mixed-format pack workload in the benchmark's launch (32 x 8192 tokens, one call): every row
    of one whole 8192-token sequence (all 8 KV heads, K and V) against the oracle, with its checks for
    the format (index flips only at a boundary, norms bit-exact; QJL signs only where the projection is
    negligible)."""
    w = W.WORKLOADS[name]
    kc, vc, kf, vf = workload_codecs(w)
    k, v, slots, layout = W.pack_batch(w, device="cuda")
    kp, vp = tq.page_pool(kc, layout.num_blocks, w.block_size), tq.page_pool(vc, layout.num_blocks, w.block_size)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, w.block_size, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    seq_len = int(layout.seq_lens[0])
    b = 21  # a sequence late in the batch
    pick = np.arange(b * seq_len, (b + 1) * seq_len)
    s = slots[pick]
    H = w.num_kv_heads
    for pages, src, f in ((kp, k, kf), (vp, v, vf)):
        sub = pages[torch.as_tensor(s // w.block_size, device="cuda")].cpu().numpy()
        rows = np.stack([O.read_rows(sub, np.arange(len(s)), h, s % w.block_size, f, w.block_size)
                         for h in range(H)], axis=1)
        x = src[torch.as_tensor(pick, device="cuda")].float().cpu().numpy().astype(np.float64)
        if f.qjl and f.groupwise:
            assert check_recipe_rows(rows, x, f, range(H)) > 0.99 * len(s) * H
        elif f.qjl:
            assert check_qjl_rows(rows, x, f, range(H)) > 0.99 * len(s) * H
        else:
            flips, total = compare_rows(rows, x, f, range(H))
            assert flips <= MAX_FLIP_FRACTION * total


def test_pack_inputs_aligned_to_8_bytes_only():
    """K and V that start 8 bytes past a 16-byte boundary (the call's own requirement is 8) take the
    general kernel, since the tensor-core packs copy 16-byte pieces of the input rows; rows match the
    oracle."""
    H, T, bs = 2, 50, 16
    kc, kf = codec_pair(H, (4,), (128,), 21)
    vc, vf = codec_pair(H, (4, 3), (64, 64), 22)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4)
    k0, v0 = random_kv(T, H, gen)
    kb = torch.empty(T * H * D + 4, dtype=torch.bfloat16, device="cuda")
    vb = torch.empty(T * H * D + 4, dtype=torch.bfloat16, device="cuda")
    k = kb[4:].view(T, H, D)
    v = vb[4:].view(T, H, D)
    k.copy_(k0)
    v.copy_(v0)
    assert k.data_ptr() % 16 == 8 and v.data_ptr() % 16 == 8
    nb = -(-T // bs) + 1
    slots = torch.arange(T, device="cuda")
    kp, vp = tq.page_pool(kc, nb, bs), tq.page_pool(vc, nb, bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.pack_kv(kc, vc, k, v, slots, kp, vp, bs, d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    s = np.arange(T)
    for pages, src, f in ((kp, k0, kf), (vp, v0, vf)):
        x = src.float().cpu().numpy().astype(np.float64)
        flips, total = compare_rows(rows_of(pages.cpu().numpy(), s, bs, f, H), x, f, range(H))
        assert flips <= max(1, MAX_FLIP_FRACTION * total)
