"""GPU parity of tq_decode_paged against the fp64 oracle on the same (GPU-written) pages."""

import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq
from quantized_paged_kv_pack_b200 import workloads as W

from helpers import D, DecodeProblem, slice_format, workload_codecs

pytestmark = pytest.mark.gpu

ATOL = 2e-3  # max-abs error of the fp32 decode vs the fp64 oracle on the same cache

U4 = ((4,), (128,), 0)
U3 = ((3,), (128,), 1)
U2 = ((2,), (128,), 2)
M35 = ((4, 3), (64, 64), 3)
M25 = ((4, 2), (32, 96), 4)


def check(prob, pairs=None):
    out = prob.run()
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    pairs = pairs if pairs is not None else [(b, hq) for b in range(prob.B) for hq in range(prob.Hq)]
    worst = scale = 0.0
    for b, hq in pairs:
        ref = prob.oracle(b, hq)
        worst = max(worst, float(np.abs(got[b, hq] - ref).max()))
        scale = max(scale, float(np.abs(ref).max()))
    assert worst <= ATOL, worst
    if any(prob.lens[b] for b, _ in pairs):
        assert scale > 0.5  # the outputs are not trivially zero
    return worst


@pytest.mark.parametrize("kspec,vspec", [(U4, U4), (M35, M35), (M25, U3), (U2, M35), (U3, U2)])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_matches_oracle_small(kspec, vspec, G):
    lens = [1, 15, 16, 17, 100, 700]
    prob = DecodeProblem(lens, 2, G, kspec, (vspec[0], vspec[1], vspec[2] + 10), window=0, block_size=16, seed=G)
    check(prob)


@pytest.mark.parametrize("window,bs", [(8, 16), (64, 16), (128, 32), (5, 7)])
def test_decode_with_window_and_ragged_lengths(window, bs):
    lens = [0, 1, window, window + 1, 3 * window + 5, 2000, 4099]
    prob = DecodeProblem(lens, 2, 4, M25, U3, window=window, block_size=bs, seed=window)
    check(prob)


def test_decode_gqa16_and_long_sequence_spans_many_splits():
    prob = DecodeProblem([9000, 300], 1, 16, U4, M35, window=16, block_size=16, seed=5)
    check(prob)


def test_decode_more_splits_than_combine_threads():
    """80,000 packed tokens in 512-token splits: 157 split records, more than the combine's 128 threads
    take in one chunk."""
    prob = DecodeProblem([80000, 700], 1, 4, U4, U4, window=8, block_size=16, seed=6)
    check(prob)


def test_decode_full_small_workload():
    """The oracle-sized workload in full: 1 sequence, GQA 8, context 4096, 4-bit."""
    w = W.WORKLOADS["decode_gqa8_4k_4bit"]
    kc, vc, kf, vf = workload_codecs(w)
    layout = W.page_layout(w)
    kp, vp = tq.page_pool(kc, layout.num_blocks, w.block_size), tq.page_pool(vc, layout.num_blocks, w.block_size)
    L = int(layout.seq_lens[0])
    k, v = W.sequence_kv(w, 0, 0, L, device="cuda")
    slots = W.slot_mapping(layout, 0, 0, L, w.block_size)
    tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, w.block_size)
    q = W.queries(w, device="cuda")
    bt = torch.as_tensor(layout.block_tables, device="cuda")
    sl = torch.as_tensor(layout.seq_lens.astype(np.int32), device="cuda")
    out = tq.decode_paged(kc, vc, q, kp, vp, w.block_size, bt, sl, L, None, None, 0, 1 / math.sqrt(D))
    torch.cuda.synchronize()
    ref = O.decode_attention(q.float().cpu().numpy().astype(np.float64), kp.cpu().numpy(), vp.cpu().numpy(),
                             layout.block_tables, layout.seq_lens, None, None, 0, 1 / math.sqrt(D), kf, vf,
                             w.block_size)
    assert np.abs(out.cpu().numpy() - ref).max() <= ATOL
    assert np.abs(ref).max() > 0.5


def test_decode_empty_batch_and_zero_lengths():
    prob = DecodeProblem([0, 0], 1, 2, U4, U4, window=4, block_size=16, seed=1)
    out = prob.run()
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_decode_bad_block_id_sets_error_without_fault():
    prob = DecodeProblem([40], 1, 2, U4, U4, window=0, block_size=16, seed=2)
    prob.block_tables[0, 1] = prob.num_blocks + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    prob.run(d_err=err)
    torch.cuda.synchronize()
    assert err.item() & tq.TQ_DERR_BLOCK


def test_decode_argument_errors():
    prob = DecodeProblem([40], 1, 2, U4, U4, window=0, block_size=16, seed=3)
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        prob.run(workspace=small)
    with pytest.raises(ValueError):
        tq.decode_paged(prob.kc, prob.vc, prob.q, prob.k_pages, prob.v_pages, prob.bs, prob.block_tables, prob.seq_lens,
                        prob.max_seq_len, None, None, 4, prob.scale)
    q3 = torch.zeros(1, 3, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.UnsupportedFormatError):  # 3 query heads per KV head
        tq.decode_paged(prob.kc, prob.vc, q3, prob.k_pages, prob.v_pages, prob.bs, prob.block_tables, prob.seq_lens,
                        prob.max_seq_len, None, None, 0, prob.scale)
    prob2 = DecodeProblem([40], 2, 2, U4, U4, window=0, block_size=16, seed=4)
    with pytest.raises(ValueError):  # 3 query heads over 2 KV heads
        tq.decode_paged(prob2.kc, prob2.vc, q3, prob2.k_pages, prob2.v_pages, prob2.bs, prob2.block_tables,
                        prob2.seq_lens,
                        prob2.max_seq_len, None, None, 0, prob2.scale)


def test_decode_phases_equal_single_call():
    prob = DecodeProblem([500, 1234], 2, 4, M35, U3, window=8, block_size=16, seed=9)
    ws = tq.alloc_workspace(prob.B, prob.Hq, prob.H, prob.max_seq_len, prob.bs)
    a = prob.run(workspace=ws).clone()
    out = torch.empty_like(a)
    prob.run(workspace=ws, phase="partials")
    prob.run(workspace=ws, phase="combine", out=out)
    torch.cuda.synchronize()
    assert torch.equal(a, out)


def _workload_problem(name, n_seq):
    """Build the named decode workload on the GPU (pages by the GPU pack kernel)."""
    w = W.WORKLOADS[name]
    kc, vc, kf, vf = workload_codecs(w)
    layout = W.page_layout(w)
    kp, vp = tq.page_pool(kc, layout.num_blocks, w.block_size), tq.page_pool(vc, layout.num_blocks, w.block_size)
    for b in range(len(layout.seq_lens)):
        P = int(layout.packed_lens[b])
        for t0 in range(0, P, 16384):
            t1 = min(P, t0 + 16384)
            k, v = W.sequence_kv(w, b, t0, t1, device="cuda")
            slots = W.slot_mapping(layout, b, t0, t1, w.block_size)
            tq.pack_kv(kc, vc, k, v, torch.as_tensor(slots, device="cuda"), kp, vp, w.block_size)
    kw, vw = W.windows(w, layout, device="cuda")
    return w, kc, vc, kf, vf, layout, kp, vp, kw, vw


def _checked_sequences(layout, bs, n=8):
    """At least n sequences: the shortest, the median, the longest, and ones whose packed length ends
    inside a block (and so inside a split: a split is a whole number of blocks)."""
    L, P = layout.seq_lens, layout.packed_lens
    order = np.argsort(L, kind="stable")
    picks = [int(order[0]), int(order[len(order) // 2]), int(order[-1])]
    for b in order:
        if len(picks) >= n:
            break
        if P[b] % bs and int(b) not in picks:
            picks.append(int(b))
    for b in order[::-1]:
        if len(picks) >= n:
            break
        if int(b) not in picks:
            picks.append(int(b))
    return picks


@pytest.mark.parametrize("name", ["decode_llama8b_4bit", "decode_llama70b_3p5bit", "decode_llama8b_2p5bit",
                                  "decode_llama8b_3p5bit_qjl", "decode_llama8b_3p5bit_groupwise",
                                  "decode_llama8b_3p5bit_recipe"])
def test_decode_full_size_workloads(name, monkeypatch):
    """Full-size workloads in the benchmark's launch: every query head of 8 sequences against the
    oracle (element by element), and, on the three headline-format workloads, every output against
    the general CUDA-core kernel on the same cache."""
    w, kc, vc, kf, vf, layout, kp, vp, kw, vw = _workload_problem(name, None)
    q = W.queries(w, device="cuda")
    bt = torch.as_tensor(layout.block_tables, device="cuda")
    sl = torch.as_tensor(layout.seq_lens.astype(np.int32), device="cuda")
    maxL = int(layout.seq_lens.max())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = tq.decode_paged(kc, vc, q, kp, vp, w.block_size, bt, sl, maxL, kw, vw, w.window, 1 / math.sqrt(D),
                          d_err=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    got = out.cpu().numpy()
    G = w.num_q_heads // w.num_kv_heads
    picks = _checked_sequences(layout, w.block_size)
    assert len(picks) >= 8
    P = layout.packed_lens
    assert any(P[b] % w.block_size for b in picks) or not np.any(P % w.block_size)
    for b in picks:
        L, Pb = int(layout.seq_lens[b]), int(P[b])
        nblk = -(-Pb // w.block_size)
        blocks = torch.as_tensor(layout.block_tables[b, :nblk].astype(np.int64), device="cuda")
        for h in range(w.num_kv_heads):
            ref = O.decode_attention(q[b:b + 1, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64),
                                     kp[blocks][:, h:h + 1].cpu().numpy(), vp[blocks][:, h:h + 1].cpu().numpy(),
                                     np.arange(nblk)[None], [L], kw[b:b + 1, h:h + 1].float().cpu().numpy(),
                                     vw[b:b + 1, h:h + 1].float().cpu().numpy(), w.window, 1 / math.sqrt(D),
                                     slice_format(kf, h), slice_format(vf, h), w.block_size)[0]
            assert np.abs(got[b, h * G:(h + 1) * G] - ref).max() <= ATOL, (b, h)
            assert np.abs(ref).max() > 0.5
    if name in ("decode_llama8b_4bit", "decode_llama70b_3p5bit", "decode_llama8b_2p5bit"):
        monkeypatch.setenv("TQ_DECODE_KERNEL", "general")
        general = tq.decode_paged(kc, vc, q, kp, vp, w.block_size, bt, sl, maxL, kw, vw, w.window,
                                  1 / math.sqrt(D), d_err=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        assert (general - out).abs().max().item() <= ATOL


def test_tensor_core_and_general_kernels_agree(monkeypatch):
    """Formats with a tensor-core instantiation against the general kernel on the same cache."""
    prob = DecodeProblem([3000, 17, 260], 2, 8, M35, M35, window=32, block_size=16, seed=21)
    fast = prob.run().clone()
    monkeypatch.setenv("TQ_DECODE_KERNEL", "general")
    general = prob.run()
    torch.cuda.synchronize()
    assert (fast - general).abs().max().item() <= ATOL
    check(prob)


# ---- KV head counts that are multiples of 8: the kernel that stages one
# 16-token tile of 8 KV heads per ring slot and gives each warp one KV head.

@pytest.mark.parametrize("kspec,vspec", [(U4, U4), (M35, M35), (M25, U3), (U2, M35), (U3, U2)])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_decode_eight_kv_heads_matches_oracle(kspec, vspec, G):
    lens = [1, 16, 17, 300, 1100]
    prob = DecodeProblem(lens, 8, G, kspec, (vspec[0], vspec[1], vspec[2] + 10), window=0, block_size=16,
                         seed=100 + G)
    rng = np.random.default_rng(G)
    pairs = [(b, int(hq)) for b in range(prob.B) for hq in rng.choice(prob.Hq, min(prob.Hq, 12), replace=False)]
    check(prob, pairs)


@pytest.mark.parametrize("window,bs", [(8, 16), (64, 32), (128, 48)])
def test_decode_eight_kv_heads_windows_and_block_sizes(window, bs):
    """Block sizes above 16 take the per-head copies of a slot; windows go to the warps directly."""
    lens = [0, 1, window, window + 1, 3 * window + 5, 2100]
    prob = DecodeProblem(lens, 8, 4, M25, U3, window=window, block_size=bs, seed=window + bs)
    pairs = [(b, hq) for b in range(prob.B) for hq in (0, 5, 13, 31)]
    check(prob, pairs)



@pytest.mark.parametrize("kspec,vspec,G,bs", [(U4, U4, 8, 16), (M35, M35, 4, 32), (M25, U3, 8, 32),
                                               (M35, U4, 2, 16)])
def test_block_kernel_and_paired_kernel_agree(kspec, vspec, G, bs, monkeypatch):
    """TQ_DECODE_PAIR=0 runs the one-warp-per-head block kernel that the paired kernel replaces (it
    remains the path when the paired kernel's ring does not fit): both against the oracle and each
    other, with ragged lengths, a window and splits cut mid-block."""
    lens = [1, bs - 1, 5 * bs + 3, 4700, 9000]
    prob = DecodeProblem(lens, 8, G, kspec, (vspec[0], vspec[1], vspec[2] + 10), window=24, block_size=bs,
                         seed=200 + G + bs)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    paired = prob.run(d_err=err).clone()
    monkeypatch.setenv("TQ_DECODE_PAIR", "0")
    block = prob.run(d_err=err).clone()
    torch.cuda.synchronize()
    assert err.item() == 0
    assert (paired - block).abs().max().item() <= ATOL
    rng = np.random.default_rng(G + bs)
    pairs = [(b, int(hq)) for b in range(prob.B) for hq in rng.choice(prob.Hq, 6, replace=False)]
    check(prob, pairs)

def test_decode_sixteen_kv_heads_gqa16():
    """Two groups of 8 KV heads, two query-head groups per KV head."""
    prob = DecodeProblem([5000, 700], 16, 16, U4, M35, window=16, block_size=16, seed=31)
    pairs = [(b, hq) for b in range(prob.B) for hq in (0, 7, 8, 15, 130, 255)]
    check(prob, pairs)


def test_decode_eight_kv_heads_all_heads():
    """Every query head of a GQA-8 cache with 8 KV heads (each warp's records)."""
    prob = DecodeProblem([2500, 40], 8, 8, M35, M35, window=32, block_size=16, seed=41)
    check(prob)


def test_decode_eight_kv_heads_bad_block_id_sets_error_without_fault():
    prob = DecodeProblem([200], 8, 2, U4, U4, window=0, block_size=16, seed=42)
    prob.block_tables[0, 3] = -7
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    prob.run(d_err=err)
    torch.cuda.synchronize()
    assert err.item() & tq.TQ_DERR_BLOCK


@pytest.mark.parametrize("H,bs", [(8, 16), (2, 32)])  # the block kernel and the per-head kernel
def test_decode_boundary_tokens_dense(H, bs):
    """Boundary-token preservation: first S and last W tokens dense, the middle packed (one window buffer)."""
    lens = [0, 3, 4, 11, 12, 700, 3000]
    prob = DecodeProblem(lens, H, 4, M35, U3, window=8, block_size=bs, seed=80 + H, sinks=4)
    assert prob.window == 12
    rng = np.random.default_rng(H)
    pairs = [(b, int(hq)) for b in range(prob.B) for hq in rng.choice(prob.Hq, min(prob.Hq, 6), replace=False)]
    check(prob, pairs)


@pytest.mark.parametrize("H", [8, 2])  # the block kernel and the per-head kernel
def test_decode_many_sequences_work_list(monkeypatch, H):
    """More sequences than the work-list scan takes in one pass (1024), many of them empty or window-only:
    the tensor-core kernels deal only the listed items; every sequence is checked against the general
    kernel and a sample against the oracle."""
    rng = np.random.default_rng(11)
    lens = rng.integers(0, 90, 1500)
    lens[::7] = 0
    lens[::11] = rng.integers(300, 700, len(lens[::11]))
    prob = DecodeProblem(lens.tolist(), H, 4, M35, M35, window=16, block_size=16, seed=12)
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
    for b in [int(i) for i in rng.choice(np.flatnonzero(lens > 0), 6, replace=False)] + [1499]:
        if lens[b] == 0:
            continue
        hq = int(rng.integers(prob.Hq))
        assert np.abs(got[b, hq] - prob.oracle(b, hq)).max() <= ATOL


def test_decode_is_reproducible_bit_for_bit_on_ragged_lengths():
    """Ragged lengths put several partial splits of one tile count in the work list; their order is a
    function of the lengths alone, so repeated calls give the same output bit for bit."""
    lens = [int(x) for x in np.random.default_rng(12).integers(1, 6000, size=48)]
    prob = DecodeProblem(lens, 8, 4, ((4,), (128,), 3), ((4, 3), (64, 64), 4), window=16, block_size=16, seed=9)
    outs = [prob.run().clone() for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
