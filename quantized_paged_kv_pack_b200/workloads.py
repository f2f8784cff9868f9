"""Seeded synthetic inputs for the pack and decode calls.

This module only draws random inputs and lays out page tables. It holds none of
the codec arithmetic (no rotation, codebook, quantizer or packer), so the CPU
oracle and the CUDA path can both be fed from it without sharing any of the
method.

Input recipe (the pages measure on LongBench and on needle / summarize / qa
prompts of 32k tokens, none of which is available here; these seeded caches
stand in for them with the KV shapes of Llama-3.1-8B and -70B and contexts up
to the 131072-token limit named on the TurboQuant Inference Server page,
"Configuration"):

* K, V ~ N(0, 1) in fp32; per KV head ``n_outliers`` distinct channels drawn
  without replacement are multiplied by 10 (independently for K and V);
  with ``token_scales`` every (token, head) vector is multiplied by
  exp(U[ln 0.5, ln 4]); the result is rounded to bf16 last.
* q ~ N(0, 1), rounded to bf16.
* Parameters (lengths, block permutations, channel sets, metadata tables) come
  from NumPy ``PCG64(seed)``; bulk tensors from ``torch.Generator`` on the
  target device, reseeded per (sequence, 1024-token chunk) so any part of a
  cache can be regenerated on its own.
"""

from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

CHUNK = 1024


@dataclass(frozen=True)
class CodecSpec:
    """Plain parameters of one codec; each side builds its own codec from them."""

    group_bits: tuple
    group_size: tuple
    seed: int
    high_coords: Optional[np.ndarray] = None  # [H_kv][group_size[0]] int16, sorted
    qjl: bool = False                         # QJL residual stage after the MSE groups
    groupwise: bool = False                   # high_coords name original channels, per-group rotation


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str               # "decode" or "pack"
    seed: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    window: int
    k_bits: tuple
    k_sizes: tuple
    v_bits: tuple
    v_sizes: tuple
    k_seed: int
    v_seed: int
    n_outliers: int
    token_scales: bool
    lengths: str            # "fixed:N", "uniform:lo:hi", "loguniform:lo:hi"
    pool_slack: float = 1.0  # page pool = ceil(slack * needed) blocks, free blocks interleaved
    description: str = ""
    k_qjl: bool = False      # keys carry the QJL residual stage
    groupwise: bool = False  # K and V: group-wise rotation with per-group norms


WORKLOADS = {
    "decode_gqa8_4k_4bit": Workload(
        "decode_gqa8_4k_4bit", "decode", 1001, 1, 8, 1, 128, 16, 0,
        (4,), (128,), (4,), (128,), 0, 0, 4, False, "fixed:4096",
        description="single decode step, 1 sequence, GQA 8 (8 query heads / 1 KV head), "
                    "context 4096, block 16, uniform 4-bit K and V, no window"),
    "pack_llama8b_4bit": Workload(
        "pack_llama8b_4bit", "pack", 1002, 32, 32, 8, 128, 16, 0,
        (4,), (128,), (4,), (128,), 0, 1, 8, True, "fixed:8192",
        description="pack 32 sequences x 8192 tokens, 8 KV heads (Llama-3.1-8B KV shapes), "
                    "block 16, shuffled slot mapping, uniform 4-bit K and V"),
    "pack_llama70b_3p5bit": Workload(
        "pack_llama70b_3p5bit", "pack", 1008, 32, 64, 8, 128, 16, 0,
        (4, 3), (64, 64), (4, 3), (64, 64), 0, 1, 8, True, "fixed:8192",
        description="pack 32 sequences x 8192 tokens, 8 KV heads (the Llama-3.1-70B decode shapes), "
                    "block 16, shuffled slot mapping, K and V 3.5-bit (64 channels at 4 bits + 64 at 3 "
                    "bits, independent tables)"),
    "pack_llama8b_2p5bit": Workload(
        "pack_llama8b_2p5bit", "pack", 1009, 32, 32, 8, 128, 32, 0,
        (4, 2), (32, 96), (3,), (128,), 0, 1, 8, True, "fixed:8192",
        description="pack 32 sequences x 8192 tokens, 8 KV heads, block 32, shuffled slot mapping, "
                    "K 2.5-bit (32 channels at 4 bits + 96 at 2 bits), V uniform 3-bit (the formats of "
                    "the batch-256 decode workload)"),
    "pack_llama8b_3p5bit_qjl": Workload(
        "pack_llama8b_3p5bit_qjl", "pack", 1011, 32, 32, 8, 128, 16, 0,
        (3, 2), (64, 64), (4, 3), (64, 64), 61, 62, 8, True, "fixed:8192", k_qjl=True,
        description="pack 32 sequences x 8192 tokens, 8 KV heads, block 16, shuffled slot mapping, the QJL "
                    "decode workload's formats (K 2.5-bit MSE plus the 1-bit QJL stage, V 3.5-bit); QJL "
                    "tensor-core pack for K, plain tensor-core pack for V"),
    "pack_llama8b_3p5bit_groupwise": Workload(
        "pack_llama8b_3p5bit_groupwise", "pack", 1012, 32, 32, 8, 128, 16, 0,
        (4, 3), (64, 64), (4, 3), (64, 64), 71, 72, 8, True, "fixed:8192", groupwise=True,
        description="pack 32 sequences x 8192 tokens, 8 KV heads, block 16, shuffled slot mapping, K and V "
                    "3.5-bit group-wise (the group-wise decode workload's formats); tensor-core group-wise "
                    "pack kernel"),
    "pack_llama8b_3p5bit_recipe": Workload(
        "pack_llama8b_3p5bit_recipe", "pack", 1013, 32, 32, 8, 128, 16, 0,
        (3, 2), (64, 64), (4, 3), (64, 64), 81, 82, 8, True, "fixed:8192", k_qjl=True, groupwise=True,
        description="pack 32 sequences x 8192 tokens, 8 KV heads, block 16, shuffled slot mapping, the recipe "
                    "decode workload's formats (K recipe rows: two group-wise groups, each with its QJL "
                    "signs and norms; V 3.5-bit group-wise); tensor-core recipe and group-wise packs"),
    "decode_llama8b_4bit": Workload(
        "decode_llama8b_4bit", "decode", 1003, 64, 32, 8, 128, 16, 64,
        (4,), (128,), (4,), (128,), 0, 1, 8, True, "uniform:1024:32768",
        description="decode batch 64, 32 query / 8 KV heads (Llama-3.1-8B), context U[1024, 32768], "
                    "block 16, uniform 4-bit K and V, 64-token bf16 window"),
    "decode_llama70b_3p5bit": Workload(
        "decode_llama70b_3p5bit", "decode", 1004, 16, 64, 8, 128, 16, 128,
        (4, 3), (64, 64), (4, 3), (64, 64), 0, 1, 8, True, "fixed:131072",
        description="decode batch 16, 64 query / 8 KV heads (Llama-3.1-70B), context 131072, "
                    "block 16, K and V 3.5-bit (64 channels at 4 bits + 64 at 3 bits, "
                    "independent tables), 128-token bf16 window"),
    "decode_llama8b_2p5bit": Workload(
        "decode_llama8b_2p5bit", "decode", 1005, 256, 32, 8, 128, 32, 128,
        (4, 2), (32, 96), (3,), (128,), 0, 1, 8, True, "loguniform:512:65536", 1.25,
        description="decode batch 256, 32 query / 8 KV heads, context log-uniform [512, 65536], "
                    "block 32, K 2.5-bit (32 channels at 4 bits + 96 at 2 bits), V uniform 3-bit, "
                    "128-token bf16 window, fragmented page pool"),
    "decode_llama8b_3p5bit_qjl": Workload(
        "decode_llama8b_3p5bit_qjl", "decode", 1006, 16, 32, 8, 128, 16, 128,
        (3, 2), (64, 64), (4, 3), (64, 64), 61, 62, 8, True, "fixed:16384", k_qjl=True,
        description="decode batch 16, 32 query / 8 KV heads (Llama-3.1-8B), context 16384, block 16, "
                    "K 2.5-bit MSE (64 channels at 3 bits + 64 at 2) plus the 1-bit QJL residual stage "
                    "(3.5 bits per channel), V 3.5-bit, 128-token bf16 window; QJL keys are scored on the tensor cores "
                    "(sign k-steps)"),
    "decode_llama8b_3p5bit_groupwise": Workload(
        "decode_llama8b_3p5bit_groupwise", "decode", 1007, 16, 32, 8, 128, 16, 128,
        (4, 3), (64, 64), (4, 3), (64, 64), 71, 72, 8, True, "fixed:16384", groupwise=True,
        description="decode batch 16, 32 query / 8 KV heads (Llama-3.1-8B), context 16384, block 16, "
                    "K and V 3.5-bit group-wise: 64 original channels (the outlier channels among them) "
                    "at 4 bits and the other 64 at 3 bits, each group rotated on its own with its own norm, "
                    "128-token bf16 window; group-wise K and V run on the tensor-core kernel "
                    "(query rotated by the dense per-head R_h)"),
    "decode_llama8b_3p5bit_recipe": Workload(
        "decode_llama8b_3p5bit_recipe", "decode", 1010, 16, 32, 8, 128, 16, 128,
        (3, 2), (64, 64), (4, 3), (64, 64), 81, 82, 8, True, "fixed:16384", k_qjl=True, groupwise=True,
        description="decode batch 16, 32 query / 8 KV heads (Llama-3.1-8B), context 16384, block 16, "
                    "K in the recipe row as printed: two group-wise groups (64 original channels, the "
                    "outliers among them, at 3 bits + 64 at 2), each with its QJL signs, norm and residual "
                    "norm (3.5 bits per channel); V 3.5-bit group-wise; 128-token bf16 window; runs on the "
                    "tensor-core decode kernel"),
}


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def codec_specs(w: Workload):
    """(K spec, V spec). High channel sets are seeded, sorted, independent for K and V.

    A group-wise workload stands in for calibration: its high set of original
    channels holds that head's outlier channels plus seeded others.
    """
    rng = _rng(w.seed * 7 + 3)
    specs = []
    for which, (bits, sizes, seed, qjl) in enumerate(((w.k_bits, w.k_sizes, w.k_seed, w.k_qjl),
                                                       (w.v_bits, w.v_sizes, w.v_seed, False))):
        high = None
        if len(bits) == 2 and w.groupwise:
            out = _outlier_channels(w, which)
            rows = []
            for h in range(w.num_kv_heads):
                rest = np.setdiff1d(np.arange(w.head_dim), out[h])
                extra = rng.choice(rest, sizes[0] - len(out[h]), replace=False)
                rows.append(np.sort(np.concatenate([out[h], extra])))
            high = np.stack(rows).astype(np.int16)
        elif len(bits) == 2:
            high = np.stack([np.sort(rng.choice(w.head_dim, sizes[0], replace=False))
                             for _ in range(w.num_kv_heads)]).astype(np.int16)
        specs.append(CodecSpec(tuple(bits), tuple(sizes), seed, high, qjl, w.groupwise))
    return specs[0], specs[1]


def seq_lens(w: Workload) -> np.ndarray:
    rng = _rng(w.seed)
    kind, *args = w.lengths.split(":")
    if kind == "fixed":
        return np.full(w.batch, int(args[0]), dtype=np.int64)
    lo, hi = int(args[0]), int(args[1])
    if kind == "uniform":
        return rng.integers(lo, hi + 1, size=w.batch).astype(np.int64)
    if kind == "loguniform":
        return np.rint(np.exp(rng.uniform(math.log(lo), math.log(hi), size=w.batch))).astype(np.int64)
    raise ValueError(w.lengths)


@dataclass
class PageLayout:
    seq_lens: np.ndarray       # [B] total tokens, window included
    packed_lens: np.ndarray    # [B] tokens held in pages
    block_tables: np.ndarray   # [B][max_blocks] int32 physical block ids (-1 past the end)
    num_blocks: int


def page_layout(w: Workload, lens: Optional[np.ndarray] = None) -> PageLayout:
    """Physical blocks: a seeded permutation of the pool; with slack > 1 a random
    subset of a larger pool is used, so free blocks sit between used ones."""
    lens = seq_lens(w) if lens is None else np.asarray(lens, dtype=np.int64)
    window = w.window if w.kind == "decode" else 0
    packed = lens - np.minimum(window, lens)
    nblk = -(-packed // w.block_size)
    needed = int(nblk.sum())
    pool = max(1, int(math.ceil(w.pool_slack * needed)))
    rng = _rng(w.seed * 7 + 5)
    order = rng.permutation(pool)[:needed]
    max_blocks = max(1, int(nblk.max()) if len(nblk) else 1)
    tables = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(nblk):
        tables[b, :n] = order[pos:pos + n]
        pos += n
    return PageLayout(lens, packed, tables, pool)


def slot_mapping(layout: PageLayout, b: int, t0: int, t1: int, block_size: int) -> np.ndarray:
    """Serving-pattern slots of tokens [t0, t1) of sequence b: block_table * bs + t % bs."""
    t = np.arange(t0, t1)
    return layout.block_tables[b, t // block_size].astype(np.int64) * block_size + t % block_size


def _chunk_generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _outlier_channels(w: Workload, which: int) -> np.ndarray:
    """[H_kv][n_outliers] original channels scaled by 10 (which: 0 = K, 1 = V)."""
    rng = _rng(w.seed * 7 + 11 + which)
    return np.stack([rng.choice(w.head_dim, w.n_outliers, replace=False) for _ in range(w.num_kv_heads)])


def _channel_gain(w: Workload, which: int, device) -> torch.Tensor:
    gain = torch.ones(w.num_kv_heads, w.head_dim, dtype=torch.float32)
    if w.n_outliers:
        ch = _outlier_channels(w, which)
        for h in range(w.num_kv_heads):
            gain[h, torch.as_tensor(ch[h], dtype=torch.long)] = 10.0
    return gain.to(device)


def sequence_kv(w: Workload, b: int, t0: int, t1: int, device="cpu"):
    """bf16 K and V [t1 - t0][H_kv][d] of tokens [t0, t1) of sequence b."""
    H, d = w.num_kv_heads, w.head_dim
    out = []
    for which in (0, 1):
        gain = _channel_gain(w, which, device)
        parts = []
        c0 = t0 // CHUNK
        for c in range(c0, -(-t1 // CHUNK)):
            g = _chunk_generator(device, ((w.seed * 1_000_003 + b) * 4099 + c) * 2 + which)
            x = torch.randn(CHUNK, H, d, generator=g, device=device, dtype=torch.float32)
            if w.token_scales:
                s = torch.rand(CHUNK, H, 1, generator=g, device=device, dtype=torch.float32)
                x = x * torch.exp(math.log(0.5) + s * (math.log(4.0) - math.log(0.5)))
            x = x * gain
            lo = max(t0, c * CHUNK) - c * CHUNK
            hi = min(t1, (c + 1) * CHUNK) - c * CHUNK
            parts.append(x[lo:hi])
        out.append(torch.cat(parts).to(torch.bfloat16) if parts else
                   torch.empty(0, H, d, dtype=torch.bfloat16, device=device))
    return out[0], out[1]


def queries(w: Workload, device="cpu", step: int = 0) -> torch.Tensor:
    g = _chunk_generator(device, w.seed * 31 + 7 + 1000 * step)
    return torch.randn(w.batch, w.num_q_heads, w.head_dim, generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def windows(w: Workload, layout: PageLayout, device="cpu"):
    """bf16 windows [B][H_kv][W][d]: the last min(W, L_b) tokens of each sequence, rest zero."""
    B, H, d, W = len(layout.seq_lens), w.num_kv_heads, w.head_dim, w.window
    kw = torch.zeros(B, H, max(W, 1), d, dtype=torch.bfloat16, device=device)
    vw = torch.zeros_like(kw)
    for b in range(B):
        L, P = int(layout.seq_lens[b]), int(layout.packed_lens[b])
        if L > P:
            k, v = sequence_kv(w, b, P, L, device)
            kw[b, :, :L - P] = k.transpose(0, 1)
            vw[b, :, :L - P] = v.transpose(0, 1)
    return kw, vw


def pack_batch(w: Workload, device="cpu"):
    """Whole pack workload: K, V [T][H][d] sequence-major, and the shuffled slot mapping."""
    layout = page_layout(w)
    ks, vs, slots = [], [], []
    for b in range(len(layout.seq_lens)):
        L = int(layout.seq_lens[b])
        k, v = sequence_kv(w, b, 0, L, device)
        ks.append(k)
        vs.append(v)
        slots.append(slot_mapping(layout, b, 0, L, w.block_size))
    return torch.cat(ks), torch.cat(vs), np.concatenate(slots), layout
