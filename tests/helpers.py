"""Shared test helpers: build both sides' codecs from plain specs, make decode problems."""

import math

import numpy as np
import torch

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq
from quantized_paged_kv_pack_b200 import workloads as W

D = 128


def random_high(H, n, seed):
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(D, n, replace=False)) for _ in range(H)]).astype(np.int16)


def codec_pair(H, bits, sizes, seed, high=None, qjl=False, groupwise=False):
    """(device Codec, oracle Format) for the same plain parameters."""
    if len(bits) == 2 and high is None:
        high = random_high(H, sizes[0], seed + 17)
    return (tq.Codec(H, bits, sizes, high, seed, qjl=qjl, groupwise=groupwise),
            O.Format(D, H, tuple(bits), tuple(sizes), high, seed, qjl=qjl, groupwise=groupwise))


def slice_format(f: O.Format, h: int) -> O.Format:
    """The oracle format of KV head h alone (metadata sliced to one head)."""
    hc = None if f.high_coords is None else np.asarray(f.high_coords)[h:h + 1]
    return O.Format(f.head_dim, 1, f.group_bits, f.group_size, hc, f.seed, qjl=f.qjl, groupwise=f.groupwise)


def random_kv(T, H, gen, scale_outliers=True):
    """bf16 K/V [T][H][128] on the GPU: N(0,1), some channels x10, per-vector scales."""
    k = torch.randn(T, H, D, generator=gen, device="cuda")
    v = torch.randn(T, H, D, generator=gen, device="cuda")
    if scale_outliers:
        k[:, :, :4] *= 10
        v[:, :, 5:9] *= 10
        k *= torch.exp(torch.rand(T, H, 1, generator=gen, device="cuda") * math.log(8) + math.log(0.5))
        v *= torch.exp(torch.rand(T, H, 1, generator=gen, device="cuda") * math.log(8) + math.log(0.5))
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


class DecodeProblem:
    """A paged cache written by the GPU pack kernel, plus queries and windows.

    With ``sinks`` = S > 0 (boundary-token preservation) the first min(S, L)
    tokens of a sequence stay dense too: the dense buffer holds them followed by
    the last ``window`` tokens, the pages hold the tokens in between, and the
    decode call's window is S + window.
    """

    def __init__(self, lens, H, G, kspec, vspec, window, block_size, seed, slack=1.3, sinks=0, kqjl=False,
                 vqjl=False, kgw=False, vgw=False):
        self.lens = np.asarray(lens, dtype=np.int64)
        self.B, self.H, self.G, self.Hq = len(lens), H, G, H * G
        self.sinks = sinks
        window = window + sinks  # dense tokens per sequence (at most)
        self.window, self.bs = window, block_size
        gen = torch.Generator(device="cuda")
        gen.manual_seed(seed)
        rng = np.random.default_rng(seed)
        self.kc, self.kf = codec_pair(H, *kspec, qjl=kqjl, groupwise=kgw)
        self.vc, self.vf = codec_pair(H, *vspec, qjl=vqjl, groupwise=vgw)
        packed = self.lens - np.minimum(window, self.lens)
        nblk = -(-packed // block_size)
        self.num_blocks = max(1, int(math.ceil(slack * nblk.sum())) + 1)
        order = rng.permutation(self.num_blocks)
        self.max_blocks = max(1, int(nblk.max()) if len(nblk) else 1)
        bt = np.full((self.B, self.max_blocks), -1, np.int32)
        pos = 0
        for b in range(self.B):
            bt[b, :nblk[b]] = order[pos:pos + nblk[b]]
            pos += nblk[b]
        self.block_tables_np = bt
        self.k_pages = tq.page_pool(self.kc, self.num_blocks, block_size)
        self.v_pages = tq.page_pool(self.vc, self.num_blocks, block_size)
        Wn = max(window, 1)
        self.k_win = torch.zeros(self.B, H, Wn, D, dtype=torch.bfloat16, device="cuda")
        self.v_win = torch.zeros_like(self.k_win)
        self.kv = []  # the original tokens, in order (for order-independent checks)
        for b in range(self.B):
            L, P = int(self.lens[b]), int(packed[b])
            k, v = random_kv(L, H, gen)
            self.kv.append((k, v))
            s0 = min(sinks, L)  # packed tokens are s0 .. s0 + P - 1
            if P:
                t = np.arange(P)
                slots = torch.as_tensor(bt[b, t // block_size].astype(np.int64) * block_size + t % block_size,
                                        device="cuda")
                tq.pack_kv(self.kc, self.vc, k[s0:s0 + P].contiguous(), v[s0:s0 + P].contiguous(), slots,
                           self.k_pages, self.v_pages, block_size)
            if L > P:
                dense = torch.cat((torch.arange(0, s0), torch.arange(s0 + P, L))).to(k.device)
                self.k_win[b, :, :L - P] = k[dense].transpose(0, 1)
                self.v_win[b, :, :L - P] = v[dense].transpose(0, 1)
        self.q = torch.randn(self.B, self.Hq, D, generator=gen, device="cuda").to(torch.bfloat16)
        self.block_tables = torch.as_tensor(bt, device="cuda")
        self.seq_lens = torch.as_tensor(self.lens.astype(np.int32), device="cuda")
        self.max_seq_len = int(self.lens.max()) if self.B else 0
        self.scale = 1.0 / math.sqrt(D)

    def run(self, **kw):
        return tq.decode_paged(self.kc, self.vc, self.q, self.k_pages, self.v_pages, self.bs, self.block_tables,
                               self.seq_lens, self.max_seq_len, self.k_win if self.window else None,
                               self.v_win if self.window else None, self.window, self.scale, **kw)

    def oracle(self, b, hq):
        """fp64 oracle output of (sequence b, query head hq) over the GPU-written pages."""
        h = hq // self.G
        L = int(self.lens[b])
        P = L - min(self.window, L)
        nblk = -(-P // self.bs)
        blocks = torch.as_tensor(self.block_tables_np[b, :nblk].astype(np.int64), device="cuda")
        if nblk:
            kp = self.k_pages[blocks][:, h:h + 1].cpu().numpy()
            vp = self.v_pages[blocks][:, h:h + 1].cpu().numpy()
        else:
            kp = np.zeros((1, 1, self.bs * self.kc.row_bytes), np.uint8)
            vp = np.zeros((1, 1, self.bs * self.vc.row_bytes), np.uint8)
        table = np.arange(max(nblk, 1))[None]
        q = self.q[b:b + 1, hq:hq + 1].float().cpu().numpy().astype(np.float64)
        kw = self.k_win[b:b + 1, h:h + 1].float().cpu().numpy().astype(np.float64)
        vw = self.v_win[b:b + 1, h:h + 1].float().cpu().numpy().astype(np.float64)
        return O.decode_attention(q, kp, vp, table, [L], kw, vw, self.window, self.scale,
                                  slice_format(self.kf, h), slice_format(self.vf, h), self.bs)[0, 0]


def workload_codecs(w):
    """(device K codec, device V codec, oracle K format, oracle V format) of a named workload."""
    ks, vs = W.codec_specs(w)
    kc = tq.Codec(w.num_kv_heads, ks.group_bits, ks.group_size, ks.high_coords, ks.seed, qjl=ks.qjl,
                  groupwise=ks.groupwise)
    vc = tq.Codec(w.num_kv_heads, vs.group_bits, vs.group_size, vs.high_coords, vs.seed, qjl=vs.qjl,
                  groupwise=vs.groupwise)
    kf = O.Format(D, w.num_kv_heads, ks.group_bits, ks.group_size, ks.high_coords, ks.seed, qjl=ks.qjl,
                  groupwise=ks.groupwise)
    vf = O.Format(D, w.num_kv_heads, vs.group_bits, vs.group_size, vs.high_coords, vs.seed, qjl=vs.qjl,
                  groupwise=vs.groupwise)
    return kc, vc, kf, vf


QJL_BOUNDARY_REL = 1e-5  # near-boundary exemption for index mismatches
SIGN_REL = 1e-4  # a sign may differ only where |(S r)_i| is this small against |r| sqrt(d)


def check_qjl_rows(rows, x, fmt, heads):
    """GPU rows [N][H][row] against the oracle's QJL quantization of x [N][H][d]."""
    compared = 0
    for h in heads:
        f1 = slice_format(fmt, h)
        idx, n16, u, signs, g16 = O.quantize_qjl(x[:, h], f1, 0)
        gidx, gn16, gsigns, gg16 = O.decode_rows(rows[:, h], f1)
        assert np.array_equal(gn16.astype(np.float16).view(np.uint16), n16.astype(np.float16).view(np.uint16))
        bad = np.any(gidx != idx, axis=-1)  # vectors with an index flip at a boundary
        if bad.any():
            margin = O.boundary_margin(u, f1)
            flips = gidx != idx
            assert np.all(margin[flips] <= QJL_BOUNDARY_REL), "index mismatch away from a codebook boundary"
        ok = ~bad
        # residual norms: fp16 of |r|, equal unless |r| sits at an fp16 rounding midpoint
        gd = gg16[ok] != g16[ok]
        if gd.any():
            rel = np.abs(gg16[ok][gd] - g16[ok][gd]) / np.maximum(g16[ok][gd], 1e-30)
            assert np.all(rel < 2e-3), "residual norm differs by more than one fp16 step"
            assert gd.sum() <= max(2, 0.002 * ok.sum())
        # signs: equal except where the projection is negligibly small
        r = np.empty(u.shape)
        perm = O.permutation(f1, 0)
        start = 0
        chat = np.empty(u.shape)
        for b, size in zip(f1.group_bits, f1.group_size):
            cb, _ = O.codebook(b, D)
            chat[:, start:start + size] = cb[idx[:, start:start + size]]
            start += size
        r[:, perm] = u - chat
        proj = r @ O.qjl_matrix(f1).T
        scale = np.linalg.norm(r, axis=-1, keepdims=True) * math.sqrt(D)
        diff = (gsigns != signs) & ok[:, None]
        assert np.all(np.abs(proj[diff]) <= SIGN_REL * np.broadcast_to(scale, proj.shape)[diff]), \
            "QJL sign mismatch away from zero"
        compared += int(ok.sum())
    return compared


RECIPE_SIGN_REL = 1e-4  # a sign may differ only where |(S_g r_g)_i| is this small against |r_g| sqrt(n_g)


def check_recipe_rows(rows, x, fmt, heads):
    """GPU rows [N][H][row] against the oracle's recipe quantization of x [N][H][d]."""
    compared = 0
    for h in heads:
        f1 = slice_format(fmt, h)
        idx, n16, u, signs, g16 = O.quantize_qjl(x[:, h], f1, 0)
        gidx, gn16, gsigns, gg16 = O.decode_rows(rows[:, h], f1)
        assert np.array_equal(gn16.astype(np.float16).view(np.uint16), n16.astype(np.float16).view(np.uint16))
        flips = gidx != idx
        if flips.any():
            margin = O.boundary_margin(u, f1)
            assert np.all(margin[flips] <= QJL_BOUNDARY_REL), "index mismatch away from a codebook boundary"
        ok = ~np.any(flips, axis=-1)
        gd = gg16[ok] != g16[ok]
        if gd.any():
            rel = np.abs(gg16[ok][gd] - g16[ok][gd]) / np.maximum(g16[ok][gd], 1e-30)
            assert np.all(rel < 2e-3), "residual norm differs by more than one fp16 step"
            assert gd.sum() <= max(2, 0.002 * gd.size)
        start = 0
        for g, (b, n) in enumerate(zip(f1.group_bits, f1.group_size)):
            c, _ = O.codebook(b, n)
            r = u[:, start:start + n] - c[idx[:, start:start + n]]
            proj = r @ O.recipe_qjl_matrix(f1, g).T
            scale = np.linalg.norm(r, axis=-1, keepdims=True) * math.sqrt(n)
            diff = (gsigns[:, start:start + n] != signs[:, start:start + n]) & ok[:, None]
            assert np.all(np.abs(proj[diff]) <= RECIPE_SIGN_REL * np.broadcast_to(scale, proj.shape)[diff]), \
                "QJL sign mismatch away from zero"
            start += n
        compared += int(ok.sum())
    return compared
