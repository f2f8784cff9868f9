"""Pins of the CPU oracle to facts outside itself (runs without a GPU).

Each test checks the oracle against something it does not compute the same
way: a value the pages print, a published table, a closed form, a library
routine, an invariant, or brute force on tiny inputs.
"""

import json
import math
import os
import struct
from fractions import Fraction

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
from scipy.special import gamma

from oracle import tq_oracle as O

D = 128


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def fmt(bits, sizes, H=1, seed=0, d=D, rng=None):
    high = None
    if len(bits) == 2:
        rng = rng or np.random.default_rng(5)
        high = np.stack([np.sort(rng.choice(d, sizes[0], replace=False)) for _ in range(H)])
    return O.Format(d, H, tuple(bits), tuple(sizes), high, seed)


FORMATS = {
    "4u": ((4,), (128,)),
    "3p5": ((4, 3), (64, 64)),
    "2p5k": ((4, 2), (32, 96)),
    "3u": ((3,), (128,)),
    "2u": ((2,), (128,)),
}


# --- rotation ---------------------------------------------------------------

@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128])
def test_hadamard_matches_library_and_is_orthogonal(d):
    H = O.hadamard_matrix(d)
    assert np.array_equal(H, scipy.linalg.hadamard(d).astype(float))
    assert np.array_equal(H @ H.T, d * np.eye(d))
    assert np.array_equal(H, H.T)
    K = np.array([[1.0]])
    while K.shape[0] < d:  # Sylvester recursion H_2n = [[H, H], [H, -H]]
        K = np.kron(np.array([[1.0, 1.0], [1.0, -1.0]]), K)
    assert np.array_equal(H, K)


def test_rotation_orthonormal_and_self_inverse():
    rng = np.random.default_rng(0)
    s = O.hadamard_signs(7, D)
    R = O.rotate(np.eye(D), s)  # row i = R e_i, so R here is the transpose of the map
    assert np.allclose(R @ R.T, np.eye(D), atol=1e-14)
    x = rng.standard_normal((50, D))
    y = O.rotate(x, s)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    assert np.allclose(O.unrotate(y, s), x, atol=1e-13)
    # rotating twice without signs is the identity up to scale 1 (H/sqrt(d) is an involution)
    ones = np.ones(D)
    assert np.allclose(O.rotate(O.rotate(x, ones), ones), x, atol=1e-13)


def test_splitmix64_reference_outputs(golden_dir):
    g = _golden(golden_dir, "splitmix64_seed0.json")
    got = O.splitmix64(g["seed"], len(g["outputs_hex"]))
    assert [f"{z:016x}" for z in got] == g["outputs_hex"]
    s = O.hadamard_signs(0, 3)
    assert list(s) == [-1.0 if int(h, 16) & 1 else 1.0 for h in g["outputs_hex"]]


# --- coordinate density and codebooks ----------------------------------------

@pytest.mark.parametrize("d", [3, 8, 128])
def test_density_mass_and_moments_match_quadrature(d):
    C = O.coord_density_const(d)
    f = lambda x: C * (1 - x * x) ** ((d - 3) / 2)  # noqa: E731
    for a, b in [(-1, 1), (-0.3, 0.05), (0.02, 0.2), (-0.9, -0.1), (0.2, 1.0)]:
        m, _ = scipy.integrate.quad(f, a, b, epsabs=1e-15, epsrel=1e-13, limit=200)
        m1, _ = scipy.integrate.quad(lambda x: x * f(x), a, b, epsabs=1e-15, epsrel=1e-13, limit=200)
        m2, _ = scipy.integrate.quad(lambda x: x * x * f(x), a, b, epsabs=1e-15, epsrel=1e-13, limit=200)
        assert O.cell_mass(a, b, d) == pytest.approx(m, rel=1e-11, abs=1e-15)
        assert O.cell_first_moment(a, b, d) == pytest.approx(m1, rel=1e-11, abs=1e-15)
        assert O.cell_second_moment(a, b, d) == pytest.approx(m2, rel=1e-11, abs=1e-15)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_d3_is_uniform_quantizer(bits):
    # A coordinate of a uniform point on S^2 is uniform on [-1, 1] (Archimedes),
    # whose Lloyd-Max quantizer is the uniform one.
    L = 1 << bits
    c = O.lloyd_max(bits, 3)
    assert np.allclose(c, -1 + (2 * np.arange(L) + 1) / L, atol=1e-12)


@pytest.mark.parametrize("d", [16, 128, 1000])
def test_codebook_one_bit_closed_form(d):
    c = O.lloyd_max(1, d)
    e_abs = gamma(d / 2) / (math.sqrt(math.pi) * gamma((d + 1) / 2)) if d < 300 else \
        math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    assert np.allclose(c, [-e_abs, e_abs], rtol=1e-13)


def test_codebook_large_d_tends_to_gaussian_table(golden_dir):
    # sqrt(d) X -> N(0, 1): the codebook tends to Max's Gaussian quantizer.
    g = _golden(golden_dir, "gaussian_lloyd_max.json")["levels"]
    d = 1 << 16
    for bits in (1, 2, 3, 4):
        ref = g[str(1 << bits)]
        c = O.lloyd_max(bits, d, tol=1e-11) * math.sqrt(d)  # betainc noise floor is higher at d = 2^16
        pos = c[len(c) // 2:]
        assert np.allclose(pos, ref["outputs"], rtol=1.5e-3, atol=6e-4)
        edges = np.concatenate(([-1.0], 0.5 * (c[:-1] + c[1:]) / math.sqrt(d), [1.0]))
        cu = c / math.sqrt(d)
        dist = (O.cell_second_moment(edges[:-1], edges[1:], d) - 2 * cu * O.cell_first_moment(edges[:-1], edges[1:], d)
                + cu * cu * O.cell_mass(edges[:-1], edges[1:], d)).sum() * d
        assert dist == pytest.approx(ref["mse"], rel=2e-3)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_optimality_conditions_d128(bits):
    c = O.lloyd_max(bits, D)
    assert np.allclose(c, -c[::-1], atol=0)
    edges = np.concatenate(([-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]))
    C = O.coord_density_const(D)
    for i in range(len(c)):
        a, b = edges[i], edges[i + 1]
        num, _ = scipy.integrate.quad(lambda x: x * C * (1 - x * x) ** 62.5, a, b, epsabs=1e-17, epsrel=1e-14)
        den, _ = scipy.integrate.quad(lambda x: C * (1 - x * x) ** 62.5, a, b, epsabs=1e-17, epsrel=1e-14)
        assert c[i] == pytest.approx(num / den, rel=1e-11, abs=1e-14)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_fp16_codebook_and_fp32_boundaries(bits):
    c, beta = O.codebook(bits, D)
    assert np.array_equal(c.astype(np.float16).astype(np.float64), c)
    assert np.array_equal(beta, 0.5 * (c[:-1] + c[1:]))
    assert np.array_equal(beta.astype(np.float32).astype(np.float64), beta)
    assert np.all(np.diff(beta) > 0)
    assert np.max(np.abs(c - O.lloyd_max(bits, D))) <= 2.0 ** -11 * np.max(np.abs(c))


# --- quantizer -----------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_boundary_count_equals_nearest_centroid(bits):
    c, beta = O.codebook(bits, D)
    rng = np.random.default_rng(bits)
    u = np.concatenate((rng.uniform(-0.4, 0.4, 4000), beta, np.nextafter(beta, 1), np.nextafter(beta, -1)))
    idx = np.searchsorted(beta, u, side="left")
    cf = [Fraction(float(ci)) for ci in c]
    for x, i in zip(u, idx):
        xf = Fraction(float(x))
        dist = [abs(xf - ci) for ci in cf]  # exact rational distances
        best = min(range(len(c)), key=lambda k: (dist[k], k))  # ties to the lower index
        assert i == best


def test_product_codeword_bruteforce_d4():
    d, bits = 4, 2
    f = O.Format(d, 1, (bits,), (d,), None, 3)
    c, _ = O.codebook(bits, d)
    grid = np.array(np.meshgrid(*[np.arange(4)] * d, indexing="ij")).reshape(d, -1).T  # 4^4 codewords
    words = c[grid]
    rng = np.random.default_rng(1)
    x = rng.standard_normal((300, d))
    idx, _, u = O.quantize(x, f, 0)
    for k in range(len(x)):
        best = np.argmin(((words - u[k]) ** 2).sum(axis=1))
        assert np.array_equal(grid[best], idx[k])


def test_norm_is_fp16_round_half_even_of_exact_norm():
    rng = np.random.default_rng(2)
    x = O.bf16_round(rng.standard_normal((400, D)) * rng.uniform(0.1, 50, (400, 1))).astype(np.float64)
    f = fmt((4,), (128,))
    _, n16, _ = O.quantize(x, f, 0)
    for k in range(len(x)):
        exact = math.sqrt(math.fsum(v * v for v in x[k]))
        ref = struct.unpack("<e", struct.pack("<e", exact))[0]  # Python's IEEE half, RNE
        assert n16[k] == ref


def test_zero_vector_row():
    f = fmt((4,), (128,))
    idx, n16, u = O.quantize(np.zeros((1, D)), f, 0)
    assert n16[0] == 0.0 and np.all(u == 0) and np.all(idx == 7)
    assert np.all(O.dequantize_rows(idx, n16, f, 0) == 0)


# --- row format ---------------------------------------------------------------------

@pytest.mark.parametrize("name,expected", [("4u", 66), ("3p5", 58), ("2p5k", 42), ("3u", 50), ("2u", 34)])
def test_row_bytes(name, expected):
    bits, sizes = FORMATS[name]
    assert O.row_bytes(fmt(bits, sizes)) == expected


@pytest.mark.parametrize("name", list(FORMATS))
def test_pack_roundtrip_exhaustive(name):
    bits, sizes = FORMATS[name]
    f = fmt(bits, sizes)
    pb = O.position_bits(f)
    L = 1 << int(pb.max())
    idx = (np.arange(D)[None, :] + np.arange(L)[:, None]) % (1 << pb)[None, :]  # every value at every position
    n16 = O.fp16_round(np.linspace(0, 300, L))
    rows = O.encode_rows(idx, n16, f)
    assert rows.shape == (L, O.row_bytes(f))
    back, nb = O.decode_rows(rows, f)
    assert np.array_equal(back, idx) and np.array_equal(nb, n16)


def test_row_bit_layout_golden(golden_dir):
    for case in _golden(golden_dir, "row_bit_layout.json")["cases"]:
        d = sum(case["group_size"])
        high = np.arange(case["group_size"][0])[None, :] if len(case["group_bits"]) == 2 else None
        qjl, gw = case.get("qjl", False), case.get("groupwise", False)
        f = O.Format(d, 1, tuple(case["group_bits"]), tuple(case["group_size"]), high, 0, qjl=qjl, groupwise=gw)
        idx = np.array([case["indices"]])
        if gw:
            row = O.encode_rows(idx, np.array([case["norms"]]), f)[0]
        elif qjl:
            row = O.encode_rows(idx, np.array([case["norm"]]), f, signs=np.array([case["signs"]]),
                                g16=np.array([case["residual_norm"]]))[0]
        else:
            row = O.encode_rows(idx, np.array([case["norm"]]), f)[0]
        assert len(row) == O.row_bytes(f)
        assert bytes(row).hex() == case["row_hex"]
        back = O.decode_rows(row[None], f)
        assert np.array_equal(back[0][0], case["indices"])


def test_permutation_puts_high_coords_first():
    f = fmt((4, 3), (64, 64), H=3)
    for h in range(3):
        p = O.permutation(f, h)
        assert sorted(p) == list(range(D))
        assert list(p[:64]) == sorted(f.high_coords[h]) and list(p[64:]) == sorted(set(range(D)) - set(p[:64]))


# --- reconstruction invariant -------------------------------------------------

@pytest.mark.parametrize("name", ["4u", "3p5", "2p5k", "3u"])
def test_reconstruction_error_matches_codebook_distortion(name):
    bits, sizes = FORMATS[name]
    f = fmt(bits, sizes)
    expected = 0.0
    for b, n in zip(bits, sizes):
        c, beta = O.codebook(b, D)
        e = np.concatenate(([-1.0], beta, [1.0]))
        per = (O.cell_second_moment(e[:-1], e[1:], D) - 2 * c * O.cell_first_moment(e[:-1], e[1:], D)
               + c * c * O.cell_mass(e[:-1], e[1:], D)).sum()
        expected += n * per
    rng = np.random.default_rng(11)
    x = rng.standard_normal((20000, D))
    idx, _, u = O.quantize(x, f, 0)
    chat = np.empty_like(u)
    start = 0
    for b, n in zip(bits, sizes):
        c, _ = O.codebook(b, D)
        chat[:, start:start + n] = c[idx[:, start:start + n]]
        start += n
    err = ((u - chat) ** 2).sum(axis=1)
    sigma = err.std() / math.sqrt(len(err))
    assert abs(err.mean() - expected) < 4 * sigma
    # reconstruction through rows and the inverse rotation gives the same error up to the fp16 norm
    xr = O.dequantize_rows(idx[:200], np.linalg.norm(x[:200], axis=1), f, 0)
    n = np.linalg.norm(x[:200], axis=1)
    assert np.allclose(((xr - x[:200]) ** 2).sum(axis=1) / n ** 2, err[:200], rtol=1e-9, atol=1e-13)


# --- pages, addressing --------------------------------------------------------

def _hand_row(pages, blk, head, off, ib, bs):
    """Row bytes read by hand from a (block, head) sub-page: index bytes, then the norm."""
    sub = bytes(pages[blk, head])
    return sub[off * ib:(off + 1) * ib] + sub[bs * ib + 2 * off: bs * ib + 2 * off + 2]


def test_pack_addressing_by_formula():
    rng = np.random.default_rng(4)
    H, bs, nb, T = 2, 4, 6, 17
    kf, vf = fmt((4,), (128,), H=H, seed=0), fmt((4, 3), (64, 64), H=H, seed=1)
    k = O.bf16_round(rng.standard_normal((T, H, D))).astype(np.float64)
    v = O.bf16_round(rng.standard_normal((T, H, D))).astype(np.float64)
    slots = rng.permutation(nb * bs)[:T]
    slots[3] = -1
    kp, vp = O.pack_kv(k, v, slots, kf, vf, nb, bs)
    for t in range(T):
        for h in range(H):
            if slots[t] < 0:
                continue
            ki, kn, _ = O.quantize(k[t, h][None], kf, h)
            vi, vn, _ = O.quantize(v[t, h][None], vf, h)
            assert np.array_equal(O.read_row(kp, slots[t], h, bs, kf), O.encode_rows(ki, kn, kf)[0])
            assert np.array_equal(O.read_row(vp, slots[t], h, bs, vf), O.encode_rows(vi, vn, vf)[0])
            # the same bytes, located by hand: index bytes at off*ib, the norm at bs*ib + 2*off
            blk, off = divmod(int(slots[t]), bs)
            row = _hand_row(kp, blk, h, off, O.index_bytes(kf), bs)
            assert row == bytes(O.encode_rows(ki, kn, kf)[0])
    written = {(s // bs, s % bs) for s in slots if s >= 0}
    for blk in range(nb):
        for off in range(bs):
            if (blk, off) not in written:
                for h in range(H):
                    assert not any(_hand_row(kp, blk, h, off, O.index_bytes(kf), bs))
    with pytest.raises(IndexError):
        O.pack_kv(k, v, np.full(T, nb * bs), kf, vf, nb, bs)


# --- attention ---------------------------------------------------------------

def _pages_for(seq_keys, seq_vals, kf, vf, bs, rng):
    """Pack one sequence's tokens into a permuted block pool."""
    P = len(seq_keys)
    nblk = max(1, -(-P // bs))
    table = rng.permutation(nblk + 2)[:nblk]
    slots = table[np.arange(P) // bs] * bs + np.arange(P) % bs
    kp, vp = O.pack_kv(seq_keys, seq_vals, slots, kf, vf, nblk + 2, bs)
    return kp, vp, table


def test_attention_single_token_returns_its_value():
    rng = np.random.default_rng(6)
    kf, vf = fmt((4,), (128,)), fmt((3,), (128,), seed=1)
    k = O.bf16_round(rng.standard_normal((1, 1, D))).astype(np.float64)
    v = O.bf16_round(rng.standard_normal((1, 1, D))).astype(np.float64)
    kp, vp, table = _pages_for(k, v, kf, vf, 16, rng)
    q = rng.standard_normal((1, 4, D))
    out = O.decode_attention(q, kp, vp, table[None], [1], None, None, 0, 0.1, kf, vf, 16)
    vi, vn = O.decode_rows(O.read_rows(vp, [table[0]], 0, [0], vf, 16), vf)
    vhat = O.dequantize_rows(vi, vn, vf, 0)[0]
    for g in range(4):
        assert np.allclose(out[0, g], vhat, atol=1e-13)


def test_attention_identical_keys_average_values():
    rng = np.random.default_rng(7)
    kf, vf = fmt((4,), (128,)), fmt((4,), (128,), seed=1)
    P = 37
    k = np.repeat(O.bf16_round(rng.standard_normal((1, 1, D))).astype(np.float64), P, axis=0)
    v = O.bf16_round(rng.standard_normal((P, 1, D))).astype(np.float64)
    kp, vp, table = _pages_for(k, v, kf, vf, 8, rng)
    q = rng.standard_normal((1, 2, D))
    out = O.decode_attention(q, kp, vp, table[None], [P], None, None, 0, 0.3, kf, vf, 8)
    vi, vn, _ = O.quantize(v[:, 0], vf, 0)
    mean = O.dequantize_rows(vi, vn, vf, 0).mean(axis=0)
    assert np.allclose(out[0, 0], mean, atol=1e-12) and np.allclose(out[0, 1], mean, atol=1e-12)


def test_attention_window_only_is_dense_softmax_by_hand():
    rng = np.random.default_rng(8)
    kf, vf = fmt((4,), (128,)), fmt((4,), (128,))
    W, L, d = 5, 3, D
    kw = np.zeros((1, 1, W, d))
    vw = np.zeros((1, 1, W, d))
    kw[0, 0, :L] = rng.standard_normal((L, d))
    vw[0, 0, :L] = rng.standard_normal((L, d))
    q = rng.standard_normal((1, 1, d))
    pages = np.zeros((1, 1, 4 * O.row_bytes(kf)), dtype=np.uint8)
    out = O.decode_attention(q, pages, pages, np.zeros((1, 1), np.int64), [L], kw, vw, W, 0.2, kf, vf, 4)
    s = [0.2 * sum(q[0, 0, j] * kw[0, 0, t, j] for j in range(d)) for t in range(L)]
    m = max(s)
    w = [math.exp(x - m) for x in s]
    ref = [sum(w[t] * vw[0, 0, t, j] for t in range(L)) / sum(w) for j in range(d)]
    assert np.allclose(out[0, 0], ref, atol=1e-12)


def test_sixteen_bit_codebook_reproduces_dense_attention():
    rng = np.random.default_rng(9)
    f16 = O.Format(D, 1, (16,), (D,), None, 5)
    P = 64
    k = rng.standard_normal((P, D)) * 3
    v = rng.standard_normal((P, D)) * 3
    q = rng.standard_normal(D)
    ki, kn, _ = O.quantize(k, f16, 0)
    vi, vn, _ = O.quantize(v, f16, 0)
    kh, vh = O.dequantize_rows(ki, kn, f16, 0), O.dequantize_rows(vi, vn, f16, 0)
    scale = 1 / math.sqrt(D)
    ref = O.dense_attention(q, k, v, scale)
    got = O.dense_attention(q, kh, vh, scale)
    # Perturbation bound: |d out| <= max_t |dv_t| + 2 max|v| max_t |d s_t|.
    dv = np.abs(vh - v).max()
    ds = scale * np.abs((kh - k) @ q).max()
    bound = dv + 2 * np.abs(v).max() * ds
    err = np.abs(got - ref).max()
    assert err <= bound
    assert err < 5e-5 * np.abs(v).max()
    # the same comparison with the 4-bit codebook is three orders of magnitude worse
    f4 = O.Format(D, 1, (4,), (D,), None, 5)
    k4 = O.dequantize_rows(*O.quantize(k, f4, 0)[:2], f4, 0)
    v4 = O.dequantize_rows(*O.quantize(v, f4, 0)[:2], f4, 0)
    assert np.abs(O.dense_attention(q, k4, v4, scale) - ref).max() > 1000 * err


def _bruteforce_row_decode(row, bits, sizes, perm):
    """Read a row bit by bit (pure Python) into (rotated-order indices, norm)."""
    idx = [0] * sum(sizes)
    bitpos = 0
    p = 0
    for b, n in zip(bits, sizes):
        for _ in range(n):
            val = 0
            for k in range(b):
                byte, bit = divmod(bitpos, 8)
                val |= ((int(row[byte]) >> bit) & 1) << k
                bitpos += 1
            idx[perm[p]] = val
            p += 1
    norm = struct.unpack("<e", bytes(row[bitpos // 8: bitpos // 8 + 2]))[0]
    return idx, norm


def test_attention_bruteforce_tiny():
    rng = np.random.default_rng(10)
    d, H, G, bs, W = 8, 2, 2, 2, 2
    high = np.stack([np.sort(rng.choice(d, 4, replace=False)) for _ in range(H)])
    kf = O.Format(d, H, (4, 2), (4, 4), high, 3)
    vf = O.Format(d, H, (3,), (d,), None, 9)
    lens = [3, 5]
    B = len(lens)
    maxb = 2
    tables = np.array([[4, 1], [0, 3]])
    nb = 5
    kp = np.zeros((nb, H, bs * O.row_bytes(kf)), np.uint8)
    vp = np.zeros((nb, H, bs * O.row_bytes(vf)), np.uint8)
    kw = np.zeros((B, H, W, d))
    vw = np.zeros((B, H, W, d))
    hist_k, hist_v = {}, {}
    for b, L in enumerate(lens):
        P = L - min(W, L)
        kk = O.bf16_round(rng.standard_normal((L, H, d)) * 2).astype(np.float64)
        vv = O.bf16_round(rng.standard_normal((L, H, d)) * 2).astype(np.float64)
        slots = tables[b, np.arange(P) // bs] * bs + np.arange(P) % bs
        O.pack_kv(kk[:P], vv[:P], slots, kf, vf, nb, bs, kp, vp)
        kw[b, :, :L - P] = kk[P:].transpose(1, 0, 2)
        vw[b, :, :L - P] = vv[P:].transpose(1, 0, 2)
        hist_k[b], hist_v[b] = kk, vv
    q = rng.standard_normal((B, H * G, d))
    out = O.decode_attention(q, kp, vp, tables, lens, kw, vw, W, 0.7, kf, vf, bs)

    def hand_dequant(row, f, h):
        perm = list(O.permutation(f, h))
        idx, norm = _bruteforce_row_decode(row, f.group_bits, f.group_size, perm)
        bits_of = {}
        p = 0
        for b_, n_ in zip(f.group_bits, f.group_size):
            for _ in range(n_):
                bits_of[perm[p]] = b_
                p += 1
        cent = [O.codebook(bits_of[j], d)[0][idx[j]] for j in range(d)]
        z = O.splitmix64(f.seed, d)
        s = [-1.0 if zz & 1 else 1.0 for zz in z]
        return [norm * s[i] * sum((-1) ** bin(i & j).count("1") * cent[j] for j in range(d)) / math.sqrt(d)
                for i in range(d)]

    for b, L in enumerate(lens):
        P = L - min(W, L)
        for hq in range(H * G):
            h = hq // G
            keys, vals = [], []
            for t in range(P):
                blk, off = tables[b][t // bs], t % bs
                keys.append(hand_dequant(_hand_row(kp, blk, h, off, O.index_bytes(kf), bs), kf, h))
                vals.append(hand_dequant(_hand_row(vp, blk, h, off, O.index_bytes(vf), bs), vf, h))
            for t in range(L - P):
                keys.append(list(kw[b, h, t]))
                vals.append(list(vw[b, h, t]))
            s = [0.7 * sum(q[b, hq, j] * kk[j] for j in range(d)) for kk in keys]
            m = max(s)
            w = [math.exp(x - m) for x in s]
            ref = [sum(w[t] * vals[t][j] for t in range(L)) / sum(w) for j in range(d)]
            assert np.allclose(out[b, hq], ref, atol=1e-12)


# --- byte ledger --------------------------------------------------------------

def test_ledger_ratios_match_server_page(golden_dir):
    g = _golden(golden_dir, "server_page_table.json")
    tol = g["printed_precision"]
    for key, (bits, sizes) in (("tq35", ((4, 3), (64, 64))), ("tq25", ((4, 2), (32, 96)))):
        f = fmt(bits, sizes, H=8)
        assert f.mean_bits == g["bits_per_channel"][key]
        led = O.byte_ledger(f, f, [4096] * 4, 0, 16, 1024)
        ratio = led.dense_bytes / led.index_bytes  # index-only ratio, as the page reports
        assert abs(ratio - g["compression_ratio"][key]) <= tol["compression_ratio"]
        equiv = g["equivalent_context_tokens_80gb_a100"]["full"] * ratio
        assert equiv == pytest.approx(g["equivalent_context_tokens_80gb_a100"][key], rel=tol["equivalent_context_relative"])
    # with the 2-byte norm included, per-row ratios are 256/66, 256/58, 256/42, 256/50
    for (bits, sizes), rb in (((4,), (128,)), 66), (((4, 3), (64, 64)), 58), (((4, 2), (32, 96)), 42), (((3,), (128,)), 50):
        f = fmt(bits, sizes, H=8)
        led = O.byte_ledger(f, f, [100], 0, 16, 7)
        assert led.dense_bytes / (led.index_bytes + led.norm_bytes) == pytest.approx(256 / rb)


def test_ledger_counts_what_the_oracle_allocates():
    rng = np.random.default_rng(12)
    H, bs, W = 2, 4, 3
    kf, vf = fmt((4, 3), (64, 64), H=H), fmt((3,), (128,), H=H, seed=2)
    lens = [2, 9, 13]
    packed = [L - min(W, L) for L in lens]
    nblk = [-(-p // bs) for p in packed]
    nb = sum(nblk) + 1
    led = O.byte_ledger(kf, vf, lens, W, bs, nb, workspace_bytes=123)
    k = O.bf16_round(rng.standard_normal((sum(packed), H, D))).astype(np.float64)
    kp, vp = O.pack_kv(k, k, np.arange(sum(packed)), kf, vf, nb, bs)
    assert led.page_pool_bytes == kp.nbytes + vp.nbytes
    assert led.index_bytes + led.norm_bytes == sum(packed) * H * (O.row_bytes(kf) + O.row_bytes(vf))
    assert led.window_bytes == 2 * np.zeros((len(lens), H, W, D), np.float16).nbytes
    assert led.block_table_bytes == np.zeros(sum(nblk), np.int32).nbytes
    cb = sum(O.codebook(b, D)[0].astype(np.float16).nbytes + O.codebook(b, D)[1].astype(np.float32).nbytes
             for f in (kf, vf) for b in f.group_bits)
    assert led.codebook_bytes == cb
    assert led.dense_bytes == 2 * np.zeros((sum(lens), H, D), np.float16).nbytes
    assert led.workspace_bytes == 123
    assert led.metadata_bytes == led.norm_bytes + led.codebook_bytes + led.transform_bytes + led.window_bytes \
        + led.block_table_bytes + 123


def test_attention_empty_history_is_zero():
    kf, vf = fmt((4,), (128,)), fmt((4,), (128,))
    pages = np.zeros((1, 1, 4 * O.row_bytes(kf)), dtype=np.uint8)
    q = np.ones((2, 2, D))
    win = np.ones((2, 1, 3, D))
    out = O.decode_attention(q, pages, pages, np.zeros((2, 1), np.int64), [0, 1], win, win, 3, 0.1, kf, vf, 4)
    assert np.all(out[0] == 0) and np.allclose(out[1], 1.0)


def test_boundary_dense_tokens_counts():
    """First S and last W tokens dense, the middle packed; short sequences are all dense."""
    for L in range(0, 30):
        for S in (0, 1, 4):
            for W in (0, 3, 8):
                dense, s0, P = O.boundary_dense_tokens(L, S, W)
                assert s0 == min(S, L) and P == max(0, L - S - W)
                packed = list(range(s0, s0 + P))
                assert sorted(dense + packed) == list(range(L))  # a partition of the tokens
                assert dense[:s0] == list(range(s0))             # the sinks lead the dense buffer
                assert all(t >= s0 + P for t in dense[s0:])      # then the most recent tokens


def test_boundary_tokens_as_window_equal_attention_in_token_order():
    """Sinks and recent tokens passed as one window give attention over the original token order."""
    rng = np.random.default_rng(44)
    d, H, G, bs = 16, 2, 2, 4
    kf = O.Format(d, H, (4,), (d,), None, 5)
    vf = O.Format(d, H, (3,), (d,), None, 6)
    S, W = 3, 5
    lens = [2, 7, 30]
    B = len(lens)
    nb = 16
    kp = np.zeros((nb, H, bs * O.row_bytes(kf)), np.uint8)
    vp = np.zeros((nb, H, bs * O.row_bytes(vf)), np.uint8)
    kw = np.zeros((B, H, S + W, d))
    vw = np.zeros((B, H, S + W, d))
    tables = np.zeros((B, 8), np.int64)
    free = list(rng.permutation(nb))
    hist = []
    for b, L in enumerate(lens):
        kk = O.bf16_round(rng.standard_normal((L, H, d)) * 2).astype(np.float64)
        vv = O.bf16_round(rng.standard_normal((L, H, d)) * 2).astype(np.float64)
        dense, s0, P = O.boundary_dense_tokens(L, S, W)
        nblk = -(-P // bs)
        tables[b, :nblk] = [free.pop() for _ in range(nblk)]
        slots = tables[b, np.arange(P) // bs] * bs + np.arange(P) % bs
        O.pack_kv(kk[s0:s0 + P], vv[s0:s0 + P], slots, kf, vf, nb, bs, kp, vp)
        kw[b, :, :len(dense)] = kk[dense].transpose(1, 0, 2)
        vw[b, :, :len(dense)] = vv[dense].transpose(1, 0, 2)
        hist.append((kk, vv, s0, P))
    q = rng.standard_normal((B, H * G, d))
    out = O.decode_attention(q, kp, vp, tables, lens, kw, vw, S + W, 0.3, kf, vf, bs)
    for b, L in enumerate(lens):
        kk, vv, s0, P = hist[b]
        for h in range(H):
            # keys in token order: dense sinks, the packed middle as stored, dense recent tokens
            ki, kn = O.decode_rows(O.read_rows(kp, tables[b, np.arange(P) // bs], h, np.arange(P) % bs, kf, bs), kf)
            vi, vn = O.decode_rows(O.read_rows(vp, tables[b, np.arange(P) // bs], h, np.arange(P) % bs, vf, bs), vf)
            keys = np.concatenate((kk[:s0, h], O.dequantize_rows(ki, kn, kf, h), kk[s0 + P:, h]))
            vals = np.concatenate((vv[:s0, h], O.dequantize_rows(vi, vn, vf, h), vv[s0 + P:, h]))
            for g in range(G):
                ref = O.dense_attention(q[b, h * G + g], keys, vals, 0.3)
                assert np.abs(out[b, h * G + g] - ref).max() < 1e-12


# ---- QJL residual stage (R16) ----------------------------------------------------------

def test_qjl_estimator_is_unbiased_over_the_projection():
    """E_S[q . (c + sqrt(pi/2)/d g S^T sign(S r))] = q . u for Gaussian S (the QJL identity).

    Averaged over many independent S, the estimate converges to the exact
    product; a wrong constant or an inverted sign convention is far outside
    the bound (the mean of S^T sign(S r) is sqrt(2/pi) d r / |r| exactly).
    """
    rng = np.random.default_rng(7)
    d = 64
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    c_hat = np.round(u * 4) / 4  # any fixed approximation; r is its residual
    r = u - c_hat
    g = np.linalg.norm(r)
    q = rng.standard_normal(d) + 5 * r / g  # a clear component along the residual
    n_draw = 4000
    est = np.empty(n_draw)
    for i in range(n_draw):
        S = rng.standard_normal((d, d))
        z = np.where(S @ r >= 0, 1.0, -1.0)
        est[i] = q @ (c_hat + math.sqrt(math.pi / 2) / d * g * (S.T @ z))
    exact = q @ u
    sem = est.std(ddof=1) / math.sqrt(n_draw)
    assert abs(est.mean() - exact) < 4.5 * sem
    # the QJL variance bound: Var <= pi/(2d) |q|^2 g^2
    assert est.var() <= 1.05 * math.pi / (2 * d) * (q @ q) * g * g
    # and the constant matters: the same draws with 1/d instead of sqrt(pi/2)/d are biased
    biased = (est - q @ c_hat) / math.sqrt(math.pi / 2) + q @ c_hat
    assert abs(biased.mean() - exact) > 10 * sem


def test_qjl_matrix_is_standard_normal():
    """S entries (Box-Muller over SplitMix64) pass a Kolmogorov-Smirnov test against N(0, 1)."""
    import scipy.stats
    fmt = O.Format(128, 1, (3,), (128,), None, 5, qjl=True)
    S = O.qjl_matrix(fmt)
    assert S.shape == (128, 128)
    assert np.all(S == S.astype(np.float32))  # held in fp32
    p = scipy.stats.kstest(S.ravel(), "norm").pvalue
    assert p > 1e-3
    assert abs(S.mean()) < 0.03 and abs(S.std() - 1) < 0.02
    # independent of the sign stream: another seed gives another matrix
    S2 = O.qjl_matrix(O.Format(128, 1, (3,), (128,), None, 6, qjl=True))
    assert abs(np.corrcoef(S.ravel(), S2.ravel())[0, 1]) < 0.03


def test_qjl_row_layout_by_hand():
    """[MSE indices][d sign bits LSB-first][fp16 norm][fp16 residual norm], decoded bit by bit."""
    rng = np.random.default_rng(12)
    d, H = 16, 1
    high = np.array([[0, 3, 5, 6, 9, 10, 12, 15]])
    fmt = O.Format(d, H, (3, 2), (8, 8), high, 4, qjl=True)
    assert O.row_bytes(fmt) == 3 + 2 + d // 8 + 4
    x = O.bf16_round(rng.standard_normal((5, d)) * 3)
    idx, n16, u, signs, g16 = O.quantize_qjl(x, fmt, 0)
    rows = O.encode_rows(idx, n16, fmt, signs, g16)
    for t in range(5):
        row = rows[t]
        bit = lambda k: (int(row[k // 8]) >> (k % 8)) & 1
        pos = 0
        for p in range(16):
            b = 3 if p < 8 else 2
            assert sum(bit(pos + j) << j for j in range(b)) == idx[t, p]
            pos += b
        assert pos == 40
        for i in range(d):
            assert bit(pos + i) == signs[t, i]
        nb = 40 // 8 + d // 8
        assert struct.unpack("<e", bytes(row[nb:nb + 2]))[0] == n16[t]
        assert struct.unpack("<e", bytes(row[nb + 2:nb + 4]))[0] == g16[t]
    back = O.decode_rows(rows, fmt)
    assert np.array_equal(back[0], idx) and np.array_equal(back[2], signs)
    assert np.array_equal(back[1], n16) and np.array_equal(back[3], g16)


def test_qjl_residual_and_signs_follow_the_definitions():
    """r = u - c[idx] in rotated order, g = |r|, bit i = [(S r)_i >= 0]; keys from rows agree."""
    rng = np.random.default_rng(13)
    d, H = 128, 2
    fmt = O.Format(d, H, (3,), (d,), None, 21, qjl=True)
    x = O.bf16_round(rng.standard_normal((6, d)) * 2)
    idx, n16, u, signs, g16 = O.quantize_qjl(x, fmt, 1)
    c, _ = O.codebook(3, d)
    r = u - c[idx]  # one group: packed order is rotated order
    assert np.allclose(g16, O.fp16_round(np.linalg.norm(r, axis=-1)))
    proj = r @ O.qjl_matrix(fmt).T
    assert np.array_equal(signs, (proj >= 0).astype(np.int64))
    # the key a row stands for: n R^T (c[idx] + sqrt(pi/2)/d g S^T z)
    key = O.dequantize_rows(idx, n16, fmt, 1, signs, g16)
    z = 2.0 * signs - 1.0
    rot = c[idx] + math.sqrt(math.pi / 2) / d * g16[:, None] * (z @ O.qjl_matrix(fmt))
    H128 = O.hadamard_matrix(d)
    s = O.hadamard_signs(fmt.seed, d)
    expect = n16[:, None] * (rot @ H128.T) * s / math.sqrt(d)
    assert np.allclose(key, expect, atol=1e-12)
    # q . key estimates q . x: over many vectors the mean error is small against the spread
    q = rng.standard_normal(d)
    xs = O.bf16_round(rng.standard_normal((400, d)))
    i2, n2, _, s2, g2 = O.quantize_qjl(xs, fmt, 0)
    est = O.dequantize_rows(i2, n2, fmt, 0, s2, g2) @ q
    err = est - xs @ q
    assert abs(err.mean()) < 4 * err.std(ddof=1) / math.sqrt(len(err))


# ---- group-wise rotation (R17) ------------------------------------------------------------

def _gw_format(bits=(4, 2), sizes=(32, 96), H=2, seed=9):
    rng = np.random.default_rng(seed)
    high = np.stack([np.sort(rng.choice(D, sizes[0], replace=False)) for _ in range(H)])
    return O.Format(D, H, bits, sizes, high, seed, groupwise=True)


def test_groupwise_rotation_is_blockwise_orthogonal():
    """R is orthogonal, keeps each group's channels inside its own rows, and its
    power-of-two blocks are the textbook Sylvester matrices (scipy) with signs."""
    f = _gw_format()
    R = O.group_rotation(f, 1)
    assert np.allclose(R @ R.T, np.eye(D), atol=1e-14)
    g0, g1 = O.group_channels(f, 1)
    assert np.all(R[:32][:, g1] == 0) and np.all(R[32:][:, g0] == 0)
    s = O.hadamard_signs(f.seed, D)
    blocks = [(0, g0[:32], 32), (32, g1[:64], 64), (96, g1[64:], 32)]  # 96 = 64 + 32
    for row, cols, m in blocks:
        ref = scipy.linalg.hadamard(m) / math.sqrt(m) * s[cols][None, :]
        assert np.allclose(R[row:row + m][:, cols], ref, atol=1e-15)
    assert O.pow2_blocks(112) == [64, 32, 16] and O.pow2_blocks(48) == [32, 16]


def test_groupwise_per_group_distortion_matches_dimension_n_g():
    """For Gaussian x each group's unit vector is uniform on its own sphere, so the
    coordinate error equals the Lloyd-Max distortion for dimension |g| (not d)."""
    f = _gw_format((4, 2), (32, 96), H=1, seed=3)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((20000, D))
    idx, n16, u = O.quantize(x, f, 0)
    start = 0
    for b, n in zip(f.group_bits, f.group_size):
        c, beta = O.codebook(b, n)
        e = np.concatenate(([-1.0], beta, [1.0]))
        per = (O.cell_second_moment(e[:-1], e[1:], n) - 2 * c * O.cell_first_moment(e[:-1], e[1:], n)
               + c * c * O.cell_mass(e[:-1], e[1:], n)).sum()
        err = ((u[:, start:start + n] - c[idx[:, start:start + n]]) ** 2).sum(axis=1)
        sigma = err.std() / math.sqrt(len(err))
        assert abs(err.mean() - n * per) < 4 * sigma
        # the same codebook for dimension d would be measurably off for the small group
        if n == 32:
            c128, beta128 = O.codebook(b, D)
            e128 = np.concatenate(([-1.0], beta128, [1.0]))
            per128 = (O.cell_second_moment(e128[:-1], e128[1:], n) - 2 * c128 * O.cell_first_moment(e128[:-1], e128[1:], n)
                      + c128 * c128 * O.cell_mass(e128[:-1], e128[1:], n)).sum()
            assert per128 > per * 1.01
        start += n
    # norms: one fp16 norm per group, of that group's channels
    g0, g1 = O.group_channels(f, 0)
    assert np.array_equal(n16[:, 0], O.fp16_round(np.linalg.norm(x[:, g0], axis=1)))
    assert np.array_equal(n16[:, 1], O.fp16_round(np.linalg.norm(x[:, g1], axis=1)))


def test_groupwise_row_layout_and_reconstruction():
    """Row = [group-0 indices][group-1 indices][n_0][n_1]; keys rebuild from the rows as
    each group's norm times R^T of its centroids."""
    f = _gw_format((3, 2), (64, 64), H=1, seed=8)
    rng = np.random.default_rng(6)
    x = O.bf16_round(rng.standard_normal((7, D)) * 2)
    idx, n16, u = O.quantize(x, f, 0)
    rows = O.encode_rows(idx, n16, f)
    assert rows.shape[-1] == O.row_bytes(f) == 24 + 16 + 4
    for t in range(7):
        assert struct.unpack("<e", bytes(rows[t, 40:42]))[0] == n16[t, 0]
        assert struct.unpack("<e", bytes(rows[t, 42:44]))[0] == n16[t, 1]
        bit = lambda k: (int(rows[t, k // 8]) >> (k % 8)) & 1
        pos = 0
        for p in range(D):
            b = 3 if p < 64 else 2
            assert sum(bit(pos + j) << j for j in range(b)) == idx[t, p]
            pos += b
    back_idx, back_n = O.decode_rows(rows, f)
    xr = O.dequantize_rows(back_idx, back_n, f, 0)
    c0, _ = O.codebook(3, 64)
    c1, _ = O.codebook(2, 64)
    chat = np.concatenate((c0[idx[:, :64]] * n16[:, :1], c1[idx[:, 64:]] * n16[:, 1:]), axis=1)
    assert np.allclose(xr, chat @ O.group_rotation(f, 0), atol=1e-12)
    # and close to x: each group within its codebook's error
    rel = np.linalg.norm(xr - x, axis=1) / np.linalg.norm(x, axis=1)
    assert np.all(rel < 0.5)


def test_qjl_oracle_key_is_unbiased_over_codec_seeds():
    """The oracle's own QJL key (quantize_qjl, then dequantize_rows) estimates q . x without bias.

    One fixed x and q; the codec seed runs over 2000 values, so S comes from
    the oracle's qjl_matrix (and the sign vector changes with it). Given the
    rotation, the QJL identity E_S[sqrt(pi/2)/d S^T sign(S r)] = r / |r| makes
    the key's expectation n R^T (c + r) = x, and its variance is bounded by
    pi/(2d) |q|^2 |r|^2 n^2 (Zandieh et al., QJL). The fp16 norm and residual
    norm add a bias of at most about 2^-11 |q . x|. The two mistakes that
    leave a single-S check near zero are shown to fail the same mean test: the
    constant sqrt(2/pi)/d in place of sqrt(pi/2)/d, and z = 1 - 2 bits.
    """
    d, n_seeds = 128, 2000
    rng = np.random.default_rng(31)
    x = O.bf16_round(rng.standard_normal(d) * 2.0)[None, :]
    # q along x plus noise: the residual is correlated with the rotated vector
    # (a Lloyd-Max error is orthogonal to the centroid, not to the input), so
    # a wrong QJL scale or sign shifts q . key by a multiple of the distortion
    q = x[0] / np.linalg.norm(x[0]) * 8.0 + rng.standard_normal(d)
    exact = float(x[0] @ q)
    est, mse_part, bound = np.empty(n_seeds), np.empty(n_seeds), np.empty(n_seeds)
    for i in range(n_seeds):
        f = O.Format(d, 1, (3,), (d,), None, 1000 + i, qjl=True)
        idx, n16, u, signs, g16 = O.quantize_qjl(x, f, 0)
        est[i] = float(O.dequantize_rows(idx, n16, f, 0, signs, g16)[0] @ q)
        mse_part[i] = float(O.dequantize_rows(idx, n16, f, 0, signs, np.zeros_like(g16))[0] @ q)
        bound[i] = math.pi / (2 * d) * float(q @ q) * float(g16[0]) ** 2 * float(n16[0]) ** 2
    qjl_part = est - mse_part
    sem = est.std(ddof=1) / math.sqrt(n_seeds)
    fp16_bias = 2.0 ** -10 * abs(exact)
    assert abs(est.mean() - exact) < 4 * sem + fp16_bias
    # second moment of the error within the QJL variance bound (averaged over the draws)
    assert np.mean((est - exact) ** 2) <= 1.1 * bound.mean()
    # the QJL term carries signal: dropping it leaves the MSE part's shrinkage bias
    assert abs(mse_part.mean() - exact) > 8 * sem + fp16_bias
    wrong_const = mse_part + (2.0 / math.pi) * qjl_part  # sqrt(2/pi)/d instead of sqrt(pi/2)/d
    wrong_sign = mse_part - qjl_part                       # z = 1 - 2 bits
    for alt in (wrong_const, wrong_sign):
        alt_sem = alt.std(ddof=1) / math.sqrt(n_seeds)
        assert abs(alt.mean() - exact) > 8 * max(sem, alt_sem) + fp16_bias


def test_ledger_transform_bytes_are_the_transforms_a_decode_holds():
    """transform_bytes = the nbytes of what the oracle builds for each codec: int8 signs, the int16
    permutation of every head, the fp32 QJL matrix S of a QJL codec, and the dense fp32 rotation
    R_h of every head of a group-wise codec ("System Invariants": the ratio counts transforms)."""
    H = 3
    rng = np.random.default_rng(4)
    high = np.stack([np.sort(rng.choice(D, 64, replace=False)) for _ in range(H)])
    cases = [O.Format(D, H, (4, 3), (64, 64), high, 5, groupwise=True),
             O.Format(D, H, (3, 2), (64, 64), high, 6, qjl=True),
             O.Format(D, H, (4,), (128,), None, 7)]
    for kf in cases:
        for vf in cases:
            if vf.qjl:
                continue
            led = O.byte_ledger(kf, vf, [40, 7], 4, 16, 5)
            expect = 0
            for f in (kf, vf):
                expect += O.hadamard_signs(f.seed, D).astype(np.int8).nbytes
                expect += sum(O.permutation(f, h).astype(np.int16).nbytes for h in range(H))
                if f.qjl:
                    expect += O.qjl_matrix(f).astype(np.float32).nbytes
                if f.groupwise:
                    expect += sum(O.group_rotation(f, h).astype(np.float32).nbytes for h in range(H))
            assert led.transform_bytes == expect, (kf, vf)


# ---- the recipe row as printed (R18): group-wise rotation with a QJL stage per group ---------

def _recipe_format(bits=(4, 3), sizes=(64, 64), H=2, seed=11, d=D):
    rng = np.random.default_rng(seed)
    high = np.stack([np.sort(rng.choice(d, sizes[0], replace=False)) for _ in range(H)])
    return O.Format(d, H, bits, sizes, high, seed, qjl=True, groupwise=True)


def test_recipe_row_layout_by_hand():
    """Two groups, each [MSE indices][QJL signs][vector norm][residual norm], decoded bit by bit."""
    rng = np.random.default_rng(21)
    d = 32
    f = _recipe_format((3, 2), (16, 16), H=1, seed=4, d=d)
    assert O.row_bytes(f) == (6 + 2 + 4) + (4 + 2 + 4)
    x = O.bf16_round(rng.standard_normal((5, d)) * 3)
    idx, n16, u, signs, g16 = O.quantize_qjl(x, f, 0)
    rows = O.encode_rows(idx, n16, f, signs, g16)
    for t in range(5):
        row = rows[t]
        bit = lambda k: (int(row[k // 8]) >> (k % 8)) & 1
        pos = 0
        for g, (b, n) in enumerate(((3, 16), (2, 16))):
            for p in range(n):
                assert sum(bit(pos + j) << j for j in range(b)) == idx[t, 16 * g + p]
                pos += b
            for p in range(n):
                assert bit(pos) == signs[t, 16 * g + p]
                pos += 1
            nb = pos // 8
            assert struct.unpack("<e", bytes(row[nb:nb + 2]))[0] == n16[t, g]
            assert struct.unpack("<e", bytes(row[nb + 2:nb + 4]))[0] == g16[t, g]
            pos += 32
        assert pos == 8 * O.row_bytes(f)
    back = O.decode_rows(rows, f)
    for a, b in zip(back, (idx, n16, signs, g16)):
        assert np.array_equal(a, b)


def test_recipe_subpage_order_and_round_trip():
    """In a sub-page: each group's [indices][signs] in the index area, each group's (norm, residual
    norm) in the norm area; rows written and read back are unchanged."""
    f = _recipe_format((4, 2), (32, 96), H=1, seed=5)
    a0, a1 = 32 * 4 // 8 + 4, 96 * 2 // 8 + 12
    order = O.subpage_byte_order(f)
    assert O.index_bytes(f) == a0 + a1 and O.norm_bytes(f) == 8
    assert np.array_equal(order[:a0], np.arange(a0))
    assert np.array_equal(order[a0:a0 + a1], np.arange(a0 + 4, a0 + 4 + a1))
    assert np.array_equal(order[a0 + a1:], np.r_[a0:a0 + 4, a0 + a1 + 4:a0 + a1 + 8])
    rng = np.random.default_rng(3)
    bs, nb = 4, 3
    pages = np.zeros((nb, 1, O.subpage_bytes(f, bs)), np.uint8)
    rows = rng.integers(0, 256, (6, O.row_bytes(f)), dtype=np.uint8)
    blocks, offs = np.array([0, 0, 1, 2, 2, 1]), np.array([0, 3, 1, 2, 0, 3])
    O.write_rows(pages, blocks, 0, offs, rows, f, bs)
    assert np.array_equal(O.read_rows(pages, blocks, 0, offs, f, bs), rows)
    # the index bytes of the row at offset 3 of block 0 sit at 3 * index_bytes, its norms after the index area
    ib = O.index_bytes(f)
    assert np.array_equal(pages[0, 0, 3 * ib:4 * ib], rows[1, order[:ib]])
    assert np.array_equal(pages[0, 0, bs * ib + 3 * 8:bs * ib + 4 * 8], rows[1, order[ib:]])


def test_recipe_matrices_are_standard_normal_and_distinct():
    import scipy.stats
    f = _recipe_format((4, 3), (64, 64), seed=8)
    S0, S1 = O.recipe_qjl_matrix(f, 0), O.recipe_qjl_matrix(f, 1)
    assert S0.shape == (64, 64) and S1.shape == (64, 64)
    assert np.all(S0 == S0.astype(np.float32)) and np.all(S1 == S1.astype(np.float32))
    for S in (S0, S1):
        assert scipy.stats.kstest(S.ravel(), "norm").pvalue > 1e-3
    assert abs(np.corrcoef(S0.ravel(), S1.ravel())[0, 1]) < 0.05
    assert abs(np.corrcoef(S0.ravel(), O.qjl_matrix(O.Format(64, 1, (4,), (64,), None, 8, qjl=True)).ravel())[0, 1]) < 0.05


def test_recipe_key_without_residual_is_the_groupwise_key():
    """With every residual norm set to 0 the recipe key is the R17 group-wise key of the same
    indices and norms (the QJL term is the only addition)."""
    rng = np.random.default_rng(9)
    f = _recipe_format((4, 3), (64, 64), H=2, seed=13)
    fg = O.Format(D, 2, (4, 3), (64, 64), f.high_coords, 13, groupwise=True)
    x = O.bf16_round(rng.standard_normal((7, D)) * 2)
    idx, n16, _, signs, g16 = O.quantize_qjl(x, f, 1)
    gi, gn, _ = O.quantize(x, fg, 1)
    assert np.array_equal(idx, gi) and np.array_equal(n16, gn)
    key0 = O.dequantize_rows(idx, n16, f, 1, signs, np.zeros_like(g16))
    assert np.allclose(key0, O.dequantize_rows(gi, gn, fg, 1), atol=1e-12)


def test_recipe_key_is_unbiased_over_codec_seeds():
    """For one fixed x and q over 1500 codec seeds (so every S_g comes from recipe_qjl_matrix):
    the mean of q.key equals q.x within 4 sigma, the mean squared error stays inside the sum of
    the groups' QJL bounds pi/(2 n_g) |q_g|^2 gamma_g^2 n_g^2, and the wrong constant
    sqrt(2/pi)/n_g or the inverted sign convention fail the same mean check."""
    d, n_seeds = D, 1500
    rng = np.random.default_rng(41)
    x = O.bf16_round(rng.standard_normal(d) * 2.0)[None, :]
    q = x[0] / np.linalg.norm(x[0]) * 8.0 + rng.standard_normal(d)
    high = np.sort(rng.choice(d, 64, replace=False))[None, :]
    exact = float(x[0] @ q)
    est, mse_part, bound = np.empty(n_seeds), np.empty(n_seeds), np.empty(n_seeds)
    for i in range(n_seeds):
        f = O.Format(d, 1, (3, 2), (64, 64), high, 500 + i, qjl=True, groupwise=True)
        idx, n16, u, signs, g16 = O.quantize_qjl(x, f, 0)
        est[i] = float(O.dequantize_rows(idx, n16, f, 0, signs, g16)[0] @ q)
        mse_part[i] = float(O.dequantize_rows(idx, n16, f, 0, signs, np.zeros_like(g16))[0] @ q)
        qg = O.group_rotation(f, 0) @ q  # the query in the groups' rotated coordinates
        bound[i] = sum(math.pi / (2 * 64) * float(qg[64 * g:64 * (g + 1)] @ qg[64 * g:64 * (g + 1)])
                       * float(g16[0, g]) ** 2 * float(n16[0, g]) ** 2 for g in range(2))
    qjl_part = est - mse_part
    sem = est.std(ddof=1) / math.sqrt(n_seeds)
    fp16_bias = 2.0 ** -10 * abs(exact)
    assert abs(est.mean() - exact) < 4 * sem + fp16_bias
    assert np.mean((est - exact) ** 2) <= 1.15 * bound.mean()
    assert abs(mse_part.mean() - exact) > 8 * sem + fp16_bias
    for alt in (mse_part + (2.0 / math.pi) * qjl_part, mse_part - qjl_part):
        alt_sem = alt.std(ddof=1) / math.sqrt(n_seeds)
        assert abs(alt.mean() - exact) > 8 * max(sem, alt_sem) + fp16_bias


def test_recipe_attention_and_ledger():
    """decode_attention over recipe pages equals dense attention over the recipe keys; the ledger
    counts 8 norm bytes per row and the two S_g and R_h as transforms."""
    rng = np.random.default_rng(17)
    H, bs = 2, 4
    kf = _recipe_format((4, 3), (64, 64), H=H, seed=2)
    vf = O.Format(D, H, (4, 3), (64, 64), kf.high_coords, 3, groupwise=True)
    T = 10
    k = O.bf16_round(rng.standard_normal((T, H, D)))
    v = O.bf16_round(rng.standard_normal((T, H, D)))
    kp, vp = O.pack_kv(k, v, np.arange(T), kf, vf, 3, bs)
    q = O.bf16_round(rng.standard_normal((1, 2 * H, D)))
    out = O.decode_attention(q, kp, vp, np.array([[0, 1, 2]]), [T], np.zeros((1, H, 1, D)),
                             np.zeros((1, H, 1, D)), 0, 0.2, kf, vf, bs)
    for h in range(H):
        idx, n16, _, signs, g16 = O.quantize_qjl(k[:, h], kf, h)
        keys = O.dequantize_rows(idx, n16, kf, h, signs, g16)
        vi, vn, _ = O.quantize(v[:, h], vf, h)
        vals = O.dequantize_rows(vi, vn, vf, h)
        for g in range(2):
            ref = O.dense_attention(q[0, 2 * h + g], keys, vals, 0.2)
            assert np.abs(out[0, 2 * h + g] - ref).max() < 1e-12
    led = O.byte_ledger(kf, vf, [T], 0, bs, 3)
    assert led.norm_bytes == T * H * (8 + 4)
    expect = 2 * (D + H * D * 2) + 4 * (64 * 64 + 64 * 64) + 2 * 4 * H * D * D
    assert led.transform_bytes == expect
