"""CPU oracle for the compressed paged KV cache: the diagnostic route, written plainly.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module. The only callers are the files under ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs
of ``bench.py``. It shares no code, tables or constants with the CUDA library:
every codebook, sign vector, permutation and byte layout below is computed here
from its definition.

What it follows (pages cited by title and section):

* TurboQuant "Design" page, "Diagnostic Route Design": dense reconstruction,
  plain loops, CPU execution and extra assertions are allowed on this route; it
  makes no throughput claim.
* TurboQuant "Design" page, "Serving Route Design": slot -> physical block ->
  token offset -> packed row bytes, with block = slot // block_size and
  offset = slot % block_size.
* TurboQuant "Design" page, "Recipe Strategy": a row holds the MSE indices of
  each channel group, then the vector norm; the high group is named by sorted
  calibration indices.
* TurboQuant "Design" page, "System Invariants": storage and metadata bytes
  are reported separately.
* TurboQuant Inference Server page, "Codebook caching": Lloyd-Max codebooks,
  computed once on the CPU.
* tattletale page (EXL3 quant): random Hadamard rotations as the transform.

Precision: fp64 throughout, except where the row format itself fixes a
narrower type (fp16 centroids and norms, fp32 decision boundaries).

Readings taken where the pages are silent (each is also listed in the design
notes of the repository):

R1  One randomized Hadamard rotation over all d coordinates per head and one
    per-token norm; channel groups are sets of *rotated* coordinates.
R2  The codebook is the Lloyd-Max quantizer of one coordinate of a uniformly
    random unit vector in R^d (density f_d below), d = head_dim, for every
    group. Centroids are rounded to fp16 (b <= 8); decision boundaries are the
    exact midpoints of adjacent fp16 centroids, held in fp32.
R3  R = H diag(s) / sqrt(d), H the natural-order Sylvester matrix,
    s_i = +1 when bit 0 of the i-th SplitMix64 output is 0, else -1. One sign
    vector per codec (shared by its heads).
R4  Norm n = ||x||_2 of the bf16 input promoted exactly; stored as fp16
    round-to-nearest-even; u = R x / n with the unrounded n; u = 0 if n = 0.
R5  idx = #{boundaries strictly below u}: nearest centroid, ties to the lower
    index.
R6  Row = [group-0 bitstream][group-1 bitstream][fp16 norm, little endian];
    each bitstream is LSB-first, index k at bits [k*b, (k+1)*b). Group 0 holds
    the high coordinates in ascending order, group 1 the rest ascending.
    Pages are [num_blocks][H_kv][block_size * row_bytes]: the sub-page of one
    (block, head) holds the index bytes of its block_size rows, row after row,
    then their block_size fp16 norms. A row is found from (block, offset)
    alone; K and V have separate pools that share block ids.
R7  The last min(W, L_b) tokens of a sequence live only in the dense bf16
    window; the first P_b = L_b - min(W, L_b) tokens are packed.
R8  slot < 0 is a padding token and is skipped; slot >= num_blocks*block_size
    raises IndexError.
R16 QJL residual stage (TurboQuant "Design" page, "Recipe Strategy": row
    [MSE indices][QJL signs][vector norm][residual norm]). With qjl set, the
    MSE part is the format's groups as above; r = u - c[idx] is the residual
    of the unit rotated vector (rotated coordinate order), g = ||r|| is
    stored as fp16 after the norm, and bit i of the d sign bits (LSB-first)
    is 1 when (S r)_i >= 0. S is d x d with iid N(0, 1) entries held in fp32
    (qjl_matrix). The key a row stands for is the unbiased inner-product
    estimate n R^T (c[idx] + sqrt(pi/2) / d * g * S^T z), z = 2 bits - 1:
    E over S of its product with q equals q . x when g is exact. In a
    sub-page the sign bytes follow the index bytes of each row and the norm
    area holds (norm, residual norm) per row.
R17 Group-wise rotation (the original-channel reading of the high/low
    recipe; "Recipe Strategy": the high channel set comes from calibration
    metadata). With groupwise set, group 0 is the set of ORIGINAL channels
    high_coords[h] (ascending) and group 1 the other channels (ascending).
    Each group is rotated on its own: y_g = B_g (s[ch_g] * x[ch_g]), B_g the
    block-diagonal of orthonormal natural-order Hadamard blocks of the
    power-of-two sizes that make up |g|, largest first (96 = 64 + 32), s the
    codec's sign vector indexed by channel. Each group has its own norm
    n_g = |x[ch_g]| (fp16) and codebook (Lloyd-Max for dimension |g|);
    u_g = y_g / n_g. Row = [group-0 indices][group-1 indices][n_0][n_1];
    the norm area of a sub-page holds (n_0, n_1) per row.
R18 The recipe row as printed (TurboQuant "Design" page, "Recipe Strategy":
    two groups, each [MSE indices][QJL signs][vector norm][residual norm]):
    groupwise and qjl together. Each group is quantized as in R17 (its own
    block-Hadamard rotation, norm n_g and dimension-n_g codebook); its
    residual r_g = u_g - c_g[idx_g] (the group's rotated order) gets fp16 norm
    gamma_g and n_g sign bits [(S_g r_g)_i >= 0], S_g an n_g x n_g matrix of
    iid N(0, 1) (recipe_qjl_matrix). The key is, per group, n_g B_g^T (c_g +
    sqrt(pi/2)/n_g gamma_g S_g^T z_g) on the group's channels. The logical
    row keeps the printed order; in a sub-page the index area holds each
    group's [indices][signs] (group 0, then group 1) and the norm area its
    (n_g, gamma_g) pairs, so index rows stay whole bytes apart from the norms
    as in R6.
R14 Boundary-token preservation: the first S and the last W tokens of a
    sequence stay dense, the ones between are packed (boundary_dense_tokens).
    Attention is a sum over keys, so the dense ones may sit in one buffer in
    any order; the decode treats them as its window.
"""

from __future__ import annotations

import functools
import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
from scipy.special import betainc, betaincinv, gammaln

__all__ = [
    "Format", "coord_density_const", "coord_cdf", "coord_tail", "cell_mass",
    "cell_first_moment", "cell_second_moment", "lloyd_max", "codebook", "boundary_dense_tokens",
    "qjl_matrix", "quantize_qjl", "norm_bytes", "mse_index_bytes", "group_rotation", "group_channels",
    "pow2_blocks",
    "splitmix64", "hadamard_signs", "hadamard_matrix", "rotate", "unrotate",
    "permutation", "position_bits", "row_bytes", "index_bytes",
    "quantize", "encode_rows", "decode_rows", "dequantize_rows",
    "pack_kv", "read_row", "read_rows", "write_rows", "subpage_bytes", "decode_attention", "dense_attention",
    "boundary_margin", "byte_ledger", "Ledger", "fp16_round", "bf16_round",
]


# ---------------------------------------------------------------------------
# Format description (oracle-side; the CUDA library has its own)
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Format:
    """One codec: head_dim, per-group bit widths and sizes, high coordinates, seed.

    ``high_coords`` is ``[num_kv_heads][group_size[0]]`` sorted rotated
    coordinates of group 0 (TurboQuant "Design" page, "Recipe Strategy":
    sorted high-precision indices from metadata); ``None`` for one group.
    """

    head_dim: int
    num_kv_heads: int
    group_bits: tuple
    group_size: tuple
    high_coords: Optional[np.ndarray] = field(default=None, compare=False)
    seed: int = 0
    qjl: bool = False
    groupwise: bool = False

    def __post_init__(self):
        d = self.head_dim
        if self.groupwise and len(self.group_bits) != 2:
            raise ValueError("group-wise rotation needs two groups")
        if self.groupwise and self.qjl and any(n % 8 for n in self.group_size):
            raise ValueError("the recipe row needs whole sign bytes per group")
        if len(self.group_bits) != len(self.group_size) or len(self.group_bits) not in (1, 2):
            raise ValueError("one or two channel groups")
        if sum(self.group_size) != d:
            raise ValueError("group sizes must sum to head_dim")
        for b in self.group_bits:
            if b not in (1, 2, 3, 4, 5, 6, 7, 8, 16):
                raise ValueError(f"unsupported bit width {b}")
        if len(self.group_bits) == 2:
            hc = np.asarray(self.high_coords)
            if hc.shape != (self.num_kv_heads, self.group_size[0]):
                raise ValueError("high_coords must be [num_kv_heads][group_size[0]]")
            for row in hc:
                if np.any(np.diff(row) <= 0) or row.min() < 0 or row.max() >= d:
                    raise ValueError("high_coords rows must be strictly ascending in [0, d)")

    @property
    def mean_bits(self) -> float:
        return sum(b * n for b, n in zip(self.group_bits, self.group_size)) / self.head_dim


# ---------------------------------------------------------------------------
# Coordinate density of a uniform unit vector (R2)
# ---------------------------------------------------------------------------

def coord_density_const(d: int) -> float:
    """C_d in f_d(x) = C_d (1 - x^2)^((d-3)/2) on [-1, 1]."""
    return math.exp(gammaln(d / 2.0) - gammaln((d - 1) / 2.0)) / math.sqrt(math.pi)


def coord_tail(x, d: int):
    """P(X > x) for x >= 0: (1/2) I_{1-x^2}((d-1)/2, 1/2)."""
    x = np.asarray(x, dtype=np.float64)
    one_minus = (1.0 - x) * (1.0 + x)
    return 0.5 * betainc((d - 1) / 2.0, 0.5, np.clip(one_minus, 0.0, 1.0))


def coord_cdf(x, d: int):
    """P(X <= x) for the coordinate density f_d."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x >= 0, 1.0 - coord_tail(np.abs(x), d), coord_tail(np.abs(x), d))


def cell_mass(a, b, d: int):
    """P(a < X <= b), written so that tail cells do not cancel."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    pos = coord_tail(np.abs(a), d) - coord_tail(np.abs(b), d)          # 0 <= a < b
    neg = coord_tail(np.abs(b), d) - coord_tail(np.abs(a), d)          # a < b <= 0
    mid = 1.0 - coord_tail(np.abs(a), d) - coord_tail(np.abs(b), d)    # a < 0 < b
    return np.where(a >= 0, pos, np.where(b <= 0, neg, mid))


def cell_first_moment(a, b, d: int):
    """Integral of x f_d(x) over [a, b]; closed form C_d/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)]."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    e = (d - 1) / 2.0
    wa = np.clip((1.0 - a) * (1.0 + a), 0.0, 1.0) ** e
    wb = np.clip((1.0 - b) * (1.0 + b), 0.0, 1.0) ** e
    return coord_density_const(d) / (d - 1) * (wa - wb)


def cell_second_moment(a, b, d: int):
    """Integral of x^2 f_d(x) over [a, b], through the incomplete beta with p = 3/2.

    Substituting t = x^2 gives int_0^x s^2 f_d(s) ds = (C_d / 2) B(3/2, (d-1)/2) I_{x^2}(3/2, (d-1)/2).
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    p, q = 1.5, (d - 1) / 2.0
    scale = 0.5 * coord_density_const(d) * math.exp(gammaln(p) + gammaln(q) - gammaln(p + q))

    def signed(x):
        return np.sign(x) * scale * betainc(p, q, np.minimum(x * x, 1.0))

    return signed(b) - signed(a)


def _quantile(p, d: int):
    """Inverse of coord_cdf, used only to start the Lloyd iteration."""
    p = np.asarray(p, dtype=np.float64)
    hi = np.sqrt(1.0 - betaincinv((d - 1) / 2.0, 0.5, np.clip(2.0 * (1.0 - p), 0.0, 1.0)))
    lo = -np.sqrt(1.0 - betaincinv((d - 1) / 2.0, 0.5, np.clip(2.0 * p, 0.0, 1.0)))
    return np.where(p >= 0.5, hi, lo)


@functools.lru_cache(maxsize=None)
def _lloyd_max_cached(bits: int, d: int, tol: float, max_iter: int):
    levels = 1 << bits
    # Start at the quantiles of the Panter-Dite point density f_d^(1/3), which is
    # f_{d'} with d' = (d + 6) / 3; f_d is log-concave, so the Lloyd fixed point
    # is unique and the start only changes how fast it is reached.
    c = _quantile((np.arange(levels) + 0.5) / levels, (d + 6) / 3.0)
    c = 0.5 * (c - c[::-1])
    converged = False
    for _ in range(max_iter):
        edges = np.concatenate(([-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]))
        c_new = cell_first_moment(edges[:-1], edges[1:], d) / cell_mass(edges[:-1], edges[1:], d)
        c_new = 0.5 * (c_new - c_new[::-1])  # the density is even
        step = float(np.max(np.abs(c_new - c)))
        c = c_new
        if step <= tol * float(np.max(np.abs(c))):
            converged = True
            break
    return c, converged


def lloyd_max(bits: int, d: int, tol: float = 1e-14, max_iter: int = 200000,
              require_convergence: bool = True) -> np.ndarray:
    """Lloyd-Max codebook (fp64, ascending) for one coordinate of a random unit vector in R^d.

    TurboQuant Inference Server page, "Codebook caching": the codebooks are
    Lloyd-Max, computed once on the CPU. Cells are [beta_{i-1}, beta_i] with
    beta the midpoints of adjacent centroids; each centroid is its cell's
    conditional mean. The iteration starts at the quantiles (i + 1/2)/L of the
    companded density and stops when no centroid moves by more than ``tol`` times the largest one.
    """
    c, converged = _lloyd_max_cached(bits, d, tol, max_iter)
    if require_convergence and not converged:
        raise RuntimeError(f"Lloyd-Max did not converge for b={bits}, d={d}")
    return c.copy()


def fp16_round(x):
    """IEEE fp16 round-to-nearest-even of fp64 values, returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def bf16_round(x):
    """bf16 round-to-nearest-even of fp32-representable values, returned as fp32."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint32).view(np.float32).copy()
    out[nan] = np.nan
    return out


def codebook(bits: int, d: int):
    """(centroids, boundaries) as used by the row format (R2).

    For b <= 8 the centroids are fp16-rounded Lloyd-Max centroids and the
    boundaries their exact midpoints (fp32-representable). For b = 16, used
    only by the diagnostic 16-bit check, centroids stay fp64: the iteration
    starts at the companded quantiles and runs a fixed number of sweeps.
    """
    if bits == 16:
        c = lloyd_max(16, d, tol=0.0, max_iter=8, require_convergence=False)
        return c, 0.5 * (c[:-1] + c[1:])
    c = fp16_round(lloyd_max(bits, d))
    beta = 0.5 * (c[:-1] + c[1:])
    assert np.all(beta.astype(np.float32).astype(np.float64) == beta)
    return c, beta


# ---------------------------------------------------------------------------
# Rotation (R3)
# ---------------------------------------------------------------------------

def splitmix64(seed: int, n: int):
    """First n outputs of SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) from ``seed``."""
    mask = (1 << 64) - 1
    state = seed & mask
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & mask
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & mask
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & mask
        out.append(z ^ (z >> 31))
    return out


def hadamard_signs(seed: int, d: int) -> np.ndarray:
    """s_i = +1 if bit 0 of the i-th SplitMix64 output is 0, else -1 (R3)."""
    return np.array([-1.0 if (z & 1) else 1.0 for z in splitmix64(seed, d)])


def hadamard_matrix(d: int) -> np.ndarray:
    """Natural-order Sylvester matrix H[i][j] = (-1)^popcount(i & j)."""
    if d <= 0 or d & (d - 1):
        raise ValueError("head_dim must be a power of two")
    i = np.arange(d)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


def rotate(x, signs):
    """y = H (s * x) / sqrt(d) along the last axis."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    return (x * signs) @ hadamard_matrix(d).T / math.sqrt(d)


def unrotate(y, signs):
    """x = s * (H y) / sqrt(d), the inverse of ``rotate``."""
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    return (y @ hadamard_matrix(d).T) * signs / math.sqrt(d)


# ---------------------------------------------------------------------------
# Channel groups and the row layout (R1, R6)
# ---------------------------------------------------------------------------

def permutation(fmt: Format, head: int) -> np.ndarray:
    """pi_h: packed position p -> rotated coordinate (high coords ascending, then the rest)."""
    d = fmt.head_dim
    if len(fmt.group_bits) == 1:
        return np.arange(d)
    high = np.asarray(fmt.high_coords[head], dtype=np.int64)
    low = np.setdiff1d(np.arange(d), high)
    return np.concatenate((high, low))


def position_bits(fmt: Format) -> np.ndarray:
    """Bit width of each packed position."""
    return np.concatenate([np.full(n, b) for b, n in zip(fmt.group_bits, fmt.group_size)])


def mse_index_bytes(fmt: Format) -> int:
    """Bytes of the groups' index bitstreams."""
    total = 0
    for b, n in zip(fmt.group_bits, fmt.group_size):
        if (b * n) % 8:
            raise ValueError("each group bitstream must fill whole bytes")
        total += b * n // 8
    return total


def index_bytes(fmt: Format) -> int:
    """Bytes of a row before its norms: the index bitstreams, then the QJL signs (R16)."""
    return mse_index_bytes(fmt) + (fmt.head_dim // 8 if fmt.qjl else 0)


def norm_bytes(fmt: Format) -> int:
    """fp16 norm, then the fp16 residual norm with QJL (R16) or the group-1 norm (R17);
    the recipe row (R18) holds (norm, residual norm) of each group."""
    if fmt.qjl and fmt.groupwise:
        return 8
    return 4 if (fmt.qjl or fmt.groupwise) else 2


def recipe(fmt: Format) -> bool:
    """The recipe row of R18: group-wise rotation with a QJL stage per group."""
    return bool(fmt.qjl and fmt.groupwise)


def pow2_blocks(n: int):
    """The power-of-two sizes that make up n, largest first (R17)."""
    return [1 << k for k in range(n.bit_length() - 1, -1, -1) if n >> k & 1]


def group_channels(fmt: Format, head: int):
    """(channels of group 0, channels of group 1), ascending (R17)."""
    d = fmt.head_dim
    high = np.asarray(fmt.high_coords[head], dtype=np.int64)
    return high, np.setdiff1d(np.arange(d), high)


def group_rotation(fmt: Format, head: int) -> np.ndarray:
    """R (d x d) with (R x)[p] = the rotated coordinate at packed position p (R17).

    Rows 0 .. n0-1 are group 0's B_0 diag(s[ch_0]) applied to x[ch_0], rows n0 ..
    d-1 group 1's; R is orthogonal.
    """
    d = fmt.head_dim
    s = hadamard_signs(fmt.seed, d)
    R = np.zeros((d, d))
    row = 0
    for ch in group_channels(fmt, head):
        col = 0
        for m in pow2_blocks(len(ch)):
            blk = hadamard_matrix(m) / math.sqrt(m)
            cols = ch[col:col + m]
            R[row:row + m, cols] = blk * s[cols][None, :]
            row += m
            col += m
    return R


def row_bytes(fmt: Format) -> int:
    """Index bytes (and QJL signs) of a row plus its fp16 norm(s)."""
    return index_bytes(fmt) + norm_bytes(fmt)


def quantize(x, fmt: Format, head: int):
    """Quantize vectors x[..., d] of one head.

    Returns (idx, n16, u): ``idx[..., p]`` is the index at packed position p,
    ``n16`` the fp16-rounded norm (fp64 value), ``u`` the fp64 unit rotated
    vector in packed order (kept for boundary accounting).
    """
    x = np.asarray(x, dtype=np.float64)
    d = fmt.head_dim
    if fmt.groupwise:
        return _quantize_groupwise(x, fmt, head)
    n = np.sqrt(np.sum(x * x, axis=-1))
    y = rotate(x, hadamard_signs(fmt.seed, d))
    safe = np.where(n > 0, n, 1.0)
    u = np.where(n[..., None] > 0, y / safe[..., None], 0.0)
    u = u[..., permutation(fmt, head)]
    idx = np.empty(u.shape, dtype=np.int64)
    start = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        _, beta = codebook(b, d)
        idx[..., start:start + size] = np.searchsorted(beta, u[..., start:start + size], side="left")
        start += size
    n16 = n if 16 in fmt.group_bits else fp16_round(n)
    return idx, n16, u


def _quantize_groupwise(x, fmt: Format, head: int):
    """quantize() under R17: n16 is [..., 2] (the two group norms, fp16-rounded)."""
    d = fmt.head_dim
    y = x @ group_rotation(fmt, head).T          # packed order
    idx = np.empty(y.shape, dtype=np.int64)
    u = np.empty(y.shape)
    norms = []
    start = 0
    for (b, size), ch in zip(zip(fmt.group_bits, fmt.group_size), group_channels(fmt, head)):
        n = np.sqrt(np.sum(x[..., ch] ** 2, axis=-1))
        safe = np.where(n > 0, n, 1.0)
        seg = np.where(n[..., None] > 0, y[..., start:start + size] / safe[..., None], 0.0)
        _, beta = codebook(b, size)
        idx[..., start:start + size] = np.searchsorted(beta, seg, side="left")
        u[..., start:start + size] = seg
        norms.append(fp16_round(n))
        start += size
    return idx, np.stack(norms, axis=-1), u


QJL_SEED_XOR = 0x51534A4C00000001  # "QSJL": the S stream is independent of the sign stream


@functools.lru_cache(maxsize=None)
def _qjl_matrix_cached(seed: int, d: int) -> np.ndarray:
    x = splitmix64(seed ^ QJL_SEED_XOR, 2 * d * d)
    a = np.array(x[0::2], dtype=np.uint64)
    b = np.array(x[1::2], dtype=np.uint64)
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53  # (0, 1]
    u2 = (b >> np.uint64(11)).astype(np.float64) * 2.0 ** -53          # [0, 1)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)         # Box-Muller, cosine branch
    return z.astype(np.float32).astype(np.float64).reshape(d, d)


def qjl_matrix(fmt: Format) -> np.ndarray:
    """S of R16: S[i][j] = N(0, 1) drawn from SplitMix64(seed ^ QJL_SEED_XOR) outputs 2k, 2k+1
    (k = i d + j) by the Box-Muller cosine branch, then rounded to fp32."""
    return _qjl_matrix_cached(int(fmt.seed), int(fmt.head_dim)).copy()


@functools.lru_cache(maxsize=None)
def _recipe_matrix_cached(seed: int, group: int, n: int) -> np.ndarray:
    x = splitmix64(seed ^ QJL_SEED_XOR ^ ((group + 1) << 56), 2 * n * n)
    a = np.array(x[0::2], dtype=np.uint64)
    b = np.array(x[1::2], dtype=np.uint64)
    u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53  # (0, 1]
    u2 = (b >> np.uint64(11)).astype(np.float64) * 2.0 ** -53          # [0, 1)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)         # Box-Muller, cosine branch
    return z.astype(np.float32).astype(np.float64).reshape(n, n)


def recipe_qjl_matrix(fmt: Format, group: int) -> np.ndarray:
    """S_g of R18 (n_g x n_g): the R16 construction on the SplitMix64 stream seeded with
    seed ^ QJL_SEED_XOR ^ ((g + 1) << 56), one stream per group."""
    return _recipe_matrix_cached(int(fmt.seed), int(group), int(fmt.group_size[group])).copy()


def _quantize_recipe(x, fmt: Format, head: int):
    """quantize_qjl() under R18: signs [..., d] (group 0's n_0 bits, then group 1's) and
    g16 [..., 2] (the groups' fp16 residual norms)."""
    idx, n16, u = _quantize_groupwise(x, fmt, head)
    signs = np.empty(idx.shape, dtype=np.int64)
    g16 = []
    start = 0
    for g, (b, size) in enumerate(zip(fmt.group_bits, fmt.group_size)):
        c, _ = codebook(b, size)
        r = u[..., start:start + size] - c[idx[..., start:start + size]]
        g16.append(fp16_round(np.sqrt(np.sum(r * r, axis=-1))))
        signs[..., start:start + size] = (r @ recipe_qjl_matrix(fmt, g).T >= 0).astype(np.int64)
        start += size
    return idx, n16, u, signs, np.stack(g16, axis=-1)


def quantize_qjl(x, fmt: Format, head: int):
    """quantize() plus the QJL stage (R16): returns (idx, n16, u, signs, g16).

    signs[..., i] in {0, 1} (1: (S r)_i >= 0), g16 = fp16(||r||), r the
    residual of u in rotated coordinate order.
    """
    if recipe(fmt):
        return _quantize_recipe(x, fmt, head)
    idx, n16, u = quantize(x, fmt, head)
    d = fmt.head_dim
    c_hat = np.empty(idx.shape, dtype=np.float64)
    start = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        c, _ = codebook(b, d)
        c_hat[..., start:start + size] = c[idx[..., start:start + size]]
        start += size
    perm = permutation(fmt, head)
    r = np.empty(u.shape, dtype=np.float64)
    r[..., perm] = u - c_hat                       # back to rotated coordinate order
    g16 = fp16_round(np.sqrt(np.sum(r * r, axis=-1)))
    proj = r @ qjl_matrix(fmt).T                    # (S r)_i
    signs = (proj >= 0).astype(np.int64)
    return idx, n16, u, signs, g16


def boundary_margin(u, fmt: Format):
    """Per position: |u - nearest boundary| / max(|boundary|, 1/sqrt(d)).

    Reading of the tolerance "within 1e-5 relative of a codebook boundary": the
    zero boundary of even codebooks is measured against 1/sqrt(d).
    """
    u = np.asarray(u, dtype=np.float64)
    d = fmt.head_dim
    out = np.empty(u.shape)
    start = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        _, beta = codebook(b, size if fmt.groupwise else d)
        seg = u[..., start:start + size, None]
        dist = np.abs(seg - beta) / np.maximum(np.abs(beta), 1.0 / math.sqrt(d))
        out[..., start:start + size] = dist.min(axis=-1)
        start += size
    return out


def _fp16_bytes(n16):
    return np.asarray(n16, dtype=np.float64).astype(np.float16).view(np.uint8).reshape(np.shape(n16) + (2,))


def _bits(seg, b):
    """LSB-first bitstream bytes of the indices seg[..., n] at b bits each."""
    seg = np.asarray(seg, dtype=np.int64)
    if np.any(seg < 0) or np.any(seg >= (1 << b)):
        raise ValueError("index out of range for its group")
    bits = (seg[..., :, None] >> np.arange(b)) & 1
    return np.packbits(bits.reshape(seg.shape[:-1] + (seg.shape[-1] * b,)).astype(np.uint8), axis=-1,
                       bitorder="little")


def _unbits(data, n, b):
    bits = np.unpackbits(np.asarray(data, dtype=np.uint8), axis=-1, bitorder="little")
    bits = bits.reshape(data.shape[:-1] + (n, b))
    return (bits.astype(np.int64) << np.arange(b)).sum(axis=-1)


def encode_rows(idx, n16, fmt: Format, signs=None, g16=None) -> np.ndarray:
    """Pack indices (packed order) and fp16 norms into rows of ``row_bytes`` (R6; R16 with QJL;
    R18 for the recipe row, in its printed field order)."""
    idx = np.asarray(idx, dtype=np.int64)
    if recipe(fmt):
        if signs is None or g16 is None:
            raise ValueError("the recipe row needs the signs and the residual norms")
        n16, g16 = np.asarray(n16, dtype=np.float64), np.asarray(g16, dtype=np.float64)
        parts, start = [], 0
        for g, (b, size) in enumerate(zip(fmt.group_bits, fmt.group_size)):
            parts.append(_bits(idx[..., start:start + size], b))
            parts.append(_bits(np.asarray(signs)[..., start:start + size], 1))
            parts += [_fp16_bytes(n16[..., g]), _fp16_bytes(g16[..., g])]
            start += size
        return np.concatenate(parts, axis=-1)
    lead = idx.shape[:-1]
    parts = []
    start = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        if b == 16:
            raise ValueError("16-bit indices are a diagnostic codebook without a row format")
        seg = idx[..., start:start + size]
        if np.any(seg < 0) or np.any(seg >= (1 << b)):
            raise ValueError("index out of range for its group")
        bits = (seg[..., :, None] >> np.arange(b)) & 1  # LSB-first within each index
        parts.append(np.packbits(bits.reshape(lead + (size * b,)).astype(np.uint8), axis=-1, bitorder="little"))
        start += size
    if fmt.qjl:
        if signs is None or g16 is None:
            raise ValueError("a QJL format needs the signs and the residual norm")
        parts.append(np.packbits(np.asarray(signs, dtype=np.uint8), axis=-1, bitorder="little"))
    if fmt.groupwise:
        n16 = np.asarray(n16, dtype=np.float64)
        parts += [_fp16_bytes(n16[..., 0]), _fp16_bytes(n16[..., 1])]
        return np.concatenate(parts, axis=-1)
    parts.append(_fp16_bytes(n16))
    if fmt.qjl:
        parts.append(_fp16_bytes(g16))
    return np.concatenate(parts, axis=-1)


def decode_rows(rows, fmt: Format):
    """Inverse of ``encode_rows``: (idx in packed order, n16 as fp64), and with QJL
    also (signs in {0, 1}, g16 as fp64)."""
    rows = np.asarray(rows, dtype=np.uint8)
    lead = rows.shape[:-1]
    if rows.shape[-1] != row_bytes(fmt):
        raise ValueError("row length does not match the format")
    if recipe(fmt):
        idx, signs, n16, g16, off = [], [], [], [], 0
        for b, size in zip(fmt.group_bits, fmt.group_size):
            idx.append(_unbits(rows[..., off:off + size * b // 8], size, b))
            off += size * b // 8
            signs.append(_unbits(rows[..., off:off + size // 8], size, 1))
            off += size // 8
            n16.append(rows[..., off:off + 2].copy().view(np.float16).reshape(lead).astype(np.float64))
            g16.append(rows[..., off + 2:off + 4].copy().view(np.float16).reshape(lead).astype(np.float64))
            off += 4
        return (np.concatenate(idx, axis=-1), np.stack(n16, axis=-1), np.concatenate(signs, axis=-1),
                np.stack(g16, axis=-1))
    idx = []
    off = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        nbytes = size * b // 8
        bits = np.unpackbits(rows[..., off:off + nbytes], axis=-1, bitorder="little").reshape(lead + (size, b))
        idx.append((bits.astype(np.int64) << np.arange(b)).sum(axis=-1))
        off += nbytes
    if fmt.qjl:
        nb = fmt.head_dim // 8
        signs = np.unpackbits(rows[..., off:off + nb], axis=-1, bitorder="little").astype(np.int64)
        off += nb
    if fmt.groupwise:
        n16 = rows[..., off:off + 4].copy().view(np.float16).reshape(lead + (2,)).astype(np.float64)
        return np.concatenate(idx, axis=-1), n16
    n16 = rows[..., off:off + 2].copy().view(np.float16).reshape(lead).astype(np.float64)
    if fmt.qjl:
        g16 = rows[..., off + 2:off + 4].copy().view(np.float16).reshape(lead).astype(np.float64)
        return np.concatenate(idx, axis=-1), n16, signs, g16
    return np.concatenate(idx, axis=-1), n16


def dequantize_rows(idx, n16, fmt: Format, head: int, signs=None, g16=None):
    """x_hat = n16 * s * (H c_hat) / sqrt(d), c_hat placed back at the rotated coordinates.

    With QJL (R16) c_hat gains sqrt(pi/2) / d * g16 * S^T z: the vector whose
    product with any q is the unbiased estimate of q . x.
    """
    idx = np.asarray(idx, dtype=np.int64)
    d = fmt.head_dim
    if recipe(fmt):  # R18: per group c_g + sqrt(pi/2)/n_g gamma_g S_g^T z_g, scaled by n_g, then R^T
        if signs is None or g16 is None:
            raise ValueError("the recipe row needs the signs and the residual norms")
        vals = np.empty(idx.shape, dtype=np.float64)
        start = 0
        for g, (b, size) in enumerate(zip(fmt.group_bits, fmt.group_size)):
            c, _ = codebook(b, size)
            z = 2.0 * np.asarray(signs, dtype=np.float64)[..., start:start + size] - 1.0
            gam = np.asarray(g16, dtype=np.float64)[..., g:g + 1]
            seg = c[idx[..., start:start + size]] + (math.sqrt(math.pi / 2.0) / size) * gam * (
                z @ recipe_qjl_matrix(fmt, g))
            vals[..., start:start + size] = seg * np.asarray(n16, dtype=np.float64)[..., g:g + 1]
            start += size
        return vals @ group_rotation(fmt, head)
    vals = np.empty(idx.shape, dtype=np.float64)
    start = 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        c, _ = codebook(b, size if fmt.groupwise else d)
        vals[..., start:start + size] = c[idx[..., start:start + size]]
        if fmt.groupwise:  # R17: each group scaled by its own norm, then R^T back to the channels
            gi = 0 if start == 0 else 1
            vals[..., start:start + size] *= np.asarray(n16, dtype=np.float64)[..., gi:gi + 1]
        start += size
    if fmt.groupwise:
        return vals @ group_rotation(fmt, head)
    rot = np.empty_like(vals)
    rot[..., permutation(fmt, head)] = vals
    if fmt.qjl:
        if signs is None or g16 is None:
            raise ValueError("a QJL format needs the signs and the residual norm")
        z = 2.0 * np.asarray(signs, dtype=np.float64) - 1.0
        rot = rot + (math.sqrt(math.pi / 2.0) / d) * np.asarray(g16, dtype=np.float64)[..., None] * (
            z @ qjl_matrix(fmt))
    return np.asarray(n16, dtype=np.float64)[..., None] * unrotate(rot, hadamard_signs(fmt.seed, d))


# ---------------------------------------------------------------------------
# Page writes (serving route contract)
# ---------------------------------------------------------------------------

def subpage_bytes(fmt: Format, block_size: int) -> int:
    return block_size * row_bytes(fmt)


def subpage_byte_order(fmt: Format) -> np.ndarray:
    """Logical row bytes in the order a sub-page stores them: the first index_bytes(fmt) go to
    the row's place in the index area, the rest to its place in the norm area (R6). For the recipe
    row (R18) that is each group's [indices][signs], then each group's (norm, residual norm)."""
    if not recipe(fmt):
        return np.arange(row_bytes(fmt))
    heads, tails, off = [], [], 0
    for b, size in zip(fmt.group_bits, fmt.group_size):
        a = size * b // 8 + size // 8
        heads.append(np.arange(off, off + a))
        tails.append(np.arange(off + a, off + a + 4))
        off += a + 4
    return np.concatenate(heads + tails)


def write_rows(pages, blocks, head: int, offsets, rows, fmt: Format, block_size: int):
    """Store logical rows at (block, offset) of one head's sub-pages (R6 layout)."""
    ib, nb = index_bytes(fmt), norm_bytes(fmt)
    blocks = np.asarray(blocks, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.uint8)[..., subpage_byte_order(fmt)]
    cols = offsets[:, None] * ib + np.arange(ib)[None, :]
    pages[blocks[:, None], head, cols] = rows[:, :ib]
    ncols = block_size * ib + nb * offsets[:, None] + np.arange(nb)[None, :]
    pages[blocks[:, None], head, ncols] = rows[:, ib:]


def read_rows(pages, blocks, head: int, offsets, fmt: Format, block_size: int):
    """Logical rows [n][row_bytes] at (block, offset) of one head's sub-pages."""
    ib, nb = index_bytes(fmt), norm_bytes(fmt)
    blocks = np.asarray(blocks, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    cols = offsets[:, None] * ib + np.arange(ib)[None, :]
    ncols = block_size * ib + nb * offsets[:, None] + np.arange(nb)[None, :]
    stored = np.concatenate((pages[blocks[:, None], head, cols], pages[blocks[:, None], head, ncols]), axis=-1)
    rows = np.empty_like(stored)
    rows[..., subpage_byte_order(fmt)] = stored
    return rows


def pack_kv(k, v, slot_mapping, kfmt: Format, vfmt: Format, num_blocks: int, block_size: int,
            k_pages=None, v_pages=None):
    """Quantize and write K and V rows into page pools.

    TurboQuant "Design" page, "Serving Route Design": rows go to
    pages[slot // block_size][head][slot % block_size]. Pools are created
    zeroed when not given; rows of padding tokens (slot < 0) are not written.
    Raises IndexError for a slot past the pool ("Error Model").
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    slots = np.asarray(slot_mapping, dtype=np.int64)
    T, H, d = k.shape
    if v.shape != k.shape or slots.shape != (T,):
        raise ValueError("k, v must be [T][H_kv][d] and slot_mapping [T]")
    if np.any(slots >= num_blocks * block_size):
        raise IndexError("slot mapping points outside the allocated pages")
    if k_pages is None:
        k_pages = np.zeros((num_blocks, H, subpage_bytes(kfmt, block_size)), dtype=np.uint8)
    if v_pages is None:
        v_pages = np.zeros((num_blocks, H, subpage_bytes(vfmt, block_size)), dtype=np.uint8)
    live = np.nonzero(slots >= 0)[0]
    blk = slots[live] // block_size
    off = slots[live] % block_size
    for h in range(H):
        for src, fmt, pages in ((k, kfmt, k_pages), (v, vfmt, v_pages)):
            if fmt.qjl:
                idx, n16, _, signs, g16 = quantize_qjl(src[live, h, :], fmt, h)
                rows = encode_rows(idx, n16, fmt, signs, g16)
            else:
                idx, n16, _ = quantize(src[live, h, :], fmt, h)
                rows = encode_rows(idx, n16, fmt)
            write_rows(pages, blk, h, off, rows, fmt, block_size)
    return k_pages, v_pages


def read_row(pages, slot: int, head: int, block_size: int, fmt: Format):
    """Row bytes of one token, by the page address formula."""
    return read_rows(pages, [slot // block_size], head, [slot % block_size], fmt, block_size)[0]


# ---------------------------------------------------------------------------
# Decode attention (dense reconstruction: diagnostic route only)
# ---------------------------------------------------------------------------

def _gather_rows(pages, block_table, count: int, head: int, block_size: int, fmt: Format):
    i = np.arange(count)
    blocks = np.asarray(block_table, dtype=np.int64)[i // block_size]
    return read_rows(pages, blocks, head, i % block_size, fmt, block_size)


def decode_attention(q, k_pages, v_pages, block_tables, seq_lens, k_win, v_win, window: int,
                     scale: float, kfmt: Format, vfmt: Format, block_size: int, batch=None):
    """Single-token decode attention over packed pages plus the dense window, in fp64.

    For each sequence b and query head g (KV head g // G), the keys and values
    are the dequantized packed tokens 0..P_b-1, read through the block table,
    followed by the bf16 window tokens (R7). out = softmax(scale q.k) @ v.
    A sequence with no tokens gets a zero output. Returns out[B][H_q][d] for
    the sequences in ``batch`` (all by default).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    H = kfmt.num_kv_heads
    if Hq % H:
        raise ValueError("H_q must be a multiple of H_kv")
    G = Hq // H
    batch = range(B) if batch is None else batch
    out = np.zeros((len(batch), Hq, d))
    for ob, b in enumerate(batch):
        L = int(seq_lens[b])
        n_win = min(window, L)
        P = L - n_win
        for h in range(H):
            kd = decode_rows(_gather_rows(k_pages, block_tables[b], P, h, block_size, kfmt), kfmt)
            vd = decode_rows(_gather_rows(v_pages, block_tables[b], P, h, block_size, vfmt), vfmt)
            keys = dequantize_rows(kd[0], kd[1], kfmt, h, *kd[2:])  # (signs, g16) follow with QJL
            vals = dequantize_rows(vd[0], vd[1], vfmt, h, *vd[2:])
            if n_win:
                keys = np.concatenate((keys, np.asarray(k_win[b, h, :n_win], dtype=np.float64)))
                vals = np.concatenate((vals, np.asarray(v_win[b, h, :n_win], dtype=np.float64)))
            if L == 0:
                continue  # an empty history attends to nothing: the output stays zero
            for g in range(G):
                out[ob, h * G + g] = dense_attention(q[b, h * G + g], keys, vals, scale)
    return out


def boundary_dense_tokens(L: int, sinks: int, window: int):
    """Token positions kept dense under boundary-token preservation (R14).

    The policy keeps some boundary tokens dense next to the recent window
    (TurboQuant "Design" page, "Format Strategy"); which tokens is not stated.
    Reading: the first min(sinks, L) tokens and the last min(window, L - that)
    tokens stay dense bf16; the tokens between them are packed. Returns
    (dense positions in order, first packed position, packed count). The dense
    positions are what the decode call's window buffer holds, in this order,
    with window = sinks + window.
    """
    s = min(sinks, L)
    w = min(window, L - s)
    P = L - s - w
    dense = list(range(s)) + list(range(s + P, L))
    return dense, s, P


def dense_attention(q, keys, vals, scale: float):
    """softmax(scale * keys @ q) @ vals in fp64 (max-subtracted)."""
    s = scale * (np.asarray(keys, dtype=np.float64) @ np.asarray(q, dtype=np.float64))
    if s.size == 0:
        raise ValueError("attention over an empty history")
    p = np.exp(s - s.max())
    return (p / p.sum()) @ np.asarray(vals, dtype=np.float64)


# ---------------------------------------------------------------------------
# Byte ledger (System Invariants: storage and metadata reported separately)
# ---------------------------------------------------------------------------

@dataclass
class Ledger:
    dense_bytes: int
    index_bytes: int
    norm_bytes: int
    codebook_bytes: int
    transform_bytes: int
    window_bytes: int
    block_table_bytes: int
    workspace_bytes: int
    page_pool_bytes: int

    @property
    def metadata_bytes(self) -> int:
        return (self.norm_bytes + self.codebook_bytes + self.transform_bytes + self.window_bytes
                + self.block_table_bytes + self.workspace_bytes)

    @property
    def all_in_ratio(self) -> float:
        return self.dense_bytes / (self.index_bytes + self.metadata_bytes)


def byte_ledger(kfmt: Format, vfmt: Format, seq_lens: Sequence[int], window: int, block_size: int,
                num_blocks: int, workspace_bytes: int = 0) -> Ledger:
    """Plain byte arithmetic for one layer's cache.

    dense: bf16 K and V of every token. index: packed index bytes (with QJL
    also the sign bytes) of the packed tokens. norms: 2 bytes per packed row
    (4 with QJL: the residual norm too), K and V. codebooks: fp16 centroids
    and fp32 boundaries of every group of both codecs. transforms: d int8 signs
    and H_kv*d int16 permutation entries per codec, plus the fp32 d x d QJL
    matrix of a QJL codec (one n_g x n_g S_g per group for the recipe row,
    R18), plus for a group-wise codec (R17) its per-head
    rotation held as a dense fp32 d x d matrix R_h per KV head ("System
    Invariants": the all-in ratio counts transforms). window: the allocated
    bf16 window, K and V. block tables: one int32 per used block.
    """
    H, d = kfmt.num_kv_heads, kfmt.head_dim
    lens = [int(x) for x in seq_lens]
    packed = [L - min(window, L) for L in lens]
    P = sum(packed)
    dense = 2 * 2 * H * d * sum(lens)
    idx = P * H * (index_bytes(kfmt) + index_bytes(vfmt))
    norms = P * H * (norm_bytes(kfmt) + norm_bytes(vfmt))
    cb = 0
    for fmt in (kfmt, vfmt):
        for b in fmt.group_bits:
            cb += (1 << b) * 2 + ((1 << b) - 1) * 4
    transforms = 2 * (d + H * d * 2)
    for fmt in (kfmt, vfmt):
        if fmt.qjl:  # S (R16), or one S_g per group for the recipe row (R18)
            transforms += sum(4 * n * n for n in fmt.group_size) if fmt.groupwise else 4 * d * d
        if fmt.groupwise:
            transforms += 4 * H * d * d
    win = 2 * 2 * len(lens) * H * window * d
    bt = 4 * sum(-(-p // block_size) for p in packed)
    pool = num_blocks * H * block_size * (row_bytes(kfmt) + row_bytes(vfmt))
    return Ledger(dense, idx, norms, cb, transforms, win, bt, int(workspace_bytes), pool)
