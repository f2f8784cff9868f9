"""Thin ctypes binding of libtq (include/tq.h): argument marshalling only.

Every step of the pack and decode path runs in the CUDA library; this module
checks tensor dtypes, shapes and devices, passes raw pointers and the current
CUDA stream, and maps status codes to exceptions following the TurboQuant
"Design" page, "Error Model" (ValueError, IndexError, FileNotFoundError,
UnsupportedFormatError). There is no fallback: if libtq.so is missing or no
CUDA device is present, the calls raise.
"""

from __future__ import annotations

import ctypes
import json
import os
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_ERR_VALUE, TQ_ERR_INDEX, TQ_ERR_NOT_FOUND, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA, TQ_ERR_TIMEOUT = range(7)
TQ_DERR_SLOT, TQ_DERR_BLOCK, TQ_DERR_TIMEOUT, TQ_DERR_LAUNCH = 1, 2, 4, 8
HEAD_DIM = 128


class UnsupportedFormatError(Exception):
    """The kernels do not implement the requested format (no silent fallback)."""


class TQTimeoutError(RuntimeError):
    """A bounded wait inside a kernel expired."""


class TQCudaError(RuntimeError):
    """A CUDA runtime call inside the library failed."""


class _FormatDesc(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("group_bits", ctypes.c_int32 * 2), ("group_size", ctypes.c_int32 * 2),
                ("high_coords", ctypes.POINTER(ctypes.c_int16)), ("hadamard_seed", ctypes.c_uint64),
                ("qjl", ctypes.c_int32), ("groupwise", ctypes.c_int32)]


class _Ledger(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "dense_bytes", "index_bytes", "norm_bytes", "codebook_bytes", "transform_bytes", "window_bytes",
        "block_table_bytes", "workspace_bytes", "page_pool_bytes", "metadata_bytes")] + \
        [("index_only_ratio", ctypes.c_double), ("all_in_ratio", ctypes.c_double)]


_lib = None
_VP, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t


def lib():
    """Load libtq.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with quantized_paged_kv_pack_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        L.tq_last_error.restype = ctypes.c_char_p
        L.tq_codec_host_tables.argtypes = [P(_FormatDesc), _VP, _VP, _VP, _VP, _VP]
        L.tq_codec_qjl_matrix.argtypes = [P(_FormatDesc), _VP]
        L.tq_codec_group_rotation.argtypes = [P(_FormatDesc), _VP]
        L.tq_make_codec.argtypes = [P(_FormatDesc), P(_VP)]
        L.tq_free_codec.argtypes = [_VP]
        L.tq_free_codec.restype = None
        L.tq_codec_row_bytes.argtypes = [_VP]
        L.tq_codec_row_bytes.restype = _I32
        L.tq_pack_kv.argtypes = [_VP, _VP, _VP, _VP, _VP, _I64, _VP, _VP, _I64, _I32, _VP, _VP]
        L.tq_decode_workspace_bytes.argtypes = [_I32, _I32, _I32, _I32, _I32]
        L.tq_decode_workspace_bytes.restype = _SZ
        dec = [_VP, _VP, _VP, _VP, _VP, _VP, _I32, _VP, _I32, _I32, _I32, _VP, _VP, _I32, ctypes.c_float, _I64, _I32]
        L.tq_decode_paged.argtypes = dec + [_VP, _VP, _SZ, _VP, _VP]
        L.tq_decode_partials.argtypes = dec + [_VP, _SZ, _VP, _VP]
        L.tq_decode_combine.argtypes = [_VP, _VP, _I32, _I32, _I32, _I32, _I32, _VP, _VP, _SZ, _VP]
        L.tq_decode_paged_static.argtypes = dec + [_VP, _VP, _VP]
        L.tq_static_workspace_bytes.argtypes = []
        L.tq_static_workspace_bytes.restype = _SZ
        L.tq_window_append.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _I32, _I32, _VP, _VP, _I32, _VP, _VP, _I64,
                                       _I32, _I32, _VP, _VP]
        L.tq_window_append_decode.argtypes = [_VP, _VP, _VP, _VP, _VP, _VP, _I32, _I32, _VP, _VP, _VP, _VP, _I32,
                                              _VP, _I32, _I32, _I32, ctypes.c_float, _I64, _I32, _VP, _VP, _SZ,
                                              _VP, _VP]
        L.tq_byte_ledger.argtypes = [P(_FormatDesc), P(_FormatDesc), _I32, _VP, _I32, _I32, _I32, _I64, _I32,
                                     P(_Ledger)]
        for name in ("tq_codec_host_tables", "tq_codec_qjl_matrix", "tq_codec_group_rotation", "tq_make_codec", "tq_pack_kv", "tq_decode_paged",
                     "tq_decode_partials", "tq_decode_combine", "tq_byte_ledger", "tq_decode_paged_static",
                     "tq_window_append", "tq_window_append_decode"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(status: int):
    if status == TQ_OK:
        return
    msg = lib().tq_last_error().decode()
    if status == TQ_ERR_VALUE:
        raise ValueError(msg)
    if status == TQ_ERR_INDEX:
        raise IndexError(msg)
    if status == TQ_ERR_NOT_FOUND:
        raise FileNotFoundError(msg)
    if status == TQ_ERR_UNSUPPORTED:
        raise UnsupportedFormatError(msg)
    if status == TQ_ERR_TIMEOUT:
        raise TQTimeoutError(msg)
    raise TQCudaError(msg or f"tq status {status}")


def _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, qjl=False, groupwise=False):
    bits, sizes = tuple(group_bits), tuple(group_size)
    d = _FormatDesc()
    d.head_dim, d.num_kv_heads, d.n_groups = head_dim, num_kv_heads, len(bits)
    if len(bits) not in (1, 2) or len(sizes) != len(bits):
        raise ValueError("one or two channel groups with matching sizes")
    for i in range(len(bits)):
        d.group_bits[i], d.group_size[i] = bits[i], sizes[i]
    keep = None
    if high_coords is not None:
        keep = np.ascontiguousarray(np.asarray(high_coords, dtype=np.int16))
        d.high_coords = keep.ctypes.data_as(ctypes.POINTER(ctypes.c_int16))
    d.hadamard_seed = int(seed) & ((1 << 64) - 1)
    d.qjl = 1 if qjl else 0
    d.groupwise = 1 if groupwise else 0
    return d, keep


def codec_host_tables(head_dim, num_kv_heads, group_bits, group_size, high_coords=None, seed=0, qjl=False,
                      groupwise=False):
    """Host-side codec tables (no CUDA call): codebooks, signs, permutation, row bytes."""
    d, keep = _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, qjl, groupwise)
    c16 = np.zeros((2, 16), np.uint16)
    bnd = np.zeros((2, 15), np.float32)
    sg = np.zeros(head_dim, np.int8)
    perm = np.zeros((num_kv_heads, head_dim), np.int16)
    rb = ctypes.c_int32()
    _check(lib().tq_codec_host_tables(ctypes.byref(d), c16.ctypes.data, bnd.ctypes.data, sg.ctypes.data,
                                      perm.ctypes.data, ctypes.addressof(rb)))
    del keep
    return {"centroids_f16": c16, "boundaries": bnd, "signs": sg, "perm": perm, "row_bytes": rb.value}


def qjl_matrix(head_dim, num_kv_heads, group_bits, group_size, high_coords=None, seed=0) -> np.ndarray:
    """The QJL matrix S of a codec (tq_codec_qjl_matrix), float32 [head_dim][head_dim]; host only."""
    d, keep = _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, True)
    out = np.zeros((head_dim, head_dim), np.float32)
    _check(lib().tq_codec_qjl_matrix(ctypes.byref(d), out.ctypes.data))
    del keep
    return out


def recipe_qjl_matrices(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed=0):
    """S_0 and S_1 of a recipe-row codec (qjl and groupwise; tq_codec_qjl_matrix), float32
    [group_size[g]][group_size[g]] each; host only."""
    d, keep = _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, True, True)
    out = np.zeros(head_dim * head_dim, np.float32)
    _check(lib().tq_codec_qjl_matrix(ctypes.byref(d), out.ctypes.data))
    del keep
    n0, n1 = group_size
    return out[:n0 * n0].reshape(n0, n0), out[n0 * n0:n0 * n0 + n1 * n1].reshape(n1, n1)


def group_rotation(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed=0) -> np.ndarray:
    """R_h of a group-wise codec (tq_codec_group_rotation), float32 [H][head_dim][head_dim]; host only."""
    d, keep = _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, False, True)
    out = np.zeros((num_kv_heads, head_dim, head_dim), np.float32)
    _check(lib().tq_codec_group_rotation(ctypes.byref(d), out.ctypes.data))
    del keep
    return out


class Codec:
    """A device codec (tq_make_codec); immutable, freed on close()."""

    def __init__(self, num_kv_heads: int, group_bits: Sequence[int], group_size: Sequence[int],
                 high_coords=None, seed: int = 0, head_dim: int = HEAD_DIM, qjl: bool = False,
                 groupwise: bool = False):
        self.head_dim, self.num_kv_heads = head_dim, num_kv_heads
        self.group_bits, self.group_size, self.seed = tuple(group_bits), tuple(group_size), seed
        self.qjl, self.groupwise = bool(qjl), bool(groupwise)
        self.high_coords = None if high_coords is None else np.asarray(high_coords, dtype=np.int16)
        d, keep = _desc(head_dim, num_kv_heads, group_bits, group_size, high_coords, seed, qjl, groupwise)
        h = _VP()
        _check(lib().tq_make_codec(ctypes.byref(d), ctypes.byref(h)))
        del keep
        self._h = h
        self.row_bytes = lib().tq_codec_row_bytes(h)

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("codec is closed")
        return self._h

    def desc(self):
        return _desc(self.head_dim, self.num_kv_heads, self.group_bits, self.group_size, self.high_coords, self.seed,
                     self.qjl, self.groupwise)

    def close(self):
        if getattr(self, "_h", None) is not None:
            lib().tq_free_codec(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def load_recipe_metadata(path: str) -> dict:
    """Read a recipe metadata JSON (sorted high-precision channel indices per KV head).

    TurboQuant "Design" page, "Recipe Strategy": activation energy -> sorted
    high-precision indices -> metadata JSON; runtime loads and validates it.
    "Error Model": a missing file raises FileNotFoundError. The keys are
    head_dim, num_kv_heads, group_bits, group_size, high_coords, hadamard_seed,
    and optionally qjl and groupwise (booleans).
    """
    if not os.path.exists(path):
        raise FileNotFoundError(f"recipe metadata not found: {path}")
    with open(path) as f:
        meta = json.load(f)
    try:
        spec = dict(head_dim=int(meta["head_dim"]), num_kv_heads=int(meta["num_kv_heads"]),
                    group_bits=tuple(meta["group_bits"]), group_size=tuple(meta["group_size"]),
                    high_coords=None if meta.get("high_coords") is None else np.asarray(meta["high_coords"], np.int16),
                    seed=int(meta.get("hadamard_seed", 0)), qjl=bool(meta.get("qjl", False)),
                    groupwise=bool(meta.get("groupwise", False)))
    except (KeyError, TypeError) as e:
        raise ValueError(f"malformed recipe metadata: {e}") from e
    codec_host_tables(spec["head_dim"], spec["num_kv_heads"], spec["group_bits"], spec["group_size"],
                      spec["high_coords"], spec["seed"], spec["qjl"], spec["groupwise"])  # validates
    return spec


def slice_recipe(spec: dict, rank: int, world: int) -> dict:
    """The recipe of one tensor-parallel partition of the KV heads.

    TurboQuant "Design" page, "Recipe Strategy": the runtime slices the
    metadata by tensor-parallel partition. KV heads are split into `world`
    contiguous ranges; partition `rank` keeps heads [rank H/world, (rank+1)
    H/world) and their rows of high_coords. The sign seed is shared, so every
    partition rotates as the whole model does.
    """
    H = int(spec["num_kv_heads"])
    if world < 1 or H % world:
        raise ValueError(f"num_kv_heads {H} does not split into {world} partitions")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    n = H // world
    out = dict(spec)
    out["num_kv_heads"] = n
    if spec.get("high_coords") is not None:
        out["high_coords"] = np.ascontiguousarray(np.asarray(spec["high_coords"])[rank * n:(rank + 1) * n])
    codec_host_tables(spec["head_dim"], n, spec["group_bits"], spec["group_size"], out.get("high_coords"),
                      spec.get("seed", 0), spec.get("qjl", False), spec.get("groupwise", False))  # validates
    return out


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def page_pool(codec: Codec, num_blocks: int, block_size: int, device="cuda") -> torch.Tensor:
    """Zeroed uint8 pool [num_blocks][H_kv][block_size * row_bytes] (one sub-page per block and head)."""
    return torch.zeros(num_blocks, codec.num_kv_heads, block_size * codec.row_bytes, dtype=torch.uint8,
                       device=device)


def _pools(kc, vc, k_pages, v_pages, block_size):
    if k_pages.dim() != 3 or v_pages.dim() != 3:
        raise ValueError("page pools must be [num_blocks][H_kv][block_size * row_bytes]")
    if block_size < 1:
        raise ValueError("block_size must be positive")
    nb = k_pages.shape[0]
    _need(k_pages, torch.uint8, (nb, kc.num_kv_heads, block_size * kc.row_bytes), "k_pages")
    _need(v_pages, torch.uint8, (nb, vc.num_kv_heads, block_size * vc.row_bytes), "v_pages")
    return nb


def pack_kv(kc: Codec, vc: Codec, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
            k_pages: torch.Tensor, v_pages: torch.Tensor, block_size: int, d_err: Optional[torch.Tensor] = None,
            stream=None):
    """Quantize and write K/V rows into the page pools (tq_pack_kv)."""
    T = k.shape[0] if k.dim() == 3 else -1
    H = kc.num_kv_heads
    _need(k, torch.bfloat16, (T, H, kc.head_dim), "k")
    _need(v, torch.bfloat16, (T, H, kc.head_dim), "v")
    _need(slot_mapping, torch.int64, (T,), "slot_mapping")
    nb = _pools(kc, vc, k_pages, v_pages, block_size)
    bs = int(block_size)
    if d_err is not None:
        _need(d_err, torch.int32, (1,), "d_err")
    _check(lib().tq_pack_kv(kc.handle, vc.handle, _ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_pages),
                            _ptr(v_pages), nb, bs, _ptr(d_err), _stream(stream)))


def window_append(kc: Codec, vc: Codec, k_new: torch.Tensor, v_new: torch.Tensor, k_win: Optional[torch.Tensor],
                  v_win: Optional[torch.Tensor], window: int, sinks: int, seq_lens: torch.Tensor,
                  block_tables: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_size: int,
                  d_err: Optional[torch.Tensor] = None, stream=None):
    """Append one token per sequence, evicting the oldest window token into the pages (tq_window_append).

    ``k_win``/``v_win`` are [B][H][sinks + window][d] dense buffers (updated in
    place); ``seq_lens`` holds the lengths before the append and is not changed.
    """
    B = k_new.shape[0] if k_new.dim() == 3 else -1
    H = kc.num_kv_heads
    _need(k_new, torch.bfloat16, (B, H, kc.head_dim), "k_new")
    _need(v_new, torch.bfloat16, (B, H, kc.head_dim), "v_new")
    dense = int(window) + int(sinks)
    if dense > 0:
        if k_win is None or v_win is None:
            raise ValueError("sinks + window > 0 needs the dense buffers")
        _need(k_win, torch.bfloat16, (B, H, dense, kc.head_dim), "k_win")
        _need(v_win, torch.bfloat16, (B, H, dense, kc.head_dim), "v_win")
    _need(seq_lens, torch.int32, (B,), "seq_lens")
    if block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("block_tables must be [batch][max_blocks_per_seq]")
    _need(block_tables, torch.int32, (B, block_tables.shape[1]), "block_tables")
    nb = _pools(kc, vc, k_pages, v_pages, block_size)
    if d_err is not None:
        _need(d_err, torch.int32, (1,), "d_err")
    _check(lib().tq_window_append(kc.handle, vc.handle, _ptr(k_new), _ptr(v_new), _ptr(k_win), _ptr(v_win),
                                  int(window), int(sinks), _ptr(seq_lens), _ptr(block_tables),
                                  int(block_tables.shape[1]), _ptr(k_pages), _ptr(v_pages), nb, int(block_size), B,
                                  _ptr(d_err), _stream(stream)))


def window_append_decode(kc: Codec, vc: Codec, k_new: torch.Tensor, v_new: torch.Tensor,
                         k_win: Optional[torch.Tensor], v_win: Optional[torch.Tensor], window: int, sinks: int,
                         q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, block_size: int,
                         block_tables: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int, softmax_scale: float,
                         out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                         d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One decode step (tq_window_append_decode): window_append, then decode_paged with window
    sinks + window and the same seq_lens, in fewer launches; returns fp32 [B][H_q][d]."""
    if q.dim() != 3:
        raise ValueError("q must be [batch][num_q_heads][head_dim]")
    B, Hq, d = q.shape
    H = kc.num_kv_heads
    _need(q, torch.bfloat16, (B, Hq, kc.head_dim), "q")
    _need(k_new, torch.bfloat16, (B, H, kc.head_dim), "k_new")
    _need(v_new, torch.bfloat16, (B, H, kc.head_dim), "v_new")
    dense = int(window) + int(sinks)
    if dense > 0:
        if k_win is None or v_win is None:
            raise ValueError("sinks + window > 0 needs the dense buffers")
        _need(k_win, torch.bfloat16, (B, H, dense, kc.head_dim), "k_win")
        _need(v_win, torch.bfloat16, (B, H, dense, kc.head_dim), "v_win")
    else:
        k_win = v_win = None
    _need(seq_lens, torch.int32, (B,), "seq_lens")
    if block_tables.dim() != 2:
        raise ValueError("block_tables must be [batch][max_blocks_per_seq]")
    _need(block_tables, torch.int32, (B, block_tables.shape[1]), "block_tables")
    nb = _pools(kc, vc, k_pages, v_pages, block_size)
    bs = int(block_size)
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (B, Hq, d), "out")
    if workspace is None:
        workspace = alloc_workspace(B, Hq, H, max_seq_len, bs, device=q.device)
    if d_err is not None:
        _need(d_err, torch.int32, (1,), "d_err")
    _check(lib().tq_window_append_decode(kc.handle, vc.handle, _ptr(k_new), _ptr(v_new), _ptr(k_win), _ptr(v_win),
                                         int(window), int(sinks), _ptr(q), _ptr(k_pages), _ptr(v_pages),
                                         _ptr(block_tables), int(block_tables.shape[1]), _ptr(seq_lens), B, Hq,
                                         int(max_seq_len), float(softmax_scale), nb, bs, _ptr(out), _ptr(workspace),
                                         workspace.numel(), _ptr(d_err), _stream(stream)))
    return out


def decode_workspace_bytes(batch: int, num_q_heads: int, num_kv_heads: int, max_seq_len: int, block_size: int) -> int:
    return int(lib().tq_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, max_seq_len, block_size))


def alloc_workspace(batch, num_q_heads, num_kv_heads, max_seq_len, block_size, device="cuda") -> torch.Tensor:
    n = decode_workspace_bytes(batch, num_q_heads, num_kv_heads, max_seq_len, block_size)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def decode_paged(kc: Codec, vc: Codec, q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                 block_size: int, block_tables: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                 k_win: Optional[torch.Tensor], v_win: Optional[torch.Tensor], window: int,
                 softmax_scale: float, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 d_err: Optional[torch.Tensor] = None, stream=None, phase: str = "all") -> torch.Tensor:
    """Decode attention over packed pages (tq_decode_paged); returns fp32 [B][H_q][d].

    ``phase`` is "all" (tq_decode_paged), "partials" or "combine" (the two
    halves, for timing them apart).
    """
    if q.dim() != 3:
        raise ValueError("q must be [batch][num_q_heads][head_dim]")
    B, Hq, d = q.shape
    H = kc.num_kv_heads
    _need(q, torch.bfloat16, (B, Hq, kc.head_dim), "q")
    nb = _pools(kc, vc, k_pages, v_pages, block_size)
    bs = int(block_size)
    if block_tables.dim() != 2:
        raise ValueError("block_tables must be [batch][max_blocks_per_seq]")
    _need(block_tables, torch.int32, (B, block_tables.shape[1]), "block_tables")
    _need(seq_lens, torch.int32, (B,), "seq_lens")
    if window > 0:
        _need(k_win, torch.bfloat16, (B, H, window, kc.head_dim), "k_win")
        _need(v_win, torch.bfloat16, (B, H, window, kc.head_dim), "v_win")
    else:
        k_win = v_win = None
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (B, Hq, d), "out")
    if workspace is None:
        workspace = alloc_workspace(B, Hq, H, max_seq_len, bs, device=q.device)
    if d_err is not None:
        _need(d_err, torch.int32, (1,), "d_err")
    L, s = lib(), _stream(stream)
    common = (kc.handle, vc.handle, _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_tables), block_tables.shape[1],
              _ptr(seq_lens), B, Hq, int(max_seq_len), _ptr(k_win), _ptr(v_win), int(window), float(softmax_scale),
              nb, bs)
    ws = (_ptr(workspace), workspace.numel())
    if phase == "all":
        _check(L.tq_decode_paged(*common, _ptr(out), *ws, _ptr(d_err), s))
    elif phase == "partials":
        _check(L.tq_decode_partials(*common, *ws, _ptr(d_err), s))
    elif phase == "combine":
        _check(L.tq_decode_combine(vc.handle, _ptr(seq_lens), B, Hq, int(max_seq_len), int(window), bs, _ptr(out),
                                   *ws, s))
    else:
        raise ValueError(f"unknown phase {phase!r}")
    return out


def static_workspace_bytes() -> int:
    """Size of the fixed scratch array behind decode_paged_static, as built into libtq.so."""
    return int(lib().tq_static_workspace_bytes())


def decode_paged_static(kc: Codec, vc: Codec, q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                        block_size: int, block_tables: torch.Tensor, seq_lens: torch.Tensor, max_seq_len: int,
                        k_win: Optional[torch.Tensor], v_win: Optional[torch.Tensor], window: int,
                        softmax_scale: float, out: Optional[torch.Tensor] = None,
                        d_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode attention that allocates no device memory in the library (tq_decode_paged_static).

    For callers that cannot call cudaMalloc (another runtime owns the device
    memory, or the path may not take cudaMalloc's implicit synchronization):
    the split-K scratch is a fixed array of static_workspace_bytes() inside the
    library, shared by every call, so calls that overlap on the GPU race. The
    first call on a device loads that array there (it reserves the memory), so
    make it at start-up, before another runtime takes the rest of the device.
    ``out`` should be preallocated by such callers; if it is None this
    wrapper creates it with torch for convenience.
    """
    if q.dim() != 3:
        raise ValueError("q must be [batch][num_q_heads][head_dim]")
    B, Hq, d = q.shape
    H = kc.num_kv_heads
    _need(q, torch.bfloat16, (B, Hq, kc.head_dim), "q")
    nb = _pools(kc, vc, k_pages, v_pages, block_size)
    if block_tables.dim() != 2:
        raise ValueError("block_tables must be [batch][max_blocks_per_seq]")
    _need(block_tables, torch.int32, (B, block_tables.shape[1]), "block_tables")
    _need(seq_lens, torch.int32, (B,), "seq_lens")
    if window > 0:
        _need(k_win, torch.bfloat16, (B, H, window, kc.head_dim), "k_win")
        _need(v_win, torch.bfloat16, (B, H, window, kc.head_dim), "v_win")
    else:
        k_win = v_win = None
    if out is None:
        out = torch.empty(B, Hq, d, dtype=torch.float32, device=q.device)
    _need(out, torch.float32, (B, Hq, d), "out")
    if d_err is not None:
        _need(d_err, torch.int32, (1,), "d_err")
    _check(lib().tq_decode_paged_static(
        kc.handle, vc.handle, _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_tables), block_tables.shape[1],
        _ptr(seq_lens), B, Hq, int(max_seq_len), _ptr(k_win), _ptr(v_win), int(window), float(softmax_scale), nb,
        int(block_size), _ptr(out), _ptr(d_err), _stream(stream)))
    return out


def byte_ledger(kc: Codec, vc: Codec, seq_lens: Sequence[int], window: int, num_q_heads: int, block_size: int,
                num_blocks: int, max_seq_len: Optional[int] = None) -> dict:
    """tq_byte_ledger for the host lengths ``seq_lens``; storage and metadata reported apart."""
    lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    max_seq_len = int(lens.max()) if max_seq_len is None and len(lens) else int(max_seq_len or 0)
    kd, kkeep = kc.desc()
    vd, vkeep = vc.desc()
    r = _Ledger()
    _check(lib().tq_byte_ledger(ctypes.byref(kd), ctypes.byref(vd), len(lens), lens.ctypes.data, window, num_q_heads,
                                block_size, num_blocks, max_seq_len, ctypes.byref(r)))
    del kkeep, vkeep
    return {name: getattr(r, name) for name, _ in _Ledger._fields_}


def host_ledger(num_kv_heads, kspec: dict, vspec: dict, seq_lens, window, num_q_heads, block_size, num_blocks,
                max_seq_len=None) -> dict:
    """tq_byte_ledger from plain codec parameters (no device needed)."""
    lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    max_seq_len = int(lens.max()) if max_seq_len is None and len(lens) else int(max_seq_len or 0)
    kd, kkeep = _desc(HEAD_DIM, num_kv_heads, kspec["group_bits"], kspec["group_size"], kspec.get("high_coords"),
                      kspec.get("seed", 0), kspec.get("qjl", False), kspec.get("groupwise", False))
    vd, vkeep = _desc(HEAD_DIM, num_kv_heads, vspec["group_bits"], vspec["group_size"], vspec.get("high_coords"),
                      vspec.get("seed", 0), vspec.get("qjl", False), vspec.get("groupwise", False))
    r = _Ledger()
    _check(lib().tq_byte_ledger(ctypes.byref(kd), ctypes.byref(vd), len(lens), lens.ctypes.data, window, num_q_heads,
                                block_size, num_blocks, max_seq_len, ctypes.byref(r)))
    del kkeep, vkeep
    return {name: getattr(r, name) for name, _ in _Ledger._fields_}
