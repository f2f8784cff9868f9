"""C-ABI checks that need no GPU: exports, host codec tables vs the oracle, errors, ledger."""

import ctypes
import json
import os
import re

import numpy as np
import pytest

from oracle import tq_oracle as O
from quantized_paged_kv_pack_b200 import tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
D = 128


def declared_functions():
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"tq_make_codec", "tq_pack_kv", "tq_decode_paged", "tq_byte_ledger"} <= set(names)
    L = ctypes.CDLL(tq.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing


def _high(H, n, seed):
    rng = np.random.default_rng(seed)
    return np.stack([np.sort(rng.choice(D, n, replace=False)) for _ in range(H)]).astype(np.int16)


CASES = [((4,), (128,), None, 0), ((3,), (128,), None, 1), ((2,), (128,), None, 7),
         ((4, 3), (64, 64), "h", 0), ((4, 2), (32, 96), "h", 1), ((3, 2), (16, 112), "h", 12345678901234)]


@pytest.mark.parametrize("bits,sizes,high,seed", CASES)
def test_host_tables_equal_oracle(bits, sizes, high, seed):
    H = 4
    hc = _high(H, sizes[0], seed % 97) if high else None
    t = tq.codec_host_tables(D, H, bits, sizes, hc, seed)
    f = O.Format(D, H, bits, sizes, hc, seed)
    for g, b in enumerate(bits):
        c, beta = O.codebook(b, D)
        L = 1 << b
        assert np.array_equal(t["centroids_f16"][g, :L], c.astype(np.float16).view(np.uint16))
        assert np.array_equal(t["boundaries"][g, :L - 1].astype(np.float64), beta)
    assert np.array_equal(t["signs"].astype(np.float64), O.hadamard_signs(seed, D))
    for h in range(H):
        assert np.array_equal(t["perm"][h], O.permutation(f, h))
    assert t["row_bytes"] == O.row_bytes(f)


@pytest.mark.parametrize("kw,err", [
    (dict(bits=(9,), sizes=(128,)), ValueError),
    (dict(bits=(1,), sizes=(128,)), tq.UnsupportedFormatError),
    (dict(bits=(5,), sizes=(128,)), tq.UnsupportedFormatError),
    (dict(bits=(4,), sizes=(64,), d=64), tq.UnsupportedFormatError),
    (dict(bits=(4,), sizes=(96,), d=96), ValueError),
    (dict(bits=(4, 3), sizes=(64, 32)), ValueError),
    (dict(bits=(4, 3), sizes=(60, 68)), tq.UnsupportedFormatError),
    (dict(bits=(4, 3), sizes=(64, 64), high="missing"), ValueError),
    (dict(bits=(4, 3), sizes=(64, 64), high="unsorted"), ValueError),
    (dict(bits=(4, 3), sizes=(64, 64), high="range"), ValueError),
    (dict(bits=(4,), sizes=(128,), high="extra"), ValueError),
    (dict(bits=(4,), sizes=(128,), H=0), ValueError),
])
def test_descriptor_validation(kw, err):
    d, H = kw.get("d", D), kw.get("H", 2)
    hc = None
    mode = kw.get("high")
    if mode in ("unsorted", "range", "extra"):
        hc = _high(max(H, 1), kw["sizes"][0], 3)
        if mode == "unsorted":
            hc[0, [0, 1]] = hc[0, [1, 0]]
        elif mode == "range":
            hc[1, -1] = 200
    elif kw.get("bits") and len(kw["bits"]) == 2 and mode != "missing":
        hc = _high(H, kw["sizes"][0], 3)
    with pytest.raises(err):
        tq.codec_host_tables(d, H, kw["bits"], kw["sizes"], hc, 0)


def test_workspace_bytes_bounded_by_shape():
    n = tq.decode_workspace_bytes(16, 64, 8, 131072, 16)
    assert 0 < n < 64 << 20
    assert tq.decode_workspace_bytes(16, 64, 8, 131072, 0) == 0
    assert tq.decode_workspace_bytes(16, 60, 8, 131072, 16) == 0
    assert tq.decode_workspace_bytes(64, 32, 8, 32768, 16) >= tq.decode_workspace_bytes(32, 32, 8, 32768, 16)


def _spec(bits, sizes, seed, H):
    return {"group_bits": bits, "group_size": sizes, "seed": seed,
            "high_coords": _high(H, sizes[0], 5) if len(bits) == 2 else None}


@pytest.mark.parametrize("kb,ks,vb,vs", [((4,), (128,), (4,), (128,)), ((4, 3), (64, 64), (4, 3), (64, 64)),
                                          ((4, 2), (32, 96), (3,), (128,))])
def test_ledger_matches_oracle(kb, ks, vb, vs):
    H, Hq, W, bs = 8, 32, 64, 16
    lens = [0, 5, 64, 65, 1000, 4097]
    ksp, vsp = _spec(kb, ks, 0, H), _spec(vb, vs, 1, H)
    nb = sum(-(-(L - min(W, L)) // bs) for L in lens) + 3
    got = tq.host_ledger(H, ksp, vsp, lens, W, Hq, bs, nb)
    kf = O.Format(D, H, kb, ks, ksp["high_coords"], 0)
    vf = O.Format(D, H, vb, vs, vsp["high_coords"], 1)
    ws = tq.decode_workspace_bytes(len(lens), Hq, H, max(lens), bs)
    ref = O.byte_ledger(kf, vf, lens, W, bs, nb, workspace_bytes=ws)
    for key in ("dense_bytes", "index_bytes", "norm_bytes", "codebook_bytes", "transform_bytes", "window_bytes",
                "block_table_bytes", "workspace_bytes", "page_pool_bytes", "metadata_bytes"):
        assert got[key] == getattr(ref, key), key
    assert got["all_in_ratio"] == pytest.approx(ref.all_in_ratio, rel=1e-12)
    assert got["index_only_ratio"] == pytest.approx(ref.dense_bytes / ref.index_bytes, rel=1e-12)


def test_recipe_metadata_loader(tmp_path):
    with pytest.raises(FileNotFoundError):
        tq.load_recipe_metadata(str(tmp_path / "absent.json"))
    hc = _high(8, 64, 9)
    p = tmp_path / "recipe.json"
    p.write_text(json.dumps({"head_dim": 128, "num_kv_heads": 8, "group_bits": [4, 3], "group_size": [64, 64],
                             "high_coords": hc.tolist(), "hadamard_seed": 3}))
    spec = tq.load_recipe_metadata(str(p))
    assert spec["group_bits"] == (4, 3) and np.array_equal(spec["high_coords"], hc)
    bad = tmp_path / "bad.json"
    bad.write_text(json.dumps({"head_dim": 128, "num_kv_heads": 8, "group_bits": [4, 3], "group_size": [64, 64],
                               "high_coords": hc[:, ::-1].tolist()}))
    with pytest.raises(ValueError):
        tq.load_recipe_metadata(str(bad))
    with pytest.raises(ValueError):
        bad.write_text(json.dumps({"head_dim": 128}))
        tq.load_recipe_metadata(str(bad))



# ---- QJL codecs (host side) ------------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 5, 2**63 + 11])
def test_qjl_matrix_equals_oracle(seed):
    """The library's S (C++ double math, rounded to float) equals the oracle's (NumPy) entry for entry."""
    got = tq.qjl_matrix(D, 2, (3,), (128,), None, seed)
    ref = O.qjl_matrix(O.Format(D, 2, (3,), (128,), None, seed, qjl=True))
    assert got.dtype == np.float32 and got.shape == (D, D)
    mismatch = np.count_nonzero(got.astype(np.float64) != ref)
    assert mismatch == 0  # an fp64 last-ulp difference could flip one fp32 rounding; none seen at these seeds


def test_qjl_row_bytes_and_ledger():
    H, Hq, W, bs = 8, 32, 64, 16
    hc = _high(H, 64, 5)
    t = tq.codec_host_tables(D, H, (3, 2), (64, 64), hc, 7, qjl=True)
    f = O.Format(D, H, (3, 2), (64, 64), hc, 7, qjl=True)
    assert t["row_bytes"] == O.row_bytes(f) == 40 + 16 + 4
    lens = [0, 5, 64, 65, 1000, 4097]
    ksp = {"group_bits": (3, 2), "group_size": (64, 64), "seed": 7, "high_coords": hc, "qjl": True}
    vsp = {"group_bits": (3,), "group_size": (128,), "seed": 1, "high_coords": None}
    nb = sum(-(-(L - min(W, L)) // bs) for L in lens) + 3
    got = tq.host_ledger(H, ksp, vsp, lens, W, Hq, bs, nb)
    ws = tq.decode_workspace_bytes(len(lens), Hq, H, max(lens), bs)
    ref = O.byte_ledger(f, O.Format(D, H, (3,), (128,), None, 1), lens, W, bs, nb, workspace_bytes=ws)
    for key in ("index_bytes", "norm_bytes", "transform_bytes", "page_pool_bytes", "metadata_bytes"):
        assert got[key] == getattr(ref, key), key



def test_groupwise_row_bytes_ledger_and_validation():
    H, Hq, W, bs = 4, 16, 32, 16
    hc = _high(H, 32, 4)
    t = tq.codec_host_tables(D, H, (4, 2), (32, 96), hc, 3, groupwise=True)
    f = O.Format(D, H, (4, 2), (32, 96), hc, 3, groupwise=True)
    assert t["row_bytes"] == O.row_bytes(f) == 16 + 24 + 4
    # codebooks of the groups' own dimensions (32 and 96)
    for g, (b, n) in enumerate(((4, 32), (2, 96))):
        c, beta = O.codebook(b, n)
        assert np.array_equal(t["centroids_f16"][g][:1 << b], c.astype(np.float16).view(np.uint16))
        assert np.array_equal(t["boundaries"][g][:(1 << b) - 1], beta.astype(np.float32))
    lens = [0, 9, 32, 33, 700]
    ksp = {"group_bits": (4, 2), "group_size": (32, 96), "seed": 3, "high_coords": hc, "groupwise": True}
    vsp = {"group_bits": (3,), "group_size": (128,), "seed": 1, "high_coords": None}
    nb = sum(-(-(L - min(W, L)) // bs) for L in lens) + 2
    got = tq.host_ledger(H, ksp, vsp, lens, W, Hq, bs, nb)
    ws = tq.decode_workspace_bytes(len(lens), Hq, H, max(lens), bs)
    ref = O.byte_ledger(f, O.Format(D, H, (3,), (128,), None, 1), lens, W, bs, nb, workspace_bytes=ws)
    for key in ("index_bytes", "norm_bytes", "transform_bytes", "page_pool_bytes", "metadata_bytes"):
        assert got[key] == getattr(ref, key), key
    with pytest.raises(ValueError):  # group-wise needs two groups
        tq.codec_host_tables(D, H, (3,), (128,), None, 3, groupwise=True)



@pytest.mark.parametrize("bits,sizes,seed", [((4, 3), (64, 64), 5), ((4, 2), (32, 96), 6), ((3, 2), (16, 112), 7),
                                             ((2, 4), (80, 48), 8)])
def test_group_rotation_equals_oracle(bits, sizes, seed):
    """The library's R_h (built from its permutation, signs and Hadamard blocks) against the oracle's."""
    H = 3
    hc = _high(H, sizes[0], seed)
    got = tq.group_rotation(D, H, bits, sizes, hc, seed)
    f = O.Format(D, H, bits, sizes, hc, seed, groupwise=True)
    for h in range(H):
        ref = O.group_rotation(f, h)
        assert np.array_equal(got[h], ref.astype(np.float32))
        assert np.allclose(got[h].astype(np.float64) @ got[h].T.astype(np.float64), np.eye(D), atol=1e-6)
    with pytest.raises(ValueError):
        tq.group_rotation(D, H, (4, 3), (64, 64), None, seed)


def test_recipe_slicing_by_tensor_parallel_partition(tmp_path):
    hc = _high(8, 32, 12)
    p = tmp_path / "recipe.json"
    p.write_text(json.dumps({"head_dim": 128, "num_kv_heads": 8, "group_bits": [4, 2], "group_size": [32, 96],
                             "high_coords": hc.tolist(), "hadamard_seed": 5, "groupwise": True}))
    spec = tq.load_recipe_metadata(str(p))
    assert spec["groupwise"] and not spec["qjl"]
    parts = [tq.slice_recipe(spec, r, 4) for r in range(4)]
    assert all(q["num_kv_heads"] == 2 for q in parts)
    assert np.array_equal(np.concatenate([q["high_coords"] for q in parts]), hc)
    # a partition's codec tables equal the corresponding heads of the whole model's
    whole = tq.codec_host_tables(128, 8, (4, 2), (32, 96), hc, 5, groupwise=True)
    part = tq.codec_host_tables(128, 2, (4, 2), (32, 96), parts[3]["high_coords"], 5, groupwise=True)
    assert np.array_equal(part["perm"], whole["perm"][6:8]) and np.array_equal(part["signs"], whole["signs"])
    with pytest.raises(ValueError):
        tq.slice_recipe(spec, 0, 3)
    with pytest.raises(ValueError):
        tq.slice_recipe(spec, 4, 4)


def test_static_workspace_size_matches_header():
    """The binding reads the static array's size from the library; it must be the header's value."""
    text = open(os.path.join(ROOT, "include", "tq.h")).read()
    m = re.search(r"#define\s+TQ_STATIC_WORKSPACE_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", text)
    assert m, "TQ_STATIC_WORKSPACE_BYTES not found in tq.h"
    assert tq.static_workspace_bytes() == int(m.group(1)) << int(m.group(2))


def test_device_allocation_and_setup_are_per_codec_and_per_device():
    """The library allocates device memory only in tq_make_codec (the header's contract), and
    device settings are made once per device, not once per process: no source under csrc/ keeps
    a process-wide device pointer or a call_once around CUDA state."""
    csrc = os.path.join(ROOT, "quantized_paged_kv_pack_b200", "csrc")
    allocs = []
    for name in sorted(os.listdir(csrc)):
        text = open(os.path.join(csrc, name)).read()
        code = re.sub(r"//[^\n]*|/\*.*?\*/", "", text, flags=re.S)
        assert "call_once" not in code and "once_flag" not in code, name
        for m in re.finditer(r"\bcudaMalloc\w*\s*\(", code):
            start, end = code.find("tq_status tq_make_codec("), code.find("void tq_free_codec(")
            allocs.append((name, 0 <= start < m.start() < end))
    assert allocs == [("tq_codec.cpp", True)], allocs
    codec = open(os.path.join(csrc, "tq_codec.cpp")).read()
    make = codec[codec.index("tq_status tq_make_codec("):codec.index("void tq_free_codec(")]
    assert "build_pack_cells" in make and "dev.cells" in make  # the pack's cell table rides in that allocation


def test_recipe_row_host_tables_matrices_and_ledger():
    """The recipe row (qjl and groupwise): row bytes, the two S_g bit for bit, and the ledger
    field by field against the oracle."""
    H, Hq, W, bs = 4, 16, 32, 16
    hc = _high(H, 64, 6)
    for bits, sizes in (((4, 3), (64, 64)), ((4, 2), (32, 96))):
        hcs = _high(H, sizes[0], 6)
        t = tq.codec_host_tables(D, H, bits, sizes, hcs, 9, qjl=True, groupwise=True)
        f = O.Format(D, H, bits, sizes, hcs, 9, qjl=True, groupwise=True)
        assert t["row_bytes"] == O.row_bytes(f)
        S0, S1 = tq.recipe_qjl_matrices(D, H, bits, sizes, hcs, 9)
        assert np.array_equal(S0.astype(np.float64), O.recipe_qjl_matrix(f, 0))
        assert np.array_equal(S1.astype(np.float64), O.recipe_qjl_matrix(f, 1))
    assert O.row_bytes(O.Format(D, H, (4, 3), (64, 64), hc, 9, qjl=True, groupwise=True)) == 32 + 8 + 24 + 8 + 8
    lens = [0, 9, 32, 33, 700]
    ksp = {"group_bits": (4, 3), "group_size": (64, 64), "seed": 9, "high_coords": hc, "qjl": True,
           "groupwise": True}
    vsp = {"group_bits": (4, 3), "group_size": (64, 64), "seed": 2, "high_coords": hc, "groupwise": True}
    nb = sum(-(-(L - min(W, L)) // bs) for L in lens) + 2
    got = tq.host_ledger(H, ksp, vsp, lens, W, Hq, bs, nb)
    ws = tq.decode_workspace_bytes(len(lens), Hq, H, max(lens), bs)
    kf = O.Format(D, H, (4, 3), (64, 64), hc, 9, qjl=True, groupwise=True)
    vf = O.Format(D, H, (4, 3), (64, 64), hc, 2, groupwise=True)
    ref = O.byte_ledger(kf, vf, lens, W, bs, nb, workspace_bytes=ws)
    for key in ("index_bytes", "norm_bytes", "transform_bytes", "page_pool_bytes", "metadata_bytes"):
        assert got[key] == getattr(ref, key), key
