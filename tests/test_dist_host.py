"""Multi-process host logic of the benchmark's replica mode, on CPU with gloo (world size 2).

The path has no exchange step: each rank runs its own seeded replica, and the
only collectives are the timing barrier and the max over ranks of the step time.
"""

import datetime
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_paged_kv_pack_b200 import workloads as WL  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        step_ms = [0.75, 1.25][rank]  # rank 1 is the slower replica
        bench.barrier(dist)
        slowest = bench.max_over_ranks(step_ms, dist)
        bench.barrier(dist)
        w = bench.rank_workload(WL.WORKLOADS["decode_llama8b_4bit"], rank)
        out.put((rank, slowest, w.seed, int(WL.seq_lens(w).sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_step_time_and_own_seeded_replicas():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict((r, rest) for r, *rest in (out.get(timeout=10) for _ in range(2)))
    assert res[0][0] == res[1][0] == 1.25                 # both ranks report the slowest replica
    assert res[0][1] != res[1][1]                          # each rank has its own seed ...
    assert res[0][2] != res[1][2]                          # ... and so its own sequence lengths
    assert res[0][1] == WL.WORKLOADS["decode_llama8b_4bit"].seed  # rank 0 runs the workload as named


def test_aggregate_is_whole_job_over_the_slowest_rank():
    one = bench.aggregate_gbs(1, 2_000_000_000, 1.0)
    assert one == pytest.approx(2000.0)
    # weak scaling: N replicas each moving the same bytes, timed by the slowest one
    assert bench.aggregate_gbs(4, 2_000_000_000, 1.0) == pytest.approx(4 * one)
    assert bench.aggregate_gbs(2, 2_000_000_000, 2.0) == pytest.approx(one)


def test_rank_workloads_keep_shapes():
    w = WL.WORKLOADS["decode_llama70b_3p5bit"]
    r3 = bench.rank_workload(w, 3)
    for f in ("batch", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "window", "k_bits", "v_bits",
              "lengths"):
        assert getattr(r3, f) == getattr(w, f)
    assert r3.seed == w.seed + 3000
    assert bench.rank_workload(w, 0) is w
    assert np.array_equal(WL.seq_lens(r3), WL.seq_lens(w))  # fixed-length workload: same lengths


def test_reference_arm_on_a_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_line_on_rank_zero():
    """The oracle reference arm on the small parity workload prints the contract's keys."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "decode_gqa8_4k_4bit", "--reference-budget", "0.5"],
                       capture_output=True, text=True, timeout=600, env=dict(os.environ, RANK="0"))
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_oracle_baseline_sample_with_one_thread():
    """The benchmark's CPU-oracle baseline, held to one thread, on the small parity workload."""
    w = WL.WORKLOADS["decode_gqa8_4k_4bit"]
    kspec, vspec = WL.codec_specs(w)
    lay = WL.page_layout(w)
    from oracle import tq_oracle as O

    rb = sum(O.row_bytes(O.Format(128, 1, s.group_bits, s.group_size, None, s.seed)) for s in (kspec, vspec))
    src = lambda b, h: bench.oracle_pages_unit(w, kspec, vspec, lay, b, h)  # noqa: E731
    gbs, tps, desc, threads = bench.oracle_decode_sample_one_thread(w, kspec, vspec, lay, src, 0.0, rb)
    assert threads == 1 and gbs > 0 and tps > 0 and "sequence 0" in desc


def test_oracle_pack_sample_and_guard():
    """The pack workload's CPU-oracle timing leg, and the guard that reports a failing leg in the line."""
    w = WL.WORKLOADS["pack_llama8b_4bit"]
    ks, vs = WL.codec_specs(w)
    gbs, tps, desc, threads = bench.oracle_pack_sample(w, ks, vs, 0.0, chunk=64)
    assert gbs > 0 and tps > 0 and "first 64 tokens" in desc and threads >= 1
    ok = bench.guarded(lambda: (1.0, 2.0, "d", 3))
    assert ok == {"GB/s": 1.0, "token_heads_per_s": 2.0, "cores": 3, "kind": "oracle", "sample": "d"}
    bad = bench.guarded(lambda: 1 / 0)
    assert bad["error"].startswith("ZeroDivisionError")


def test_pack_launch_count_follows_the_dispatch():
    """The benchmark's claim of kernels per tq_pack_kv call: one for uniform 4-bit K and V (one grid for
    both), two (one per side) when both sides have a tensor-core pack, one general launch otherwise."""
    expect = {"pack_llama8b_4bit": 1, "pack_llama70b_3p5bit": 2, "pack_llama8b_2p5bit": 2,
              "pack_llama8b_3p5bit_qjl": 2, "pack_llama8b_3p5bit_groupwise": 2, "pack_llama8b_3p5bit_recipe": 2}
    assert {n for n, w in WL.WORKLOADS.items() if w.kind == "pack"} == set(expect)
    for name, n in expect.items():
        setup = object.__new__(bench.PackSetup)
        setup.w = WL.WORKLOADS[name]
        assert setup.launches() == n, name
    # a block size that is not a multiple of 8, or a format without a tensor-core pack: the general kernel
    w = WL.WORKLOADS["pack_llama70b_3p5bit"]
    for changed in ({"block_size": 12}, {"k_bits": (3, 2), "k_sizes": (16, 112)}):
        setup = object.__new__(bench.PackSetup)
        setup.w = WL.Workload(**{**w.__dict__, **changed})
        assert setup.launches() == 1, changed
