"""Benchmark of the compressed paged KV cache on B200: one JSON line on rank 0.

A step is one serving decode step of the whole hot path over the workload's
batch, one tq_window_append_decode call: the window append packs the token
that leaves each (sequence, KV head)'s dense window into its page slot, then
the decode attends every query head over the packed history plus the bf16
window. Inputs are resident in HBM before timing; the page pools are far
larger than L2, so no flush is needed between steps. Each timed step replays
a CUDA graph of the call when the replay reproduces the eager call's output
bit for bit (else the eager call runs); `config.step_launch` says which.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

--impl reference times the CPU oracle (fp64 NumPy) on a bounded sample of the
same workload: it is a deliberately slow baseline, not a target.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from quantized_paged_kv_pack_b200 import tq  # noqa: E402
from quantized_paged_kv_pack_b200 import workloads as WL  # noqa: E402

HEADLINE = "decode_llama70b_3p5bit"
SMALL = "decode_gqa8_4k_4bit"
DECODE_LAUNCHES = 3  # per step: prologue (work list, query rotation, windows, the append), decode, combine
EXTRA = ["decode_llama8b_4bit", "decode_llama8b_2p5bit", "decode_llama8b_3p5bit_qjl",
         "decode_llama8b_3p5bit_groupwise", "decode_llama8b_3p5bit_recipe",
         "pack_llama8b_4bit", "pack_llama70b_3p5bit", "pack_llama8b_2p5bit", "pack_llama8b_3p5bit_qjl",
         "pack_llama8b_3p5bit_groupwise", "pack_llama8b_3p5bit_recipe"]
D = 128
METRIC = "paged TQ decode HBM GB/s (algorithmic bytes / step time)"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash(name):
    with open(os.path.join(ROOT, "quantized_paged_kv_pack_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def stored_traffic(workload, kernel_file):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        t = json.load(f)
    e = t.get(workload)
    if not e or e.get("source_sha256_16") != kernel_source_hash(kernel_file):
        return None
    return e.get("bytes_per_launch")


# --------------------------------------------------------------------------- workload setup

class DecodeSetup:
    """A decode workload resident on the GPU, with the pages written by tq_pack_kv."""

    def __init__(self, w: WL.Workload, seed_offset: int = 0):
        w = rank_workload(w, seed_offset)
        self.w = w
        ks, vs = WL.codec_specs(w)
        self.kspec, self.vspec = ks, vs
        self.kc = tq.Codec(w.num_kv_heads, ks.group_bits, ks.group_size, ks.high_coords, ks.seed,
                           qjl=ks.qjl, groupwise=ks.groupwise)
        self.vc = tq.Codec(w.num_kv_heads, vs.group_bits, vs.group_size, vs.high_coords, vs.seed,
                           qjl=vs.qjl, groupwise=vs.groupwise)
        lay = WL.page_layout(w)
        B = len(lay.seq_lens)
        # one spare block per sequence, next in its block table, takes the rows the
        # step's window eviction packs when the packed length ends on a block boundary
        self.num_blocks = lay.num_blocks + B
        self.append_block = np.arange(lay.num_blocks, lay.num_blocks + B)
        self.layout = lay
        bs = w.block_size
        self.kp = tq.page_pool(self.kc, self.num_blocks, bs)
        self.vp = tq.page_pool(self.vc, self.num_blocks, bs)
        for b in range(B):
            P = int(lay.packed_lens[b])
            for t0 in range(0, P, 32768):
                t1 = min(P, t0 + 32768)
                k, v = WL.sequence_kv(w, b, t0, t1, device="cuda")
                slots = torch.as_tensor(WL.slot_mapping(lay, b, t0, t1, bs), device="cuda")
                tq.pack_kv(self.kc, self.vc, k, v, slots, self.kp, self.vp, bs)
        self.kw, self.vw = WL.windows(w, lay, device="cuda")
        if w.window:
            # ring order for tq_window_append: token t of the window in slot t % W
            for b in range(B):
                shift = int(lay.packed_lens[b]) % w.window
                n = int(min(w.window, lay.seq_lens[b]))
                if shift and n == w.window:
                    self.kw[b] = torch.roll(self.kw[b], shifts=shift, dims=1)
                    self.vw[b] = torch.roll(self.vw[b], shifts=shift, dims=1)
        self.q = WL.queries(w, device="cuda")
        nblk = -(-lay.packed_lens // bs)
        bt = np.concatenate((lay.block_tables, np.zeros((B, 1), lay.block_tables.dtype)), axis=1)
        bt[np.arange(B), nblk] = self.append_block
        self.bt = torch.as_tensor(bt.astype(np.int32), device="cuda")
        self.sl = torch.as_tensor(lay.seq_lens.astype(np.int32), device="cuda")
        self.max_len = int(lay.seq_lens.max())
        self.scale = 1.0 / math.sqrt(D)
        self.ws = tq.alloc_workspace(B, w.num_q_heads, w.num_kv_heads, self.max_len, bs)
        self.out = torch.empty(B, w.num_q_heads, D, dtype=torch.float32, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        # the step's new token per (sequence, head); the token it replaces in the window is packed
        g = torch.Generator(device="cuda")
        g.manual_seed(w.seed + 99)
        self.new_k = (torch.randn(B, w.num_kv_heads, D, generator=g, device="cuda") * 2).to(torch.bfloat16)
        self.new_v = (torch.randn(B, w.num_kv_heads, D, generator=g, device="cuda") * 2).to(torch.bfloat16)
        torch.cuda.synchronize()

    # algorithmic bytes -----------------------------------------------------
    def decode_split_bytes(self):
        w, lay = self.w, self.layout
        rows = int(lay.packed_lens.sum()) * w.num_kv_heads * (self.kc.row_bytes + self.vc.row_bytes)
        win = int(np.minimum(w.window, lay.seq_lens).sum()) * w.num_kv_heads * D * 2 * 2
        bt = 4 * int((-(-lay.packed_lens // w.block_size)).sum())
        q = len(lay.seq_lens) * w.num_q_heads * D * 2
        return rows + win + bt + q

    def out_bytes(self):
        return len(self.layout.seq_lens) * self.w.num_q_heads * D * 4

    def pack_bytes(self):
        """Window eviction with append: new K/V read, evicted K/V read, window slot written, rows written."""
        B, H = len(self.layout.seq_lens), self.w.num_kv_heads
        win = 2 * (B * H * D * 2 * 2) if self.w.window else 0
        return B * H * D * 2 * 2 + win + B * H * (self.kc.row_bytes + self.vc.row_bytes) + B * 8

    def step_bytes(self):
        return self.decode_split_bytes() + self.out_bytes() + self.pack_bytes()

    def kv_tokens(self):
        return int(self.layout.seq_lens.sum())

    # the step ---------------------------------------------------------------
    def pack(self, k=None, v=None):
        """The step's write side: tq_window_append of one new token per sequence.

        The lengths are not advanced, so every step evicts into the same packed
        position and each timed step does the same work over the same history.
        """
        w = self.w
        tq.window_append(self.kc, self.vc, self.new_k if k is None else k, self.new_v if v is None else v,
                         self.kw if w.window else None, self.vw if w.window else None, w.window, 0, self.sl,
                         self.bt, self.kp, self.vp, w.block_size, d_err=self.err)

    def step(self, k=None, v=None, q=None, out=None):
        """The whole step in one call: tq_window_append_decode (the append runs in the decode's first
        kernel; the results are those of pack() then decode())."""
        w = self.w
        return tq.window_append_decode(self.kc, self.vc, self.new_k if k is None else k,
                                       self.new_v if v is None else v, self.kw if w.window else None,
                                       self.vw if w.window else None, w.window, 0, self.q if q is None else q,
                                       self.kp, self.vp, w.block_size, self.bt, self.sl, self.max_len, self.scale,
                                       out=self.out if out is None else out, workspace=self.ws, d_err=self.err)

    def decode(self, phase="all", q=None, out=None):
        w = self.w
        return tq.decode_paged(self.kc, self.vc, self.q if q is None else q, self.kp, self.vp, w.block_size,
                               self.bt, self.sl,
                               self.max_len, self.kw if w.window else None, self.vw if w.window else None, w.window,
                               self.scale, out=self.out if out is None else out, workspace=self.ws, d_err=self.err,
                               phase=phase)


class PackSetup:
    def __init__(self, w: WL.Workload):
        self.w = w
        ks, vs = WL.codec_specs(w)
        self.kc = tq.Codec(w.num_kv_heads, ks.group_bits, ks.group_size, ks.high_coords, ks.seed,
                           qjl=ks.qjl, groupwise=ks.groupwise)
        self.vc = tq.Codec(w.num_kv_heads, vs.group_bits, vs.group_size, vs.high_coords, vs.seed,
                           qjl=vs.qjl, groupwise=vs.groupwise)
        self.k, self.v, slots, lay = WL.pack_batch(w, device="cuda")
        self.slots = torch.as_tensor(slots, device="cuda")
        self.kp = tq.page_pool(self.kc, lay.num_blocks, w.block_size)
        self.vp = tq.page_pool(self.vc, lay.num_blocks, w.block_size)
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()

    def bytes(self):
        T, H = self.k.shape[0], self.w.num_kv_heads
        return T * H * D * 2 * 2 + T * H * (self.kc.row_bytes + self.vc.row_bytes) + T * 8

    def launches(self):
        """Kernels per tq_pack_kv call, as the library dispatches them: one for uniform 4-bit K and V
        (both sides in one grid); one per side when both sides have a tensor-core pack (plain 3/4-bit,
        4+3 and 4+2 mixes; group-wise 4+3 and 4+2; QJL 3+2, 4+3, uniform 3 and 2 bits; recipe rows
        3+2 and 4+3); else one general launch."""
        ks, vs = WL.codec_specs(self.w)

        def fast(spec):
            shape = (tuple(spec.group_bits), tuple(spec.group_size))
            mixes = {((4, 3), (64, 64)), ((4, 2), (32, 96))}
            if spec.qjl and spec.groupwise:
                return shape in {((3, 2), (64, 64)), ((4, 3), (64, 64))}
            if spec.qjl:
                return shape in {((3, 2), (64, 64)), ((4, 3), (64, 64)), ((3,), (128,)), ((2,), (128,))}
            if spec.groupwise:
                return shape in mixes
            return shape in mixes | {((4,), (128,)), ((3,), (128,))}

        if self.w.block_size % 8 or not (fast(ks) and fast(vs)):
            return 1
        u4 = all(tuple(sp.group_bits) == (4,) and not sp.qjl for sp in (ks, vs))
        return 1 if u4 else 2

    def step(self):
        tq.pack_kv(self.kc, self.vc, self.k, self.v, self.slots, self.kp, self.vp, self.w.block_size, d_err=self.err)


# --------------------------------------------------------------------------- measurement

class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs.

    NVML (read-only queries) from a thread every 2 ms, so that a timed region of
    tens of milliseconds still gets several samples; nvidia-smi (-lms 100) when
    NVML is not importable. Nothing here changes a GPU setting.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, device_index=0):
        self.proc = None
        self.thread = None
        self.samples = []  # (sm MHz, max MHz, reasons)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            sel = str(device_index)
        self.sel = sel

    def _nvml_loop(self, nv, handle, stop):
        mx = None
        while not stop.is_set():
            try:
                if mx is None:
                    mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((float(sm), float(mx), {n for n, b in self.REASON_BITS.items() if bits & b}))
            except Exception:
                pass  # a failed query is skipped, not fatal
            stop.wait(0.002)

    def __enter__(self):
        try:
            import threading

            import pynvml as nv

            nv.nvmlInit()
            handle = (nv.nvmlDeviceGetHandleByUUID(self.sel) if self.sel.startswith("GPU-")
                      else nv.nvmlDeviceGetHandleByIndex(int(self.sel)))
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, handle, self.stop), daemon=True)
            self.thread.start()
            time.sleep(0.02)
            self.first = len(self.samples)  # samples from here on fall inside the timed region
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        time.sleep(0.15)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in out.splitlines():
                parts = [q.strip() for q in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm, mx = float(parts[1]), float(parts[2])
                except ValueError:
                    continue
                self.samples.append((sm, mx, {n for n, v in zip(names, parts[5:9]) if v.lower() == "active"}))

    def summary(self):
        inside = self.samples[getattr(self, "first", 0):]
        where = "timed region"
        if not inside:  # a region shorter than the sampling interval: the samples just before it
            inside, where = self.samples[-3:], "just before the timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set().union(*(r for _, _, r in inside))
        return {"sm_mhz": statistics.median(sm for sm, _, _ in inside), "sm_max_mhz": inside[-1][1],
                "reasons": sorted(reasons), "samples": len(inside), "sampled": where,
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


def time_steps(fns, steps, stream):
    """Run `steps` iterations of the callables in `fns` with events between them.

    Returns (total ms, [per-callable mean ms], [per-step ms]). Events are
    recorded on the stream the library launches on (torch's current stream).
    """
    n = len(fns)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        ev[s][0].record(stream)
        for i, f in enumerate(fns):
            f()
            ev[s][i + 1].record(stream)
    torch.cuda.synchronize()
    per_step = [ev[s][0].elapsed_time(ev[s][n]) for s in range(steps)]
    parts = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) / steps for i in range(n)]
    return sum(per_step), parts, per_step


def capture_step(step, outputs):
    """The step as a CUDA graph, so that a replay is one launch and a stall of the host thread
    between the step's own launches cannot leave the GPU idle inside a timed step. The graph is
    kept only if a replay, from zeroed outputs, gives the eager step's outputs bit for bit; else
    (or if capture fails) the step runs eagerly. Returns (callable, how)."""
    torch.cuda.synchronize()
    step()
    torch.cuda.synchronize()
    ref = [o.clone() for o in outputs]
    try:
        g = torch.cuda.CUDAGraph()
        # thread-local: other threads' CUDA calls (NCCL's watchdog under torchrun) stay legal during capture
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            step()
    except Exception as e:  # the library's launches could not be captured: time the eager step
        torch.cuda.synchronize()
        try:
            step()  # clears a launch error a failed capture may have left for the next call
        except Exception:
            pass
        torch.cuda.synchronize()
        return step, f"eager (capture failed: {type(e).__name__})"
    for o in outputs:
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    if not all(torch.equal(o, r) for o, r in zip(outputs, ref)):
        return step, "eager (graph replay differed)"
    return g.replay, "cuda_graph"


def percentiles(xs):
    q = np.percentile(np.asarray(xs, dtype=np.float64), [10, 50, 90])
    return {"p10": float(q[0]), "p50": float(q[1]), "p90": float(q[2])}


def measure_decode(setup: DecodeSetup, steps, warmup, dist_ctx=None, clocks=True):
    """The step (tq_window_append_decode: the window append and the decode call in three launches)
    timed with events only between steps, as a caller runs it: an event between two kernels would stop
    the later one from launching while the earlier one ends. The phase breakdown (append, partials,
    combine, as three separate calls) comes from a second pass with events between the phases."""
    stream = torch.cuda.current_stream()
    phases = [setup.pack, lambda: setup.decode("partials"), lambda: setup.decode("combine")]
    step = setup.step

    for _ in range(warmup):
        step()
        for f in phases:
            f()
    torch.cuda.synchronize()
    if setup.err.item():
        raise RuntimeError(f"device error word {setup.err.item()} during warm-up")
    timed, how = capture_step(step, [setup.out])
    barrier(dist_ctx)
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.__enter__()
    total_ms, _, per_step = time_steps([timed], steps, stream)
    if sampler:
        sampler.__exit__(None, None, None)
    if setup.err.item():
        raise RuntimeError(f"device error word {setup.err.item()} in the timed steps")
    _, parts, _ = time_steps(phases, steps, stream)
    barrier(dist_ctx)
    total_ms = max_over_ranks(total_ms, dist_ctx)
    return total_ms / steps, parts, (sampler.summary() if sampler else None), per_step, how


def measure_latency(setup: DecodeSetup, reps, warmup, cold):
    """Decode-call latency (partials + combine) in microseconds, p10 / p50 / p90.

    cold: before every repetition, outside the event pair, a buffer of twice
    the L2 size is written, so the call starts with none of its data in L2.
    Before the first event a spin kernel of about 100 us keeps the GPU busy
    while the host enqueues the call's launches, so the pair times the GPU's
    work, not the host's launch latency.
    """
    stream = torch.cuda.current_stream()
    l2 = int(getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "L2_cache_size", 0)) or (126 << 20)
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device="cuda") if cold else None
    for _ in range(warmup):
        setup.decode()
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(200_000)  # the spacer (about 100 us at ~2 GHz)
        e0.record(stream)
        setup.decode()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
    del flush
    return percentiles(times)


def measure_decode_e2e(setup: DecodeSetup, steps, warmup):
    """Same step through the public API from pinned host buffers (H2D in, D2H out, inside the timing)."""
    B, Hq, H = setup.q.shape[0], setup.q.shape[1], setup.w.num_kv_heads
    hq = setup.q.cpu().pin_memory()
    hk = setup.new_k.cpu().pin_memory()
    hv = setup.new_v.cpu().pin_memory()
    hout = torch.empty(B, Hq, D, dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(setup.q), torch.empty_like(setup.new_k), torch.empty_like(setup.new_v)
    dout = torch.empty_like(setup.out)

    def step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        setup.step(dk, dv, q=dq, out=dout)
        hout.copy_(dout, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    total, _, _ = time_steps([step], steps, torch.cuda.current_stream())
    h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
    d2h = hout.numel() * 4
    return total / steps, h2d, d2h


def measure_pack(setup: PackSetup, steps, warmup, clocks=False):
    """Returns (ms per step, clock summary or None, how the step was launched)."""
    for _ in range(warmup):
        setup.step()
    torch.cuda.synchronize()
    timed, how = capture_step(setup.step, [setup.kp, setup.vp])
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.__enter__()
    total, _, _ = time_steps([timed], steps, torch.cuda.current_stream())
    if sampler:
        sampler.__exit__(None, None, None)
    if setup.err.item():
        raise RuntimeError(f"device error word {setup.err.item()} in the timed steps")
    return total / steps, (sampler.summary() if sampler else None), how


# --------------------------------------------------------------------------- distributed plumbing

def init_dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return None
    import datetime

    import torch.distributed as dist

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    return dist


def barrier(dist_ctx):
    if dist_ctx is not None:
        dist_ctx.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x, dist_ctx):
    """The largest x over the ranks (step times: the job is as slow as its slowest replica)."""
    if dist_ctx is None:
        return x
    dev = "cuda" if dist_ctx.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist_ctx.all_reduce(t, op=dist_ctx.ReduceOp.MAX)
    return float(t.item())


def guarded(sample):
    """Run an oracle timing leg; a failure is reported in the line instead of ending the benchmark."""
    try:
        gbs, tps, desc, threads = sample()
        return {"GB/s": gbs, "token_heads_per_s": tps, "cores": threads, "kind": "oracle", "sample": desc}
    except Exception as e:  # noqa: BLE001 - a secondary, reported leg
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def rank_workload(w: WL.Workload, rank: int) -> WL.Workload:
    """Rank r's replica of a workload: the same shapes, its own seeded data (weak scaling)."""
    return WL.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank}) if rank else w


def aggregate_gbs(world: int, bytes_per_rank_step: int, max_step_ms: float) -> float:
    """Whole-job GB/s: the bytes every rank moved in a step over the slowest rank's step time."""
    return world * bytes_per_rank_step / (max_step_ms * 1e-3) / 1e9


# --------------------------------------------------------------------------- CPU oracle legs

def _oracle_formats(w, kspec, vspec, h):
    from oracle import tq_oracle as O

    hk = None if kspec.high_coords is None else kspec.high_coords[h:h + 1]
    hv = None if vspec.high_coords is None else vspec.high_coords[h:h + 1]
    return (O.Format(D, 1, kspec.group_bits, kspec.group_size, hk, kspec.seed, qjl=kspec.qjl,
                     groupwise=kspec.groupwise),
            O.Format(D, 1, vspec.group_bits, vspec.group_size, hv, vspec.seed, qjl=vspec.qjl,
                     groupwise=vspec.groupwise))


def _median_sequence(lay):
    order = np.argsort(lay.seq_lens, kind="stable")
    return int(order[len(order) // 2])


def gpu_pages_unit(setup: "DecodeSetup", b: int, h: int):
    """(kp, vp, table, q, kw, vw) of unit (b, h) from the GPU-written cache."""
    w, lay = setup.w, setup.layout
    G = w.num_q_heads // w.num_kv_heads
    P = int(lay.packed_lens[b])
    nblk = -(-P // w.block_size)
    blocks = torch.as_tensor(lay.block_tables[b, :max(nblk, 1)].astype(np.int64).clip(0), device="cuda")
    return (setup.kp[blocks][:, h:h + 1].cpu().numpy(), setup.vp[blocks][:, h:h + 1].cpu().numpy(),
            np.arange(max(nblk, 1))[None], setup.q[b:b + 1, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64),
            setup.kw[b:b + 1, h:h + 1].float().cpu().numpy(), setup.vw[b:b + 1, h:h + 1].float().cpu().numpy())


def oracle_pages_unit(w, kspec, vspec, lay, b, h, cache={}):
    """(kp, vp, table, q, kw, vw) of unit (b, h) built on the CPU by the oracle's own pack."""
    from oracle import tq_oracle as O

    key = (w.name, b)
    if key not in cache:
        cache.clear()
        L = int(lay.seq_lens[b])
        k, v = WL.sequence_kv(w, b, 0, L, device="cpu")
        cache[key] = (k.float().numpy(), v.float().numpy(), WL.queries(w, device="cpu").float().numpy())
    k, v, q = cache[key]
    G = w.num_q_heads // w.num_kv_heads
    L, P = int(lay.seq_lens[b]), int(lay.packed_lens[b])
    kf1, vf1 = _oracle_formats(w, kspec, vspec, h)
    nblk = max(1, -(-P // w.block_size))
    kp, vp = O.pack_kv(k[:P, h:h + 1], v[:P, h:h + 1], np.arange(P), kf1, vf1, nblk, w.block_size)
    Wn = max(w.window, 1)
    kw = np.zeros((1, 1, Wn, D))
    vw = np.zeros((1, 1, Wn, D))
    kw[0, 0, :L - P] = k[P:L, h]
    vw[0, 0, :L - P] = v[P:L, h]
    return kp, vp, np.arange(nblk)[None], q[b:b + 1, h * G:(h + 1) * G].astype(np.float64), kw, vw


def oracle_decode_sample(w, kspec, vspec, lay, unit_source, budget_s: float, row_bytes):
    """Time the oracle's decode attention on (sequence, KV head) units until ~budget_s of CPU work.

    Returns (GB/s of algorithmic bytes, KV token-heads/s, description, threads).
    """
    from oracle import tq_oracle as O

    G = w.num_q_heads // w.num_kv_heads
    b = _median_sequence(lay)
    L, P = int(lay.seq_lens[b]), int(lay.packed_lens[b])
    done_bytes = done_tok = 0
    elapsed = 0.0
    units = 0
    for h in range(w.num_kv_heads):
        kp, vp, table, q, kw, vw = unit_source(b, h)
        kf1, vf1 = _oracle_formats(w, kspec, vspec, h)
        t0 = time.perf_counter()
        O.decode_attention(q, kp, vp, table, [L], kw, vw, w.window, 1.0 / math.sqrt(D), kf1, vf1, w.block_size)
        elapsed += time.perf_counter() - t0
        units += 1
        n_win = min(w.window, L)
        done_bytes += P * row_bytes + n_win * D * 4 + 4 * (-(-P // w.block_size)) + G * D * 6
        done_tok += L
        if elapsed >= budget_s:
            break
    threads = len(os.sched_getaffinity(0))
    desc = (f"oracle decode of sequence {b} (L={L}, the median length), {units} of {w.num_kv_heads} KV heads, "
            f"all {G} query heads of each")
    return done_bytes / elapsed / 1e9, done_tok / elapsed, desc, threads


def oracle_pack_sample(w, kspec, vspec, budget_s: float, chunk: int = 512):
    """Time the oracle's pack (quantize, encode, page write) on 512-token chunks of sequence 0 until
    ~budget_s of CPU work. Rows go to a pool of the chunk's own size: the per-row work is the same.

    Returns (GB/s of algorithmic bytes, token-heads/s, description, threads).
    """
    from oracle import tq_oracle as O

    H, bs = w.num_kv_heads, w.block_size
    kf, vf = (O.Format(D, H, s.group_bits, s.group_size, s.high_coords, s.seed, qjl=s.qjl, groupwise=s.groupwise)
              for s in (kspec, vspec))
    per_token = H * D * 2 * 2 + H * (O.row_bytes(kf) + O.row_bytes(vf)) + 8
    L = int(WL.seq_lens(w)[0])
    done = 0
    elapsed = 0.0
    for t0 in range(0, L, chunk):
        t1 = min(L, t0 + chunk)
        k, v = WL.sequence_kv(w, 0, t0, t1, device="cpu")
        k, v = k.float().numpy(), v.float().numpy()
        slots = np.arange(t1 - t0, dtype=np.int64)
        t_start = time.perf_counter()
        O.pack_kv(k, v, slots, kf, vf, -(-(t1 - t0) // bs), bs)
        elapsed += time.perf_counter() - t_start
        done += t1 - t0
        if elapsed >= budget_s:
            break
    desc = f"oracle pack of the first {done} tokens of sequence 0, all {H} KV heads, K and V"
    return done * per_token / elapsed / 1e9, done * H / elapsed, desc, len(os.sched_getaffinity(0))


def oracle_decode_sample_one_thread(w, kspec, vspec, lay, unit_source, budget_s: float, row_bytes):
    """The same oracle sample with NumPy's BLAS and OpenMP pools held to one thread."""
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=1):
        gbs, tps, desc, _ = oracle_decode_sample(w, kspec, vspec, lay, unit_source, budget_s, row_bytes)
    return gbs, tps, desc, 1


# --------------------------------------------------------------------------- main

def run_reference(args):
    """--impl reference: the CPU oracle as the reference arm (rank 0 only, no GPU code)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload_of(args)
    kspec, vspec = WL.codec_specs(w)
    lay = WL.page_layout(w)
    from oracle import tq_oracle as O

    rb = sum(O.row_bytes(O.Format(D, 1, s.group_bits, s.group_size,
                                  None if s.high_coords is None else s.high_coords[:1], s.seed, qjl=s.qjl,
                                  groupwise=s.groupwise))
             for s in (kspec, vspec))
    src = lambda b, h: oracle_pages_unit(w, kspec, vspec, lay, b, h)  # noqa: E731
    for _ in range(args.warmup):
        oracle_decode_sample(w, kspec, vspec, lay, src, 0.0, rb)
    vals, desc, threads = [], None, None
    for _ in range(args.steps):
        gbs, tps, desc, threads = oracle_decode_sample(w, kspec, vspec, lay, src, args.reference_budget, rb)
        vals.append(gbs)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "description": w.description},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_of(args):
    w = WL.WORKLOADS[args.workload]
    if args.batch:
        w = WL.Workload(**{**w.__dict__, "batch": args.batch})
    return w


def run_pack(args, w, dist_ctx, rank, world):
    """Headline on the pack workload: one step = tq_pack_kv over the whole batch."""
    setup = PackSetup(w)
    ms, clocks, how = measure_pack(setup, args.steps, args.warmup, clocks=True)
    ms = max_over_ranks(ms, dist_ctx)
    peak, peak_kind = peaks()
    nbytes = setup.bytes()
    hk, hv, hs = setup.k.cpu().pin_memory(), setup.v.cpu().pin_memory(), setup.slots.cpu().pin_memory()
    herr = torch.zeros(1, dtype=torch.int32).pin_memory()

    def e2e_step():
        setup.k.copy_(hk, non_blocking=True)
        setup.v.copy_(hv, non_blocking=True)
        setup.slots.copy_(hs, non_blocking=True)
        setup.step()
        herr.copy_(setup.err, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    total, _, _ = time_steps([e2e_step], max(3, args.steps // 2), torch.cuda.current_stream())
    e2e_ms = max_over_ranks(total / max(3, args.steps // 2), dist_ctx)
    gbs = world * nbytes / (ms * 1e-3) / 1e9
    line = {"metric": "TQ pack HBM GB/s (algorithmic bytes / step time)", "value": gbs, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
            "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                       "l2": f"no flush: {nbytes / 1e9:.2f} GB moved per step, L2 is 126 MB",
                       "step_launch": how},
            "tokens_per_s": world * setup.k.shape[0] / (ms * 1e-3),
            "roofline": {"bound": "hbm", "kernel": "pack", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": nbytes / (ms * 1e-3) / 1e9 / peak,
                         "traffic": None if args.batch else stored_traffic(w.name, "tq_pack_mma.cu")},
            "e2e": {"value": world * nbytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": hk.numel() * 2 + hv.numel() * 2 + hs.numel() * 8,
                    "d2h_bytes_per_step": 4},
            "gpu_launches": setup.launches() * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    dist_ctx = init_dist()
    rank = dist_ctx.get_rank() if dist_ctx else 0
    world = dist_ctx.get_world_size() if dist_ctx else 1
    if world == 1:
        torch.cuda.set_device(0)
    w = workload_of(args)
    if w.kind == "pack":
        rc = run_pack(args, w, dist_ctx, rank, world)
        if dist_ctx is not None:
            dist_ctx.barrier()
            dist_ctx.destroy_process_group()
        return rc
    setup = DecodeSetup(w, seed_offset=rank)
    step_ms, parts, clocks, per_step, how = measure_decode(setup, args.steps, args.warmup, dist_ctx)
    e2e_ms, h2d, d2h = measure_decode_e2e(setup, max(3, args.steps // 2), args.warmup)
    e2e_ms = max_over_ranks(e2e_ms, dist_ctx)
    peak, peak_kind = peaks()
    split_bytes = setup.decode_split_bytes()
    achieved = split_bytes / (parts[1] * 1e-3) / 1e9
    step_bytes = setup.step_bytes()
    value = aggregate_gbs(world, step_bytes, step_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
        "config": {"workload": w.name, "description": w.description, "batch": w.batch,
                   "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads, "head_dim": D,
                   "block_size": w.block_size, "window": w.window,
                   "k_format": {"bits": list(w.k_bits), "sizes": list(w.k_sizes)},
                   "v_format": {"bits": list(w.v_bits), "sizes": list(w.v_sizes)},
                   "parallelism": f"{world} independent replicas (no collective)",
                   "l2": f"no flush: {split_bytes / 1e9:.2f} GB of pages read per step, L2 is 126 MB",
                   "step_launch": how},
        "kv_tokens_per_s": world * setup.kv_tokens() / (step_ms * 1e-3),
        "step_ms_percentiles": percentiles(per_step),
        "step_breakdown_ms": {"window_append": parts[0], "decode_partials": parts[1], "decode_combine": parts[2]},
        "algorithmic_bytes_per_step": step_bytes,
        "roofline": {"bound": "hbm", "kernel": "decode partials phase (decode_prologue_kernel + decode_pair_kernel)",
                     "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_8TBs": achieved / 8000.0,
                     "traffic": None if args.batch else stored_traffic(w.name, "tq_decode_mma.cu")},
        "e2e": {"value": aggregate_gbs(world, step_bytes, e2e_ms), "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        # window append, work list, query rotation, window, decode partials, combine
        "gpu_launches": DECODE_LAUNCHES * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline:
        gbs, tps, desc, threads = oracle_decode_sample(
            w, setup.kspec, setup.vspec, setup.layout, lambda b, h: gpu_pages_unit(setup, b, h), args.cpu_budget,
            setup.kc.row_bytes + setup.vc.row_bytes)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc,
                                "kv_token_heads_per_s": tps}
        gbs1, tps1, desc1, _ = oracle_decode_sample_one_thread(
            w, setup.kspec, setup.vspec, setup.layout, lambda b, h: gpu_pages_unit(setup, b, h),
            args.cpu_budget / 2, setup.kc.row_bytes + setup.vc.row_bytes)
        line["cpu_baseline"]["one_thread"] = {"value": gbs1, "unit": "GB/s", "cores": 1, "sample": desc1,
                                              "kv_token_heads_per_s": tps1}
        line["cpu_baseline"]["note"] = ("cores = the host threads NumPy's thread pools may use; the oracle is "
                                        "mostly element-wise NumPy, and one_thread is its serial rate")
    if world == 1 and not args.no_extra:
        extra = {}
        for name in EXTRA:
            ew = WL.WORKLOADS[name]
            if ew.kind == "decode":
                del setup
                torch.cuda.empty_cache()
                setup = DecodeSetup(ew)
                n_steps = max(5, args.steps // 2)
                ms, p, _, _, how_x = measure_decode(setup, n_steps, args.warmup, None, clocks=False)
                line["gpu_launches"] += DECODE_LAUNCHES * n_steps
                sb = setup.decode_split_bytes()
                extra[name] = {"GB/s": setup.step_bytes() / (ms * 1e-3) / 1e9,
                               "kv_tokens_per_s": setup.kv_tokens() / (ms * 1e-3), "ms_per_step": ms,
                               "step_breakdown_ms": {"window_append": p[0], "decode_partials": p[1],
                                                     "decode_combine": p[2]},
                               "decode_partials_GB/s": sb / (p[1] * 1e-3) / 1e9,
                               "decode_partials_frac": sb / (p[1] * 1e-3) / 1e9 / peak,
                               "traffic": stored_traffic(name, "tq_decode_mma.cu"), "step_launch": how_x}
                if not args.no_cpu_baseline:
                    extra[name]["cpu_oracle"] = guarded(lambda: oracle_decode_sample(
                        ew, setup.kspec, setup.vspec, setup.layout, lambda b, h: gpu_pages_unit(setup, b, h),
                        args.cpu_budget / 4, setup.kc.row_bytes + setup.vc.row_bytes))
            else:
                del setup
                torch.cuda.empty_cache()
                setup = PackSetup(ew)
                ms, _, how_x = measure_pack(setup, max(5, args.steps // 2), args.warmup)
                gbs = setup.bytes() / (ms * 1e-3) / 1e9
                extra[name] = {"GB/s": gbs, "tokens_per_s": setup.k.shape[0] / (ms * 1e-3), "ms_per_step": ms,
                               "frac": gbs / peak, "traffic": stored_traffic(name, "tq_pack_mma.cu"),
                               "step_launch": how_x}
                if not args.no_cpu_baseline:
                    ks, vs = WL.codec_specs(ew)
                    extra[name]["cpu_oracle"] = guarded(lambda: oracle_pack_sample(ew, ks, vs, args.cpu_budget / 4))
                line["gpu_launches"] += setup.launches() * max(5, args.steps // 2)
        # the small parity case: a latency, hot and with L2 flushed before each call
        del setup
        torch.cuda.empty_cache()
        setup = DecodeSetup(WL.WORKLOADS[SMALL])
        reps = max(20, args.steps)
        extra[SMALL] = {"latency_us_hot": measure_latency(setup, reps, args.warmup, cold=False),
                        "latency_us_cold": measure_latency(setup, reps, args.warmup, cold=True),
                        "note": "decode call (prologue, partials, combine); launch- and latency-bound"}
        line["per_workload"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_ctx is not None:
        dist_ctx.barrier()
        dist_ctx.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WL.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (small profiling cases)")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--reference-budget", type=float, default=4.0, help="seconds of oracle work per reference step")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
