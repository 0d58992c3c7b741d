#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200: one step = copy-on-write
block copies (when the workload forks), append of the step's new K/V, and
decode attention over the paged context, all through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...   (the fp64 CPU oracle as the reference arm)

Prints ONE JSON line (rank 0). ``value`` is algorithmic HBM bytes of the whole
step (decode K/V + q + out, append read+write, block copy read+write) per second
of device time, summed over ranks (weak scaling: each rank owns its own batch;
sequences are independent, so no data-path collective exists). Inputs are
resident in HBM and every step is timed with its own CUDA events on the
launching stream. Between timed steps L2 is not flushed when the step's unique
input bytes exceed twice the 126 MB L2 (every benched configuration: 0.3 to 6.8
GB); a smaller workload is flushed by writing a 512 MiB buffer. A write flush
leaves ~126 MB of dirty lines that the next step must write back, which is why
it is not used where the inputs alone already evict L2.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); seq-steps/s"
UNIT = "GB/s"
DEFAULT_CONFIG = "llama13b_bs16"
# (label, workload name, partition_size override or None = the workload's own)
# (label, workload, partition size (None: the workload's), sequences decoded together,
#  grouped consumer (None: the run's))
EXTRA_CONFIGS = [("llama7b", "llama7b", None, 1, None),
                 ("llama13b_bs16", "llama13b_bs16", None, 1, None),
                 ("llama13b_bs32", "llama13b_bs32", None, 1, None),
                 ("llama70b_gqa", "llama70b_gqa", None, 1, None),
                 ("llama70b_gqa_policy", "llama70b_gqa", 0, 1, None),
                 ("cow_beam4", "cow_beam4", None, 1, None),
                 ("cow_beam4_grouped", "cow_beam4", 0, 4, None),
                 ("cow_beam4_grouped_tcgen05", "cow_beam4", 0, 4, "tcgen05"),
                 ("llama70b_verify4", "llama70b_verify4", 0, 1, None),
                 ("llama70b_verify4_tcgen05", "llama70b_verify4", 0, 1, "tcgen05"),
                 ("llama13b_bs16_fp8", "llama13b_bs16_fp8", None, 1, None),
                 ("llama13b_bs16_int8", "llama13b_bs16_int8", None, 1, None),
                 ("llama70b_gqa_policy_fp8", "llama70b_gqa_fp8", 0, 1, None),
                 ("cow_beam4_grouped_fp8", "cow_beam4_fp8", 0, 4, None),
                 ("llama70b_verify4_fp8", "llama70b_verify4_fp8", 0, 1, None)]
# pa_test_last_decode_kernel() -> the decode kernel a call enqueued
KERNEL_NAMES = {0: "decode_tma_simt_kernel (CUDA-core)",
                1: "decode_tma_mma_kernel (persistent, tensor-core GQA)",
                2: "decode_tma_grouped_kernel (persistent, grouped sequences)",
                3: "decode_umma_grouped_kernel (tcgen05, grouped sequences)"}
FALLBACK_HBM_GBS = 6650.0
DATASHEET_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 512 << 20          # > 2x the 126 MB L2
STREAM_BYTES = 4 << 30


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--partition-size", type=int, default=None,
                    help="override the workload's partition size (0 = library policy)")
    ap.add_argument("--group-size", type=int, default=1,
                    help="decode sequences [k g, (k+1) g) together (pa_decode_grouped) when > 1")
    ap.add_argument("--grouped-consumer", choices=["mma_sync", "tcgen05"], default="mma_sync",
                    help="consumer of the grouped / multi-token decode (pa_set_grouped_consumer)")
    ap.add_argument("--no-extra-configs", action="store_true",
                    help="skip the per-configuration table")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def dist_max(x: float, device) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(step_bytes: int, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job GB/s: every rank moved step_bytes per step; the job took the
    slowest rank's time."""
    return world * step_bytes * steps / (max_total_ms / 1e3) / 1e9


def pct(xs, scale=1.0, nd=2):
    """p10 / p50 / p90 of a list of timings (same unit as xs x scale)."""
    ys = sorted(x * scale for x in xs)
    def q(f):
        k = (len(ys) - 1) * f
        lo, hi = int(math.floor(k)), int(math.ceil(k))
        return ys[lo] + (ys[hi] - ys[lo]) * (k - lo)
    return {"p10": round(q(0.1), nd), "p50": round(q(0.5), nd), "p90": round(q(0.9), nd)}


def stream_read_gbs(device, reps=20):
    """Read bandwidth of the library's read-only streaming kernel over 4 GiB: the
    best of `reps` back-to-back launches (a roof is the most the hardware gives;
    decode fractions of it take the decode's typical launch)."""
    import torch

    import paged_kv_cache_335_b200 as pa
    lib = pa.load_library()
    buf = torch.empty(STREAM_BYTES, dtype=torch.uint8, device=device)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    ctas = sms * 2                      # two 96 KiB rings per SM
    part = torch.empty(ctas, dtype=torch.int32, device=device)
    st = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = (ctypes.c_void_p(buf.data_ptr()), ctypes.c_size_t(STREAM_BYTES),
            ctypes.c_void_p(part.data_ptr()), ctas, st)
    for _ in range(3):
        if lib.pa_stream_read(*args) != 0:
            raise RuntimeError("pa_stream_read failed")
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for e0, e1 in evs:
        e0.record()
        if lib.pa_stream_read(*args) != 0:
            raise RuntimeError("pa_stream_read failed")
        e1.record()
    torch.cuda.synchronize()
    times = [e0.elapsed_time(e1) for e0, e1 in evs]
    del buf
    return STREAM_BYTES / (min(times) / 1e3) / 1e9


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", d
    except Exception:
        return FALLBACK_HBM_GBS, "fallback", {}


def host_cores():
    return len(os.sched_getaffinity(0))


class ClockSampler:
    """nvidia-smi samples (100 ms) of SM clock, power and throttle reasons."""
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.windows = []

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "100", "-i", str(self.gpu_id)],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()

    def samples(self, t0, t1):
        rows = []
        if not self.path or not os.path.exists(self.path):
            return rows
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append((ts, float(parts[1]), float(parts[2]), parts[3], parts[4:]))
            except Exception:
                continue
        return [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]

    def summary(self, t0, t1):
        rows = self.samples(t0, t1)
        if not rows:
            return {"unavailable": "no nvidia-smi samples in the window"}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[4]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": max(r[2] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def bad_clocks(c):
    if "sm_mhz" not in c:
        return False
    if set(c["reasons"]) & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    return c["sm_mhz"] < 0.6 * c["sm_max_mhz"] and not c["reasons"]


def profile_traffic(kernel_file, workload):
    """dram bytes per launch from a committed ncu summary of this exact kernel
    source (matched by sha256), or None."""
    try:
        sha = hashlib.sha256(open(kernel_file, "rb").read()).hexdigest()
    except OSError:
        return None, None
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None, sha
    for name in sorted(os.listdir(pdir)):
        if not name.endswith((".md", ".txt")):
            continue
        text = open(os.path.join(pdir, name), encoding="utf-8").read()
        lines = text.splitlines()
        if f"source_sha256: {sha}" not in lines or f"workload: {workload}" not in lines:
            continue
        m = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
        if m:
            return float(m.group(1)), sha
    return None, sha


# ---------------------------------------------------------------------------
# one configuration on the GPU
# ---------------------------------------------------------------------------
class Step:
    """Device-resident inputs of one workload and pre-marshalled C-ABI calls."""

    def __init__(self, wl, device, seed_offset=0, partition_size=None, group_size=1):
        import torch

        import paged_kv_cache_335_b200 as pa
        from paged_kv_cache_335_b200 import workloads as W
        self.wl = wl
        self.torch = torch
        self.lib = pa.load_library()
        self.vals = W.make_values(wl, device, poison=False, seed_offset=seed_offset)
        v = self.vals
        self.tables = torch.as_tensor(wl.block_tables, device=device)
        self.ctx = torch.as_tensor(wl.context_lens, device=device)
        self.slots = torch.as_tensor(wl.slot_mapping, device=device)
        self.pairs = torch.as_tensor(wl.copy_pairs, device=device)
        self.out = torch.empty_like(v["q"])
        self.desc = pa.cache_desc(v["k_cache"])
        self.ps = wl.partition_size if partition_size is None else partition_size
        self.group_size = group_size
        self.multi = wl.query_start is not None
        if self.multi:
            self.query_start = torch.as_tensor(wl.query_start, device=device)
            self.num_partitions = pa.pa_decode_multi_num_partitions(
                wl.num_seqs, wl.num_query_rows, wl.max_query_len, wl.num_heads,
                wl.max_context_len, v["k_cache"], self.ps)
            need = pa.pa_decode_multi_workspace_size(
                wl.num_seqs, wl.num_query_rows, wl.max_query_len, wl.num_heads,
                wl.max_context_len, v["k_cache"], self.ps)
        else:
            self.num_partitions = pa.pa_decode_grouped_num_partitions(
                wl.num_seqs, wl.num_heads, wl.max_context_len, v["k_cache"], group_size, self.ps)
            need = pa.pa_decode_grouped_workspace_size(
                wl.num_seqs, wl.num_heads, wl.max_context_len, v["k_cache"], group_size, self.ps)
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
        self.ws_bytes = need
        self.stream = torch.cuda.current_stream(device)
        P = ctypes.c_void_p
        self.sp = P(self.stream.cuda_stream)
        self.args_copy = (P(self.pairs.data_ptr()), int(self.pairs.shape[0]),
                          P(v["k_cache"].data_ptr()), P(v["v_cache"].data_ptr()),
                          ctypes.byref(self.desc), self.sp)
        self.args_append = (P(v["k_new"].data_ptr()), P(v["v_new"].data_ptr()),
                            P(self.slots.data_ptr()), wl.num_tokens, P(v["k_cache"].data_ptr()),
                            P(v["v_cache"].data_ptr()), ctypes.byref(self.desc), self.sp)
        self.append_fn = self.lib.pa_kv_append
        if wl.kv_quant:                                  # quantised cache: codes + scales
            self.args_append = self.args_append[:6] + (P(v["k_scale"].data_ptr()),
                                                       P(v["v_scale"].data_ptr())) + \
                self.args_append[6:]
            self.append_fn = self.lib.pa_kv_append_quant
        self.args_decode = (P(self.out.data_ptr()), P(v["q"].data_ptr()),
                            P(v["k_cache"].data_ptr()), P(v["v_cache"].data_ptr()),
                            P(self.tables.data_ptr()), int(self.tables.shape[1]),
                            P(self.ctx.data_ptr()), wl.max_context_len, wl.num_seqs,
                            wl.num_heads, ctypes.c_float(wl.scale), ctypes.byref(self.desc)) + \
            ((group_size,) if group_size > 1 else ()) + \
            (self.ps, P(self.ws.data_ptr()), ctypes.c_size_t(self.ws_bytes), self.sp)
        self.decode_fn = self.lib.pa_decode_grouped if group_size > 1 else self.lib.pa_decode
        scales = (P(v["k_scale"].data_ptr()), P(v["v_scale"].data_ptr())) if wl.kv_quant else ()
        if wl.kv_quant:
            self.args_decode = self.args_decode[:4] + scales + self.args_decode[4:]
            self.decode_fn = (self.lib.pa_decode_grouped_quant if group_size > 1
                              else self.lib.pa_decode_quant)
        if self.multi:
            self.args_decode = (P(self.out.data_ptr()), P(v["q"].data_ptr()),
                                P(v["k_cache"].data_ptr()), P(v["v_cache"].data_ptr())) + \
                scales + (P(self.tables.data_ptr()), int(self.tables.shape[1]),
                          P(self.ctx.data_ptr()), P(self.query_start.data_ptr()),
                          wl.max_context_len, wl.num_seqs, wl.num_query_rows,
                          wl.max_query_len, wl.num_heads, ctypes.c_float(wl.scale),
                          ctypes.byref(self.desc), self.ps, P(self.ws.data_ptr()),
                          ctypes.c_size_t(self.ws_bytes), self.sp)
            self.decode_fn = self.lib.pa_decode_multi_quant if wl.kv_quant else self.lib.pa_decode_multi
        self.has_copy = wl.copy_pairs.shape[0] > 0
        self.has_append = wl.num_tokens > 0
        self.launches_per_step = (self.num_partitions > 1) + 1 + int(self.has_append) + \
            (-(-int(wl.copy_pairs.shape[0]) // 65535) if self.has_copy else 0)
        self.step_bytes = wl.decode_bytes() + wl.append_bytes() + wl.copy_bytes()

    def run(self, ev=None):
        """Enqueue one step; ev = (start, after_moves, end) events or None."""
        lib = self.lib
        if ev:
            ev[0].record(self.stream)
        if self.has_copy:
            rc = lib.pa_block_copy(*self.args_copy)
            if rc:
                raise RuntimeError(lib.pa_get_last_error().decode())
        if self.has_append:
            rc = self.append_fn(*self.args_append)
            if rc:
                raise RuntimeError(lib.pa_get_last_error().decode())
        if ev:
            ev[1].record(self.stream)
        rc = self.decode_fn(*self.args_decode)
        if rc:
            raise RuntimeError(lib.pa_get_last_error().decode())
        if ev:
            ev[2].record(self.stream)

    def release(self):
        del self.vals, self.out, self.ws


L2_BYTES = 126 * 10**6


def needs_flush(wl) -> bool:
    """Flush L2 between steps only when the step's inputs could stay in it."""
    unique = wl.unique_kv_bytes() if wl.copy_pairs.shape[0] else wl.kv_bytes()
    return unique < 2 * L2_BYTES


def time_steps(step, steps, warmup, flush, barrier=None):
    """Device time of `steps` steps with per-step events; `flush` (a tensor or
    None) is overwritten before each step to evict L2."""
    torch = step.torch
    for _ in range(warmup):
        if flush is not None:
            flush.zero_()
        step.run()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if barrier:
        barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        step.run(evs[i])
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if barrier:
        barrier()
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    mov_ms = [e[0].elapsed_time(e[1]) for e in evs]
    lib = step.lib
    rc = lib.pa_sync_check(step.sp)
    if rc:
        raise RuntimeError("kernel status: " + lib.pa_get_last_error().decode())
    return {"step_ms": step_ms, "decode_ms": dec_ms, "moves_ms": mov_ms,
            "wall": (t_wall0, t_wall1)}


def swap_bandwidth(device, blocks=1024, reps=5):
    """pa_block_swap of `blocks` scattered blocks of the 13B pool shape (40 kv heads
    x 16 slots x 128 dims, bf16: 160 KiB per block per cache) to a pinned host pool
    and back, next to the copy engine moving one contiguous buffer of the same size."""
    import torch

    import paged_kv_cache_335_b200 as pa
    shape = (40, 16, 128)
    dev_blocks, host_blocks = 2 * blocks + 64, blocks + 16
    kd = torch.randn((dev_blocks,) + shape, device=device).to(torch.bfloat16)
    vd = torch.randn((dev_blocks,) + shape, device=device).to(torch.bfloat16)
    kh = torch.empty((host_blocks,) + shape, dtype=torch.bfloat16).pin_memory()
    vh = torch.empty((host_blocks,) + shape, dtype=torch.bfloat16).pin_memory()
    g = torch.Generator().manual_seed(5)
    src = torch.randperm(dev_blocks, generator=g)[:blocks]
    dst = torch.randperm(host_blocks, generator=g)[:blocks]
    out_pairs = torch.stack([src, dst], 1).to(device)
    in_pairs = torch.stack([dst, torch.randperm(dev_blocks, generator=g)[:blocks]], 1).to(device)
    nbytes = 2 * blocks * kd[0].numel() * kd.element_size()
    flat_d = torch.empty(nbytes // 2, dtype=torch.bfloat16, device=device)
    flat_h = torch.empty(nbytes // 2, dtype=torch.bfloat16).pin_memory()

    def timed(fn):
        ts = []
        for i in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i:
                ts.append(e0.elapsed_time(e1) / 1e3)
        return nbytes / statistics.median(ts) / 1e9

    res = {
        "blocks": blocks, "bytes_per_direction": nbytes,
        "out_gbs": round(timed(lambda: pa.pa_block_swap(out_pairs, kd, vd, kh, vh)), 1),
        "in_gbs": round(timed(lambda: pa.pa_block_swap(in_pairs, kh, vh, kd, vd)), 1),
        "copy_engine_d2h_gbs": round(timed(lambda: flat_h.copy_(flat_d, non_blocking=True)), 1),
        "copy_engine_h2d_gbs": round(timed(lambda: flat_d.copy_(flat_h, non_blocking=True)), 1),
    }
    pa.pa_sync_check()
    del kd, vd, kh, vh, flat_d, flat_h
    torch.cuda.empty_cache()
    return res


def measure_config(w2, device, ps, gs, consumer, args, flush_buf, hbm_peak, read_gbs):
    """Decode figures of one extra configuration (same step timing as the headline)."""
    import paged_kv_cache_335_b200 as pa
    prev = None
    if consumer == "tcgen05":
        prev = pa.pa_set_grouped_consumer(pa.PA_GROUPED_TCGEN05)
    try:
        st = Step(w2, device, partition_size=ps, group_size=gs)
        try:
            r2 = time_steps(st, min(args.steps, 50), 3, flush_buf if needs_flush(w2) else None)
            sm = statistics.median(r2["step_ms"])
            dm = statistics.median(r2["decode_ms"])
            gbs = w2.decode_bytes() / (dm / 1e3) / 1e9
            return {
                "decode_gbs": round(gbs, 1),
                "decode_frac_of_peak": round(gbs / hbm_peak, 4),
                "decode_frac_of_datasheet": round(gbs / DATASHEET_HBM_GBS, 4),
                "decode_frac_of_stream_read": round(gbs / read_gbs, 4) if read_gbs else None,
                "decode_us": round(dm * 1e3, 2),
                "decode_us_pct": pct(r2["decode_ms"], 1e3),
                "step_us": round(sm * 1e3, 2),
                "moves_us": round(statistics.median(r2["moves_ms"]) * 1e3, 2),
                "seq_steps_per_s": round(w2.num_seqs / (sm / 1e3), 1),
                "partitions": st.num_partitions,
                "partition_size": "library policy" if st.ps == 0 else st.ps,
                "group_size": gs,
                "grouped_consumer": consumer or args.grouped_consumer,
                "decode_bytes": w2.decode_bytes(),
                "unique_kv_bytes": w2.unique_kv_bytes() if w2.name.startswith("cow") else None,
            }
        finally:
            st.release()
            del st
    finally:
        if prev is not None:
            pa.pa_set_grouped_consumer(prev)


def e2e_steps(step, steps, warmup):
    """The same step through the Python binding of the C ABI with inputs in
    pinned HOST memory: the H2D copy of every step's inputs and the D2H read of
    its output are inside the timed region. As a serving loop would issue them,
    the copies run on two copy streams against double-buffered device inputs and
    outputs, so step i's inputs cross the link while step i - 1 decodes and its
    output comes back while step i + 1 decodes; events order every buffer reuse
    (a buffer is refilled only after the kernels and the read of two steps back
    are done)."""
    import paged_kv_cache_335_b200 as pa
    torch = step.torch
    wl, v = step.wl, step.vals
    host = {"q": v["q"].cpu().pin_memory(), "k_new": v["k_new"].cpu().pin_memory(),
            "v_new": v["v_new"].cpu().pin_memory(),
            "tables": step.tables.cpu().pin_memory(), "ctx": step.ctx.cpu().pin_memory(),
            "slots": step.slots.cpu().pin_memory(), "pairs": step.pairs.cpu().pin_memory()}
    if step.multi:
        host["query_start"] = step.query_start.cpu().pin_memory()
    devs = [{k: torch.empty_like(t, device=v["q"].device) for k, t in host.items()} for _ in range(2)]
    outs = [step.out, torch.empty_like(step.out)]
    outs_host = [torch.empty_like(step.out, device="cpu").pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    in_ready, in_free = [ev(), ev()], [ev(), ev()]
    out_ready, out_free = [ev(), ev()], [ev(), ev()]

    def one(i):
        b = i % 2
        dev, out = devs[b], outs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(in_free[b])          # the kernels of step i - 2 read these
            for k in host:
                dev[k].copy_(host[k], non_blocking=True)
            in_ready[b].record(s_in)
        comp.wait_event(in_ready[b])
        comp.wait_event(out_free[b])             # the read of step i - 2's output is done
        if wl.copy_pairs.shape[0]:
            pa.pa_block_copy(dev["pairs"], v["k_cache"], v["v_cache"])
        if wl.num_tokens and wl.kv_quant:
            pa.pa_kv_append_quant(dev["k_new"], dev["v_new"], dev["slots"], v["k_cache"],
                                  v["v_cache"], v["k_scale"], v["v_scale"])
        elif wl.num_tokens:
            pa.pa_kv_append(dev["k_new"], dev["v_new"], dev["slots"], v["k_cache"], v["v_cache"])
        if wl.kv_quant and step.multi:
            pa.pa_decode_multi_quant(out, dev["q"], v["k_cache"], v["v_cache"], v["k_scale"],
                                     v["v_scale"], dev["tables"], dev["ctx"], dev["query_start"],
                                     wl.scale, max_context_len=wl.max_context_len,
                                     max_query_len=wl.max_query_len, partition_size=step.ps,
                                     workspace=step.ws)
        elif wl.kv_quant and step.group_size > 1:
            pa.pa_decode_grouped_quant(out, dev["q"], v["k_cache"], v["v_cache"],
                                       v["k_scale"], v["v_scale"], dev["tables"], dev["ctx"],
                                       wl.scale, step.group_size,
                                       max_context_len=wl.max_context_len,
                                       partition_size=step.ps, workspace=step.ws)
        elif wl.kv_quant:
            pa.pa_decode_quant(out, dev["q"], v["k_cache"], v["v_cache"], v["k_scale"],
                               v["v_scale"], dev["tables"], dev["ctx"], wl.scale,
                               max_context_len=wl.max_context_len, partition_size=step.ps,
                               workspace=step.ws)
        elif step.multi:
            pa.pa_decode_multi(out, dev["q"], v["k_cache"], v["v_cache"], dev["tables"],
                               dev["ctx"], dev["query_start"], wl.scale,
                               max_context_len=wl.max_context_len,
                               max_query_len=wl.max_query_len, partition_size=step.ps,
                               workspace=step.ws)
        elif step.group_size > 1:
            pa.pa_decode_grouped(out, dev["q"], v["k_cache"], v["v_cache"], dev["tables"],
                                 dev["ctx"], wl.scale, step.group_size,
                                 max_context_len=wl.max_context_len, partition_size=step.ps,
                                 workspace=step.ws)
        else:
            pa.pa_decode(out, dev["q"], v["k_cache"], v["v_cache"], dev["tables"],
                         dev["ctx"], wl.scale, max_context_len=wl.max_context_len,
                         partition_size=step.ps, workspace=step.ws)
        in_free[b].record(comp)
        out_ready[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(out_ready[b])
            outs_host[b].copy_(out, non_blocking=True)
            out_free[b].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        one(i)
    for b in range(2):
        comp.wait_event(out_free[b])             # every output is back in host memory
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return ms, h2d, d2h


# ---------------------------------------------------------------------------
# oracle (CPU) timing
# ---------------------------------------------------------------------------
def oracle_sample(wl, target_s, threads):
    """Time the oracle's step (copies, append, decode) on a bounded sample of the
    workload's sequences; returns (GB/s, seconds, sample description, bytes)."""
    import numpy as np
    import torch

    import oracle
    from paged_kv_cache_335_b200 import workloads as W

    def run(ids):
        sub = W.restrict(wl, ids)
        vals = W.make_values(sub, "cpu", poison=False)
        host = {k: (t.numpy().copy() if t.dtype == torch.float32 and t.dim() == 1
                    else W.to_numpy(t).copy()) for k, t in vals.items()}
        t0 = time.perf_counter()
        if sub.copy_pairs.shape[0]:
            oracle.block_copy(sub.copy_pairs, host["k_cache"], host["v_cache"])
        if sub.num_tokens and sub.kv_quant:
            oracle.kv_append_quant(host["k_new"], host["v_new"], sub.slot_mapping,
                                   host["k_cache"], host["v_cache"], host["k_scale"],
                                   host["v_scale"], sub.kv_quant)
        elif sub.num_tokens:
            oracle.kv_append(host["k_new"], host["v_new"], sub.slot_mapping, host["k_cache"],
                             host["v_cache"])
        if sub.kv_quant and sub.query_start is not None:
            # each query token as a row of its own, at its causal end
            qs = np.asarray(sub.query_start)
            rows_t, rows_c = [], []
            for s in range(sub.num_seqs):
                n = int(qs[s + 1] - qs[s])
                for j in range(n):
                    rows_t.append(sub.block_tables[s])
                    rows_c.append(int(sub.context_lens[s]) - n + j + 1)
            oracle.decode_quant(host["q"], host["k_cache"], host["v_cache"], host["k_scale"],
                                host["v_scale"],
                                np.asarray(rows_t, np.int32).reshape(len(rows_c), -1),
                                np.asarray(rows_c, np.int32), sub.scale, sub.kv_quant,
                                num_threads=threads)
        elif sub.kv_quant:
            oracle.decode_quant(host["q"], host["k_cache"], host["v_cache"], host["k_scale"],
                                host["v_scale"], sub.block_tables, sub.context_lens, sub.scale,
                                sub.kv_quant, num_threads=threads)
        elif sub.query_start is not None:
            oracle.decode_multi(host["q"], host["k_cache"], host["v_cache"], sub.block_tables,
                                sub.context_lens, sub.query_start, sub.scale,
                                num_threads=threads)
        else:
            oracle.decode(host["q"], host["k_cache"], host["v_cache"], sub.block_tables,
                          sub.context_lens, sub.scale, num_threads=threads)
        dt = time.perf_counter() - t0
        return dt, sub.decode_bytes() + sub.append_bytes() + sub.copy_bytes(), sub

    rng = np.random.default_rng(12345)
    order = rng.permutation(wl.num_seqs)
    probe = max(1, min(wl.num_seqs, threads // max(1, wl.num_heads) + 1))
    dt, _, _ = run(order[:probe])
    per_seq = dt / probe
    n = int(min(wl.num_seqs, max(probe, math.ceil(target_s / max(per_seq, 1e-6)))))
    dt, nbytes, sub = run(order[:n])
    desc = (f"oracle step on {n} of {wl.num_seqs} sequences (all {wl.num_heads} heads, "
            f"{int(sub.context_lens.sum())} context tokens), {threads} threads")
    return nbytes / dt / 1e9, dt, desc, nbytes


def reference_arm(args):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    from paged_kv_cache_335_b200 import workloads as W
    wl = W.make(args.config)
    threads = host_cores()
    per_step = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, per_step, threads)
    vals, secs, desc = [], [], ""
    for _ in range(args.steps):
        gbs, dt, desc, _ = oracle_sample(wl, per_step, threads)
        vals.append(gbs)
        secs.append(dt)
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(wl, needs_flush(wl)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl, flush=False):
    return {"workload": wl.name, "num_seqs": wl.num_seqs, "num_heads": wl.num_heads,
            "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
            "block_size": wl.block_size, "dtype": wl.dtype,
            "context_tokens": int(wl.context_lens.sum()),
            "max_context_len": wl.max_context_len, "copy_pairs": int(wl.copy_pairs.shape[0]),
            "appended_tokens": wl.num_tokens, "pool_blocks": wl.num_blocks,
            "l2": ("flushed between timed steps (512 MiB write)" if flush else
                   f"not flushed: inputs larger than L2 ({(wl.unique_kv_bytes() if wl.copy_pairs.shape[0] else wl.kv_bytes()) / 1e9:.2f} GB unique K/V per step vs 126 MB L2)"),
            "description": wl.description}


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------
def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    import torch
    import torch.distributed as dist

    import paged_kv_cache_335_b200 as pa
    from paged_kv_cache_335_b200 import build as pbuild
    from paged_kv_cache_335_b200 import workloads as W

    rank, local_rank, world = dist_env()
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if rank == 0:
        pbuild.build()
    if world > 1:
        dist.barrier()
    pa.load_library()
    hbm_peak, peak_kind, peak_doc = peaks()

    def barrier():
        if world > 1:
            dist.barrier()

    flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    wl = W.make(args.config)
    if args.partition_size is not None:
        wl.partition_size = args.partition_size
    import paged_kv_cache_335_b200 as pa
    pa.pa_set_grouped_consumer(pa.PA_GROUPED_TCGEN05 if args.grouped_consumer == "tcgen05"
                               else pa.PA_GROUPED_MMA_SYNC)
    step = Step(wl, device, seed_offset=rank, group_size=args.group_size)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        uuid = str(local_rank)
    clocks = ClockSampler(uuid)
    clocks.start()
    flush = flush_buf if needs_flush(wl) else None
    res = time_steps(step, args.steps, args.warmup, flush, barrier)
    t0, t1 = res["wall"]
    # the timed region is short: continue the same (untimed) loop for >= 1.5 s so
    # the 100 ms clock samples describe the clocks under this load
    probe_t1 = t1
    if t1 - t0 < 1.5:
        t_end = time.time() + 1.5
        while time.time() < t_end:
            for _ in range(20):
                if flush is not None:
                    flush.zero_()
                step.run()
            torch.cuda.synchronize()
        probe_t1 = time.time()
    clk = clocks.summary(t0, probe_t1)
    remeasured = False
    if bad_clocks(clk):
        res = time_steps(step, args.steps, args.warmup, flush, barrier)
        t0, t1 = res["wall"]
        clk = clocks.summary(t0, max(t1, t0 + 0.3))
        remeasured = True
    clocks.stop()
    clk["window"] = ("timed region" if probe_t1 == t1 else
                     "timed region + untimed continuation of the same step loop")
    if remeasured:
        clk["remeasured"] = True

    total_ms = dist_max(sum(res["step_ms"]), device)
    ms_per_step = total_ms / args.steps
    value = weak_scaling_value(step.step_bytes, args.steps, world, total_ms)
    dec_ms = statistics.mean(res["decode_ms"])
    dec_gbs = wl.decode_bytes() / (dec_ms / 1e3) / 1e9
    kernel_file = os.path.join(ROOT, "paged_kv_cache_335_b200", "csrc", "pa_decode_tma.cu")
    kernel_name = KERNEL_NAMES.get(step.lib.pa_test_last_decode_kernel(), "unknown")
    if step.num_partitions > 1:
        kernel_name += " + partition_reduce_kernel"
    tag = wl.name if args.group_size == 1 else f"{wl.name}_grouped{args.group_size}"
    if step.lib.pa_test_last_decode_kernel() == pa.PA_KERNEL_GROUPED_TCGEN05:
        tag += "_tcgen05"
    traffic, sha = profile_traffic(kernel_file, tag)

    # end to end through the public binding with host buffers
    e2e_ms, h2d, d2h = e2e_steps(step, args.steps, max(3, args.warmup))
    e2e_ms = dist_max(e2e_ms, device)
    e2e_value = weak_scaling_value(step.step_bytes, args.steps, world, e2e_ms)
    launches = step.launches_per_step * args.steps
    step_ps, step_np = step.ps, step.num_partitions
    step.release()
    del step
    torch.cuda.empty_cache()

    read_gbs = stream_read_gbs(device) if world == 1 else None
    per_config = {}
    if world == 1 and not args.no_extra_configs:
        for label, name, ps, gs, consumer in EXTRA_CONFIGS:
            try:
                per_config[label] = measure_config(W.make(name), device, ps, gs, consumer, args,
                                                   flush_buf, hbm_peak, read_gbs)
            except Exception as e:  # one configuration failing must not lose the others
                print(f"bench: configuration {label} failed: {e!r}", file=sys.stderr)
                per_config[label] = {"error": repr(e)[:300]}
            torch.cuda.empty_cache()
        per_config["swap_llama13b_blocks"] = swap_bandwidth(device)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = host_cores()
        gbs, secs, desc, _ = oracle_sample(wl, args.cpu_seconds, threads)
        gbs1, secs1, desc1, _ = oracle_sample(wl, args.cpu_seconds / 2, 1)
        cpu = {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc, "seconds": round(secs, 2),
               "single_thread": {"value": gbs1, "unit": UNIT, "cores": 1, "sample": desc1,
                                 "seconds": round(secs1, 2)}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic (seeded N(0,1) values, seeded shapes)",
            "config": config_dict(wl, flush is not None),
            "launch": {"group_size": args.group_size, "grouped_consumer": args.grouped_consumer,
                       "partition_size": "library policy" if step_ps == 0 else step_ps,
                       "partitions": step_np},
            "step_us_pct": pct(res["step_ms"], 1e3),
            "decode_us_pct": pct(res["decode_ms"], 1e3),
            "seq_steps_per_s": round(world * wl.num_seqs / (ms_per_step / 1e3), 1),
            "frac_of_hbm_peak": round(value / world / hbm_peak, 4),
            "reference_bandwidths_gbs": {
                "measured_copy_hbm_gbs": hbm_peak, "datasheet": DATASHEET_HBM_GBS,
                "stream_read_this_run": round(read_gbs, 1) if read_gbs else None},
            "decode_frac_of_stream_read": round(dec_gbs / read_gbs, 4) if read_gbs else None,
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm_peak,
                         "unit": "GB/s", "frac": round(dec_gbs / hbm_peak, 4),
                         "frac_of_datasheet": round(dec_gbs / DATASHEET_HBM_GBS, 4),
                         "traffic": traffic,
                         "kernel": kernel_name,
                         "algorithmic_bytes_per_launch": wl.decode_bytes(),
                         "avg_launch_us": round(dec_ms * 1e3, 2),
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"
                         if peak_kind == "measured" else "fallback 6.65 TB/s",
                         "kernel_source_sha256": sha},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clk,
            "configs": per_config or None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
