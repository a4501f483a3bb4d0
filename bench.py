#!/usr/bin/env python
"""Benchmark of the fused QK-norm + RoPE + quant + paged-append path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one fused call (one kernel: validation, Q/K RMSNorm, RoPE, FP8
quantisation, paged K/V scatter, last-page tail zeroing, flags) over one batch
of the ragged FP8 prefill workload: 16 requests with U[0, 2048] new tokens
each (two empty; 9,212 tokens in all) on U[0, 4096] prior context, Hq 64 /
Hkv 8, head_dim 128, page 16, static FP8 E4M3 Q/K/V.  Inputs are synthetic
and seeded (workloads.py).  Each step uses its own replica of the step inputs
(packed QKV, metadata, page table, out_q: the same token counts with other
data, positions and pages), and a step's data (288 MB) is larger than L2
(126 MB); the timed launches are replayed from CUDA graphs.

Rank 0 prints one JSON line.  The timed region (exactly K launches) is
repeated; `ms_per_step` and `value` come from the median region.  `value` =
tokens/s over all ranks (the max-over-ranks device time of a region);
`roofline` = algorithmic bytes per launch / median launch time, against the
measured HBM copy bandwidth; `e2e` = the same metric through the public API
with pinned host buffers (host->device copies of the step's inputs and
device->host copies of out_q and flags inside the timed region);
`cpu_baseline` = the CPU oracle on a bounded sample, single-threaded
(`cpu_baseline_all_cores`: one process per host core on disjoint requests);
`per_config` (last, compact) adds every named workload measured the same way
outside the timed region: microseconds per launch, fraction of the peak, the
two schedules forced, and the floor -- a plain copy kernel moving the same
bytes in one launch (libfqr_floor.so).

--impl reference times the CPU oracle (the reference arm of this build) on
the host cores on the same workload, metric and unit.
"""
from __future__ import annotations

import argparse
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused QKnorm+RoPE+quant+paged-append tokens/s and HBM GB/s (% of peak), 1 B200"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
MAIN_WORKLOAD = "ragged_prefill_fp8"
MIN_TIMED_LAUNCHES = 200
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--repeats", type=int, default=None,
                    help="timed regions of exactly --steps launches each (default: at least 5, "
                         "and at least 200 launches in all); the median region is reported")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=MAIN_WORKLOAD, choices=sorted(workloads.APPEND_CONFIGS))
    ap.add_argument("--replicas", type=int, default=None, help="override the replica count")
    ap.add_argument("--schedule", type=int, default=0, choices=[0, 1, 2],
                    help="0 automatic, 1 latency, 2 streaming")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU budget of the oracle baseline sample")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--profile", action="store_true",
                    help="profiling run: only --workload (or mla_decode), --steps eager launches, "
                         "no graphs, no e2e / per-config / CPU legs, no JSON line")
    ap.add_argument("--mla", action="store_true", help="with --profile: the MLA workload")
    ap.add_argument("--mla-workload", default="mla_decode", choices=sorted(workloads.MLA_CONFIGS),
                    help="with --profile --mla: which MLA workload")
    ap.add_argument("--small-cache", action="store_true",
                    help="with --profile: wrap sequence lengths to 1024 (same bytes per call, "
                         "a cache of 1024 slots per request)")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ helpers

def describe_plan(plan: dict) -> str:
    """The launch fqr_append_plan_query reports, in words."""
    if plan["schedule"] == 2:
        return (f"fqr::pipe_append_kernel (streaming schedule: {plan['grid']} blocks of "
                f"{plan['block_threads']} threads, {plan['tasks']} units; chosen automatically)")
    extra = [("warp-level batch check" if plan["warp_check"] else "block batch prologue"),
             "quad-major head tasks"]
    if plan["bulk_tails"]:
        extra.append("bulk-copy tails")
    if plan["request_tails"]:
        extra.append("request tasks own the tails")
    return (f"fqr::warp_append_kernel (latency schedule: {plan['grid']} blocks of "
            f"{plan['block_threads']} threads, {plan['tasks']} warp tasks, " + ", ".join(extra) +
            "; chosen automatically)")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs: copy, read+write)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


# The sources the fused append's kernels are built from (the MLA kernels, the
# host entry points and the runtime are not among them).
APPEND_KERNEL_SOURCES = ("fqr_append.cu", "fqr_append_pipe.cu", "fqr_append_warp.cu",
                         "fqr_device.cuh", "fqr_head.cuh", "fqr_launch.h")


def _code_tokens(text: str) -> str:
    """A source file without its comments and with whitespace collapsed (the
    sources hold no string literal with a comment marker)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(names=APPEND_KERNEL_SOURCES) -> str:
    """Hash of the append kernels' code: comments and layout do not change it."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "qk_norm_rope_token_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update((name + "\n" + _code_tokens(f.read())).encode())
    return h.hexdigest()[:16]


TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "traffic.json")


def profiled_traffic(workload: str):
    """Measured memory traffic per launch of this workload's kernel, from the
    committed ncu record profiles/traffic.json, if it was captured on the
    current append-kernel sources.  Returns (traffic bytes or None, details).

    traffic = dram__bytes_read.sum + 32 x lts__t_sectors_srcnode_gpc_op_write.sum:
    reads counted at DRAM, writes where the SMs issue them into L2 (a
    write-back cache: a launch's last writes are still in L2 when it ends, so
    dram__bytes_write undercounts them; every sector written reaches DRAM
    once).  lts__t_sectors_op_write.sum would count again the writes that
    cross the die-to-die fabric to their home L2 slice."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None, {"note": "no traffic record"}
    if rec.get("kernel_sources") != kernel_source_hash():
        return None, {"note": "traffic record taken on other kernel sources"}
    e = rec.get("workloads", {}).get(workload)
    if not e:
        return None, {"note": f"no traffic record for {workload}"}
    t = int(e["dram_read_bytes"]) + int(e["gpc_write_bytes"])
    return t, {"dram_read": int(e["dram_read_bytes"]), "sm_write_into_l2": int(e["gpc_write_bytes"]),
               "dram_write": int(e["dram_write_bytes"]),
               "basis": "ncu: dram__bytes_read.sum + 32 x lts__t_sectors_srcnode_gpc_op_write.sum "
                        "per launch (profiles/traffic.json)"}


class ClockSampler:
    """nvidia-smi sampling of one GPU during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fd, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = self.t1 = None

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        os.close(self.fd)
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[1]), float(parts[2]), parts[3], parts[5:9]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if self.t0 and self.t1 and self.t0 - 0.15 <= r[0] <= self.t1 + 0.15]
        window = "timed region"
        if len(inside) < 3:
            inside, window = rows, "warm-up and timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in inside for n, v in zip(names, r[4]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "window": window}


def gpu_smi_id(torch, dev) -> str:
    """nvidia-smi --id of the GPU torch calls `dev` (its UUID)."""
    props = torch.cuda.get_device_properties(dev)
    u = str(getattr(props, "uuid", ""))
    if u and not u.startswith("GPU-"):
        u = "GPU-" + u
    return u or str(dev.index)


# -------------------------------------------------------- device workloads

def replica_workloads(name, min_bytes=3 * L2_BYTES, max_replicas=64, seed_offset=0,
                      small_cache=False):
    """The replicas a bench of workload `name` rotates over: enough that one
    cycle moves at least `min_bytes` (at least 2, at most `max_replicas`).
    Replica r is the workload drawn with seed base + seed_offset + 7919 r; a
    workload that draws its token counts (the ragged prefill) keeps the first
    replica's counts, so that every step has the same tokens and shape."""
    make = workloads.APPEND_CONFIGS[name]
    if small_cache:
        def make(seed=None, _f=workloads.APPEND_CONFIGS[name], **kw):
            return workloads.shrink_cache(_f(**kw) if seed is None else _f(seed=seed, **kw))
    base = make()
    R = replica_count(base, min_bytes, max_replicas)
    base_n = np.diff(base.q_indptr)
    ws = []
    for r in range(R):
        sd = base.seed + seed_offset + 7919 * r
        rep = base if sd == base.seed else make(seed=sd)
        if rep.T != base.T:
            rep = make(seed=sd, n_new=base_n)
        ws.append(rep)
    return ws


class AppendBench:
    """R replicas of one append workload sharing one pair of KV caches."""

    def __init__(self, name, torch, fqr, device, min_bytes=3 * L2_BYTES, max_replicas=64,
                 seed_offset=0, schedule=0, small_cache=False):
        self.torch, self.fqr, self.dev = torch, fqr, device
        self.schedule = schedule
        ws = replica_workloads(name, min_bytes, max_replicas, seed_offset, small_cache)
        self.R = len(ws)
        base = ws[0]
        self.name = base.name
        self.ws = ws
        self.bytes = [workloads.append_bytes(w)["total"] for w in ws]
        self.T = base.T
        w0 = ws[0]
        es = w0.kv_esize
        dt = torch.int16 if es == 2 else torch.uint8
        shape = (w0.num_pages, w0.page_size, w0.Hkv, 128)
        self.k_cache = torch.empty(shape, dtype=dt, device=device)
        self.v_cache = torch.empty(shape, dtype=dt, device=device)
        self.cs = self._d(w0.cos_sin)
        self.qw = self._d(w0.q_norm_w)
        self.kw = self._d(w0.k_norm_w)
        self.scales = {k: torch.tensor([v], dtype=torch.float32, device=device)
                       for k, v in (("q_scale_inv", w0.q_scale_inv), ("k_scale", w0.k_scale),
                                    ("v_scale", w0.v_scale))}
        self.reps = []
        for w in ws:
            st = dict(qkv=self._d(w.qkv), q_indptr=self._d(w.q_indptr),
                      seq_lens=self._d(w.seq_lens), page_table=self._d(w.page_table),
                      out_q=torch.empty((w.T, w.Hq, 128), dtype=dt if w.quant_policy == 0
                                        else torch.uint8, device=device),
                      q_scale=torch.empty(w.q_scale_shape if w.T else (1, w.Hq),
                                          dtype=torch.float32, device=device),
                      flags=torch.empty((w.B,), dtype=torch.int32, device=device))
            if w.out_kv:   # caller-owned K/V rows instead of the paged caches
                kdt = dt if w.quant_policy == 0 else torch.uint8
                st["out_k"] = torch.empty((w.T, w.Hkv, 128), dtype=kdt, device=device)
                st["out_v"] = torch.empty((w.T, w.Hkv, 128), dtype=kdt, device=device)
            st["params"] = self._params(w, st)
            self.reps.append(st)

    def _d(self, a):
        if a is None:
            return None
        t = self.torch.from_numpy(np.ascontiguousarray(a))
        if t.dtype == self.torch.uint16:
            t = t.view(self.torch.int16)
        return t.to(self.dev)

    def kw_for(self, w, st):
        return dict(q_norm_w=self.qw, k_norm_w=self.kw, eps=w.eps, rope_style=w.rope_style,
                    rot_dim=w.rot_dim, quant_policy=w.quant_policy,
                    q_scale=st["q_scale"] if w.quant_policy == 1 else None,
                    q_scale_inv=self.scales["q_scale_inv"] if w.quant_policy == 2 else None,
                    k_scale=self.scales["k_scale"] if w.quant_policy else None,
                    v_scale=self.scales["v_scale"] if w.quant_policy else None,
                    upper_max=w.upper_max, schedule=self.schedule, max_seqlen=w.max_seqlen,
                    norm_style=w.norm_style, out_k=st.get("out_k"), out_v=st.get("out_v"))

    def _params(self, w, st):
        return self.fqr.append_params(st["qkv"], self.cs, st["q_indptr"], st["seq_lens"],
                                      st["page_table"], self.k_cache, self.v_cache, st["out_q"],
                                      st["flags"], **self.kw_for(w, st))

    def launch(self, i, stream_handle):
        rc = self.fqr.append_paged_raw(self.reps[i % self.R]["params"], stream_handle)
        if rc != 0:
            raise self.fqr.FqrError(rc)

    def check_flags(self):
        for st in self.reps:
            assert int(st["flags"].abs().max()) == 0, "a replica was flagged"


class MlaBench:
    def __init__(self, torch, fqr, device, min_bytes=3 * L2_BYTES, max_replicas=256,
                 name="mla_decode"):
        self.torch, self.fqr, self.dev = torch, fqr, device
        base = workloads.MLA_CONFIGS[name]()
        self.name = base.name
        per = workloads.mla_bytes(base)["total"]
        self.R = int(min(max_replicas, max(2, math.ceil(min_bytes / per))))
        self.ws = [base] + [workloads.make_mla(seed=base.seed + 7919 * r, n_new=[1] * base.B,
                                               seq_lens=base.seq_lens, Hq=base.Hq,
                                               block_size=base.block_size,
                                               max_blocks=base.max_blocks,
                                               cos_sin_rows=base.cos_sin_rows,
                                               q_quant=base.q_quant,
                                               q_scale_inv=base.q_scale_inv,
                                               upper_max=base.upper_max,
                                               q_group=base.q_group)
                            for r in range(1, self.R)]
        self.bytes = [workloads.mla_bytes(w)["total"] for w in self.ws]
        self.T = base.T
        self.latent = torch.empty((base.num_blocks, base.block_size, base.width),
                                  dtype=torch.uint8, device=device)
        self.cs = self._d(base.cos_sin)
        self.scale = torch.tensor([base.kv_scale], dtype=torch.float32, device=device)
        self.params = []
        self.keep = []
        self.qsi = torch.tensor([base.q_scale_inv], dtype=torch.float32, device=device)
        for w in self.ws:
            q, kv_c, k_pe = self._d(w.q), self._d(w.kv_c), self._d(w.k_pe)
            ind, sl, bt = self._d(w.q_indptr), self._d(w.seq_lens), self._d(w.block_table)
            flags = torch.empty((w.B,), dtype=torch.int32, device=device)
            qq = {}
            if w.q_quant:   # Q quantised into q_out / q_scale (q read-only)
                q_out = torch.empty((w.T, w.Hq, w.nope_dim + w.rope_dim), dtype=torch.uint8,
                                    device=device)
                q_scale = torch.empty(w.q_scale_shape, dtype=torch.float32, device=device)
                qq = dict(q_quant=w.q_quant, q_scale_inv=self.qsi, upper_max=w.upper_max,
                          q_out=q_out, q_scale=q_scale, q_group=w.q_group)
            self.keep.append((q, kv_c, k_pe, ind, sl, bt, flags, qq))
            self.params.append(fqr.mla_params(q, kv_c, k_pe, self.cs, ind, sl, bt, self.latent,
                                              flags, nope_dim=w.nope_dim,
                                              rope_style=w.rope_style, kv_scale=self.scale,
                                              **qq))

    _d = AppendBench._d

    def launch(self, i, stream_handle):
        rc = self.fqr.concat_mla_cache_raw(self.params[i % self.R], stream_handle)
        if rc != 0:
            raise self.fqr.FqrError(rc)


class FloorBench:
    """The plain copy kernel of libfqr_floor.so moving a workload's read and
    write bytes (workloads.append_bytes) in one launch, over replicas of its
    source and destination buffers (a cycle larger than L2), launched like
    the fused kernel (programmatic dependent launch).  Its time per launch is
    the floor the fused kernel is compared with on small workloads."""

    def __init__(self, torch, device, read_bytes, write_bytes, min_bytes=3 * L2_BYTES,
                 max_replicas=64):
        import ctypes
        path = os.path.join(ROOT, "qk_norm_rope_token_b200", "libfqr_floor.so")
        self.lib = ctypes.CDLL(path)
        self.lib.fqr_floor_copy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint64,
                                            ctypes.c_uint64, ctypes.c_int, ctypes.c_void_p]
        self.lib.fqr_floor_copy.restype = ctypes.c_int
        self.rb = -(-int(read_bytes) // 16) * 16
        self.wb = -(-int(write_bytes) // 16) * 16
        per = self.rb + self.wb
        self.R = int(min(max_replicas, max(2, math.ceil(min_bytes / per))))
        self.src = [torch.randint(0, 1 << 30, (max(4, self.rb // 4),), dtype=torch.int32,
                                  device=device) for _ in range(self.R)]
        self.dst = [torch.empty(max(4, self.wb // 4), dtype=torch.int32, device=device)
                    for _ in range(self.R)]
        self.bytes = [per] * self.R
        vec = max(self.rb, self.wb) // 16
        self.blocks = int(min(4 * 148, max(1, -(-vec // 256))))

    def launch(self, i, stream_handle):
        k = i % self.R
        rc = self.lib.fqr_floor_copy(self.src[k].data_ptr(), self.dst[k].data_ptr(), self.rb,
                                     self.wb, self.blocks, stream_handle)
        if rc != 0:
            raise RuntimeError(f"fqr_floor_copy failed: {rc}")


def time_launches(torch, bench, steps, warmup, repeats=1, graph_chunk=1000, barrier=None,
                  marks=None):
    """Warm up, then time `repeats` regions of exactly `steps` launches each
    (replayed from CUDA graphs of up to `graph_chunk` launches, cycling over
    the replicas) with CUDA events on the launching stream, each region
    bracketed by a barrier and a device synchronisation.  Returns (the list of
    region times in ms, the algorithmic bytes of one region)."""
    stream = torch.cuda.current_stream()
    h = stream.cuda_stream
    for i in range(warmup):
        bench.launch(i, h)
    torch.cuda.synchronize()

    def capture(n, first):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            hs = torch.cuda.current_stream().cuda_stream
            for i in range(n):
                bench.launch(first + i, hs)
        return g

    chunk = max(1, min(graph_chunk, steps))
    # a chunk that is a multiple of R keeps every replay's replica set identical
    if chunk >= bench.R:
        chunk -= chunk % bench.R
    full, rest = divmod(steps, chunk)
    g_full = capture(chunk, 0) if full else None
    g_rest = capture(rest, 0) if rest else None
    # replay once untimed (graph upload)
    for g in (g_full, g_rest):
        if g is not None:
            g.replay()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if marks is not None:
        marks(True)
    times = []
    for _ in range(repeats):
        if barrier is not None:
            barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rest is not None:
            g_rest.replay()
        end.record(stream)
        torch.cuda.synchronize()
        if barrier is not None:
            barrier()
        times.append(start.elapsed_time(end))
    if marks is not None:
        marks(False)
    nbytes = sum(bench.bytes[i % bench.R] for i in range(chunk)) * full + \
        sum(bench.bytes[i % bench.R] for i in range(rest))
    del g_full, g_rest
    return times, nbytes


def e2e_measure(torch, fqr, bench, steps):
    """Same metric through the public API with pinned host buffers: every
    step copies its inputs host->device, runs the kernel and copies out_q and
    flags device->host (StagedAppend: copy-in of step i+1, kernel of step i
    and copy-out of step i-1 overlap on three streams)."""
    w0 = bench.ws[0]
    dev = bench.dev
    R = min(bench.R, 8)
    in_shapes = {"qkv": ((w0.T, w0.row_stride), torch.int16),
                 "q_indptr": ((w0.B + 1,), torch.int32), "seq_lens": ((w0.B,), torch.int32),
                 "page_table": (tuple(w0.page_table.shape), torch.int32)}
    out_shapes = {"out_q": (tuple(bench.reps[0]["out_q"].shape), bench.reps[0]["out_q"].dtype),
                  "flags": ((w0.B,), torch.int32)}
    if w0.quant_policy == 1:
        out_shapes["q_scale"] = (tuple(w0.q_scale_shape), torch.float32)
    kw = bench.kw_for(w0, {"q_scale": None})
    kw.pop("q_scale", None)
    sa = fqr.StagedAppend(in_shapes, out_shapes, dev, depth=3, cos_sin_cache=bench.cs,
                          k_cache=bench.k_cache, v_cache=bench.v_cache, **kw)
    host_in, host_out = [], []
    for w in bench.ws[:R]:
        hi, ho = sa.new_host_buffers()
        hi["qkv"].copy_(torch.from_numpy(w.qkv.view(np.int16)))
        hi["q_indptr"].copy_(torch.from_numpy(w.q_indptr))
        hi["seq_lens"].copy_(torch.from_numpy(w.seq_lens))
        hi["page_table"].copy_(torch.from_numpy(w.page_table))
        host_in.append(hi)
        host_out.append(ho)
    h2d = int(host_in[0]["_flat"].numel())
    d2h = int(host_out[0]["_flat"].numel())

    for i in range(20):
        sa.submit(host_in[i % R], host_out[i % R])
    sa.synchronize()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    sa.fork(stream)           # the pipeline's streams start after `start`
    for i in range(steps):
        sa.submit(host_in[i % R], host_out[i % R])
    sa.join(stream)           # `end` follows every step's copy-out
    end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    assert int(host_out[(steps - 1) % R]["flags"].abs().max()) == 0
    # the host outputs of the first replica's last step, for the check in the
    # cpu_baseline leg (outside the timed region)
    sample = {k: v.clone() for k, v in host_out[0].items() if not k.startswith("_")}
    sa.close()
    return {"value": bench.T * steps / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "api": "qk_norm_rope_token_b200.StagedAppend over the library's native pipeline "
                   "(fqr_pipeline_*: 3 streams, 3 staging slots, one copy each way per step)"}, sample


# ----------------------------------------------------------- CPU baselines

def oracle_sample(w, budget_s, max_calls=None, outputs=None):
    """Time the oracle as it stands on whole calls of workload w (host caches
    allocated lazily: only the pages a call touches are materialised).
    outputs: a dict that receives the last call's out_q, q_scale and flags."""
    import oracle
    es = w.kv_esize
    dt = np.uint16 if es == 2 else np.uint8
    shape = (w.num_pages, w.page_size, w.Hkv, 128)
    kc = np.zeros(shape, dt)
    vc = np.zeros(shape, dt)
    oq, qs, fl = oracle.new_outputs(w)
    calls, t0 = 0, time.perf_counter()
    while True:
        rc = oracle.append_paged(w, kc, vc, oq, qs if w.quant_policy == 1 else None, fl)
        assert rc == 0
        calls += 1
        el = time.perf_counter() - t0
        if (max_calls and calls >= max_calls) or (not max_calls and el >= budget_s):
            break
    if outputs is not None:
        outputs.update(out_q=oq, q_scale=qs, flags=fl)
    return calls, el


def cpu_baseline(w, budget_s, e2e_sample=None):
    """The oracle on whole calls of w for about budget_s; with e2e_sample (the
    e2e leg's host outputs of one step on w), also whether they are
    bit-identical to the oracle's."""
    outs = {}
    calls, el = oracle_sample(w, budget_s, outputs=outs)
    res = {"value": w.T * calls / el, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{calls} whole calls of {w.name} ({w.T} tokens each), "
                     f"{el:.1f} s single-threaded C oracle (fp32, -O2, no FMA)"}
    if e2e_sample is not None:
        same = {}
        for k in ("out_q", "q_scale", "flags"):
            if k in e2e_sample:
                got = e2e_sample[k].numpy()
                same[k] = bool(got.shape == outs[k].shape
                               and got.tobytes() == np.ascontiguousarray(outs[k]).tobytes())
        res["e2e_check"] = {"against": "the oracle's outputs of the same call", "identical": same}
    return res


def _oracle_worker(job):
    """One process of the all-cores baseline: whole calls of a sub-batch."""
    w, budget_s = job
    calls, el = oracle_sample(w, budget_s)
    return w.T * calls, el


def cpu_baseline_all_cores(w, budget_s, cores=None):
    """The oracle as it stands, one process per host core, each on its own
    whole requests of the workload (disjoint sub-batches are valid calls of
    their own) for budget_s seconds; throughput = all tokens / the longest
    worker's time.  Processes are spawned (never forked after CUDA use)."""
    import multiprocessing as mp
    n = max(1, min(cores or os.cpu_count() or 1, w.B))
    per = -(-w.B // n)
    subs = [_sub_batch(w, b0, min(w.B, b0 + per)) for b0 in range(0, w.B, per)]
    with mp.get_context("spawn").Pool(len(subs)) as pool:
        res = pool.map(_oracle_worker, [(sb, budget_s) for sb in subs])
    tokens = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    return {"value": tokens / el, "unit": UNIT, "cores": len(subs), "kind": "oracle",
            "sample": f"{len(subs)} processes, each whole calls of {per} requests of {w.name} "
                      f"for {budget_s:.0f} s ({tokens} tokens in all); single-threaded C oracle "
                      f"per process (fp32, -O2, no FMA)"}


def _reference_worker(job):
    """One process of the reference arm: W warm-up and K timed steps, each
    one whole oracle call over the next of this worker's sub-batches."""
    subs, warmup, steps = job
    import oracle
    w = subs[0]
    dt = np.uint16 if w.kv_esize == 2 else np.uint8
    kc = np.zeros((w.num_pages, w.page_size, w.Hkv, 128), dt)
    vc = np.zeros_like(kc)
    outs = [oracle.new_outputs(sb) for sb in subs]

    def step(i):
        sb = subs[i % len(subs)]
        oq, qs, fl = outs[i % len(subs)]
        assert oracle.append_paged(sb, kc, vc, oq, qs if sb.quant_policy == 1 else None, fl) == 0
        return sb.T

    for i in range(warmup):
        step(i)
    t0 = time.perf_counter()
    toks = sum(step(i) for i in range(steps))
    return toks, time.perf_counter() - t0


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = workloads.APPEND_CONFIGS[args.workload]()
    # the oracle as it stands on the host cores: one spawned process per core,
    # each on its own whole requests; every step, each process runs one call
    # over a sample of its requests, sized so the whole run stays within a
    # few minutes
    n = max(1, min(os.cpu_count() or 1, w.B))
    calls, el = oracle_sample(w, 0.0, max_calls=2)
    per_token = el / calls / max(w.T, 1)
    budget = 120.0
    per_worker = -(-w.B // n)
    tokens = int(max(1, min(per_worker, budget / max(1, args.steps + args.warmup) / per_token)))
    jobs = []
    for j in range(n):
        lo, hi = j * per_worker, min(w.B, (j + 1) * per_worker)
        if lo >= hi:
            break
        subs = [_sub_batch(w, b0, min(hi, b0 + tokens)) for b0 in range(lo, hi, tokens)]
        jobs.append((subs, args.warmup, args.steps))
    import multiprocessing as mp
    with mp.get_context("spawn").Pool(len(jobs)) as pool:
        res = pool.map(_reference_worker, jobs)
    toks = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    value = toks / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_block(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": len(jobs), "kind": "oracle",
                         "sample": f"{len(jobs)} processes x {args.steps} steps, each step one "
                                   f"call over {tokens} request(s) of the process's own share of "
                                   f"{w.name}; single-threaded C oracle per process"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _sub_batch(w, b0, b1):
    """Requests [b0, b1) of an append workload as a workload of their own."""
    import copy
    s = copy.copy(w)
    lo, hi = int(w.q_indptr[b0]), int(w.q_indptr[b1])
    s.B = b1 - b0
    s.T = hi - lo
    s.qkv = w.qkv[lo:hi]
    s.q_indptr = (w.q_indptr[b0:b1 + 1] - lo).astype(np.int32)
    s.seq_lens = w.seq_lens[b0:b1].copy()
    s.page_table = w.page_table[b0:b1].copy()
    s.positions = None if w.positions is None else w.positions[lo:hi]
    return s


def max_over_ranks(torch, dist, x: float, device) -> float:
    """The maximum of a per-rank time over all ranks (x itself on one rank)."""
    if dist is None or not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_count(w, min_bytes=3 * L2_BYTES, max_replicas=64) -> int:
    """Replicas a bench of workload w rotates over (replica_workloads)."""
    per = workloads.append_bytes(w)["total"]
    return int(min(max_replicas, max(2, math.ceil(min_bytes / per))))


def config_block(w):
    """The workload of a line, identical for both arms: its shape, and how the
    GPU arm keeps the timed steps' inputs out of L2 (derived from w alone)."""
    R = replica_count(w)
    per = workloads.append_bytes(w)["total"]
    return {"workload": w.name, "tokens_per_step": w.T, "requests": w.B, "Hq": w.Hq,
            "Hkv": w.Hkv, "head_dim": 128, "page_size": w.page_size,
            "quant_policy": w.quant_policy,
            "io_dtype": "bf16 in, " + ("bf16" if w.quant_policy == 0 else "e4m3") + " out",
            "parallelism": "replicas", "replicas": R,
            "seeds": f"{w.seed} (+7919 per replica); the replicas keep the first draw's token counts",
            "l2": (f"inputs larger than L2: each step uses its own replica of the step inputs "
                   f"({R} replicas, about {R * per / 1e6:.0f} MB rotated per cycle)")}


# --------------------------------------------------------------------- main

def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import qk_norm_rope_token_b200 as fqr

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.profile:
        return run_profile(args, torch, fqr, dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    peak, peak_src = load_peaks()
    bench = AppendBench(args.workload, torch, fqr, dev, seed_offset=1000 * rank,
                        schedule=args.schedule)
    repeats = args.repeats or max(5, math.ceil(MIN_TIMED_LAUNCHES / max(args.steps, 1)))
    sampler = ClockSampler(gpu_smi_id(torch, dev)) if rank == 0 else None
    if sampler is not None:
        time.sleep(1.0)   # let nvidia-smi start sampling before the warm-up
    region_ms, nbytes = time_launches(torch, bench, args.steps, args.warmup, repeats=repeats,
                                      barrier=barrier, marks=sampler.mark if sampler else None)
    bench.check_flags()
    clocks = sampler.stop() if sampler else None
    region_max = [max_over_ranks(torch, dist, m, dev) for m in region_ms]
    ms_max = statistics.median(region_max)
    ms_local = statistics.median(region_ms)
    value = world * bench.T * args.steps / (ms_max / 1e3)
    per_launch_s = ms_local / 1e3 / args.steps
    achieved = nbytes / args.steps / per_launch_s / 1e9
    traffic, traffic_parts = profiled_traffic(args.workload)

    e2e, e2e_sample = e2e_measure(torch, fqr, bench, min(args.e2e_steps, max(args.steps, 1)))
    e2e_ms = max_over_ranks(torch, dist, e2e["ms_per_step"], dev)
    e2e["value"] = world * bench.T / (e2e_ms / 1e3)
    per_config = None
    if rank == 0 and not args.no_per_config:
        per_config = measure_per_config(torch, fqr, dev, peak)
    cpu = cpu_all = None
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(bench.ws[0], args.cpu_seconds, e2e_sample)
        e2e["check"] = cpu.pop("e2e_check")
        cpu_all = cpu_baseline_all_cores(bench.ws[0], args.cpu_seconds)
    if dist is not None:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    us = [m * 1e3 / args.steps for m in region_ms]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "gpu_launches": args.steps,
        "config": config_block(bench.ws[0]),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "traffic_over_algorithmic": (traffic / (nbytes / args.steps)
                                                  if traffic else None),
                     "bytes_per_launch": nbytes / args.steps,
                     "us_per_launch": per_launch_s * 1e6,
                     "timing": f"median of {repeats} regions of exactly {args.steps} launches "
                               f"(CUDA events, CUDA-graph replays of back-to-back launches); "
                               f"region us/launch min {min(us):.2f} max {max(us):.2f}",
                     "peak_source": peak_src, "traffic_parts": traffic_parts,
                     "kernel": describe_plan(fqr.append_plan(bench.reps[0]["params"]))},
        "e2e": e2e, "clocks": clocks, "cpu_baseline": cpu,
        "cpu_baseline_all_cores": cpu_all,
        "per_config": per_config,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_profile(args, torch, fqr, dev):
    """A few eager launches of one workload for ncu (small device footprint)."""
    if args.mla:
        b = MlaBench(torch, fqr, dev, max_replicas=args.replicas or 2, name=args.mla_workload)
    else:
        b = AppendBench(args.workload, torch, fqr, dev, max_replicas=args.replicas or 2,
                        schedule=args.schedule, small_cache=args.small_cache)
    h = torch.cuda.current_stream().cuda_stream
    for i in range(args.warmup + args.steps):
        b.launch(i, h)
    torch.cuda.synchronize()
    if not args.mla:
        b.check_flags()
    print(f"profile: {b.name} x {args.warmup + args.steps} launches, {b.R} replicas, "
          f"{max(b.bytes) / 1e6:.1f} MB per launch")
    return 0


def _short(x, digits=3):
    return float(f"{x:.{digits}g}")


def measure_per_config(torch, fqr, dev, peak, warmup=50, repeats=3):
    """Every named workload, timed like the headline (median of `repeats`
    regions), in a compact form: us = microseconds per launch (automatic
    schedule), frac = algorithmic bytes / time / peak, lat / str = us per
    launch with the latency / streaming schedule forced, floor = us per
    launch of a plain copy kernel moving the same read and write bytes
    (FloorBench), MB = algorithmic megabytes per launch, T = tokens per
    launch."""
    out = {}

    def timed(b):
        n = max(200, min(4000, int(4e9 / max(b.bytes))))
        reg, nbytes = time_launches(torch, b, n, warmup, repeats=repeats)
        return statistics.median(reg) * 1e3 / n, nbytes / n

    for name in sorted(workloads.APPEND_CONFIGS):
        b = AppendBench(name, torch, fqr, dev)
        us, per = timed(b)
        b.check_flags()
        e = {"us": _short(us), "frac": _short(per / (us * 1e-6) / 1e9 / peak),
             "MB": _short(per / 1e6), "T": b.T}
        for sched, label in ((1, "lat"), (2, "str")):   # both schedules, for tuning
            for st in b.reps:
                st["params"].schedule = sched
            e[label] = _short(timed(b)[0])
        nb = workloads.append_bytes(b.ws[0])
        del b
        torch.cuda.empty_cache()
        f = FloorBench(torch, dev, nb["read"], nb["write"])
        e["floor"] = _short(timed(f)[0])     # the plain copy of the same bytes
        out[name] = e
        del f
        torch.cuda.empty_cache()
    for name in workloads.MLA_CONFIGS:
        m = MlaBench(torch, fqr, dev, name=name)
        us, per = timed(m)
        out[name] = {"us": _short(us), "frac": _short(per / (us * 1e-6) / 1e9 / peak),
                     "MB": _short(per / 1e6), "T": m.T}
        del m
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
