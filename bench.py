"""Benchmark of the TPA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: the 8 x 2048-token prefill of a d_model=1024, h=16, d_h=64,
R_Q=6, R_K=R_V=2 layer (bf16).  One step = project (+RoPE) -> cache append -> causal
prefill for the batch, then one decode token per sequence (project the new token,
append it, decode over 2049 keys), i.e. every step of the hot path once.  The
value is whole-job algorithmic TFLOP/s.  The same line carries the decode leg on
the 64 x 32768-token factor cache (GB/s of factor bytes), the roofline of the
dominant kernel, the fp64 oracle timed on the host cores, an end-to-end number
through the public API with host buffers, and SM clocks sampled during the timed
region.

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch (sequences
are independent, no data-path collective), so scaling is weak; the time is the max
over ranks.  `--impl reference` times the fp64 oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tensor_product_attention_b200 import inputs as I  # noqa: E402

METRIC = "TPA decode factor-cache GB/s (% HBM peak); prefill TFLOP/s (% bf16 peak)"
DEFAULT = "prefill_b8_s2048_d1024"
LAYER_LEG = "layer_prefill_b4_s8192_d2048"
DECODE_LEG = "decode_b64_ctx32k"
KVONLY_DECODE_LEG = "kvonly_decode_b16_ctx64k_128k"
SHARED_DECODE_LEG = "shared_basis_decode_b64_ctx32k"
FLUSH_BYTES = 256 << 20          # > 126 MB L2

# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture of
# the kernel as it stands (dram__bytes_read.sum + dram__bytes_write.sum); None where no
# capture of the current kernel exists.  The 32K decode was captured on 16 of its 64
# sequences and the KV-only decode on 4 of its 16, each scaled by the keys processed
# (traffic grows in proportion); the b8 x s2048 prefill (query-major kernel) at full size.
PROFILED_TRAFFIC = {
    ("prefill_b8_s2048_d1024", "tpa_prefill"): 26284288 + 9728,
    ("prefill_b8_s2048_d1024", "tpa_project"): 35785216 + 922112,
    ("decode_b64_ctx32k", "tpa_decode"): 4 * (604.104192e6 + 6.208e6),
    ("kvonly_decode_b16_ctx64k_128k", "tpa_decode"): 1602374 / 428112 * (548.204288e6 + 9.393664e6),
    ("shared_basis_decode_b64_ctx32k", "tpa_decode"): 287.670784e6 + 7.064576e6,
}


# ------------------------------------------------------------------ accounting

def attn_flops_per_pair(wl) -> int:
    """Algorithmic flops per (query, key) pair, all heads: the B-space score
    contraction 2 R_Q R_K d_h, its per-head a_Q a_K weighting 2 h R_Q R_K, and the
    weighted sum of values 2 h d_h.  TPA-KVonly: the per-head query against each
    B_K row, 2 h R_K d_h, the a_K weighting 2 h R_K, and the values 2 h d_h."""
    if wl.rank_q == 0:
        return 2 * wl.n_heads * wl.rank_k * wl.head_dim + 2 * wl.n_heads * wl.rank_k \
            + 2 * wl.n_heads * wl.head_dim
    return 2 * wl.rank_q * wl.rank_k * wl.head_dim + 2 * wl.n_heads * wl.rank_q * wl.rank_k \
        + 2 * wl.n_heads * wl.head_dim


def proj_flops(wl, tokens: int) -> int:
    n = (wl.rank_q + wl.rank_k + wl.rank_v) * (wl.n_heads + wl.head_dim)
    if wl.rank_q == 0:
        n += wl.n_heads * wl.head_dim              # TPA-KVonly: the plain W_Q
    if wl.shared_basis:
        n -= (wl.rank_k + wl.rank_v) * wl.head_dim  # no W_B_k, W_B_v
    return 2 * tokens * n * wl.d_model


def causal_pairs(batch: int, S: int, start: int = 0) -> int:
    return batch * (S * start + S * (S + 1) // 2)


def cache_bytes_per_token(wl) -> int:
    """Per-token cache bytes: (R_K + R_V)(h + d_h) elements, or (R_K + R_V) h with a
    shared basis (its B side is one per-layer table, counted once per launch)."""
    es = 2 if wl.dtype == "bf16" else 4
    per_rank = wl.n_heads + (0 if wl.shared_basis else wl.head_dim)
    return (wl.rank_k + wl.rank_v) * per_rank * es


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------ helpers

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, value: float) -> float:
    """The slowest rank's time: every rank gets the max (timing plumbing only)."""
    if ws == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(ws: int, work_per_rank: float, ms_max: float) -> float:
    """Weak scaling: every rank processes its own batch of `work_per_rank` units; the
    job rate is all ranks' units over the slowest rank's time (per second)."""
    return ws * work_per_rank / (ms_max * 1e-3)


class Events:
    """CUDA events on the launching stream, one pair per named region per step."""

    def __init__(self):
        self.pairs = {}

    def start(self, name):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs.setdefault(name, []).append([e, None])

    def stop(self, name):
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        self.pairs[name][-1][1] = e

    def mean_ms(self, name):
        v = [a.elapsed_time(b) for a, b in self.pairs.get(name, [])]
        return sum(v) / len(v) if v else float("nan")

    def total_ms(self, name):
        return sum(a.elapsed_time(b) for a, b in self.pairs.get(name, []))


# ------------------------------------------------------------------ prefill workload

class PrefillStep:
    """Buffers and the calls of one prefill step (+ one decode token per sequence)."""

    def __init__(self, wl, tpa):
        self.wl, self.tpa = wl, tpa
        B, S = wl.batch, wl.seqlen
        dt = tpa.BF16 if wl.dtype == "bf16" else tpa.F32
        self.dims = tpa.Dims(wl.d_model, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v, dt)
        self.cap = S + 1
        self.cs = torch.empty((self.cap, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
        tpa.tpa_rope_table(self.dims, wl.rope_base, self.cap, self.cs)
        self.x_host = torch.cat([I.prefill_x(wl, b) for b in range(B)]).pin_memory()
        self.xn_host = torch.stack([I.prefill_x(wl, b, S + 1)[S] for b in range(B)]).pin_memory()
        self.x = self.x_host.cuda()
        self.xn = self.xn_host.cuda()
        self.w = I.prefill_w(wl).cuda()
        self.fac = tpa.alloc_factors(self.dims, B * S)
        self.cache = tpa.alloc_cache(self.dims, B, self.cap)
        tdt = self.dims.torch_dtype
        self.out = torch.empty((B * S, wl.n_heads, wl.head_dim), dtype=tdt, device="cuda")
        self.out1 = torch.empty((B, wl.n_heads, wl.head_dim), dtype=tdt, device="cuda")
        self.pre = [S] * B                     # lengths before the decode step
        self.ws = tpa.alloc_step_workspace(self.dims, self.pre)
        self.out_host = torch.empty(self.out.shape, dtype=tdt).pin_memory()
        self.out1_host = torch.empty(self.out1.shape, dtype=tdt).pin_memory()
        # a second set of step inputs / outputs for the pipelined end-to-end timing
        self.slots = [(self.x, self.xn, self.out, self.out1, self.out_host, self.out1_host),
                      (torch.empty_like(self.x), torch.empty_like(self.xn), torch.empty_like(self.out),
                       torch.empty_like(self.out1), torch.empty_like(self.out_host).pin_memory(),
                       torch.empty_like(self.out1_host).pin_memory())]
        self.launches_per_step = 6   # project, append, prefill; decode step: project, decode, combine

    def flops(self):
        wl = self.wl
        B, S = wl.batch, wl.seqlen
        f = proj_flops(wl, B * (S + 1))
        f += attn_flops_per_pair(wl) * (causal_pairs(B, S) + B * (S + 1))
        return f

    def run(self, ev: Events | None = None, slot: int = 0):
        t, wl, d = self.tpa, self.wl, self.dims
        B, S = wl.batch, wl.seqlen
        zero = [0] * B
        x, xn, out, out1 = self.slots[slot][:4]
        mark = (lambda n: ev.start(n)) if ev else (lambda n: None)
        done = (lambda n: ev.stop(n)) if ev else (lambda n: None)
        mark("project"); t.tpa_project(d, x, self.w, B, S, zero, self.cs, self.cap, self.fac); done("project")
        mark("append"); t.tpa_cache_append(d, self.cache, self.fac, B, S, zero); done("append")
        mark("prefill"); t.tpa_prefill(d, self.fac, self.cache, B, S, zero, out); done("prefill")
        mark("decode_step")
        t.tpa_decode_step(d, xn, self.w, self.cs, self.cap, self.cache, self.pre, out1, self.ws)
        done("decode_step")

    def e2e_inputs(self, slot):
        """(pinned host, device) pairs each step copies in."""
        return [(self.x_host, self.slots[slot][0]), (self.xn_host, self.slots[slot][1])]

    def e2e_outputs(self, slot):
        """(device, pinned host) pairs each step copies out."""
        return [(self.slots[slot][2], self.slots[slot][4]), (self.slots[slot][3], self.slots[slot][5])]


    def io_bytes(self):
        h2d = self.x_host.numel() * self.x_host.element_size() + self.xn_host.numel() * self.xn_host.element_size()
        d2h = self.out_host.numel() * self.out_host.element_size() + self.out1_host.numel() * self.out1_host.element_size()
        return h2d, d2h


# ------------------------------------------------------------------ decode workload

class DecodeStep:
    def __init__(self, wl, tpa):
        self.wl, self.tpa = wl, tpa
        self.dims = tpa.Dims(0, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v,
                             tpa.BF16 if wl.dtype == "bf16" else tpa.F32, int(wl.shared_basis))
        self.lengths = [int(v) for v in I.decode_lengths(wl)]
        B = wl.batch
        self.cache = tpa.alloc_cache(self.dims, B, max(self.lengths))
        if wl.shared_basis:
            # the layer's per-position basis tables: built once, like the weights
            cap = max(self.lengths)
            basis = I.shared_basis(wl)
            cs = torch.empty((cap, wl.head_dim // 2, 2), dtype=torch.float32, device="cuda")
            tpa.tpa_rope_table(self.dims, wl.rope_base, cap, cs)
            tpa.tpa_shared_basis_tables(self.dims, basis["b_k"].cuda(), basis["b_v"].cuda(), cs, cap,
                                        self.cache.b_k, self.cache.b_v)
            torch.cuda.synchronize()
            del cs
        per_seq = ("a_k", "a_v") if wl.shared_basis else ("a_k", "a_v", "b_k", "b_v")
        qa, qb = [], []
        for b, L in enumerate(self.lengths):
            seq = I.decode_sequence(wl, b, L)
            for n in per_seq:
                getattr(self.cache, n)[b, :L].copy_(seq[n])
            if wl.rank_q:
                qa.append(seq["a_q"]); qb.append(seq["b_q"])
            else:
                qb.append(seq["q"])
            del seq
        self.qa_host = torch.stack(qa).pin_memory() if qa else None
        self.qb_host = torch.stack(qb).pin_memory()
        self.q_a = self.qa_host.cuda() if qa else None
        self.q_b = self.qb_host.cuda()
        tdt = self.dims.torch_dtype
        self.out = torch.empty((B, wl.n_heads, wl.head_dim), dtype=tdt, device="cuda")
        self.out_host = torch.empty(self.out.shape, dtype=tdt).pin_memory()
        # a second set of step inputs / outputs for the pipelined end-to-end timing
        like = lambda t: None if t is None else torch.empty_like(t)
        self.slots = [(self.q_a, self.q_b, self.out, self.out_host),
                      (like(self.q_a), like(self.q_b), like(self.out), like(self.out_host).pin_memory())]
        self.ws = tpa.alloc_workspace(self.dims, self.lengths)
        self.launches_per_step = 2   # decode, combine

    def factor_bytes(self):
        """Cache bytes one launch must read: every key's factors, plus (shared basis)
        the key table rows up to the longest context and one value tile, once."""
        n = sum(self.lengths) * cache_bytes_per_token(self.wl)
        if self.wl.shared_basis:
            es = 2 if self.wl.dtype == "bf16" else 4
            n += max(self.lengths) * self.wl.rank_k * self.wl.head_dim * es
            n += self.wl.rank_v * self.wl.head_dim * es
        return n

    def bytes(self):
        q = self.q_b.numel() * self.q_b.element_size() + (0 if self.q_a is None else self.q_a.numel() * self.q_a.element_size())
        return self.factor_bytes() + q + self.out.numel() * self.out.element_size()

    def run(self, ev: Events | None = None, slot: int = 0):
        q_a, q_b, out = self.slots[slot][:3]
        if ev:
            ev.start("decode")
        self.tpa.tpa_decode(self.dims, q_a, q_b, self.cache, self.lengths, out, self.ws)
        if ev:
            ev.stop("decode")

    def e2e_inputs(self, slot):
        pairs = [(self.qb_host, self.slots[slot][1])]
        if self.qa_host is not None:
            pairs.append((self.qa_host, self.slots[slot][0]))
        return pairs

    def e2e_outputs(self, slot):
        return [(self.slots[slot][2], self.slots[slot][3])]

    def io_bytes(self):
        h2d = self.qb_host.numel() * self.qb_host.element_size()
        if self.qa_host is not None:
            h2d += self.qa_host.numel() * self.qa_host.element_size()
        return h2d, self.out_host.numel() * self.out_host.element_size()


# ------------------------------------------------------------------ timing

def timed(step, steps, warmup, ws, flush: torch.Tensor | None, graph: bool = True):
    """W untimed steps, then exactly K timed steps between barrier+sync, each timed
    with CUDA events on the launching stream.  With `graph`, the step's launches are
    captured once into a CUDA graph and the K timed steps are graph replays (the
    host-side argument checks and launch overhead stay out of the step).  The L2
    flush, when used, sits between steps and outside the events.  Returns the mean
    per-step ms (max over ranks)."""
    for _ in range(warmup):
        step.run()
    torch.cuda.synchronize()
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step.run()
        torch.cuda.synchronize()
    ev = Events()
    barrier(ws)
    torch.cuda.synchronize()
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        ev.start("step")
        if g is not None:
            g.replay()
        else:
            step.run()
        ev.stop("step")
    torch.cuda.synchronize()
    barrier(ws)
    ms = ev.total_ms("step") / steps
    del g
    return max_over_ranks(ws, ms)


def timed_legs(step, steps, flush: torch.Tensor | None):
    """Per-call CUDA events for each leg of the step (direct calls, not a graph)."""
    ev = Events()
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        step.run(ev)
    torch.cuda.synchronize()
    return ev


class E2EPipeline:
    """Each step copies its inputs in from pinned host memory, runs, and copies its
    outputs out, as a serving loop would: two copy streams and two buffer sets let the
    upload of step k+1 and the download of step k-1 overlap the compute of step k.
    Events keep every buffer from being overwritten before it is consumed."""

    def __init__(self, step):
        self.step = step
        self.comp = torch.cuda.current_stream()
        self.h2d, self.d2h = torch.cuda.Stream(), torch.cuda.Stream()
        self.in_ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.comp_done = [torch.cuda.Event(), torch.cuda.Event()]
        self.out_done = [torch.cuda.Event(), torch.cuda.Event()]
        self.k = 0

    def one(self):
        s, k = self.k % 2, self.k
        with torch.cuda.stream(self.h2d):
            if k >= 2:
                self.h2d.wait_event(self.comp_done[s])     # step k-2 has read these inputs
            for host, dev in self.step.e2e_inputs(s):
                dev.copy_(host, non_blocking=True)
            self.in_ready[s].record(self.h2d)
        self.comp.wait_event(self.in_ready[s])
        if k >= 2:
            self.comp.wait_event(self.out_done[s])         # step k-2's outputs are out
        self.step.run(slot=s)
        self.comp_done[s].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.comp_done[s])
            for dev, host in self.step.e2e_outputs(s):
                host.copy_(dev, non_blocking=True)
            self.out_done[s].record(self.d2h)
        self.k += 1

    def drain(self):
        for e in self.out_done:
            self.comp.wait_event(e)


def timed_e2e(step, steps, warmup, ws):
    """End to end through the public calls, host buffers in and out every step (see
    E2EPipeline); the events on the compute stream bracket all three streams' work."""
    pipe = E2EPipeline(step)
    for _ in range(warmup):
        pipe.one()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(pipe.comp)
    pipe.h2d.wait_event(a)
    pipe.d2h.wait_event(a)
    for _ in range(steps):
        pipe.one()
    pipe.drain()
    b.record(pipe.comp)
    torch.cuda.synchronize()
    barrier(ws)
    return max_over_ranks(ws, a.elapsed_time(b) / steps)


# ------------------------------------------------------------------ CPU oracle baseline

def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def oracle_prefill_sample(wl, n_seq: int = 1, seqlen: int | None = None):
    """Time the oracle's forward (project + RoPE + causal attention, fp64) on n_seq
    sequences of the workload; returns (seconds, flops of that sample)."""
    import oracle
    S = seqlen or wl.seqlen
    od = oracle.Dims(wl.d_model, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v,
                     shared_basis=wl.shared_basis)
    basis = {k: v.double().numpy() for k, v in I.shared_basis(wl).items()} if wl.shared_basis else None
    x = np.stack([I.prefill_x(wl, b, S).double().numpy() for b in range(n_seq)])
    w = I.prefill_w(wl).double().numpy()
    t0 = time.perf_counter()
    oracle.tpa_forward(x, w, od, wl.rope_base, basis=basis)
    dt = time.perf_counter() - t0
    return dt, proj_flops(wl, n_seq * S) + attn_flops_per_pair(wl) * causal_pairs(n_seq, S)


def oracle_decode_sample(wl, n_seq: int = 1, length: int | None = None):
    """Time the oracle's decode on n_seq sequences; returns (seconds, factor bytes)."""
    import oracle
    od = oracle.Dims(0, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v,
                     shared_basis=wl.shared_basis)
    lengths = I.decode_lengths(wl)
    total = 0
    seqs = []
    for b in range(n_seq):
        L = int(length or lengths[b])
        seqs.append(({k: v.double().numpy() for k, v in I.decode_sequence(wl, b, L).items()}, L))
        total += L * cache_bytes_per_token(wl)
    basis = {k: v.double().numpy() for k, v in I.shared_basis(wl).items()} if wl.shared_basis else None
    t0 = time.perf_counter()
    for s, L in seqs:
        kv = s
        if basis is not None:       # the per-layer tables are part of the timed work
            kv = {"a_k": s["a_k"], "a_v": s["a_v"], **oracle.shared_basis_tables(basis, od, L, wl.rope_base)}
        oracle.decode_attention(s, kv, od, L)
    return time.perf_counter() - t0, total


# The bounded oracle samples: the first PREFILL_SAMPLE tokens of one sequence for the
# prefill workloads (the fp64 scores alone are h * S^2 * 8 bytes), two whole sequences
# for decode.  The reference arm times the same samples.
PREFILL_SAMPLE = 2048
PREFILL_SAMPLE_1T = 512          # the single-thread run: a quarter of the tokens


def oracle_sample(wl, one_thread=False):
    """(rate, unit, seconds, description) of the oracle on the workload's bounded sample."""
    if wl.kind == "prefill":
        S = min(wl.seqlen, PREFILL_SAMPLE_1T if one_thread else PREFILL_SAMPLE)
        dt, fl = oracle_prefill_sample(wl, 1, seqlen=S)
        return fl / dt / 1e12, "TFLOP/s", dt, (
            f"fp64 oracle forward of the first {S} tokens of 1 of {wl.batch} sequences "
            f"({wl.seqlen} tokens each): projection, RoPE, causal attention")
    dt, by = oracle_decode_sample(wl, 1 if one_thread else 2)
    return by / dt / 1e9, "GB/s", dt, f"fp64 oracle decode of {1 if one_thread else 2} of {wl.batch} sequences"


def cpu_baseline(wl):
    """The oracle on the host cores (all BLAS threads), plus a one-thread run."""
    v, unit, dt, what = oracle_sample(wl)
    out = {"value": v, "unit": unit, "cores": cpu_threads(), "kind": "oracle",
           "sample": f"{what}; {dt:.1f} s", "cpu_model": cpu_model(), "threads": cpu_threads(),
           "host_cpus": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            v1, _, dt1, what1 = oracle_sample(wl, one_thread=True)
        out["one_thread"] = {"value": v1, "unit": unit, "threads": 1, "sample": f"{what1}; {dt1:.1f} s"}
    except ImportError:
        out["one_thread"] = None
    return out


# ------------------------------------------------------------------ main

def workload_config(wl, args, ws):
    """The `config` object of the JSON line: the workload by name and shape, and how it
    was timed.  Both arms print the same object for the same workload."""
    timing = "CUDA-graph replay of the step" if not getattr(args, "no_graph", False) else "direct calls"
    if wl.kind == "prefill":
        return {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seqlen, "d_model": wl.d_model,
                "n_heads": wl.n_heads, "head_dim": wl.head_dim, "rank_q": wl.rank_q,
                "rank_k": wl.rank_k, "rank_v": wl.rank_v,
                "step": "project+RoPE -> append -> causal prefill, then 1 decode token per sequence",
                "l2": "flushed between steps (256 MiB write outside the step events)",
                "timing": timing, "parallelism": f"dp{ws} (independent sequences per rank)"}
    return {"workload": wl.name, "batch": wl.batch, "context": list(wl.context),
            "n_heads": wl.n_heads, "head_dim": wl.head_dim, "rank_q": wl.rank_q,
            "rank_k": wl.rank_k, "rank_v": wl.rank_v, "shared_basis": bool(wl.shared_basis),
            "l2": "inputs larger than L2", "timing": timing,
            "parallelism": f"dp{ws} (independent sequences per rank)"}


def prefill_rooflines(wl, ev, pk):
    """Rooflines of the prefill step's two tensor-core kernels from their per-launch
    CUDA-event times: the causal prefill (algorithmic flops per causal pair) and the
    factor projection (2 T N D)."""
    pre_ms = ev.mean_ms("prefill")
    pre_fl = attn_flops_per_pair(wl) * causal_pairs(wl.batch, wl.seqlen)
    ach = pre_fl / (pre_ms * 1e-3) / 1e12
    pre = {"kernel": "tpa_prefill (causal attention from factors)", "bound": "tensor",
           "achieved": ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
           "frac": ach / pk["bf16_tflops"], "traffic": PROFILED_TRAFFIC.get((wl.name, "tpa_prefill")),
           "peak_kind": f"bf16 dense, burst, {pk['source']}",
           "algorithmic_per_launch": f"{pre_fl:.4g} flop = {attn_flops_per_pair(wl)} flop/pair x "
                                     f"{causal_pairs(wl.batch, wl.seqlen)} causal pairs",
           "launch_ms": pre_ms}
    pj_ms = ev.mean_ms("project")
    pj_fl = proj_flops(wl, wl.batch * wl.seqlen)
    pach = pj_fl / (pj_ms * 1e-3) / 1e12
    proj = {"kernel": "tpa_project (factor projection GEMM + RoPE epilogue)", "bound": "tensor",
            "achieved": pach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": pach / pk["bf16_tflops"],
            "traffic": PROFILED_TRAFFIC.get((wl.name, "tpa_project")),
            "peak_kind": f"bf16 dense, burst, {pk['source']}",
            "algorithmic_per_launch": f"{pj_fl:.4g} flop = 2 T N D", "launch_ms": pj_ms}
    return pre, proj


def assert_tensor_core_path(tpa, wl):
    """bf16 workloads must run on the tcgen05 kernels: the bench measures those."""
    if wl.dtype != "bf16":
        return
    dims = tpa.Dims(wl.d_model or 64, wl.n_heads, wl.head_dim, wl.rank_q, wl.rank_k, wl.rank_v, tpa.BF16,
                    int(wl.shared_basis))
    calls = [tpa.CALL_DECODE] if wl.kind == "decode" else [tpa.CALL_PROJECT, tpa.CALL_PREFILL, tpa.CALL_DECODE]
    for call in calls:
        fam = tpa.tpa_kernel_family(dims, call)
        if fam != "tensor_core":
            raise SystemExit(f"{wl.name}: call {call} would take the {fam} kernels, not the tensor-core path")


def run_reference(args, wl, ws, rank):
    """The fp64 oracle on the host cores, timed per step on a bounded sample."""
    if rank != 0:
        return
    vals = []
    for _ in range(args.warmup + args.steps):
        v, unit, _, what = oracle_sample(wl)
        vals.append(v)
    v = statistics.mean(vals[args.warmup:])
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, workload distributions)",
        "config": workload_config(wl, args, ws),
        "cpu_baseline": {"value": v, "unit": unit, "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"{what}, per step", "cpu_model": cpu_model()},
        "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def measure_prefill(step, args, ws, pk, flush, clk_ok=True):
    """Time one prefill workload: the graph-replayed step, per-call legs, and the
    pipelined end-to-end step.  Returns the pieces of its JSON entry."""
    wl = step.wl
    ms = timed(step, args.steps, args.warmup, ws, flush, graph=not args.no_graph)
    ev = timed_legs(step, args.steps, flush)
    e2e_ms = timed_e2e(step, args.steps, args.warmup, ws)
    work = step.flops()
    pre, proj = prefill_rooflines(wl, ev, pk)
    h2d, d2h = step.io_bytes()
    return {
        "value": whole_job_rate(ws, work, ms) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
        "roofline": pre, "roofline_project": proj,
        "legs_ms": {n: round(ev.mean_ms(n), 4) for n in ("project", "append", "prefill", "decode_step")},
        "e2e": {"value": whole_job_rate(ws, work, e2e_ms) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "each step copies its inputs in and its outputs out (pinned host memory); "
                              "the upload of step k+1 and the download of step k-1 overlap step k"},
        "gpu_launches": step.launches_per_step * args.steps,
    }


def measure_decode(step, args, ws, pk):
    wl = step.wl
    ms = timed(step, args.steps, args.warmup, ws, None, graph=not args.no_graph)
    ev = timed_legs(step, args.steps, None)
    e2e_ms = timed_e2e(step, args.steps, args.warmup, ws)
    ach = step.factor_bytes() / (ev.mean_ms("decode") * 1e-3) / 1e9
    h2d, d2h = step.io_bytes()
    return {
        "value": whole_job_rate(ws, step.bytes(), ms) / 1e9, "unit": "GB/s", "ms_per_step": ms,
        "roofline": {"kernel": "tpa_decode (split-K decode + combine)", "bound": "hbm", "achieved": ach,
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                     "traffic": PROFILED_TRAFFIC.get((wl.name, "tpa_decode")),
                     "peak_kind": f"HBM copy, {pk['source']}",
                     "algorithmic_per_launch": f"{step.factor_bytes()} factor bytes",
                     "launch_ms": ev.mean_ms("decode")},
        "legs_ms": {"decode": round(ev.mean_ms("decode"), 4)},
        "e2e": {"value": whole_job_rate(ws, step.bytes(), e2e_ms) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": step.launches_per_step * args.steps,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode-leg", action="store_true", help="skip the decode and full-layer legs")
    ap.add_argument("--no-graph", action="store_true", help="time direct calls instead of graph replays")
    ap.add_argument("--capture", action="store_true",
                    help="for an ncu capture: run --warmup untimed steps and one more, print no bench line")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --capture: the first N sequences of the workload (a capture-sized case)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.batch and not args.capture:
        ap.error("--batch only sizes --capture runs")
    wl = I.WORKLOADS[args.workload]
    if args.batch:
        wl = I.custom(wl.name, wl, batch=min(args.batch, wl.batch))

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, wl, ws, rank)
        return

    ws, rank, local = dist_setup()
    from tensor_product_attention_b200 import binding as tpa
    pk = peaks()
    assert_tensor_core_path(tpa, wl)

    step = PrefillStep(wl, tpa) if wl.kind == "prefill" else DecodeStep(wl, tpa)
    if args.capture:
        # direct calls (no graph, no events), so that ncu -k/-s/-c select launches plainly
        for _ in range(args.warmup + 1):
            step.run()
        torch.cuda.synchronize()
        assert tpa.tpa_get_device_error() == 0
        if rank == 0:
            print(f"captured workload {wl.name}: {args.warmup + 1} steps of {step.launches_per_step} launches")
        return
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda") if wl.kind == "prefill" else None
    with ClockSampler(local) as clk:
        m = measure_prefill(step, args, ws, pk, flush) if wl.kind == "prefill" else measure_decode(step, args, ws, pk)
    clocks = clk.summary()
    assert tpa.tpa_get_device_error() == 0
    line = {
        "metric": METRIC, "value": m["value"], "unit": m["unit"], "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded, workload distributions)",
        "config": workload_config(wl, args, ws), "roofline": m["roofline"], "legs_ms": m["legs_ms"],
        "clocks": clocks, "e2e": m["e2e"], "gpu_launches": m["gpu_launches"],
    }
    if "roofline_project" in m:
        line["roofline_project"] = m["roofline_project"]
    del step
    torch.cuda.empty_cache()

    # The full-layer prefill (the largest single-GPU prefill workload) and the decode
    # workloads ride along with the default step as legs, each with its own numbers.
    legs_to_run = [] if (wl.kind != "prefill" or args.no_decode_leg) else \
        [("layer_prefill_leg", LAYER_LEG), ("decode_leg", DECODE_LEG),
         ("kvonly_decode_leg", KVONLY_DECODE_LEG), ("shared_basis_decode_leg", SHARED_DECODE_LEG)]
    for key, name in legs_to_run:
        if name == wl.name:
            continue
        lw = I.WORKLOADS[name]
        assert_tensor_core_path(tpa, lw)
        lstep = PrefillStep(lw, tpa) if lw.kind == "prefill" else DecodeStep(lw, tpa)
        with ClockSampler(local) as lclk:
            lm = measure_prefill(lstep, args, ws, pk, flush) if lw.kind == "prefill" else measure_decode(lstep, args, ws, pk)
        entry = {"workload": lw.name, "config": workload_config(lw, args, ws), **lm, "clocks": lclk.summary()}
        if lw.kind == "decode":
            entry["frac_of_hbm"] = lm["roofline"]["frac"]
            entry["factor_bytes"] = lstep.factor_bytes()
        line[key] = entry
        line["gpu_launches"] += lm["gpu_launches"]
        assert tpa.tpa_get_device_error() == 0
        del lstep
        torch.cuda.empty_cache()

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
        if "layer_prefill_leg" in line:
            line["layer_prefill_leg"]["cpu_baseline"] = cpu_baseline(I.WORKLOADS[LAYER_LEG])
    if rank == 0:
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
