#!/usr/bin/env python
"""Benchmark of the MLA layer step on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the hot path over one synthetic batch: for decode
workloads mla_decode_qkv + mla_decode_attn (front-fold, scatter, absorbed
attention, V extraction, o_proj) for `batch` tokens; for the prefill workloads
one mla_prefill of the whole sequence; for v4_qkv_bf16 one mla_v4_qkv (the
DeepSeek-V4 QKV projection) of 8192 tokens. Inputs are resident in HBM when the
timed region starts; the step is replayed from a CUDA graph; L2 is flushed
(256 MiB write, outside the timed events) before every timed step. `e2e`
times the same step through the C-ABI from pinned host buffers with the
host<->device copies inside the timed region.

Multi-GPU: independent replicas (one process per GPU, each with its own batch;
no collective on the data path), value = all ranks' tokens / max rank time.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (the reference arm of this tier); rank 0 only.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
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

import head_latent_attention_decode_b200 as mla  # noqa: E402
from head_latent_attention_decode_b200 import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "v3_fp8"
METRIC_DECODE = "MLA decode tokens/s (one layer step: front-fold + absorbed paged attention + o_proj)"
METRIC_PREFILL = "MLA prefill TFLOP/s (causal expanded path)"
METRIC_V4 = "MLA DeepSeek-V4 QKV projection TFLOP/s"


# ---------------------------------------------------------------------------
# algorithmic work (bytes / FLOPs the step must move / do)
# ---------------------------------------------------------------------------

def weight_bytes(s: wl.MlaShape) -> int:
    esz = {"f32": 4, "bf16": 2, "fp8": 1}[s.weight_dtype]
    rq, H, dn, dr, dv, rkv, D = (s.q_lora_rank, s.n_heads, s.qk_nope, s.qk_rope, s.v_dim,
                                 s.kv_lora_rank, s.hidden)
    n1 = (rq if rq else H * (dn + dr)) + rkv + dr
    params = n1 * D + (H * (dn + dr) * rq if rq else 0) + H * rkv * dn + H * dv * rkv + D * H * dv
    b = params * esz
    if s.weight_dtype == "fp8":       # fp32 block scales
        b += 4 * (params // (128 * 128) + 64)
    return b


def decode_work(s: wl.MlaShape, lens: np.ndarray) -> dict:
    a = 4 if s.act_dtype == "f32" else 2
    n = len(lens)
    R = s.kv_row_dim
    cache_read = int(lens.sum()) * R * a
    act = n * s.hidden * a * 2 + n * R * a + n * s.qk_rope * 4
    q_bytes = n * s.n_heads * R * a
    return dict(step_bytes=weight_bytes(s) + cache_read + act,
                attn_bytes=cache_read + q_bytes,
                attn_flops=2 * s.n_heads * int(lens.sum()) * (R + s.kv_lora_rank))


def prefill_flops(s: wl.MlaShape, S: int) -> dict:
    H, dn, dr, dv, rq, rkv, D = (s.n_heads, s.qk_nope, s.qk_rope, s.v_dim, s.q_lora_rank,
                                 s.kv_lora_rank, s.hidden)
    R = rkv + dr
    pairs = S * (S + 1) // 2                      # causal: query i sees i+1 keys
    proj = 2 * S * D * ((rq if rq else H * (dn + dr)) + R)
    proj += 2 * S * rq * H * (dn + dr) if rq else 0
    proj += 2 * S * rkv * H * (dn + dv)
    attn = 2 * H * pairs * (dn + dr) + 2 * H * pairs * dv
    oproj = 2 * S * H * dv * D
    return dict(total=proj + attn + oproj, attn=attn)


def v4_flops(s: wl.MlaShape, S: int) -> dict:
    """x @ [wq_a | wkv_a] and qn @ wq_b (the two GEMMs of the V4 projection)."""
    qb = 2 * S * s.q_lora_rank * s.n_heads * (s.qk_nope + s.qk_rope)
    return dict(total=2 * S * s.hidden * (s.q_lora_rank + s.kv_row_dim) + qb, qb=qb)


# ---------------------------------------------------------------------------
# DRAM traffic of the dominant kernel, from the committed ncu summary
# ---------------------------------------------------------------------------

KERNEL_SOURCES = {
    "tc_attn_decode_kernel": "tc_attn.cuh",
    "tc_attn_pair_kernel": "tc_attn_pair.cuh",
    "tc_prefill_attn_kernel": "tc_prefill_attn.cuh",
    "tc_gemm_kernel": "tc_gemm.cuh",
}


def dominant_kernel(w: wl.Workload) -> str:
    if w.mode == "prefill":
        return "tc_prefill_attn_kernel"
    if w.mode == "v4qkv":
        return "tc_gemm_kernel"
    return "tc_attn_pair_kernel" if w.shape.n_heads <= 32 else "tc_attn_decode_kernel"


def measured_traffic(kernel: str, workload: str):
    """dram read + write bytes per launch from profiles/ncu_<kernel>_<workload>.md,
    or None when there is no capture or the kernel source changed since it."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"ncu_{kernel}_{workload}.md")
    src = os.path.join(ROOT, "head_latent_attention_decode_b200", "csrc", KERNEL_SOURCES.get(kernel, ""))
    if not os.path.exists(path) or not os.path.isfile(src):
        return None
    text = open(path).read()
    m_b = re.search(r"dram bytes per launch: (\d+)", text)
    m_h = re.search(r"kernel source sha256: ([0-9a-f]{64})", text)
    if not m_b or not m_h:
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_h.group(1):
        return None
    return int(m_b.group(1))


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={CLOCK_FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for r in csv.reader(f):
                if len(r) >= 9:
                    rows.append([x.strip() for x in r])
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; barrier + max only)
# ---------------------------------------------------------------------------

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                    device_id=torch.device("cuda", local))
        else:   # the replica plumbing on CPU ranks (its tests); no step runs there
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class DecodeStep:
    def __init__(self, w: wl.Workload, rank: int):
        from head_latent_attention_decode_b200.layer import MlaLayer
        self.w = w
        s = self.s = w.shape
        self.weights = wl.make_weights(s, w.seed)
        self.inp = inp = wl.make_decode_inputs(w, seed_offset=100 + 1000 * rank)
        self.layer = layer = MlaLayer(s, self.weights)
        act = layer.act
        self.cache = torch.from_numpy(inp.cache).to(act).cuda()
        if inp.fill_hidden is not None:      # earlier rows: project N(0,1) hidden states
            xs = np.concatenate(inp.fill_hidden)
            sl = np.concatenate(inp.fill_slots)
            pos = np.concatenate([np.arange(len(f), dtype=np.int32) for f in inp.fill_slots])
            for i in range(0, len(sl), 8192):
                c, sn = layer.rope(torch.from_numpy(pos[i:i + 8192]).cuda())
                layer.decode_qkv(torch.from_numpy(xs[i:i + 8192]).to(act).cuda(), c, sn, self.cache,
                                 torch.from_numpy(sl[i:i + 8192]).cuda())
            torch.cuda.synchronize()
        n = len(inp.hidden)
        self.n = n
        self.hidden = torch.from_numpy(inp.hidden).to(act).cuda()
        self.positions = torch.from_numpy(inp.positions).cuda()
        self.cos, self.sin = layer.rope(self.positions)
        self.slot = torch.from_numpy(inp.slot_mapping).cuda()
        self.table = torch.from_numpy(inp.block_table).cuda()
        self.ctx = torch.from_numpy(inp.context_lens).cuda()
        self.max_ctx = int(inp.context_lens.max())
        self.q_abs = torch.empty((n, s.n_heads, s.kv_lora_rank), dtype=act, device="cuda")
        self.q_pe = torch.empty((n, s.n_heads, s.qk_rope), dtype=act, device="cuda")
        self.out = torch.empty((n, s.hidden), dtype=act, device="cuda")
        self.ws = layer.workspace(n, self.max_ctx)
        self.work = decode_work(s, inp.context_lens)
        self.tokens = n

    def run(self):
        mla.mla_decode_qkv(self.layer.handle, self.hidden, self.cos, self.sin, self.cache, self.slot,
                           self.q_abs, self.q_pe, self.ws)
        mla.mla_decode_attn(self.layer.handle, self.q_abs, self.q_pe, self.cache, self.table,
                            self.ctx, self.max_ctx, self.out, self.ws)

    # end to end through the C-ABI from pinned host buffers: one call copies the
    # step's inputs in, runs RoPE tables, front-fold and attention, and copies
    # the output back
    def e2e_setup(self):
        pin = lambda t: t.cpu().contiguous().pin_memory()
        self.h_hidden, self.h_pos, self.h_slot = pin(self.hidden), pin(self.positions), pin(self.slot)
        self.h_table, self.h_ctx = pin(self.table), pin(self.ctx)
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        h = self.layer.handle
        self.stage = torch.empty(mla.mla_decode_step_host_bytes(h, self.n, self.table.shape[1]),
                                 dtype=torch.uint8, device="cuda")
        h2d = sum(t.numel() * t.element_size() for t in (self.h_hidden, self.h_pos, self.h_slot,
                                                         self.h_table, self.h_ctx))
        return h2d, self.h_out.numel() * self.h_out.element_size()

    def run_e2e(self):
        mla.mla_decode_step_host(self.layer.handle, self.h_hidden, self.h_pos, self.h_slot, self.h_table,
                                 self.h_ctx, self.max_ctx, self.s.rope_theta, self.cache, self.h_out,
                                 self.stage, self.ws)


class PrefillStep:
    def __init__(self, w: wl.Workload, rank: int):
        from head_latent_attention_decode_b200.layer import MlaLayer
        self.w = w
        s = self.s = w.shape
        self.weights = wl.make_weights(s, w.seed)
        x, pos = wl.make_prefill_inputs(w, seed_offset=200 + 1000 * rank)
        self.layer = layer = MlaLayer(s, self.weights)
        self.S = S = x.shape[0]
        self.hidden = torch.from_numpy(x).to(layer.act).cuda()
        self.positions = torch.from_numpy(pos).cuda()
        self.cos, self.sin = layer.rope(self.positions)
        self.out = torch.empty((S, s.hidden), dtype=layer.act, device="cuda")
        self.ws = layer.workspace(S, 1)
        self.flops = prefill_flops(s, S)
        self.tokens = S

    def run(self):
        mla.mla_prefill(self.layer.handle, self.hidden, self.cos, self.sin, self.out, self.ws)

    def e2e_setup(self):
        self.h_hidden = self.hidden.cpu().pin_memory()
        self.h_pos = self.positions.cpu().pin_memory()
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.d_hidden, self.d_pos = torch.empty_like(self.hidden), torch.empty_like(self.positions)
        return (self.h_hidden.numel() * self.h_hidden.element_size() + self.h_pos.numel() * 4,
                self.h_out.numel() * self.h_out.element_size())

    def run_e2e(self):
        self.d_hidden.copy_(self.h_hidden, non_blocking=True)
        self.d_pos.copy_(self.h_pos, non_blocking=True)
        s = self.s
        cos = torch.empty((self.S, s.qk_rope // 2), dtype=torch.float32, device="cuda")
        sin = torch.empty_like(cos)
        mla.mla_rope_cos_sin(self.d_pos, s.qk_rope, s.rope_theta, cos, sin)
        mla.mla_prefill(self.layer.handle, self.d_hidden, cos, sin, self.out, self.ws)
        self.h_out.copy_(self.out, non_blocking=True)


class V4QkvStep:
    def __init__(self, w: wl.Workload, rank: int):
        from head_latent_attention_decode_b200.layer import MlaLayer
        self.w = w
        s = self.s = w.shape
        self.weights = wl.make_weights(s, w.seed)
        x, pos = wl.make_prefill_inputs(w, seed_offset=200 + 1000 * rank)
        self.layer = layer = MlaLayer(s, self.weights)
        self.S = S = x.shape[0]
        self.hidden = torch.from_numpy(x).to(layer.act).cuda()
        self.positions = torch.from_numpy(pos).cuda()
        self.cos, self.sin = layer.rope(self.positions)
        g = 1.0 + np.random.default_rng(w.seed + 300).uniform(-0.3, 0.3, s.kv_row_dim)
        self.kv_w = torch.from_numpy(g.astype(np.float32)).cuda()
        self.q = torch.empty((S, s.n_heads, s.qk_nope + s.qk_rope), dtype=layer.act, device="cuda")
        self.kv = torch.empty((S, s.kv_row_dim), dtype=layer.act, device="cuda")
        self.ws = layer.workspace(S, 1)
        self.flops = v4_flops(s, S)
        self.tokens = S

    def run(self):
        mla.mla_v4_qkv(self.layer.handle, self.hidden, self.cos, self.sin, self.kv_w, self.q, self.kv, self.ws)

    def e2e_setup(self):
        self.h_hidden = self.hidden.cpu().pin_memory()
        self.h_pos = self.positions.cpu().pin_memory()
        self.h_q = torch.empty(self.q.shape, dtype=self.q.dtype).pin_memory()
        self.h_kv = torch.empty(self.kv.shape, dtype=self.kv.dtype).pin_memory()
        self.d_hidden, self.d_pos = torch.empty_like(self.hidden), torch.empty_like(self.positions)
        return (self.h_hidden.numel() * self.h_hidden.element_size() + self.h_pos.numel() * 4,
                self.h_q.numel() * self.h_q.element_size() + self.h_kv.numel() * self.h_kv.element_size())

    def run_e2e(self):
        self.d_hidden.copy_(self.h_hidden, non_blocking=True)
        self.d_pos.copy_(self.h_pos, non_blocking=True)
        s = self.s
        cos = torch.empty((self.S, s.qk_rope // 2), dtype=torch.float32, device="cuda")
        sin = torch.empty_like(cos)
        mla.mla_rope_cos_sin(self.d_pos, s.qk_rope, s.rope_theta, cos, sin)
        mla.mla_v4_qkv(self.layer.handle, self.d_hidden, cos, sin, self.kv_w, self.q, self.kv, self.ws)
        self.h_q.copy_(self.q, non_blocking=True)
        self.h_kv.copy_(self.kv, non_blocking=True)


def capture(step, stream):
    """CUDA graph of one step (and the number of library launches in it)."""
    g = torch.cuda.CUDAGraph()
    before = mla.mla_kernel_launch_count()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
        step.run()
    return g, mla.mla_kernel_launch_count() - before


def timed_replays(g, k, flush, stream):
    """Replay k times, L2 flushed before each; per-replay device ms (events)."""
    ts = []
    for _ in range(k):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ts]


def kernel_time(step, kernel, k, flush, stream):
    """Average device ms of one library kernel inside the step (graph with event
    nodes around that kernel's launch)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)          # torch creates the CUDA events on first record
    b.record(stream)
    torch.cuda.synchronize()
    mla.mla_set_kernel_timer(kernel, a, b)
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            step.run()
    finally:
        mla.mla_set_kernel_timer(None)
    ms = []
    for _ in range(k):
        flush.zero_()
        g.replay()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(b))
    del g
    return float(np.mean(ms))


def cpu_oracle_sample(w: wl.Workload, budget_s: float = 12.0, max_reps: int = 1000) -> dict:
    """The fp64 oracle, as it stands, on a bounded sample of the workload."""
    from oracle import mla_ref as ref
    from threadpoolctl import threadpool_info
    s = w.shape
    weights = wl.make_weights(s, w.seed)
    W = ref.weights_fp64(weights)
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    if w.mode == "v4qkv":
        # the oracle on a block of tokens, repeated within the budget
        x, pos = wl.make_prefill_inputs(w, seq_len=64)
        g = 1.0 + np.random.default_rng(w.seed + 300).uniform(-0.3, 0.3, s.kv_row_dim)
        cos, sin = ref.rope_cos_sin(pos, s.qk_rope, s.rope_theta)
        reps, t0 = 0, time.perf_counter()
        while True:
            ref.v4_qkv(s, W, x, cos, sin, g)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s or reps >= max_reps:
                break
        f = v4_flops(s, len(x))["total"] * reps
        return dict(value=f / dt / 1e12, unit="TFLOP/s", cores=threads, kind="oracle",
                    sample=f"{len(x)} of {w.seq_len} tokens, {reps} oracle passes in {dt:.1f} s", seconds=dt)
    if w.mode == "prefill":
        S = w.seq_len
        x, pos = wl.make_prefill_inputs(w)
        rows = np.linspace(0, S - 1, 4).astype(int)
        cos, sin = ref.rope_cos_sin(pos, s.qk_rope, s.rope_theta)
        t0 = time.perf_counter()
        ref.prefill(s, W, x, cos, sin, rows=rows)
        dt = time.perf_counter() - t0
        # FLOPs actually done: K/V for all S, Q / attention / o_proj for the sampled rows
        H, dn, dr, dv = s.n_heads, s.qk_nope, s.qk_rope, s.v_dim
        f = 2 * S * s.hidden * s.kv_row_dim + 2 * S * s.kv_lora_rank * H * (dn + dv)
        f += len(rows) * (2 * s.hidden * s.q_lora_rank + 2 * s.q_lora_rank * H * (dn + dr)
                          + 2 * H * dv * s.hidden)
        f += sum(2 * H * (int(i) + 1) * (dn + dr + dv) for i in rows)
        return dict(value=f / dt / 1e12, unit="TFLOP/s", cores=threads, kind="oracle",
                    sample=f"K/V expansion of all {S} tokens + {len(rows)} query rows, one pass "
                           f"({dt:.1f} s)", seconds=dt)
    nseq = 4 if s.n_heads <= 16 else 2
    inp = wl.make_decode_inputs(w, batch=nseq)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    cache = np.asarray(inp.cache, np.float64)
    if inp.fill_hidden is not None:
        cache = ref.fill_cache_by_projection(s, W, cache, inp.fill_hidden, inp.fill_slots)
    cos, sin = ref.rope_cos_sin(inp.positions, s.qk_rope, s.rope_theta)
    reps, t0 = 0, time.perf_counter()
    while True:
        qa, qp, c2 = ref.decode_qkv(s, W, inp.hidden, cos, sin, cache, inp.slot_mapping)
        ref.decode_attn(s, W, qa, qp, c2, inp.block_table, inp.context_lens)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s or reps >= max_reps:
            break
    return dict(value=reps * nseq / dt, unit="tokens/s", cores=threads, kind="oracle",
                sample=f"{nseq} of {w.batch} sequences (contexts {inp.context_lens.tolist()}), "
                       f"{reps} oracle steps in {dt:.1f} s", seconds=dt)


def selected_workload(args) -> wl.Workload:
    """The workload named on the command line, with the profiling-slice overrides
    (--batch, --context) applied; the line's config then records the slice."""
    import dataclasses
    w = wl.WORKLOADS[args.workload]
    if getattr(args, "batch", 0) and w.mode == "decode":
        w = dataclasses.replace(w, batch=args.batch, name=f"{w.name}[batch={args.batch}]")
    if getattr(args, "context", 0) and w.mode == "decode":
        w = dataclasses.replace(w, ctx_lo=args.context, ctx_hi=args.context, name=f"{w.name}[context={args.context}]")
    return w


def run_ours(args, world, rank, local):
    w = selected_workload(args)
    peaks = {}
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        peaks = json.load(open(pk))
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    tc_peak = peaks.get("bf16_tflops", 1590.0)
    peak_src = "measured" if peaks else "fallback"
    step = {"decode": DecodeStep, "prefill": PrefillStep, "v4qkv": V4QkvStep}[w.mode](w, rank)
    stream = torch.cuda.Stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g, launches_per_step = capture(step, stream)
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        clocks = ClockSampler(local)
        t_soak = time.perf_counter()            # keep the GPU busy long enough for the
        while time.perf_counter() - t_soak < 1.0:   # clock sampler to see it under load
            g.replay()
            torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("mla_timed_steps")
        times = timed_replays(g, args.steps, flush, stream)
        torch.cuda.nvtx.range_pop()
        clk = clocks.stop()
        barrier(world)
        torch.cuda.synchronize()
        ms = all_max(float(np.mean(times)), world)
        # dominant kernel, timed live with event nodes around its launch
        kname = {"decode": "attn", "prefill": "prefill_attn", "v4qkv": "v4_qb"}[w.mode]
        kms = all_max(kernel_time(step, kname, max(3, args.steps), flush, stream), world)
        kern = dominant_kernel(w) if torch.cuda.get_device_capability()[0] == 10 else kname
        # end to end through the C-ABI with host buffers
        h2d, d2h = step.e2e_setup()
        for _ in range(2):
            step.run_e2e()
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step.run_e2e()
            b.record(stream)
            b.synchronize()
            e2e_ms.append(a.elapsed_time(b))
        e2e = all_max(float(np.mean(e2e_ms)), world)
    toks = step.tokens * world
    s = w.shape
    line = {"impl": "ours"}
    if w.mode == "decode":
        work = step.work
        value, unit = toks / (ms / 1e3), "tokens/s"
        achieved = work["attn_bytes"] / (kms / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": kern, "achieved": round(achieved, 1),
                "peak": hbm_peak, "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                "peak_source": peak_src, "kernel_ms": round(kms, 4),
                "algorithmic_bytes": work["attn_bytes"], "traffic": measured_traffic(kern, w.name)}
        extra = {"step_hbm_gbs": round(work["step_bytes"] / (ms / 1e3) / 1e9, 1),
                 "step_hbm_frac": round(work["step_bytes"] / (ms / 1e3) / 1e9 / hbm_peak, 4),
                 "step_algorithmic_bytes": work["step_bytes"]}
        e2e_val = toks / (e2e / 1e3)
        metric = METRIC_DECODE
        cfg = workload_config(w, world, step.inp.context_lens)
    elif w.mode == "v4qkv":
        fl = step.flops
        value, unit = fl["total"] * world / (ms / 1e3) / 1e12, "TFLOP/s"
        achieved = fl["qb"] / (kms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": kern, "achieved": round(achieved, 2),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
                "peak_source": peak_src, "kernel_ms": round(kms, 4),
                "algorithmic_flops": fl["qb"], "traffic": measured_traffic(kern, w.name)}
        extra = {"tokens_per_s": round(toks / (ms / 1e3), 1), "step_flops": fl["total"]}
        e2e_val = fl["total"] * world / (e2e / 1e3) / 1e12
        metric = METRIC_V4
        cfg = workload_config(w, world)
    else:
        fl = step.flops
        value, unit = fl["total"] * world / (ms / 1e3) / 1e12, "TFLOP/s"
        achieved = fl["attn"] / (kms / 1e3) / 1e12
        roof = {"bound": "tensor", "kernel": kern, "achieved": round(achieved, 2),
                "peak": tc_peak, "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 4),
                "peak_source": peak_src, "kernel_ms": round(kms, 4),
                "algorithmic_flops": fl["attn"], "traffic": measured_traffic(kern, w.name)}
        extra = {"tokens_per_s": round(toks / (ms / 1e3), 1), "step_flops": fl["total"]}
        e2e_val = fl["total"] * world / (e2e / 1e3) / 1e12
        metric = METRIC_PREFILL
        cfg = workload_config(w, world)
    line.update({"metric": metric, "value": round(value, 3), "unit": unit, "n_gpus": world,
                 "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
                 "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                 "dtype": "bf16" if s.act_dtype == "bf16" else "f32",
                 "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
                 "config": cfg, "roofline": roof, **extra,
                 "e2e": {"value": round(e2e_val, 3), "unit": unit, "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e, 4)},
                 "gpu_launches": launches_per_step * args.steps, "clocks": clk})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_oracle_sample(w)
        cb.pop("seconds", None)
        line["cpu_baseline"] = cb
    flag = mla.mla_read_device_flag(step.ws)
    if flag:
        line["device_flag"] = flag
    return line


def workload_config(w: wl.Workload, world: int, context_lens=None) -> dict:
    """The `config` object of a bench line (both arms)."""
    s = w.shape
    l2 = "flushed before each timed step (256 MiB write, outside the events)"
    if w.mode in ("prefill", "v4qkv"):
        return {"workload": w.name, "seq_len": w.seq_len, "batch": 1, "weights": s.weight_dtype, "heads": s.n_heads,
                "hidden": s.hidden, "l2": l2, "parallelism": f"replicas x{world}"}
    if context_lens is None:
        context_lens = wl._context_lens(w, np.random.default_rng(w.seed + 100))   # as make_decode_inputs draws them
    return {"workload": w.name, "batch": w.batch, "context": [int(context_lens.min()), int(context_lens.max())],
            "mean_context": float(np.mean(context_lens)), "block_size": s.block_size, "weights": s.weight_dtype,
            "heads": s.n_heads, "hidden": s.hidden, "l2": l2, "parallelism": f"replicas x{world}"}


def run_reference(args, world, rank):
    """The oracle timed as the reference arm: each step is one oracle pass over a
    bounded sample of the workload (set up once, outside the timing)."""
    if rank != 0:
        return None
    w = selected_workload(args)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, budget_s=0.0, max_reps=1)
    vals, secs, cb = [], [], None
    for _ in range(args.steps):
        cb = cpu_oracle_sample(w, budget_s=0.0, max_reps=1)
        vals.append(cb["value"])
        secs.append(cb.pop("seconds"))
    v = float(np.mean(vals))
    cb["value"] = v
    cb["sample"] = cb["sample"] + f"; {args.steps} bench steps, each one oracle pass (set-up excluded)"
    line = {"impl": "reference", "metric": {"decode": METRIC_DECODE, "prefill": METRIC_PREFILL, "v4qkv": METRIC_V4}[w.mode],
            "value": round(v, 4), "unit": cb["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(float(np.mean(secs)) * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
            "config": workload_config(w, world), "cpu_baseline": cb,
            "e2e": {"value": round(v, 4), "unit": cb["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # profiling slices of a decode workload (fewer sequences, or one context for all); not bench lines
    ap.add_argument("--batch", type=int, default=0, help="override the decode workload's sequence count")
    ap.add_argument("--context", type=int, default=0, help="give every sequence this context length")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    from head_latent_attention_decode_b200.build import build
    world, rank, local = dist_init()
    if rank == 0:
        build()
    barrier(world)
    line = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
