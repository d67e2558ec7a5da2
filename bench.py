#!/usr/bin/env python
"""Benchmark of the QK4V8 hot path on B200; prints ONE JSON line (rank 0).

Default: both halves of the metric in one line. The headline workload is the long-context
causal prefill with GQA (batch 1, 32 query / 8 KV heads, 32768 tokens, head_dim 128, bf16
inputs); a step = quantize Q and K (NVFP4), quantize V (MXFP8), QK4V8 attention forward. The
``decode`` object of the same line measures the paged decode workload (64 sequences of
8192-32768 tokens, 32 / 8 heads, 64-token pages): a step = quantize the step's Q, paged
split-K decode, split merge; with it, the quantize-on-append kernel. Other workloads
(--workload): prefill_h16_n4096, mixed_prefill_n16384 (tile scoring + FP16 tiles in the
step), paged_decode_s64 alone.

Timing: inputs resident in HBM; W warm-up steps; then K steps, each bracketed by CUDA events
on the launching stream, with a 256 MB L2 flush between steps (outside the events); barrier +
synchronize on both sides; max over ranks. `e2e` repeats the step through the same public
API with the inputs copied from pinned host memory and the output read back inside the timed
region, one after another; `e2e_overlapped` runs the same with each step's copies on copy
streams of their own, overlapped with the neighbouring steps' compute. Multi-GPU (torchrun): independent replicas, one per GPU (no collective in the path).
`--impl reference` times the CPU oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import threading
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_block_scaled_nvfp4_b200 import workloads  # noqa: E402

METRIC = "QK4V8 attention TFLOPS & % of FP4 tensor peak; decode KV GB/s & % of HBM peak"

# DRAM bytes (read + write) of one launch of the dominant kernel, from an ncu capture of that
# kernel on the workload (dram__bytes_read.sum + dram__bytes_write.sum). Only workloads with a
# capture of the current kernel have an entry; the others report null.
NCU_TRAFFIC_BYTES = {
    "prefill_h16_n4096": 18_167_040 + 1_280,
    "prefill_gqa_n32768": 154_096_128 + 217_831_168,
    "mixed_prefill_n16384": 185_389_824 + 80_766_464,
    "paged_decode_s64": 2_170_382_000 + 13_552_384,
}
KERNEL_TIMING = "CUDA graph of the kernel(s) alone, replayed after a 256 MB L2 flush, CUDA events"
FP4_OVER_BF16 = 4.0          # nominal dense ratio 9 PF / 2.25 PF
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


def prefill_flops(cfg):
    """Algorithmic FLOPs: 4 d per visible (query, key) pair (QK^T and PV)."""
    B, H, N, d = cfg["B"], cfg["Hq"], cfg["N"], cfg["d"]
    pairs = N * (N + 1) // 2 if cfg["causal"] else N * N
    return 4.0 * d * pairs * B * H


def decode_bytes(lay):
    """Algorithmic KV bytes of one decode step: per token and KV head 64 + 8 (K codes,
    scales) + 128 + 4 (V codes, scales) at d = 128, whole pages counted, plus Q, page table,
    lengths and the output."""
    cfg = lay.cfg
    d, hkv, hq, S = cfg["d"], cfg["Hkv"], cfg["Hq"], cfg["S"]
    per_tok = d // 2 + d // 16 + d + d // 32
    pages = ((lay.lens.long() + 63) // 64).sum().item()
    kv = pages * 64 * hkv * per_tok
    other = S * hq * (d // 2 + d // 16) + lay.page_table.numel() * 4 + S * 4 + S * hq * d * 2
    return float(kv), float(kv + other)


class Clocks:
    """SM clock and throttle-reason sampler running during the timed region: NVML polled every
    2 ms from a thread (the device matched by PCI bus id), else an nvidia-smi loop."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.nvml = None
        self.samples = []          # (sm MHz, max MHz, reason names)
        self.out = ""

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        p = torch.cuda.get_device_properties(self.idx)
        bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _poll(self, nv, h):
        bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), [n for n, bit in zip(self.NAMES, bits) if r & bit]))
            except Exception:
                break
            self.stop.wait(0.002)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.stop = threading.Event()
            self.nvml = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.nvml.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.nvml is not None:
            self.stop.set()
            self.nvml.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], None, set()
        for s_mhz, m_mhz, names in self.samples:
            sm.append(s_mhz)
            mx = m_mhz
            reasons.update(names)
        for ln in (self.out or "").splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml" if self.samples else "nvidia-smi"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------------------
# The steps (our arm)
# ---------------------------------------------------------------------------------------
def make_prefill_step(name):
    from bit_block_scaled_nvfp4_b200 import api
    w = workloads.make_prefill(name)
    cfg = w.cfg
    q, k, v = w.q.cuda(), w.k.cuda(), w.v.cuda()
    mixed = cfg.get("frac_bp", 0) > 0
    scale = 1.0 / math.sqrt(cfg["d"])

    def quant(q=q, k=k, v=v):
        # Q, K (NVFP4) and V (MXFP8) in two launches: the amax pass of Q and K, then one encode
        # (with FP16 tiles also V's fp16 copy; their Q and K are the inputs themselves)
        return api.quantize_qkv(q, k, v, want_fp16_v=mixed)

    def step(q=q, k=k, v=v):
        q4, k4, v8 = quant(q, k, v)
        bitmap = None
        if mixed:
            _, _, bitmap = api.tile_score_select(q4, k4, cfg["causal"], cfg["frac_bp"])
        return api.attn_qk4v8_fwd(q4, k4, v8, cfg["causal"], scale, q.dtype, fp16_bitmap=bitmap,
                                  q16=q if mixed else None, k16=k if mixed else None)

    prep = {}

    def prepared():
        # inputs quantized (and scored) once, outside the graphs that time single kernels
        if not prep:
            prep["in"] = quant()
            prep["bm"] = (api.tile_score_select(prep["in"][0], prep["in"][1], cfg["causal"],
                                                cfg["frac_bp"])[2] if mixed else None)
        return prep

    def attn_only():
        # the attention kernel alone
        q4, k4, v8 = prepared()["in"]
        return api.attn_qk4v8_fwd(q4, k4, v8, cfg["causal"], scale, q.dtype, fp16_bitmap=prep["bm"],
                                  q16=q if mixed else None, k16=k if mixed else None)

    def score_only():
        # tile scoring and top-fraction selection alone
        q4, k4, _ = prepared()["in"]
        return api.tile_score_select(q4, k4, cfg["causal"], cfg["frac_bp"])

    launches = 3 + (3 if mixed else 0)
    host = [w.q.pin_memory(), w.k.pin_memory(), w.v.pin_memory()]
    # algorithmic quantize bytes: bf16 read once, NVFP4 codes + E4M3 scales (Q, K) and MXFP8
    # codes + E8M0 scales (V) written, plus V's fp16 copy that the FP16 tiles read
    nq, nk, nv = q.numel(), k.numel(), v.numel()
    qbytes = (nq + nk) * (2 + 0.5 + 1 / 16) + nv * (2 + 1 + 1 / 32) + (2 * nv if mixed else 0)
    # algorithmic scoring bytes: the Q and K codes and E4M3 scales read once
    sbytes = (nq + nk) * (0.5 + 1 / 16)
    return dict(cfg=cfg, step=step, step_on=lambda ins: step(*ins), inputs=(q, k, v), host=host,
                launches=launches, flops=prefill_flops(cfg), kind="prefill", quant=quant,
                quant_bytes=qbytes, device_bytes=sum(t.numel() * t.element_size() for t in (q, k, v)),
                score=(score_only, sbytes) if mixed else None,
                attn_only=attn_only)


def make_decode_step(name):
    from bit_block_scaled_nvfp4_b200 import api, paged
    lay = workloads.make_decode_layout(name)
    cfg = lay.cfg
    cache = paged.empty_cache(lay.num_pages, cfg["Hkv"], cfg["d"], workloads.DECODE_K_TENSOR_SCALE, "cuda")
    lens = lay.lens.tolist()
    for s in range(cfg["S"]):
        k, v = workloads.make_decode_sequence(lay, s)
        paged.write_sequence(cache, k.cuda(), v.cuda(), lay.page_table[s, :(lens[s] + 63) // 64])
    q = workloads.make_decode_query(lay).cuda()
    table, ctx = lay.page_table.cuda(), lay.lens.cuda()
    split = 4096
    # a serving loop's shape: the fixed buffers checked and allocated once (the decode plan, the
    # query's NVFP4 buffers and workspace), so a step is its launches
    plan = api.DecodePlan(cache, table, ctx, max(lens), split, cfg["S"], cfg["Hq"])
    q4buf = api.quantize_nvfp4(q)
    qws = torch.empty(api._lib.load().quantize_nvfp4_workspace_size(), dtype=torch.uint8, device="cuda")

    def quant(q=q):
        return api.quantize_nvfp4(q, workspace=qws, out=q4buf)

    def step(q=q):
        return plan.run(quant(q))

    plans = {table.data_ptr(): plan}

    def step_on(ins):
        # one step on another set of device inputs (query, page table, lengths): a plan per set
        q_, t_, c_ = ins
        if t_.data_ptr() not in plans:
            plans[t_.data_ptr()] = api.DecodePlan(cache, t_, c_, max(lens), split, cfg["S"], cfg["Hq"])
        return plans[t_.data_ptr()].run(quant(q_))

    prep = {}

    def attn_only():
        # decode + merge alone, on a query quantized once beforehand
        if not prep:
            prep["q4"] = api.quantize_nvfp4(q)
        return plan.run(prep["q4"])

    kv, total = decode_bytes(lay)
    host = [workloads.make_decode_query(lay).pin_memory(), lay.page_table.pin_memory(), lay.lens.pin_memory()]
    return dict(cfg=cfg, step=step, step_on=step_on, inputs=(q, table, ctx), host=host, launches=4,
                kv_bytes=kv, device_bytes=kv,
                bytes=total, kind="decode", split=split, lay=lay, quant=quant, attn_only=attn_only,
                quant_bytes=q.numel() * (2 + 0.5 + 1 / 16))


def make_append(cfg, chunk=512, seed=7):
    """The KV producer side of decode: quantize-on-append into a paged cache of the decode
    workload's shape (its sequences, KV heads and head_dim), one token per sequence (a decode
    step) and a chunk of ``chunk`` tokens per sequence (a prompt chunk). Each call appends at
    fixed positions (the lengths are not advanced), so repeated calls rewrite the same bytes.
    Algorithmic bytes: the new K/V read (2 x Hkv x d x 2 B per token), K codes + scales written
    (Hkv x (d/2 + d/16) B per token) and the V codes + scale of every touched 32-token group
    (Hkv x d x (32 + 1) B per group)."""
    from bit_block_scaled_nvfp4_b200 import api, paged
    S, hkv, d = cfg["S"], cfg["Hkv"], cfg["d"]
    g = torch.Generator().manual_seed(seed)
    lens0 = torch.randint(0, 64, (S,), generator=g, dtype=torch.int32)
    per = (64 + chunk + 63) // 64 + 1
    cache = paged.empty_cache(S * per, hkv, d, workloads.DECODE_K_TENSOR_SCALE, "cuda")
    table = torch.randperm(S * per, generator=g).view(S, per).to(torch.int32).cuda()
    tail = paged.empty_tail(S, hkv, d, torch.bfloat16, "cuda")
    lens = lens0.cuda()
    out = {}
    for name, n in (("step", 1), ("chunk", chunk)):
        k = torch.randn(S * n, hkv, d, generator=g).to(torch.bfloat16).cuda()
        v = torch.randn(S * n, hkv, d, generator=g).to(torch.bfloat16).cuda()
        cu = (torch.arange(S + 1, dtype=torch.int32) * n).cuda()
        groups = sum(((int(l) + n + 31) // 32 - int(l) // 32) for l in lens0)
        nbytes = S * n * hkv * (2 * d * 2 + d // 2 + d // 16) + groups * hkv * d * 33

        def fn(k=k, v=v, cu=cu, n=n):
            api.kv_append_paged(cache, k, v, cu, lens, table, tail, max_new=n)
        out[name] = (fn, nbytes, S * n)
    return out


def time_graph(fn, K):
    """Mean time (ms) of ``fn`` captured as a CUDA graph and replayed K times after an L2 flush."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    graph, _ = capture_step(fn)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in ev:
        flush.zero_()
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in ev) / K


def capture_step(step):
    """The whole step (quantize + attention, or quantize + decode + merge) as one CUDA graph, so
    that a timed step is the device work alone, without host launch gaps between kernels."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = step()
    torch.cuda.synchronize()
    return graph, out


def time_steps(st, K, W, world):
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    step = st["step"]
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    graph, st["graph_out"] = capture_step(step)
    for _ in range(W):
        graph.replay()
    s_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    k0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    k1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    q0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    q1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    qgraph, _ = capture_step(st["quant"])      # the quantize kernels alone, as one graph
    kgraph, _ = capture_step(st["attn_only"])  # the attention (or decode) kernels alone
    barrier(world)
    torch.cuda.synchronize()
    for i in range(K):                  # the step: one graph replay per step
        flush.zero_()
        s_ev[i].record()
        graph.replay()
        e_ev[i].record()
    torch.cuda.synchronize()
    for i in range(K):                  # the dominant kernel alone, as a graph of its own
        flush.zero_()
        k0[i].record()
        kgraph.replay()
        k1[i].record()
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()
        q0[i].record()
        qgraph.replay()
        q1[i].record()
    torch.cuda.synchronize()
    barrier(world)
    step_ms = sum(s.elapsed_time(e) for s, e in zip(s_ev, e_ev)) / K
    kern_ms = sum(a.elapsed_time(b) for a, b in zip(k0, k1)) / K
    st["quant_ms"] = sum(a.elapsed_time(b) for a, b in zip(q0, q1)) / K
    return step_ms, kern_ms


L2_BYTES = 126 << 20


def time_e2e_overlapped(st, K, world):
    """The same steps through the public API as a streaming caller runs them: each step's inputs
    copied from pinned host memory on a copy stream into one of two device input sets used in
    turn, the step on the compute stream once its copy has landed, and its output read back into
    pinned memory on a third stream, so that one step's copies overlap its neighbours' compute.
    A set is refilled only after the step that read it, and a step's output buffer is reused
    only after its read-back. Device time from the first copy in to the last copy out over K
    steps (after one untimed pass that allocates); ms per step. Inputs smaller than twice the
    L2 get a 256 MB flush on the compute stream before each step, inside the timed region."""
    host = st["host"]
    sets = [list(st["inputs"]), [t.clone() for t in st["inputs"]]]
    run = st["step_on"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if st["device_bytes"] < 2 * L2_BYTES else None
    cs = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    out_host = [None, None]

    def one_pass(n, timed):
        freed = [None, None]          # the compute stream has finished the step that read set b
        read_back = [None, None]      # the read-back of the last output made from set b is done
        t0 = t1 = None
        if timed:
            t0 = torch.cuda.Event(enable_timing=True)
            t0.record(s_in)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                if freed[b] is not None:
                    s_in.wait_event(freed[b])
                for d_, h_ in zip(sets[b], host):
                    d_.copy_(h_, non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(s_in)
            cs.wait_event(landed)
            if read_back[b] is not None:
                cs.wait_event(read_back[b])
            if flush is not None:
                flush.zero_()
            out = run(sets[b])
            out = out[0] if isinstance(out, tuple) else out
            done = torch.cuda.Event()
            done.record(cs)
            freed[b] = done
            with torch.cuda.stream(s_out):
                s_out.wait_event(done)
                if out_host[b] is None:
                    out_host[b] = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
                out_host[b].copy_(out, non_blocking=True)
                rb = torch.cuda.Event()
                rb.record(s_out)
                read_back[b] = rb
            out.record_stream(s_out)
        if timed:
            t1 = torch.cuda.Event(enable_timing=True)
            t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n if timed else None

    barrier(world)
    one_pass(2, False)
    ms = one_pass(K, True)
    barrier(world)
    return ms


def time_e2e(st, K, world):
    """Same step through the public API with H2D of the inputs (into the device tensors the
    step reads) and D2H of the output."""
    host = st["host"]
    dev = list(st["inputs"])
    out_host = None
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = 0
    tot = 0.0
    barrier(world)
    for i in range(K + 1):
        flush.zero_()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for d_, h_ in zip(dev, host):
            d_.copy_(h_, non_blocking=True)
        out = st["step"]()
        if out_host is None:
            out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        out_host.copy_(out, non_blocking=True)
        b.record()
        torch.cuda.synchronize()
        if i > 0:                       # the first pass allocates the pinned output
            tot += a.elapsed_time(b)
        d2h = out.numel() * out.element_size()
    barrier(world)
    return tot / K, h2d, d2h


# ---------------------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------------------
_INPUTS = {}


def _inputs(name):
    """The workload's seeded inputs (CPU), drawn once per process: drawing them is set-up, not
    part of a timed oracle sample."""
    if name not in _INPUTS:
        _INPUTS[name] = (workloads.make_decode_layout(name) if name == "paged_decode_s64"
                         else workloads.make_prefill(name))
    return _INPUTS[name]


def oracle_sample(name, rows=256, heads=1, seqs=1):
    """Time the oracle, as it stands, on a bounded sample of the workload: ``heads`` query
    heads x ``rows`` query rows spread over the sequence (prefill; the whole-tensor scales
    are computed once), or one decode step of the ``seqs`` shortest sequences (decode).
    Returns (seconds, algorithmic units (FLOPs or bytes) done, description)."""
    from oracle import attention as OA
    from oracle import quant as OQ
    from oracle import paged as OP
    if name == "paged_decode_s64":
        lay = _inputs(name)
        cfg = lay.cfg
        q = workloads.make_decode_query(lay).float().numpy()
        lens = lay.lens.numpy()
        picked = [int(i) for i in np.argsort(lens, kind="stable")[:max(1, seqs)]]
        seqs_kv = [workloads.make_decode_sequence(lay, s) for s in picked]
        per_tok = cfg["d"] // 2 + cfg["d"] // 16 + cfg["d"] + cfg["d"] // 32
        g = cfg["Hq"] // cfg["Hkv"]
        t0 = time.perf_counter()
        qc, qs, qt = OQ.nvfp4_quantize(q)
        qh = OQ.nvfp4_dequantize(qc, qs, qt)
        units = 0
        for s, (k, v) in zip(picked, seqs_kv):
            n = int(lens[s])
            kc, ks, vc, vs = OP.quantize_sequence(k.float().numpy(), v.float().numpy(),
                                                  workloads.DECODE_K_TENSOR_SCALE)
            kh = OQ.nvfp4_dequantize(kc, ks, np.float32(workloads.DECODE_K_TENSOR_SCALE))
            vh = OQ.mxfp8_dequantize_v(vc, vs, n)
            for h in range(cfg["Hkv"]):
                OA.decode_rows(qh[s, h * g:(h + 1) * g], kh[h], vh[h], n,
                               1 / math.sqrt(cfg["d"]), 4096)
            units += ((n + 63) // 64) * 64 * cfg["Hkv"] * per_tok
        dt = time.perf_counter() - t0
        toks = "+".join(str(int(lens[s])) for s in picked)
        return dt, float(units), (f"{len(picked)} sequence(s) ({toks} tokens) x {cfg['Hkv']} "
                                  f"KV heads of one decode step")
    w = _inputs(name)
    cfg = w.cfg
    N, d = cfg["N"], cfg["d"]
    rng = np.random.default_rng(0)
    row_idx = np.sort(rng.choice(N, size=min(rows, N), replace=False))
    scale = 1 / math.sqrt(d)
    q32 = w.q.float().numpy()
    k32 = w.k.float().numpy()
    t0 = time.perf_counter()
    sq = OQ.nvfp4_tensor_scale(q32)
    sk = OQ.nvfp4_tensor_scale(k32)
    flops = 0.0
    for hq in range(heads):
        hk = hq // (cfg["Hq"] // cfg["Hkv"])
        qh = OQ.nvfp4_dequantize(*OQ.nvfp4_quantize(q32[0, hq, row_idx], tensor_scale=sq))
        kh = OQ.nvfp4_dequantize(*OQ.nvfp4_quantize(k32[0, hk], tensor_scale=sk))
        vc, vs = OQ.mxfp8_quantize_v(w.v[0, hk].float().numpy())
        vh = OQ.mxfp8_dequantize_v(vc, vs, N)
        OA.attention_rows(qh, row_idx, kh, vh, cfg["causal"], scale)
        vis = (row_idx + 1).sum() if cfg["causal"] else len(row_idx) * N
        flops += 4.0 * d * float(vis)
    dt = time.perf_counter() - t0
    return dt, flops, f"{heads} query head(s) x {len(row_idx)} seeded query rows (of {N})"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def config_of(name):
    """The workload as both arms name it: its name and its sizes."""
    return {"workload": name, **dict(workloads.WORKLOADS[name])}


def run_reference(args, world, rank):
    if rank != 0:
        return
    name = args.workload
    is_decode = name == "paged_decode_s64"
    vals = []
    desc = ""
    for i in range(args.warmup + args.steps):
        dt, units, desc = oracle_sample(name, rows=64, heads=1)
        if i >= args.warmup:
            vals.append(units / dt / (1e9 if is_decode else 1e12))
    v = statistics.mean(vals)
    unit = "GB/s" if is_decode else "TFLOP/s"
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(name),
            "cpu_baseline": {"value": v, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure(name, args, world):
    """Time one workload: the step, its dominant kernel alone, its quantize kernels alone and the
    step end to end from host buffers (all max over ranks). Returns the pieces of a line, or
    None when a device wait timed out twice."""
    from bit_block_scaled_nvfp4_b200 import api
    st = make_decode_step(name) if name == "paged_decode_s64" else make_prefill_step(name)
    # A run in which a device wait timed out (status != 0) produced no valid result: report
    # where, take the measurement once more, and give up without a number if it repeats.
    for attempt in range(2):
        with Clocks(torch.cuda.current_device()) as clk:
            step_ms, kern_ms = time_steps(st, args.steps, args.warmup, world)
        e2e_ms, h2d, d2h = time_e2e(st, max(3, args.steps // 3), world)
        e2e_ov_ms = time_e2e_overlapped(st, max(4, args.steps // 3), world)
        status = api.check_status()
        # every rank takes the same decision, so that all of them run the same collectives
        agreed = max_over_ranks(float(status), world)
        if agreed == 0:
            break
        print(f"bench: {name}: device status {status} (worst over ranks {agreed:g}), first "
              f"timed-out wait {api.timeout_site()} (attempt {attempt + 1})", file=sys.stderr)
    if agreed != 0:
        return None
    step_ms = max_over_ranks(step_ms, world)
    kern_ms = max_over_ranks(kern_ms, world)
    e2e_ms = max_over_ranks(e2e_ms, world)
    e2e_ov_ms = max_over_ranks(e2e_ov_ms, world)
    quant_ms = max_over_ranks(st["quant_ms"], world)
    pk, src = peaks()
    if st["kind"] == "prefill":
        units = st["flops"]
        value = units * world / (step_ms * 1e-3) / 1e12
        e2e_v = units * world / (e2e_ms * 1e-3) / 1e12
        e2e_ov = units * world / (e2e_ov_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
        ach = units / (kern_ms * 1e-3) / 1e12
        peak = pk["bf16_tflops"] * FP4_OVER_BF16
        roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": NCU_TRAFFIC_BYTES.get(name),
                # FP16-tile workloads run the FP16-tile instance; FP4-only ones the paired kernel
                "kernel": "attn_fwd_kernel" if st["cfg"].get("frac_bp", 0) > 0 else "attn_pp_kernel",
                "kernel_ms": kern_ms, "timing": KERNEL_TIMING,
                "peak_source": f"{src} bf16 x {FP4_OVER_BF16:g} (FP4 dense)",
                "mixed_fp4_fp8_bound_tflops": peak / 1.5}
    else:
        units = st["bytes"]
        value = units * world / (step_ms * 1e-3) / 1e9
        e2e_v = units * world / (e2e_ms * 1e-3) / 1e9
        e2e_ov = units * world / (e2e_ov_ms * 1e-3) / 1e9
        unit = "GB/s"
        ach = st["kv_bytes"] / (kern_ms * 1e-3) / 1e9
        peak = pk["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": NCU_TRAFFIC_BYTES.get(name), "traffic_kernel": "decode_kernel",
                "kernel": "decode_kernel + decode_merge_kernel", "kernel_ms": kern_ms,
                "timing": KERNEL_TIMING, "peak_source": f"{src} hbm_gbs"}
    out = {"value": value, "unit": unit, "ms_per_step": step_ms, "config": config_of(name),
           "roofline": roof,
           "e2e": {"value": e2e_v, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
           # the same with each step's copies overlapped with its neighbours' compute
           "e2e_overlapped": {"value": e2e_ov, "unit": unit, "ms_per_step": e2e_ov_ms,
                              "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                              "streams": "copy in, compute, copy out; two input sets in turn"},
           "gpu_launches": st["launches"] * args.steps,
           # the quantize kernels of the step, timed as a graph of their own after an L2 flush
           # (algorithmic bytes: the amax pass's second read of each input is not counted)
           "quantize": {"achieved_gbs": st["quant_bytes"] / (quant_ms * 1e-3) / 1e9,
                        "peak_gbs": pk["hbm_gbs"],
                        "frac": st["quant_bytes"] / (quant_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                        "ms": quant_ms, "bytes": st["quant_bytes"]},
           "device_status": status, "clocks": clk.summary()}
    if st["kind"] == "decode":
        # the producer side of the decode path: quantize-on-append into the paged cache
        app = {}
        for nm, (fn, nbytes, ntok) in make_append(st["cfg"]).items():
            ms = max_over_ranks(time_graph(fn, max(3, args.steps // 3)), world)
            app[nm] = {"ms": ms, "tokens": ntok, "bytes": nbytes,
                       "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                       "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
        out["append"] = {"kernel": "kv_append_kernel", "timing": KERNEL_TIMING,
                         "peak_gbs": pk["hbm_gbs"], **app}
    if st.get("score") is not None:
        # tile scoring and selection of the FP16-tile workload, against the HBM peak
        fn, nbytes = st["score"]
        ms = max_over_ranks(time_graph(fn, max(3, args.steps // 3)), world)
        out["score"] = {"kernel": "row_norm_tile_max_kernel + tile_select_kernel",
                        "timing": KERNEL_TIMING, "ms": ms, "bytes": nbytes,
                        "achieved_gbs": nbytes / (ms * 1e-3) / 1e9, "peak_gbs": pk["hbm_gbs"],
                        "frac": nbytes / (ms * 1e-3) / 1e9 / pk["hbm_gbs"]}
    if world == 1 and not args.no_cpu_baseline:          # the oracle is timed at N = 1 only
        # about ten seconds of host work on 16 cores: 5 query heads x 4096 rows, or 8 sequences
        dt, u, desc = oracle_sample(name, rows=4096, heads=5, seqs=8)
        cv = u / dt / (1e12 if st["kind"] == "prefill" else 1e9)
        out["cpu_baseline"] = {"value": cv, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                               "sample": desc, "seconds": dt}
    del st
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill_gqa_n32768",
                    choices=[n for n in workloads.WORKLOADS if n != "tiny_prefill"])
    ap.add_argument("--no-decode", action="store_true",
                    help="leave out the decode object (paged_decode_s64) of a prefill line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if world > 1:                   # no collective was used; release the group
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    name = args.workload
    try:
        apps = subprocess.run(["nvidia-smi", "--query-compute-apps=pid,process_name,used_memory",
                               "--format=csv,noheader"], capture_output=True, text=True, timeout=20).stdout
        print(f"bench: compute apps on the GPUs before the run: {apps.strip() or 'none'}", file=sys.stderr)
    except (OSError, subprocess.TimeoutExpired):
        pass
    head = measure(name, args, world)
    dec = None
    if head is not None and name != "paged_decode_s64" and not args.no_decode:
        dec = measure("paged_decode_s64", args, world)
    if head is None or (dec is None and name != "paged_decode_s64" and not args.no_decode):
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        raise SystemExit(3)
    line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "nvfp4/mxfp8 (fp32 accumulate)", "data": "synthetic",
            "config": head["config"],
            "parallelism": f"replicas x{world}",
            "timing": {"l2": "256 MB flush between timed steps",
                       "step": "one CUDA graph replay (all kernels of the step)"},
            **{k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step", "config")}}
    if dec is not None:
        # the other half of the metric: decode KV GB/s against the HBM peak, timed the same way
        line["decode"] = dec
        line["gpu_launches"] += dec["gpu_launches"]
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
