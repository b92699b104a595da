#!/usr/bin/env python
"""Benchmark of the Diagonal KDN memory recurrence on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|long|varlen] [--no-cpu-baseline]

Primary metric: prefill tokens/s of kdn_forward_chunkwise on the chunkwise-prefill
workload (B=4, H=16, T=4096, d_k=d_v=128, bf16 inputs, fp32 state, chunk 64); a step
is one forward over the whole batch (uncertainty/gain, chunk algebra, state carry and
readout -- every step of the hot path), timed with CUDA events on the launching stream.
The JSON line also carries the decode rate (steps/s on 256 sequences x 32 heads,
d = 128, fp32 state, 1024 steps), the long-context (B=1, H=32, T=65536, key pool) and
packed-varlen (262144 tokens, d_v = 256) prefill rates, the gain scan and the backward,
each with its roofline fraction against the measured HBM copy bandwidth, the end-to-end
rate through the C ABI with host buffers, and the fp64 oracle timed on the host cores.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent batch
(weak scaling, no data-path collective); timings are the max over ranks.

--impl reference times the fp64 CPU oracle (rank 0 only) on a bounded sample of the
same workload per step.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_BYTES = 126 * 1024 * 1024


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def workload(name, seed_offset=0):
    from kalman_delta_rule_b200 import inputs
    if name == "prefill":
        w = inputs.prefill_4x4096(seed=1 if not seed_offset else (1, seed_offset))
    elif name == "long":
        w = inputs.long_context_65536(seed=3 if not seed_offset else (3, seed_offset))
    elif name == "varlen":
        w = inputs.varlen_262144(seed=4 if not seed_offset else (4, seed_offset))
    else:
        raise ValueError(name)
    return w


def algorithmic_bytes(w, state_out=True):
    """Bytes a forward must move at least: every input once, o once, final S and P."""
    esz = 2 if w.bf16 else 4
    per_tok_head = (4 * w.dk + 2 * w.dv) * esz + esz       # q, k, alpha, sigma, v, o, r
    n = w.ntok * w.H * per_tok_head
    if state_out:
        n += w.num_seqs * w.H * (w.dk * w.dv + w.dk) * 4
    return n


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the GPU is loaded."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        top = sorted(sm)[len(sm) // 4:] or sm   # under load: drop the idle tail
        return {"sm_mhz": statistics.median(top), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        torch.cuda.synchronize()


def max_over_ranks(x, world, device="cuda"):
    """The largest of the ranks' values (each rank's device-timed duration); one scalar
    all-reduce, the only collective of the benchmark."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_per_step, steps, local_ms, world, device="cuda"):
    """Weak scaling: every rank processes its own batch; the job's rate is all ranks' units
    divided by the slowest rank's time.  Returns (rate per second, max ms)."""
    ms = max_over_ranks(local_ms, world, device)
    return world * units_per_rank_per_step * steps / (ms / 1e3), ms


# ------------------------------------------------------------------ our arm
def to_dev(a, dev):
    import torch
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    if a.dtype == np.int32:
        return torch.from_numpy(a).to(dev)
    return torch.from_numpy(a.astype(np.float32)).to(dev)


def bench_prefill(args, world, rank, dev, kdn):
    import torch
    w = workload(args.workload, seed_offset=rank)
    B = w.B if w.B else 1
    shp = lambda x: x.reshape((B, w.ntok // B) + x.shape[1:])
    names = ("q", "k", "v", "alpha", "sigma", "r")
    host = {n: shp(getattr(w, n)) for n in names}
    d = {n: to_dev(host[n], dev) for n in names}
    cu = to_dev(w.cu_seqlens, dev) if (w.B == 1 and w.num_seqs > 1) else None
    o = torch.empty(d["q"].shape[:3] + (w.dv,), dtype=d["q"].dtype, device=dev)
    S_out = torch.empty((w.num_seqs, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    P_out = torch.empty((w.num_seqs, w.H, w.dk), dtype=torch.float32, device=dev)
    max_seqlen = int(np.diff(w.cu_seqlens).max()) if cu is not None else 0
    prob = kdn.make_problem(d["q"], d["v"], cu_seqlens=cu, mu=w.mu, chunk=w.chunk, max_seqlen=max_seqlen)
    ws_bytes = kdn.kdn_workspace_size(prob)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    path = kdn.PATH_NAMES[kdn.kdn_execution_path(prob)]
    launches_per_step = 2 if path == "chunk_tcgen05_two_phase" else 1
    stream = torch.cuda.current_stream()

    def step():
        kdn.forward(d["q"], d["k"], d["v"], d["alpha"], d["sigma"], d["r"], cu_seqlens=cu, mu=w.mu, chunk=w.chunk,
                    o=o, S_out=S_out, P_out=P_out, workspace=ws, max_seqlen=max_seqlen)

    for _ in range(args.warmup):
        step()
    kdn.last_device_error()
    # sustained run for the clock record (same kernel, same inputs), then the timed region
    with ClockSampler(dev.index) as clk:
        t_end = time.time() + args.clock_seconds
        while time.time() < t_end:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        barrier(world)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    kdn.last_device_error()
    per_step_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    tokens = w.ntok  # per rank, all heads included
    value, total_ms = whole_job_rate(tokens, args.steps, evs[0].elapsed_time(evs[-1]), world)
    ms_step = total_ms / args.steps

    # the isotropic variant (one uncertainty per head) on the same inputs and path
    iso = None
    if path.startswith("chunk_tcgen05"):
        P_iso = torch.empty((w.num_seqs, w.H), dtype=torch.float32, device=dev)

        def step_iso():
            kdn.forward(d["q"], d["k"], d["v"], d["alpha"], d["sigma"], d["r"], cu_seqlens=cu, mu=w.mu,
                        chunk=w.chunk, o=o, S_out=S_out, P_out=P_iso, workspace=ws, max_seqlen=max_seqlen,
                        variant="isotropic")
        for _ in range(2):
            step_iso()
        barrier(world)
        i0, i1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_iso = max(3, min(args.steps, 5))
        i0.record(stream)
        for _ in range(n_iso):
            step_iso()
        i1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        kdn.last_device_error()
        i_value, i_ms = whole_job_rate(w.ntok, n_iso, i0.elapsed_time(i1), world)
        iso = dict(value=i_value, ms_per_step=i_ms / n_iso, gpu_launches=n_iso * launches_per_step,
                   path=kdn.execution_path(d["q"], d["v"], cu_seqlens=cu, chunk=w.chunk, variant="isotropic"))

    # end to end through the C ABI: every step copies its inputs from pinned host memory to the
    # device, runs the forward and copies o back to pinned host memory.  Steps are pipelined over
    # three streams and two device buffer sets: the copy-in of step n+1 and the copy-out of step
    # n-1 overlap the forward of step n (the two copy directions use separate copy engines).
    pinned = {n: torch.from_numpy(np.ascontiguousarray(host[n]).view(np.int16) if host[n].dtype == np.uint16
                                  else np.ascontiguousarray(host[n])).pin_memory() for n in names}
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = o_host[0].numel() * o_host[0].element_size()
    dd = [d, {n: torch.empty_like(d[n]) for n in names}]
    oo = [o, torch.empty_like(o)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    fwd_done = [ev(), ev()]     # the forward of the slot's previous step has read its inputs
    out_done = [ev(), ev()]     # the slot's previous o has reached the host
    for sl in range(2):
        fwd_done[sl].record(stream)
        out_done[sl].record(stream)

    def e2e_step(n):
        sl = n % 2
        di, do_, in_ready, o_ready = dd[sl], oo[sl], ev(), ev()
        with torch.cuda.stream(s_in):
            s_in.wait_event(fwd_done[sl])
            for nm in names:
                dst = di[nm].view(torch.int16) if di[nm].dtype == torch.bfloat16 else di[nm]
                dst.copy_(pinned[nm], non_blocking=True)
            in_ready.record(s_in)
        stream.wait_event(in_ready)
        stream.wait_event(out_done[sl])
        kdn.forward(di["q"], di["k"], di["v"], di["alpha"], di["sigma"], di["r"], cu_seqlens=cu, mu=w.mu,
                    chunk=w.chunk, o=do_, S_out=S_out, P_out=P_out, workspace=ws, max_seqlen=max_seqlen, stream=stream)
        fwd_done[sl].record(stream)
        o_ready.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(o_ready)
            o_host[sl].copy_(do_, non_blocking=True)
            out_done[sl].record(s_out)

    for i in range(max(2, args.warmup // 2)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(4, min(args.steps, 10))
    e0.record(stream)
    s_in.wait_event(e0)
    for i in range(e_steps):
        e2e_step(i)
    stream.wait_event(out_done[(e_steps - 1) % 2])
    stream.wait_event(out_done[(e_steps - 2) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_value, e2e_ms = whole_job_rate(tokens, e_steps, e0.elapsed_time(e1), world)

    # the uncertainty / gain scan on its own, over the same inputs (g fp32, k^T g, final P)
    scan = None
    if not args.no_scan:
        ws_scan = torch.empty(max(kdn.kdn_workspace_size(prob), 1), dtype=torch.uint8, device=dev)
        g_out = torch.empty(d["k"].shape, dtype=torch.float32, device=dev)
        b_out = torch.empty(d["k"].shape[:3], dtype=torch.float32, device=dev)
        p_out = torch.empty((w.num_seqs, w.H, w.dk), dtype=torch.float32, device=dev)
        sp = kdn.make_problem(d["k"], d["k"], cu_seqlens=cu, mu=w.mu, chunk=w.chunk, max_seqlen=max_seqlen)
        sargs = [d[n].data_ptr() for n in ("k", "alpha", "sigma", "r")]
        sh = stream.cuda_stream or None

        def scan_step():
            st = kdn.kdn_gain_scan(sp, *sargs, None, g_out.data_ptr(), b_out.data_ptr(), p_out.data_ptr(),
                                   ws_scan.data_ptr(), ws_scan.numel(), sh)
            if st != kdn.KDN_OK:
                raise kdn.KdnError(st, "kdn_gain_scan")

        for _ in range(args.warmup):
            scan_step()
        kdn.last_device_error()
        barrier(world)
        sev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        sev[0].record(stream)
        for i in range(args.steps):
            scan_step()
            sev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        kdn.last_device_error()
        s_ms = max_over_ranks(sev[0].elapsed_time(sev[-1]), world) / args.steps
        esz = 2 if w.bf16 else 4
        s_bytes = w.ntok * w.H * (3 * w.dk * esz + esz + w.dk * 4 + 4) + w.num_seqs * w.H * w.dk * 4
        scan = dict(value=world * w.ntok / (s_ms / 1e3), ms_step=s_ms, bytes=s_bytes, launches=args.steps)

    # the backward pass (gradients of <o, d_o> with respect to every input, S0 and P0) on the
    # same inputs, d_o drawn once on the device; both uncertainty variants
    def bwd_leg(variant):
        gen = torch.Generator(device=dev)
        gen.manual_seed(1234 + rank)
        d_o = torch.randn(o.shape, generator=gen, device=dev).to(o.dtype)
        f32 = dict(dtype=torch.float32, device=dev)
        p_shape = (w.num_seqs, w.H) + ((w.dk,) if variant == "diagonal" else ())
        grads = dict(dq=torch.empty(d["q"].shape, **f32), dk=torch.empty(d["k"].shape, **f32),
                     dv=torch.empty(d["v"].shape, **f32), dalpha=torch.empty(d["alpha"].shape, **f32),
                     dsigma=torch.empty(d["sigma"].shape, **f32), dr=torch.empty(d["r"].shape, **f32),
                     dS0=torch.empty((w.num_seqs, w.H, w.dk, w.dv), **f32), dP0=torch.empty(p_shape, **f32))
        bp = kdn.make_problem(d["q"], d["v"], cu_seqlens=cu, mu=w.mu, chunk=0, max_seqlen=max_seqlen, variant=variant)
        ws_bwd = torch.empty(kdn.kdn_backward_workspace_size(bp), dtype=torch.uint8, device=dev)
        bargs = [d[n].data_ptr() for n in names]
        gptr = [grads[n].data_ptr() for n in ("dq", "dk", "dv", "dalpha", "dsigma", "dr", "dS0", "dP0")]
        sh = stream.cuda_stream or None

        def bwd_step():
            st = kdn.kdn_backward(bp, *bargs, None, None, d_o.data_ptr(), None, None, *gptr,
                                  ws_bwd.data_ptr(), ws_bwd.numel(), sh)
            if st != kdn.KDN_OK:
                raise kdn.KdnError(st, "kdn_backward")

        for _ in range(2):
            bwd_step()
        kdn.last_device_error()
        barrier(world)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_bwd = 3
        b0.record(stream)
        for _ in range(n_bwd):
            bwd_step()
        b1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        kdn.last_device_error()
        b_ms = max_over_ranks(b0.elapsed_time(b1), world) / n_bwd
        esz = 2 if w.bf16 else 4
        b_bytes = (w.ntok * w.H * ((4 * w.dk + 2 * w.dv + 1) * esz + (4 * w.dk + w.dv + 1) * 4)
                   + w.num_seqs * w.H * (w.dk * w.dv + (w.dk if variant == "diagonal" else 1)) * 4)
        del ws_bwd
        return dict(value=world * w.ntok / (b_ms / 1e3), ms_step=b_ms, bytes=b_bytes, variant=variant)

    bwd = bwd_iso = None
    if not args.no_backward:
        bwd = bwd_leg("diagonal")
        bwd_iso = bwd_leg("isotropic")

    nbytes = algorithmic_bytes(w)
    return dict(w=w, value=value, ms_step=ms_step, per_step_ms=per_step_ms, clocks=clk.summary(), path=path, scan=scan,
                iso=iso, bwd=bwd, bwd_iso=bwd_iso,
                e2e=dict(value=e2e_value, unit="tokens/s", h2d_bytes_per_step=h2d, d2h_bytes_per_step=d2h,
                         steps=e_steps),
                bytes=nbytes, launches=args.steps * launches_per_step)


def bench_prefill_other(args, world, rank, dev, kdn, name, steps=5):
    """Another prefill workload (long context, packed varlen) timed like the headline one: inputs
    resident in HBM, CUDA events around `steps` forwards after the warm-up."""
    import torch
    w = workload(name, seed_offset=rank)
    B = w.B if w.B else 1
    names = ("q", "k", "v", "alpha", "sigma", "r")
    d = {n: to_dev(getattr(w, n).reshape((B, w.ntok // B) + getattr(w, n).shape[1:]), dev) for n in names}
    cu = to_dev(w.cu_seqlens, dev) if (w.B == 1 and w.num_seqs > 1) else None
    o = torch.empty(d["q"].shape[:3] + (w.dv,), dtype=d["q"].dtype, device=dev)
    S_out = torch.empty((w.num_seqs, w.H, w.dk, w.dv), dtype=torch.float32, device=dev)
    P_out = torch.empty((w.num_seqs, w.H, w.dk), dtype=torch.float32, device=dev)
    max_seqlen = int(np.diff(w.cu_seqlens).max()) if cu is not None else 0
    prob = kdn.make_problem(d["q"], d["v"], cu_seqlens=cu, mu=w.mu, chunk=w.chunk, max_seqlen=max_seqlen)
    ws = torch.empty(max(kdn.kdn_workspace_size(prob), 1), dtype=torch.uint8, device=dev)
    path = kdn.PATH_NAMES[kdn.kdn_execution_path(prob)]
    stream = torch.cuda.current_stream()

    def step():
        kdn.forward(d["q"], d["k"], d["v"], d["alpha"], d["sigma"], d["r"], cu_seqlens=cu, mu=w.mu, chunk=w.chunk,
                    o=o, S_out=S_out, P_out=P_out, workspace=ws, max_seqlen=max_seqlen)

    for _ in range(args.warmup):
        step()
    kdn.last_device_error()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    kdn.last_device_error()
    value, ms = whole_job_rate(w.ntok, steps, e0.elapsed_time(e1), world)
    out = dict(workload=w.name, value=value, unit="tokens/s", ms_per_step=ms / steps, steps=steps,
               gpu_launches=steps * (2 if path == "chunk_tcgen05_two_phase" else 1), path=path,
               bytes=algorithmic_bytes(w))
    del d, o, S_out, P_out, ws
    torch.cuda.empty_cache()
    return out


def bench_decode(args, world, rank, dev, kdn, steps=1024, N=256, H=32, d=128):
    """1024 decode steps on 256 sequences x 32 heads (inputs resident, drawn on the device)."""
    import torch
    from kalman_delta_rule_b200 import inputs
    dv = inputs.decode_inputs_device(2_000 + rank, steps, N, H, d, device=dev)
    S, P = dv["S0"], dv["P0"]
    q, k, v, al, sg, r = (dv[n] for n in ("q", "k", "v", "alpha", "sigma", "r"))
    o = torch.empty((N, H, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def run(n):
        for s in range(n):
            kdn.decode_step(q[s], k[s], v[s], al[s], sg[s], r[s], S, P, o=o)

    run(min(steps, max(3, args.warmup)))
    kdn.last_device_error()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    kdn.last_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    # the same tokens four per launch (multi-token decode: one state read/write per 4 tokens)
    multi = None
    if steps % 4 == 0:
        q4, k4, v4, a4, s4, r4 = [x.view((steps // 4, 4) + x.shape[1:]).transpose(0, 1) for x in (q, k, v, al, sg, r)]
        groups = [tuple(t[:, j].transpose(0, 1).contiguous() for t in (q4, k4, v4, a4, s4, r4)) for j in range(steps // 4)]
        o4 = torch.empty((N, 4, H, d), dtype=torch.bfloat16, device=dev)

        def run4(n):
            for j in range(n):
                kdn.decode_tokens(*groups[j], S, P, o=o4)
        run4(min(len(groups), 3))
        barrier(world)
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        run4(len(groups))
        m1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        kdn.last_device_error()
        mms = max_over_ranks(m0.elapsed_time(m1), world)
        # per launch: S and P read and written once, four tokens' inputs and outputs
        b4 = N * H * (2 * d * d * 4 + 2 * d * 4 + 4 * ((4 * d + d) * 2 + 2 + d * 2))
        multi = dict(value=world * steps / (mms / 1e3), ms_per_launch=mms / len(groups), launches=len(groups),
                     bytes=b4)
    per_step = ms / steps
    head_step_bytes = 2 * d * d * 4 + 2 * d * 4 + (4 * d + d) * 2 + 2 + d * 2
    nbytes = N * H * head_step_bytes
    return dict(value=world * steps / (ms / 1e3), ms_step=per_step, bytes=nbytes, steps=steps, N=N, H=H, d=d,
                multi=multi)


def cpu_baseline_prefill(w, min_seconds=10.0, max_reps=50):
    """The fp64 oracle on the host cores over the whole workload (every (sequence, head)
    chain, full length), repeated until about `min_seconds` of wall time have passed."""
    import oracle
    cores = os.cpu_count() or 1
    chains = [(s, h) for s in range(w.num_seqs) for h in range(w.H)]
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.diag_chains(w, chains, threads=cores)
        reps += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds or reps >= max_reps:
            break
    tok = reps * w.ntok
    return {"value": tok / dt, "unit": "tokens/s", "cores": min(cores, len(chains)), "kind": "oracle",
            "sample": f"the whole workload ({len(chains)} (sequence, head) chains x full length) run {reps} times "
                      f"by the fp64 C oracle, {dt:.1f} s wall"}


def kernel_hash():
    h = hashlib.sha1()
    for fn in ("kdn_chunk_2p.cu", "kdn_tc.cuh", "kdn_common.cuh"):
        with open(os.path.join(ROOT, "kalman_delta_rule_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def recorded_traffic(workload_name):
    """dram bytes of one forward step (its prep and state launches) from the committed ncu
    summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = kernel_hash()
    for line in open(p):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == workload_name and parts[2] == cur:
            return float(parts[1])
    return None


def ours(args):
    import torch
    from kalman_delta_rule_b200 import binding as kdn
    kdn.load()
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    pk, pk_kind = peaks()
    pre = bench_prefill(args, world, rank, dev, kdn)
    dec = bench_decode(args, world, rank, dev, kdn, steps=args.decode_steps) if not args.no_decode else None
    others = []
    if not args.no_other_workloads:
        for name in ("long", "varlen"):
            if name != args.workload:
                others.append(bench_prefill_other(args, world, rank, dev, kdn, name))
    w = pre["w"]
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_prefill(w)
    if rank == 0:
        kern_s = statistics.mean(pre["per_step_ms"]) / 1e3
        ach = pre["bytes"] / kern_s / 1e9
        hbm = float(pk["hbm_gbs"])
        traffic = recorded_traffic(w.name)
        line = {
            "metric": "KDN prefill tokens/s + decode steps/s on 1 B200; % of HBM/tensor roofline",
            "value": pre["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": pre["ms_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded; shapes and distributions of the workload recipe)",
            "config": {"workload": w.name, "B": w.B, "T": w.ntok // (w.B or 1), "H": w.H, "d_k": w.dk, "d_v": w.dv,
                       "chunk": w.chunk, "mu": w.mu, "state": "fp32", "kernel_path": pre["path"],
                       "l2": f"inputs larger than L2 ({pre['bytes'] / 1e9:.2f} GB > 0.13 GB), no flush",
                       "parallelism": f"replicas x{world} (independent batches, no collective)"},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "traffic": traffic if pre["path"] == "chunk_tcgen05_two_phase" else None,
                         "peak_kind": f"{pk_kind} copy bandwidth",
                         "algorithmic_bytes_per_launch": pre["bytes"],
                         "unit_of_measure": "one forward step = the prep and the state launch of the "
                                            "two-launch tensor-core path; achieved and traffic are per step"},
            "cpu_baseline": cpu,
            "e2e": pre["e2e"],
            "gpu_launches": pre["launches"],
            "clocks": pre["clocks"],
        }
        if pre["iso"] is not None:
            it = pre["iso"]
            it["metric"] = "isotropic KDN prefill tokens/s"
            it["unit"] = "tokens/s"
            it["roofline_frac"] = pre["bytes"] / (it["ms_per_step"] / 1e3) / 1e9 / hbm
            line["prefill_isotropic"] = it
        if pre["scan"] is not None:
            sc = pre["scan"]
            sach = sc["bytes"] / (sc["ms_step"] / 1e3) / 1e9
            line["gain_scan"] = {"metric": "gain scan tokens/s (P^-, gain, k^T g, final P)", "value": sc["value"],
                                 "unit": "tokens/s", "ms_per_step": sc["ms_step"], "gpu_launches": sc["launches"],
                                 "roofline": {"bound": "hbm", "achieved": sach, "peak": hbm, "unit": "GB/s",
                                              "frac": sach / hbm, "traffic": None,
                                              "algorithmic_bytes_per_launch": sc["bytes"]}}
        for key, bw, launches in (("backward", pre["bwd"], 4), ("backward_isotropic", pre["bwd_iso"], 7)):
            if bw is None:
                continue
            bach = bw["bytes"] / (bw["ms_step"] / 1e3) / 1e9
            line[key] = {"metric": f"{bw['variant']} backward tokens/s (gradients of o w.r.t. q, k, v, alpha, sigma, r, S0, P0)",
                         "value": bw["value"], "unit": "tokens/s", "ms_per_step": bw["ms_step"],
                         "gpu_launches": 3 * launches, "dtype": "f32 (bf16 inputs widened)",
                         "roofline": {"bound": "hbm", "achieved": bach, "peak": hbm, "unit": "GB/s",
                                      "frac": bach / hbm, "traffic": None,
                                      "algorithmic_bytes_per_launch": bw["bytes"],
                                      "unit_of_measure": f"one backward call = its {launches} launches"}}
        for ot in others:
            oach = ot["bytes"] / (ot["ms_per_step"] / 1e3) / 1e9
            key = "prefill_long" if ot["workload"].startswith("long") else "prefill_varlen"
            line[key] = {"metric": "KDN prefill tokens/s", "workload": ot["workload"], "value": ot["value"],
                         "unit": "tokens/s", "ms_per_step": ot["ms_per_step"], "steps": ot["steps"],
                         "gpu_launches": ot["gpu_launches"], "kernel_path": ot["path"],
                         "roofline": {"bound": "hbm", "achieved": oach, "peak": hbm, "unit": "GB/s",
                                      "frac": oach / hbm, "traffic": None,
                                      "algorithmic_bytes_per_launch": ot["bytes"],
                                      "unit_of_measure": "one forward step (prep + state launch)"}}
        if dec is not None:
            dach = dec["bytes"] / (dec["ms_step"] / 1e3) / 1e9
            line["decode"] = {"metric": "decode steps/s", "value": dec["value"], "unit": "steps/s",
                              "ms_per_step": dec["ms_step"], "steps": dec["steps"],
                              "workload": f"decode_N{dec['N']}_H{dec['H']}_d{dec['d']}_bf16_fp32state",
                              "gpu_launches": dec["steps"],
                              "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm, "unit": "GB/s",
                                           "frac": dach / hbm, "traffic": None,
                                           "algorithmic_bytes_per_launch": dec["bytes"]}}
            if dec["multi"] is not None:
                line["decode"]["four_tokens_per_launch"] = {
                    "metric": "decode steps/s, 4 tokens per launch", "value": dec["multi"]["value"], "unit": "steps/s",
                    "ms_per_launch": dec["multi"]["ms_per_launch"], "gpu_launches": dec["multi"]["launches"]}
                m = dec["multi"]
                mach = m["bytes"] / (m["ms_per_launch"] / 1e3) / 1e9
                line["decode"]["four_tokens_per_launch"]["roofline"] = {
                    "bound": "hbm", "achieved": mach, "peak": hbm, "unit": "GB/s", "frac": mach / hbm,
                    "traffic": None, "algorithmic_bytes_per_launch": m["bytes"]}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------ reference arm (the oracle)
def reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    w = workload(args.workload)
    cores = os.cpu_count() or 1
    n = max(1, min(cores, w.num_seqs * w.H, 8))
    chains = [(s, h) for s in range(w.num_seqs) for h in range(w.H)][:n]
    # each step: the oracle over n whole chains, cut to a bounded token count
    max_tok = int(os.environ.get("KDN_REF_TOKENS", "1024"))

    class Sub:
        pass
    sub = Sub()
    for nm in ("q", "k", "v", "alpha", "sigma", "r"):
        setattr(sub, nm, getattr(w, nm))
    cu = np.array([0] + [min(int(w.cu_seqlens[s + 1] - w.cu_seqlens[s]), max_tok) for s in range(w.num_seqs)])
    # rebuild a token array holding the first max_tok tokens of each sequence
    idx = np.concatenate([np.arange(int(w.cu_seqlens[s]), int(w.cu_seqlens[s]) + cu[s + 1]) for s in range(w.num_seqs)])
    for nm in ("q", "k", "v", "alpha", "sigma", "r"):
        setattr(sub, nm, getattr(w, nm)[idx])
    sub.cu_seqlens = np.concatenate([[0], np.cumsum(cu[1:])]).astype(np.int64)
    sub.H, sub.mu = w.H, w.mu
    for _ in range(args.warmup):
        oracle.diag_chains(sub, chains[:1], threads=1)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.diag_chains(sub, chains, threads=cores)
    dt = time.perf_counter() - t0
    tok = sum(int(sub.cu_seqlens[s + 1] - sub.cu_seqlens[s]) for s, _ in chains) / w.H * args.steps
    value = tok / dt
    line = {"impl": "reference", "metric": "KDN prefill tokens/s + decode steps/s on 1 B200; % of HBM/tensor roofline",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": w.name, "B": w.B, "T": w.ntok // (w.B or 1), "H": w.H, "d_k": w.dk, "d_v": w.dv,
                       "chunk": w.chunk},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(cores, len(chains)), "kind": "oracle",
                             "sample": f"per step: {len(chains)} (sequence, head) chains x first {max_tok} tokens"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=["prefill", "long", "varlen"])
    ap.add_argument("--clock-seconds", type=float, default=2.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-scan", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the long-context and packed-varlen prefill lines")
    ap.add_argument("--decode-steps", type=int, default=1024)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
