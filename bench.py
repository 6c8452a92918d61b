#!/usr/bin/env python
"""Benchmark of the Taylor-series attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one causal prefill of the main workload (B=1, H=8, N=4096,
d_k=16, d_v=64, n=3, tau=2, bf16 q/k/v, fp32 out and state) through the C ABI,
inputs resident in HBM; the L2 is flushed (a 2 x L2 write) before every timed
step.  The same JSON line carries the decode step (B=64, H=16 states of
65,536-token prefixes; one token per head per step, timed back to back over
six independent batches of states whose 245 MB exceed the L2, so each step
pays for its own state reads and for the write-back of earlier steps'
updates), the order sweep (n = 1..5 at B=1 H=8 N=8192, normalised and
un-normalised q, k), the large-head prefill, the roofline of each dominant
kernel (device time from CUDA events recorded around each launch), an
end-to-end figure with pinned host buffers, the float64 CPU oracle timed on
the host cores (prefill and decode), and the SM clocks sampled during the run.
After every timed block the library's device error word is read; a bounded
wait that ran out marks the line invalid and the exit status non-zero.

Under torchrun (N > 1) every rank runs an independent replica on its own GPU
(the path has no exchange step); times are maxed over ranks and the value is
the tokens of all ranks over that time.  ``--impl reference`` times the
float64 CPU oracle instead, on rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "causal prefill Mtok/s (n=3,d_k16,d_v64) & decode µs/step; % of roofline"
MAIN = dict(B=1, H=8, N=4096, d_k=16, d_v=64, n=3, tau=2.0)
DECODE = dict(B=64, H=16, d_k=16, d_v=64, n=3, tau=2.0, prefix=65536)
LARGE = dict(B=4, H=16, N=32768, d_k=64, d_v=64, n=3, tau=2.0)
SWEEP = dict(B=1, H=8, N=8192, d_k=16, d_v=64, tau=2.0, orders=(1, 2, 3, 4, 5))
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# decode is timed back to back over this many independent batches of states
# (6 x 40.8 MB > the 126 MB L2)
DECODE_BUFFERS = 6
DECODE_GRAPH_STEPS = 100  # dependent decode steps per CUDA-graph replay
E2E_GROUPS = 2  # head groups of the end-to-end pipeline
LEAD_CYCLES_PER_STEP = 400_000  # spin ahead of device-timed loops: about 0.2 ms of host enqueue time a step


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a
# kernel on its bench workload, from ncu captures of the kernels as committed
# (python -m recurrent_states_b200.profile_cases <case>).  ncu empties the
# caches before the launch, and what a kernel writes stays in L2 until after it
# ends, so these are mostly reads.  To be retaken whenever a kernel changes.
DRAM_BYTES = {
    "tc_fused_prefill_kernel": 6_390_784 + 0,           # main prefill
    "decode_ws_kernel": 40_992_000 + 15_104,            # decode step
    "centred_decode_ws_kernel": 41_000_704 + 22_528,    # centred decode step
    "decode_multi_ws_kernel": 41_591_296 + 98_048,      # 4 tokens per call
    "decode_multi_tc_kernel": 43_977_472 + 243_712,     # 16 tokens per call
    # one eighth of the large head (8 of 64 heads) scaled by 8: traffic grows with the heads
    "tcf_out_kernel": 8 * (184_387_328 + 50_061_568),
}
DECODE_WS_DRAM_BYTES = DRAM_BYTES["decode_ws_kernel"]

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"taylor_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.index)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# ---------------------------------------------------------------- helpers

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def allmax(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def kernel_algorithmic(name: str, w: dict, launches: int):
    """Algorithmic bytes and flops of one launch of a kernel of the path."""
    from recurrent_states_b200 import taylor_attn as TA
    F = TA.taylor_attn_num_features(w["d_k"], w["n"])
    stride = TA.taylor_attn_state_stride(w["d_k"], w["d_v"], w["n"])
    BH = w["B"] * w["H"]
    if name.startswith("decode"):
        state = 2 * F * (w["d_v"] + 1) * 4
        io = (2 * w["d_k"] + w["d_v"]) * 2 + w["d_v"] * 4
        return BH * (state + io), BH * 4 * F * (w["d_v"] + 1)
    # prefill: q, k, v read once (bf16), out written once (fp32), final state written once
    T = BH * w["N"]
    byts = T * ((2 * w["d_k"] + w["d_v"]) * 2 + w["d_v"] * 4) + BH * stride * 4
    return byts, T * 4 * F * (w["d_v"] + 1)


def ridge_bound(byts: float, flops: float, pk: dict) -> str:
    """'tensor' when the arithmetic intensity exceeds the ridge point of the
    measured peaks (bf16 flop/s over HBM byte/s), else 'hbm'."""
    return "tensor" if flops / byts > pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9) else "hbm"


def dominant(kern: dict):
    name, (launches, total) = max(kern.items(), key=lambda kv: kv[1][1])
    return name, launches, total / launches


class DeviceErrors:
    """Reads (and clears) the library's device error word after each timed
    block; any bit set means a bounded wait ran out and that block's outputs
    are incomplete."""

    def __init__(self):
        from recurrent_states_b200 import taylor_attn as TA
        self.TA = TA
        TA.taylor_attn_device_errors(clear=True)
        self.seen = {}

    def check(self, block: str):
        torch.cuda.synchronize()
        flags = self.TA.taylor_attn_device_errors(clear=True)
        if flags:
            self.seen[block] = flags


# ---------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    from recurrent_states_b200 import synth
    from recurrent_states_b200 import taylor_attn as TA

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()
    hbm_peak = pk["hbm_gbs"]
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 << 20) or (126 << 20)
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)
    errs = DeviceErrors()

    def flush_l2():
        # write a buffer of twice the L2 size, then read it back: the L2 ends
        # up holding clean lines of the flush buffer, so the timed step finds
        # none of its data cached and no dirty lines to write back
        flush.zero_()
        flush.sum()

    def ev_pair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def lead(steps):
        # a spin kernel ahead of the timed work, outside every event pair, so
        # that the host has enqueued the steps before the device reaches them:
        # the events then time the device's work, not the host's launch rate
        if hasattr(torch.cuda, "_sleep"):
            torch.cuda._sleep(int(LEAD_CYCLES_PER_STEP * steps))

    def timed(run, steps, flushed=True, kernels=False):
        """Enqueues run(i) for i < steps, each bracketed by events (L2 flushed
        before each when `flushed`); returns the per-step device ms and, with
        `kernels`, the library's per-kernel launch timing of those steps."""
        ev = [ev_pair() for _ in range(steps)]
        TA.taylor_attn_timing_read()
        torch.cuda.synchronize()
        TA.taylor_attn_timing_enable(kernels)
        lead(steps)
        for i in range(steps):
            if flushed:
                flush_l2()
            ev[i][0].record(stream)
            run(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        TA.taylor_attn_timing_enable(False)
        kern = TA.taylor_attn_timing_read()
        return [a.elapsed_time(b) for a, b in ev], (kern if kernels else None)

    def unit_dev(g, shape):
        x = torch.randn(shape, device=dev, generator=g, dtype=torch.float32)
        return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)

    blocks = {"decode", "centred_prefill", "sweep", "large"} if args.blocks == "all" else set(args.blocks.split(","))
    w = MAIN
    B, H, N, d, dv, n, tau = w["B"], w["H"], w["N"], w["d_k"], w["d_v"], w["n"], w["tau"]
    qh, kh, vh = synth.qkv(B, H, N, d, dv, seed=rank, dtype="bf16")
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    stride = TA.taylor_attn_state_stride(d, dv, n)
    out = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    st = torch.empty((B, H, stride), dtype=torch.float32, device=dev)

    def step(i=0):
        TA.taylor_attn_prefill(q, k, v, n, tau, out=out, state_out=st)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.2)
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    # ---- timed prefill: K steps, L2 flushed before each, events around each.
    # Kernels run back to back with programmatic dependent launch; per-kernel
    # events would serialise them, so the kernel split is taken in a second
    # pass of K steps (same inputs, same flushes) with per-launch events on.
    barrier(world)
    tw = time.perf_counter()
    step_ms, _ = timed(step, args.steps)
    t_wall = time.perf_counter() - tw
    barrier(world)
    step_ms_k, kern = timed(step, args.steps, kernels=True)
    errs.check("main_prefill")
    ms = statistics.mean(step_ms)
    ms_max = allmax(ms, world, dev)
    tokens = B * N
    value = world * tokens / (ms_max * 1e-3) / 1e6

    launches = sum(c for c, _ in kern.values())
    dom_name, _, per_launch_ms = dominant(kern)
    byts, flops = kernel_algorithmic("prefill", w, 1)
    achieved = byts / (per_launch_ms * 1e-3) / 1e9

    # ---- end to end through the public call with pinned host buffers: the
    # heads in E2E_GROUPS groups, each copied in, prefilled and copied out on
    # one of two streams, so that one group's copies overlap another group's
    # compute and the copies in the other direction (PCIe is full duplex)
    qp, kp, vp = qh.pin_memory(), kh.pin_memory(), vh.pin_memory()
    outp = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    stp = torch.empty(st.shape, dtype=torch.float32).pin_memory()
    BHn = B * H
    n_groups = E2E_GROUPS if BHn % E2E_GROUPS == 0 else 1
    gh = BHn // n_groups
    flat = lambda t: t.view(BHn, *t.shape[2:])  # noqa: E731
    host = [flat(t) for t in (qp, kp, vp, outp, stp)]
    devt = [flat(t) for t in (q, k, v, out, st)]
    side = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    e2e_ev = [ev_pair() for _ in range(args.steps)]
    for i in range(args.steps + args.warmup):
        if i >= args.warmup:
            flush_l2()
            e2e_ev[i - args.warmup][0].record(stream)
        for s_ in side:
            s_.wait_stream(stream)
        for gi in range(n_groups):
            sl = slice(gi * gh, (gi + 1) * gh)
            with torch.cuda.stream(side[gi % 2]):
                for dt, ht in zip(devt[:3], host[:3]):
                    dt[sl].copy_(ht[sl], non_blocking=True)
                gq, gk, gv = (t[sl].view(1, gh, *t.shape[1:]) for t in devt[:3])
                TA.taylor_attn_prefill(gq, gk, gv, n, tau, out=devt[3][sl].view(1, gh, N, dv),
                                       state_out=devt[4][sl].view(1, gh, stride))
                host[3][sl].copy_(devt[3][sl], non_blocking=True)
                host[4][sl].copy_(devt[4][sl], non_blocking=True)
        for s_ in side:
            stream.wait_stream(s_)
        if i >= args.warmup:
            e2e_ev[i - args.warmup][1].record(stream)
    torch.cuda.synchronize()
    errs.check("e2e")
    e2e_ms = allmax(statistics.mean(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = out.numel() * 4 + st.numel() * 4

    g = torch.Generator(device=dev)  # device-side inputs of the later blocks
    g.manual_seed(rank)
    if "decode" in blocks:
        # ---- decode: states of 65,536-token random prefixes built by the library
        dw = DECODE
        dB, dH = dw["B"], dw["H"]
        dstride = TA.taylor_attn_state_stride(dw["d_k"], dw["d_v"], dw["n"])
        dstate = torch.zeros((dB, dH, dstride), dtype=torch.float32, device=dev)
        seg = 4096
        tmp_state = torch.empty_like(dstate)
        for s0 in range(0, dw["prefix"], seg):
            pq_ = unit_dev(g, (dB, dH, seg, dw["d_k"]))
            pk_ = unit_dev(g, (dB, dH, seg, dw["d_k"]))
            pv_ = torch.randn((dB, dH, seg, dw["d_v"]), device=dev, generator=g).to(torch.bfloat16)
            po = torch.empty((dB, dH, seg, dw["d_v"]), dtype=torch.float32, device=dev)
            TA.taylor_attn_prefill(pq_, pk_, pv_, dw["n"], dw["tau"], out=po, state_out=tmp_state)
            TA.taylor_attn_state_merge(dstate, tmp_state, dw["d_k"], dw["d_v"], dw["n"], out=dstate)
            del pq_, pk_, pv_, po
        del tmp_state
        errs.check("decode_prefix")
        dsteps = max(args.steps, 24)
        toks = [synth.decode_tokens(dB, dH, dw["d_k"], dw["d_v"], s, seed=rank) for s in range(dsteps)]
        toks = [(a.to(dev), b.to(dev), c.to(dev)) for a, b, c in toks]
        dout = torch.empty((dB, dH, dw["d_v"]), dtype=torch.float32, device=dev)
        # six independent batches of 1,024 carried states (245 MB > L2): step s
        # updates batch s % 6, so its states were last touched six steps earlier
        dstates = [dstate] + [dstate.clone() for _ in range(DECODE_BUFFERS - 1)]

        def dec(i):
            TA.taylor_attn_decode(*toks[i], dstates[i % DECODE_BUFFERS], dw["n"], dw["tau"], out=dout)

        for s in range(max(args.warmup, 3) + DECODE_BUFFERS):
            dec(s % dsteps)
        torch.cuda.synchronize()
        # steady state: back to back, one pair of events around the whole run
        # (its device time over the steps), then per-launch events in a second run
        e0, e1 = ev_pair()
        lead(dsteps)
        e0.record(stream)
        for s in range(dsteps):
            dec(s)
        e1.record(stream)
        torch.cuda.synchronize()
        dec_us = e0.elapsed_time(e1) * 1e3 / dsteps
        _, dkern = timed(dec, dsteps, flushed=False, kernels=True)
        dk_name, _, dk_ms = dominant(dkern)
        dec_kernel_us = dk_ms * 1e3
        # one step after an L2 flush (cold reads, write-back after the kernel), context
        dflush_ms, _ = timed(dec, dsteps, flushed=True)
        # warm L2: the same batch of states step after step (it fits in L2), context
        lead(dsteps)
        e0.record(stream)
        for s in range(dsteps):
            TA.taylor_attn_decode(*toks[s], dstate, dw["n"], dw["tau"], out=dout)
        e1.record(stream)
        torch.cuda.synchronize()
        dec_warm_us = e0.elapsed_time(e1) * 1e3 / dsteps
        # 100 dependent steps over the six batches captured in one CUDA graph
        # and replayed (no host work between launches), total / 100
        dec_graph_us = None
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for s in range(DECODE_GRAPH_STEPS):
                    dec(s % dsteps)
            graph.replay()
            torch.cuda.synchronize()
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            dec_graph_us = e0.elapsed_time(e1) * 1e3 / DECODE_GRAPH_STEPS
            del graph
        except RuntimeError as ex:  # capture refused: report the reason, keep the rest of the line
            dec_graph_us = f"unavailable: {str(ex).splitlines()[0][:120]}"
        errs.check("decode")
        dec_us_max = allmax(dec_us, world, dev)
        dbytes, dflops = kernel_algorithmic("decode", dw, 1)

        # ---- the mean-centred softmax expansion (order 2) on the same carried
        # states: same state traffic, a three-way read-out; timed like decode
        def cen(i):
            TA.taylor_attn_centred_decode(*toks[i], dstates[i % DECODE_BUFFERS], 2, dw["tau"], out=dout)

        for s in range(DECODE_BUFFERS + 3):
            cen(s)
        torch.cuda.synchronize()
        lead(dsteps)
        e0.record(stream)
        for s in range(dsteps):
            cen(s)
        e1.record(stream)
        torch.cuda.synchronize()
        cen_us = e0.elapsed_time(e1) * 1e3 / dsteps
        _, ckern = timed(cen, dsteps, flushed=False, kernels=True)
        ck_name, _, ck_ms = dominant(ckern)
        cen_kernel_us = ck_ms * 1e3
        errs.check("centred_decode")

    if "centred_prefill" in blocks:
        # ---- the mean-centred expansion's prefill (order 2) on the main workload's inputs
        cout = torch.empty_like(out)
        cst = torch.empty_like(st)

        def cstep(i=0):
            TA.taylor_attn_centred_prefill(q, k, v, 2, tau, out=cout, state_out=cst)

        for _ in range(3):
            flush_l2()
            cstep()
        cp_ms, _ = timed(cstep, 10)
        _, cpkern = timed(cstep, 5, kernels=True)
        errs.check("centred_prefill")
        cp_med = statistics.median(cp_ms)
        cp_name, _, cp_dom_ms = dominant(cpkern)
        del cout, cst

    if "decode" in blocks:
        # ---- batched multi-token decode: T new tokens per head per call, in place
        multi = {}
        for T in (4, 16):
            mtoks = [(unit_dev(g, (dB, dH, T, dw["d_k"])), unit_dev(g, (dB, dH, T, dw["d_k"])),
                      torch.randn((dB, dH, T, dw["d_v"]), device=dev, generator=g).to(torch.bfloat16))
                     for _ in range(dsteps)]
            mout = torch.empty((dB, dH, T, dw["d_v"]), dtype=torch.float32, device=dev)

            def mdec(i):
                sb = dstates[i % DECODE_BUFFERS]
                TA.taylor_attn_prefill_from_state(*mtoks[i], sb, dw["n"], dw["tau"], out=mout, state_out=sb)

            for s_ in range(DECODE_BUFFERS + 3):
                mdec(s_)
            torch.cuda.synchronize()
            lead(dsteps)
            e0.record(stream)
            for s_ in range(dsteps):
                mdec(s_)
            e1.record(stream)
            torch.cuda.synchronize()
            m_us = e0.elapsed_time(e1) * 1e3 / dsteps
            _, mk = timed(mdec, dsteps, flushed=False, kernels=True)
            mk_name, _, mk_ms = dominant(mk)
            mk_us = mk_ms * 1e3
            Fd = TA.taylor_attn_num_features(dw["d_k"], dw["n"])
            m_bytes = dB * dH * (2 * Fd * (dw["d_v"] + 1) * 4 + T * ((2 * dw["d_k"] + dw["d_v"]) * 2 + dw["d_v"] * 4))
            multi[str(T)] = {"us_per_call": round(m_us, 3), "kernel": mk_name, "kernel_us": round(mk_us, 3),
                             "Mtok_s": round(dB * dH * T / (m_us * 1e-6) / 1e6, 2),
                             "hbm_frac": round(m_bytes / (mk_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_launch": m_bytes, "traffic": DRAM_BYTES.get(mk_name)}
            del mtoks, mout
        errs.check("multi_token_decode")
        del dstates

    if "sweep" in blocks:
        # ---- order sweep: n = 1..5 at B1 H8 N8192 d_k16 d_v64, q, k unit-normalised
        # and (second arm) q, k ~ N(0, 4) as drawn
        sw = SWEEP
        sweep = {}
        for arm, normalised in (("normalised", True), ("unnormalised_var4", False)):
            sq, sk, sv = synth.qkv(sw["B"], sw["H"], sw["N"], sw["d_k"], sw["d_v"], seed=rank, dtype="bf16",
                                   normalise=normalised, qk_var=1.0 if normalised else 4.0)
            sq, sk, sv = sq.to(dev), sk.to(dev), sv.to(dev)
            sout = torch.empty((sw["B"], sw["H"], sw["N"], sw["d_v"]), dtype=torch.float32, device=dev)
            res = {}
            for sn in sw["orders"]:
                sst = torch.empty((sw["B"], sw["H"], TA.taylor_attn_state_stride(sw["d_k"], sw["d_v"], sn)),
                                  dtype=torch.float32, device=dev)

                def sstep(i, sn=sn, sst=sst):
                    TA.taylor_attn_prefill(sq, sk, sv, sn, sw["tau"], out=sout, state_out=sst)

                for _ in range(3):
                    sstep(0)
                s_ms, _ = timed(sstep, 10)
                _, skern = timed(sstep, 5, kernels=True)
                s_med = statistics.median(s_ms)
                sbytes, sflops = kernel_algorithmic("prefill", dict(sw, n=sn), 1)
                bound = ridge_bound(sbytes, sflops, pk)
                entry = {"F": TA.taylor_attn_num_features(sw["d_k"], sn), "ms_per_step": round(s_med, 5),
                         "Mtok_s": round(sw["B"] * sw["N"] / (s_med * 1e-3) / 1e6, 3),
                         "algorithmic_bytes": sbytes, "algorithmic_flops": sflops,
                         "kernels_ms": {k_: round(t / c, 5) for k_, (c, t) in skern.items()}}
                if bound == "hbm":
                    a = sbytes / (s_med * 1e-3) / 1e9
                    entry["roofline"] = {"bound": "hbm", "scope": "whole step", "achieved": round(a, 2),
                                         "peak": hbm_peak, "unit": "GB/s", "frac": round(a / hbm_peak, 4)}
                else:
                    a = sflops / (s_med * 1e-3) / 1e12
                    entry["roofline"] = {"bound": "tensor", "scope": "whole step", "achieved": round(a, 3),
                                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                                         "frac": round(a / pk["bf16_tflops"], 4)}
                res[str(sn)] = entry
                del sst
            sweep[arm] = res
            del sq, sk, sv, sout
        errs.check("order_sweep")

    if "large" in blocks:
        # ---- large-head prefill (F = 2,145): the contraction-bound configuration
        lw = LARGE
        lB, lH, lN, ld, ldv, ln = lw["B"], lw["H"], lw["N"], lw["d_k"], lw["d_v"], lw["n"]
        lF = TA.taylor_attn_num_features(ld, ln)
        lq, lk = unit_dev(g, (lB, lH, lN, ld)), unit_dev(g, (lB, lH, lN, ld))
        lv = torch.randn((lB, lH, lN, ldv), device=dev, generator=g).to(torch.bfloat16)
        lout = torch.empty((lB, lH, lN, ldv), dtype=torch.float32, device=dev)
        lst = torch.empty((lB, lH, TA.taylor_attn_state_stride(ld, ldv, ln)), dtype=torch.float32, device=dev)

        def lstep(i=0):
            TA.taylor_attn_prefill(lq, lk, lv, ln, lw["tau"], out=lout, state_out=lst)

        for _ in range(3):
            lstep()
        torch.cuda.synchronize()
        l_steps_ms, _ = timed(lstep, 10)
        l_ms = statistics.median(l_steps_ms)
        _, lkern = timed(lstep, 5, kernels=True)
        errs.check("large_head_prefill")
        l_tokens = lB * lH * lN
        l_alg = l_tokens * 4 * lF * (ldv + 1)                      # state update + read-out, 2 F Dv each
        lk_name, _, lk_ms = dominant(lkern)
        # the dominant kernel's algorithmic work: the read-out contraction of every
        # query past the first group, 2 F Dv per head-token
        l_dom_alg = l_tokens * 2 * lF * (ldv + 1)
        del lq, lk, lv, lout, lst

    clk = clocks.stop()

    cpu = cpu_dec = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_leg(target_s=args.cpu_seconds)
        if "decode" in blocks:
            cpu_dec = cpu_oracle_decode_leg(target_s=min(args.cpu_seconds, 8.0))

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "Mtok/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_max, 5),
            "ms_per_step_median": round(statistics.median(step_ms), 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32" if dom_name.startswith("cc_") else "bf16",
            "data": "synthetic (seeded normal q,k unit-normalised, v normal; bf16)",
            "config": {
                "workload": "main_prefill: causal prefill B=1 H=8 N=4096 d_k=16 d_v=64 n=3 (F=153) tau=2, "
                            "bf16 q/k/v, fp32 out+state; tokens = B*N per step",
                "B": B, "H": H, "N": N, "d_k": d, "d_v": dv, "n": n, "tau": tau,
                "parallelism": f"replicas{world}",
                "l2": "flushed before each timed step: write of a 2x L2 buffer, then a read of it (clean cold L2)",
            },
            "roofline": {
                "bound": "hbm", "kernel": dom_name,
                "achieved": round(achieved, 2), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "peak_source": pk["_source"] + " (hbm_gbs, burst copy)",
                "traffic": DRAM_BYTES.get(dom_name),
                "algorithmic_bytes_per_launch": byts,
                "kernel_us_per_launch": round(per_launch_ms * 1e3, 3),
                "timing": "CUDA events around each launch of the kernel, second pass of K steps",
                "step_frac": round(byts / (ms * 1e-3) / 1e9 / hbm_peak, 4),
                "tensor_tflops": round(flops / (per_launch_ms * 1e-3) / 1e12, 3),
                "tensor_frac_of_bf16_peak": round(flops / (per_launch_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 5),
            },
            "kernels": {k_: {"launches": c, "total_ms": round(t, 4)} for k_, (c, t) in kern.items()},
            "ms_per_step_with_kernel_events": round(statistics.mean(step_ms_k), 5),
            "e2e": {"value": round(world * tokens / (e2e_ms * 1e-3) / 1e6, 3), "unit": "Mtok/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4),
                    "pipeline": f"{n_groups} head groups of {gh} on 2 streams: pinned host -> device copies, "
                                "taylor_attn_prefill, device -> pinned host copies of outputs and state"},
            "gpu_launches": launches,
            "clocks": clk,
            "wall_s_timed_region": round(t_wall, 4),
        }
        if "decode" in blocks:
            line["decode"] = {
                "workload": "decode: B=64 H=16 d_k=16 d_v=64 n=3, states of 65,536-token random prefixes, "
                            "one token per head per step; steps back to back over 6 independent batches of "
                            "states (6 x 40.8 MB > L2), so each step reads its states from HBM and the "
                            "write-back of earlier steps' updated states falls inside the timed region",
                "us_per_step": round(dec_us_max, 3),
                "kernel_us": round(dec_kernel_us, 3),
                "us_per_step_l2_flushed": round(statistics.mean(dflush_ms) * 1e3, 3),
                "us_per_step_warm_l2": round(dec_warm_us, 3),
                "us_per_step_cuda_graph": round(dec_graph_us, 3) if isinstance(dec_graph_us, float) else dec_graph_us,
                "cuda_graph_steps": DECODE_GRAPH_STEPS,
                "roofline": {"bound": "hbm", "kernel": dk_name,
                             "achieved": round(dbytes / (dec_kernel_us * 1e-6) / 1e9, 2),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(dbytes / (dec_kernel_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "step_frac": round(dbytes / (dec_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_launch": dbytes,
                             "traffic": DECODE_WS_DRAM_BYTES if dk_name == "decode_ws_kernel" else None,
                             "traffic_note": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of "
                                             "this kernel on this workload: ncu empties the caches first and the "
                                             "updated states are written back after the launch, so it holds the "
                                             "state reads only; in the back-to-back timing above each launch "
                                             "also carries earlier launches' write-backs"},
            }
        if "decode" in blocks:
            line["centred_decode"] = {
                "workload": "mean-centred softmax expansion, order 2, one token per head per step on the decode "
                            "workload's carried n=3 states (B=64 H=16 d_k=16 d_v=64), timed like decode",
                "kernel": ck_name,
                "us_per_step": round(cen_us, 3),
                "kernel_us": round(cen_kernel_us, 3),
                "roofline": {"bound": "hbm", "kernel": ck_name,
                             "achieved": round(dbytes / (cen_kernel_us * 1e-6) / 1e9, 2),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(dbytes / (cen_kernel_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_launch": dbytes, "traffic": DRAM_BYTES.get(ck_name)},
            }
        if "centred_prefill" in blocks:
            line["centred_prefill"] = {
                "workload": "mean-centred softmax expansion, order 2, causal prefill of the main workload's inputs "
                            "(B=1 H=8 N=4096 d_k=16 d_v=64, bf16 in, fp32 out + n=3 state), L2 flushed before each "
                            "step, median of 10 steps",
                "ms_per_step": round(cp_med, 5),
                "Mtok_s": round(tokens / (cp_med * 1e-3) / 1e6, 3),
                "kernels_ms": {k_: round(t / c, 5) for k_, (c, t) in cpkern.items()},
                "roofline": {"bound": "hbm", "scope": "whole step", "achieved": round(byts / (cp_med * 1e-3) / 1e9, 2),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(byts / (cp_med * 1e-3) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_step": byts,
                             "note": "same inputs, outputs and state as the main prefill; chunk states, scan "
                                     "and an output kernel with three per-degree TMEM accumulators (tcgen05), "
                                     "three launches"},
            }
        if "decode" in blocks:
            line["multi_token_decode"] = {
                "workload": "B=64 H=16 d_k=16 d_v=64 n=3, T new tokens per head per call against the carried "
                            "states (taylor_attn_prefill_from_state in place), timed like decode",
                "by_tokens_per_call": multi,
            }
        if "sweep" in blocks:
            line["order_sweep"] = {
                "workload": "causal prefill B=1 H=8 N=8192 d_k=16 d_v=64 tau=2, n = 1..5 (F = 1, 17, 153, 969, "
                            "4845), bf16 q/k/v, fp32 out+state, L2 flushed before each step, median of 10 "
                            "steps; q, k unit-normalised, and q, k ~ N(0, 4) as drawn",
                "bound_rule": "tensor when algorithmic flops / bytes exceeds the measured peaks' ridge point",
                "by_arm_and_order": sweep,
            }
        if "large" in blocks:
            line["large_head_prefill"] = {
                "workload": "causal prefill B=4 H=16 N=32768 d_k=64 d_v=64 n=3 (F=2145) tau=2, bf16 q/k/v, "
                            "fp32 out+state, L2 flushed before each step, median of 10 steps",
                "ms_per_step": round(l_ms, 4),
                "ms_per_step_mean": round(statistics.mean(l_steps_ms), 4),
                "Mtok_s": round(lB * lN / (l_ms * 1e-3) / 1e6, 3),
                "algorithmic_tflops": round(l_alg / (l_ms * 1e-3) / 1e12, 3),
                "frac_of_bf16_peak": round(l_alg / (l_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                "kernels": {k_: {"launches": c, "total_ms": round(t, 4)} for k_, (c, t) in lkern.items()},
                "roofline": {"bound": "tensor", "kernel": lk_name,
                             "achieved": round(l_dom_alg / (lk_ms * 1e-3) / 1e12, 3),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(l_dom_alg / (lk_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                             "algorithmic_flops_per_launch": l_dom_alg, "traffic": DRAM_BYTES.get(lk_name),
                             "traffic_note": "one eighth of the workload captured, scaled by heads",
                             "note": "read-out contraction 2 F Dv per head-token; hi/lo bf16 operands execute "
                                     "3x these MMA flops, padded to 80 columns"},
            }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if cpu_dec is not None and "decode" in blocks:
            line["decode"]["cpu_baseline"] = cpu_dec
        if errs.seen:
            line["device_errors"] = errs.seen
            line["valid"] = False
        print(json.dumps(line), flush=True)
    if errs.seen:
        raise SystemExit(3)


# ---------------------------------------------------------------- CPU oracle legs

def _oracle_threads(units: int) -> int:
    """Threads the oracle actually runs on: its OpenMP loop is over heads."""
    from oracle import c_oracle as C
    return max(1, min(units, C.default_threads()))


def cpu_oracle_leg(target_s: float = 12.0, reps_max: int = 50, threads: int = 0):
    """The float64 C oracle (recurrent form, OpenMP over heads) on the main
    workload, repeated until about target_s seconds of CPU work."""
    from oracle import c_oracle as C
    from recurrent_states_b200 import synth

    w = MAIN
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    cores = threads or _oracle_threads(w["B"] * w["H"])
    reps, t0 = 0, time.perf_counter()
    while True:
        C.recurrent(qd, kd, vd, w["n"], w["tau"], threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= reps_max:
            break
    tokens = reps * w["B"] * w["N"]
    return {"value": round(tokens / el / 1e6, 6), "unit": "Mtok/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} full passes of main_prefill (B1 H8 N4096, all 8 heads), float64 recurrent form, "
                      f"OpenMP over heads on {cores} thread(s), {el:.1f} s"}


def cpu_oracle_decode_leg(target_s: float = 8.0, reps_max: int = 200):
    """The float64 C oracle's decode step (one token per head from a carried
    state: rank-one update, read-out, division) over the decode workload's
    1,024 heads, OpenMP over heads, repeated until about target_s seconds."""
    from oracle import c_oracle as C
    from recurrent_states_b200 import synth

    w = DECODE
    BH = w["B"] * w["H"]
    cores = _oracle_threads(BH)
    # carried states of short random prefixes: the step's cost is the state's
    # size, not the length of the prefix that built it
    pq, pk_, pv = synth.qkv(1, BH, 64, w["d_k"], w["d_v"], seed=0, dtype="bf16")
    S = C.state(pk_.double().numpy()[0], pv.double().numpy()[0], w["n"], threads=cores)
    toks = [synth.decode_tokens(1, BH, w["d_k"], w["d_v"], s) for s in range(4)]
    toks = [tuple(t.double().numpy()[0][:, None, :] for t in tk) for tk in toks]
    reps, t0 = 0, time.perf_counter()
    while True:
        qs, ks, vs = toks[reps % len(toks)]
        _, S = C.recurrent(qs, ks, vs, w["n"], w["tau"], state_in=S, threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= reps_max:
            break
    return {"value": round(el / reps * 1e6, 1), "unit": "us/step", "cores": cores, "kind": "oracle",
            "sample": f"{reps} decode steps of all 1,024 heads (B64 H16 d_k16 d_v64 n3), float64, OpenMP over "
                      f"heads on {cores} thread(s), {el:.1f} s; states from 64-token random prefixes"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    from oracle import c_oracle as C
    from recurrent_states_b200 import synth

    w = MAIN
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    cores = _oracle_threads(w["B"] * w["H"])

    # one step = one full prefill of the workload (all heads), float64
    # recurrent form, OpenMP over the heads
    def step():
        C.recurrent(qd, kd, vd, w["n"], w["tau"], threads=cores)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    val = args.steps * w["B"] * w["N"] / el / 1e6
    # the same oracle on one thread, one head per step (the pages time a
    # single-threaded CPU implementation)
    h_steps = max(2, args.steps)
    t1 = time.perf_counter()
    for i in range(h_steps):
        h = i % w["H"]
        C.recurrent(qd[:, h:h + 1], kd[:, h:h + 1], vd[:, h:h + 1], w["n"], w["tau"], threads=1)
    el1 = time.perf_counter() - t1
    val1 = h_steps * w["B"] * w["N"] / w["H"] / el1 / 1e6
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(val, 6), "unit": "Mtok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded normal q,k unit-normalised, v normal; bf16 values in float64)",
        "config": {"workload": "main_prefill: causal prefill B=1 H=8 N=4096 d_k=16 d_v=64 n=3 (F=153) tau=2; "
                               "each step is one full prefill (all 8 heads) on the host cores",
                   "B": w["B"], "H": w["H"], "N": w["N"], "d_k": w["d_k"], "d_v": w["d_v"], "n": w["n"],
                   "tau": w["tau"], "parallelism": f"host, OpenMP over the 8 heads on {cores} thread(s)"},
        "cpu_baseline": {"value": round(val, 6), "unit": "Mtok/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} full prefills (8 heads x 4096 tokens), float64 recurrent form"},
        "cpu_single_thread": {"value": round(val1, 6), "unit": "Mtok/s", "cores": 1, "kind": "oracle",
                              "sample": f"{h_steps} single heads x 4096 tokens on one thread; Mtok/s of the "
                                        "8-head workload at that rate"},
        "e2e": {"value": round(val, 6), "unit": "Mtok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--blocks", default="all",
                    help="all (default), or a comma list of decode, centred_prefill, sweep, large: the main "
                         "prefill (with its end-to-end figure) always runs; a shorter list serves profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
