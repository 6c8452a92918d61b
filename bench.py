#!/usr/bin/env python
"""Benchmark of the Taylor-series attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one causal prefill of the main workload (B=1, H=8, N=4096,
d_k=16, d_v=64, n=3, tau=2, bf16 q/k/v, fp32 out and state) through the C ABI,
inputs resident in HBM; the L2 is flushed (a 2 x L2 write) before every timed
step.  The same JSON line carries the decode step (B=64, H=16 states of
65,536-token prefixes; one token per head per step), the roofline of the
dominant kernel (device time from CUDA events recorded around each launch),
an end-to-end figure with pinned host buffers, the float64 CPU oracle timed on
the host cores, and the SM clocks sampled during the run.

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
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes of one decode_ws_kernel launch on the decode workload, from an ncu
# capture (read 40,991,488 + write 38,400); to be retaken whenever the kernel changes.
DECODE_WS_DRAM_BYTES = 41_029_888

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


# ---------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    from recurrent_states_b200 import synth
    from recurrent_states_b200 import taylor_attn as TA

    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    pk = peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 << 20) or (126 << 20)
    flush = torch.empty(2 * l2 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer of twice the L2 size, then read it back: the L2 ends
        # up holding clean lines of the flush buffer, so the timed step finds
        # none of its data cached and no dirty lines to write back
        flush.zero_()
        flush.sum()

    w = MAIN
    B, H, N, d, dv, n, tau = w["B"], w["H"], w["N"], w["d_k"], w["d_v"], w["n"], w["tau"]
    qh, kh, vh = synth.qkv(B, H, N, d, dv, seed=rank, dtype="bf16")
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    stride = TA.taylor_attn_state_stride(d, dv, n)
    out = torch.empty((B, H, N, dv), dtype=torch.float32, device=dev)
    st = torch.empty((B, H, stride), dtype=torch.float32, device=dev)

    def step():
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
    def timed_pass(kernel_events: bool):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        TA.taylor_attn_timing_read()
        barrier(world)
        torch.cuda.synchronize()
        TA.taylor_attn_timing_enable(kernel_events)
        tw = time.perf_counter()
        for i in range(args.steps):
            flush_l2()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        tw = time.perf_counter() - tw
        TA.taylor_attn_timing_enable(False)
        barrier(world)
        return statistics.mean(a.elapsed_time(b) for a, b in ev), tw, TA.taylor_attn_timing_read()

    ms, t_wall, _ = timed_pass(False)
    ms_k, _, kern = timed_pass(True)
    ms_max = allmax(ms, world, dev)
    tokens = B * N
    value = world * tokens / (ms_max * 1e-3) / 1e6

    launches = sum(c for c, _ in kern.values())
    dom_name, (dom_launch, dom_ms) = max(kern.items(), key=lambda kv: kv[1][1])
    per_launch_ms = dom_ms / dom_launch
    byts, flops = kernel_algorithmic("prefill", w, 1)
    hbm_peak = pk["hbm_gbs"]
    achieved = byts / (per_launch_ms * 1e-3) / 1e9

    # ---- decode: states of 65,536-token random prefixes built by the library
    dw = DECODE
    dB, dH = dw["B"], dw["H"]
    dstride = TA.taylor_attn_state_stride(dw["d_k"], dw["d_v"], dw["n"])
    dstate = torch.zeros((dB, dH, dstride), dtype=torch.float32, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(rank)
    seg = 4096
    tmp_state = torch.empty_like(dstate)
    for s0 in range(0, dw["prefix"], seg):
        def unit(shape):
            x = torch.randn(shape, device=dev, generator=g, dtype=torch.float32)
            return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        pq_ = unit((dB, dH, seg, dw["d_k"]))
        pk_ = unit((dB, dH, seg, dw["d_k"]))
        pv_ = torch.randn((dB, dH, seg, dw["d_v"]), device=dev, generator=g).to(torch.bfloat16)
        po = torch.empty((dB, dH, seg, dw["d_v"]), dtype=torch.float32, device=dev)
        TA.taylor_attn_prefill(pq_, pk_, pv_, dw["n"], dw["tau"], out=po, state_out=tmp_state)
        TA.taylor_attn_state_merge(dstate, tmp_state, dw["d_k"], dw["d_v"], dw["n"], out=dstate)
        del pq_, pk_, pv_, po
    dsteps = max(args.steps, 20)
    toks = [synth.decode_tokens(dB, dH, dw["d_k"], dw["d_v"], s, seed=rank) for s in range(dsteps)]
    toks = [(a.to(dev), b.to(dev), c.to(dev)) for a, b, c in toks]
    dout = torch.empty((dB, dH, dw["d_v"]), dtype=torch.float32, device=dev)
    for s in range(max(args.warmup, 3)):
        flush_l2()
        TA.taylor_attn_decode(*toks[s], dstate, dw["n"], dw["tau"], out=dout)
    torch.cuda.synchronize()
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(dsteps)]
    TA.taylor_attn_timing_read()
    TA.taylor_attn_timing_enable(True)
    for s in range(dsteps):
        flush_l2()
        dev_ev[s][0].record(stream)
        TA.taylor_attn_decode(*toks[s], dstate, dw["n"], dw["tau"], out=dout)
        dev_ev[s][1].record(stream)
    torch.cuda.synchronize()
    TA.taylor_attn_timing_enable(False)
    dkern = TA.taylor_attn_timing_read()
    dec_us = statistics.mean(a.elapsed_time(b) for a, b in dev_ev) * 1e3
    dk_name, (dk_launch, dk_ms) = max(dkern.items(), key=lambda kv: kv[1][1])
    dbytes, dflops = kernel_algorithmic("decode", dw, 1)
    dec_kernel_us = dk_ms / dk_launch * 1e3
    # warm-L2 decode (no flush), for context
    warm_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    warm_ev[0].record(stream)
    for s in range(dsteps):
        TA.taylor_attn_decode(*toks[s], dstate, dw["n"], dw["tau"], out=dout)
    warm_ev[1].record(stream)
    torch.cuda.synchronize()
    dec_warm_us = warm_ev[0].elapsed_time(warm_ev[1]) * 1e3 / dsteps
    dec_us_max = allmax(dec_us, world, dev)

    # ---- the mean-centred softmax expansion (order 2) on the same carried
    # states: same state traffic, a three-way read-out
    for s in range(3):
        flush_l2()
        TA.taylor_attn_centred_decode(*toks[s], dstate, 2, dw["tau"], out=dout)
    torch.cuda.synchronize()
    TA.taylor_attn_timing_read()
    TA.taylor_attn_timing_enable(True)
    for s in range(dsteps):
        flush_l2()
        TA.taylor_attn_centred_decode(*toks[s], dstate, 2, dw["tau"], out=dout)
    torch.cuda.synchronize()
    TA.taylor_attn_timing_enable(False)
    ckern = TA.taylor_attn_timing_read()
    ck_name, (ck_launch, ck_ms) = max(ckern.items(), key=lambda kv: kv[1][1])
    cen_kernel_us = ck_ms / ck_launch * 1e3

    # ---- batched multi-token decode: T new tokens per head per call, in place
    multi = {}
    for T in (4, 16):
        def unit_t(shape):
            x = torch.randn(shape, device=dev, generator=g, dtype=torch.float32)
            return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        mtoks = [(unit_t((dB, dH, T, dw["d_k"])), unit_t((dB, dH, T, dw["d_k"])),
                  torch.randn((dB, dH, T, dw["d_v"]), device=dev, generator=g).to(torch.bfloat16))
                 for _ in range(dsteps)]
        mout = torch.empty((dB, dH, T, dw["d_v"]), dtype=torch.float32, device=dev)
        for s_ in range(3):
            flush_l2()
            TA.taylor_attn_prefill_from_state(*mtoks[s_], dstate, dw["n"], dw["tau"], out=mout, state_out=dstate)
        torch.cuda.synchronize()
        TA.taylor_attn_timing_read()
        TA.taylor_attn_timing_enable(True)
        m_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(dsteps)]
        for s_ in range(dsteps):
            flush_l2()
            m_ev[s_][0].record(stream)
            TA.taylor_attn_prefill_from_state(*mtoks[s_], dstate, dw["n"], dw["tau"], out=mout, state_out=dstate)
            m_ev[s_][1].record(stream)
        torch.cuda.synchronize()
        TA.taylor_attn_timing_enable(False)
        mk = TA.taylor_attn_timing_read()
        m_us = statistics.mean(a.elapsed_time(b) for a, b in m_ev) * 1e3
        mk_name, (mk_launch, mk_ms) = max(mk.items(), key=lambda kv: kv[1][1])
        mk_us = mk_ms / mk_launch * 1e3
        Fd = TA.taylor_attn_num_features(dw["d_k"], dw["n"])
        m_bytes = dB * dH * (2 * Fd * (dw["d_v"] + 1) * 4 + T * ((2 * dw["d_k"] + dw["d_v"]) * 2 + dw["d_v"] * 4))
        multi[str(T)] = {"us_per_call": round(m_us, 3), "kernel": mk_name, "kernel_us": round(mk_us, 3),
                         "Mtok_s": round(dB * dH * T / (m_us * 1e-6) / 1e6, 2),
                         "hbm_frac": round(m_bytes / (mk_us * 1e-6) / 1e9 / hbm_peak, 4),
                         "algorithmic_bytes_per_launch": m_bytes}
        del mtoks, mout

    # ---- large-head prefill (F = 2,145): the contraction-bound configuration
    lw = LARGE
    lB, lH, lN, ld, ldv, ln = lw["B"], lw["H"], lw["N"], lw["d_k"], lw["d_v"], lw["n"]
    lF = TA.taylor_attn_num_features(ld, ln)

    def unit_dev(shape):
        x = torch.randn(shape, device=dev, generator=g, dtype=torch.float32)
        return (x / x.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    lq, lk = unit_dev((lB, lH, lN, ld)), unit_dev((lB, lH, lN, ld))
    lv = torch.randn((lB, lH, lN, ldv), device=dev, generator=g).to(torch.bfloat16)
    lout = torch.empty((lB, lH, lN, ldv), dtype=torch.float32, device=dev)
    lst = torch.empty((lB, lH, TA.taylor_attn_state_stride(ld, ldv, ln)), dtype=torch.float32, device=dev)
    lsteps = 3
    for _ in range(2):
        TA.taylor_attn_prefill(lq, lk, lv, ln, lw["tau"], out=lout, state_out=lst)
    torch.cuda.synchronize()
    l_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(lsteps)]
    for s_ in range(lsteps):
        flush_l2()
        l_ev[s_][0].record(stream)
        TA.taylor_attn_prefill(lq, lk, lv, ln, lw["tau"], out=lout, state_out=lst)
        l_ev[s_][1].record(stream)
    torch.cuda.synchronize()
    l_ms = statistics.mean(a.elapsed_time(b) for a, b in l_ev)
    TA.taylor_attn_timing_read()
    TA.taylor_attn_timing_enable(True)
    for s_ in range(lsteps):
        flush_l2()
        TA.taylor_attn_prefill(lq, lk, lv, ln, lw["tau"], out=lout, state_out=lst)
    torch.cuda.synchronize()
    TA.taylor_attn_timing_enable(False)
    lkern = TA.taylor_attn_timing_read()
    l_tokens = lB * lH * lN
    l_alg = l_tokens * 4 * lF * (ldv + 1)                      # state update + read-out, 2 F Dv each
    lk_name, (lk_launch, lk_total) = max(lkern.items(), key=lambda kv: kv[1][1])
    lk_ms = lk_total / lk_launch
    # the dominant kernel's algorithmic work: the read-out contraction of every
    # query past the first group, 2 F Dv per head-token
    l_dom_alg = l_tokens * 2 * lF * (ldv + 1)
    del lq, lk, lv, lout, lst

    # ---- end to end through the public call with pinned host buffers
    qp, kp, vp = qh.pin_memory(), kh.pin_memory(), vh.pin_memory()
    outp = torch.empty(out.shape, dtype=torch.float32).pin_memory()
    stp = torch.empty(st.shape, dtype=torch.float32).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps + args.warmup):
        if i >= args.warmup:
            flush_l2()
            e2e_ev[i - args.warmup][0].record(stream)
        q.copy_(qp, non_blocking=True)
        k.copy_(kp, non_blocking=True)
        v.copy_(vp, non_blocking=True)
        step()
        outp.copy_(out, non_blocking=True)
        stp.copy_(st, non_blocking=True)
        if i >= args.warmup:
            e2e_ev[i - args.warmup][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = allmax(statistics.mean(a.elapsed_time(b) for a, b in e2e_ev), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = out.numel() * 4 + st.numel() * 4

    clk = clocks.stop()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_leg(target_s=args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "Mtok/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_max, 5),
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
                "traffic": None,
                "algorithmic_bytes_per_launch": byts,
                "kernel_us_per_launch": round(per_launch_ms * 1e3, 3),
                "timing": "CUDA events around each launch of the kernel, second pass of K steps",
                "tensor_tflops": round(flops / (per_launch_ms * 1e-3) / 1e12, 3),
                "tensor_frac_of_bf16_peak": round(flops / (per_launch_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 5),
            },
            "kernels": {k_: {"launches": c, "total_ms": round(t, 4)} for k_, (c, t) in kern.items()},
            "ms_per_step_with_kernel_events": round(ms_k, 5),
            "decode": {
                "workload": "decode: B=64 H=16 d_k=16 d_v=64 n=3, states of 65,536-token random prefixes, "
                            "one token per head per step, L2 flushed (write 2x L2, read back) before each step",
                "us_per_step": round(dec_us_max, 3),
                "us_per_step_warm_l2": round(dec_warm_us, 3),
                "kernel_us": round(dec_kernel_us, 3),
                "roofline": {"bound": "hbm", "kernel": dk_name,
                             "achieved": round(dbytes / (dec_kernel_us * 1e-6) / 1e9, 2),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(dbytes / (dec_kernel_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_launch": dbytes,
                             "traffic": DECODE_WS_DRAM_BYTES if dk_name == "decode_ws_kernel" else None,
                             "traffic_note": "dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of "
                                             "this kernel on this workload (cold caches): the states are read "
                                             "once, their updates stay in L2 within the step"},
            },
            "centred_decode": {
                "workload": "mean-centred softmax expansion, order 2, one token per head per step on the decode "
                            "workload's carried n=3 states (B=64 H=16 d_k=16 d_v=64), L2 flushed before each step",
                "kernel": ck_name,
                "kernel_us": round(cen_kernel_us, 3),
                "roofline": {"bound": "hbm", "kernel": ck_name,
                             "achieved": round(dbytes / (cen_kernel_us * 1e-6) / 1e9, 2),
                             "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(dbytes / (cen_kernel_us * 1e-6) / 1e9 / hbm_peak, 4),
                             "algorithmic_bytes_per_launch": dbytes, "traffic": None},
            },
            "multi_token_decode": {
                "workload": "B=64 H=16 d_k=16 d_v=64 n=3, T new tokens per head per call against the carried "
                            "states (taylor_attn_prefill_from_state in place), L2 flushed before each call",
                "by_tokens_per_call": multi,
            },
            "large_head_prefill": {
                "workload": "causal prefill B=4 H=16 N=32768 d_k=64 d_v=64 n=3 (F=2145) tau=2, bf16 q/k/v, "
                            "fp32 out+state, L2 flushed before each step",
                "ms_per_step": round(l_ms, 4),
                "Mtok_s": round(lB * lN / (l_ms * 1e-3) / 1e6, 3),
                "algorithmic_tflops": round(l_alg / (l_ms * 1e-3) / 1e12, 3),
                "frac_of_bf16_peak": round(l_alg / (l_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                "kernels": {k_: {"launches": c, "total_ms": round(t, 4)} for k_, (c, t) in lkern.items()},
                "roofline": {"bound": "tensor", "kernel": lk_name,
                             "achieved": round(l_dom_alg / (lk_ms * 1e-3) / 1e12, 3),
                             "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": round(l_dom_alg / (lk_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                             "algorithmic_flops_per_launch": l_dom_alg, "traffic": None,
                             "note": "read-out contraction 2 F Dv per head-token; hi/lo bf16 operands execute "
                                     "3x these MMA flops, padded to 80 columns"},
            },
            "e2e": {"value": round(world * tokens / (e2e_ms * 1e-3) / 1e6, 3), "unit": "Mtok/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": launches,
            "clocks": clk,
            "wall_s_timed_region": round(t_wall, 4),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- CPU oracle legs

def cpu_oracle_leg(target_s: float = 12.0, reps_max: int = 50):
    """The float64 C oracle (recurrent form, OpenMP over heads, all host cores)
    on the main workload, repeated until about target_s seconds of CPU work."""
    from oracle import c_oracle as C
    from recurrent_states_b200 import synth

    w = MAIN
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    cores = C.default_threads()
    reps, t0 = 0, time.perf_counter()
    while True:
        C.recurrent(qd, kd, vd, w["n"], w["tau"], threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= reps_max:
            break
    tokens = reps * w["B"] * w["N"]
    return {"value": round(tokens / el / 1e6, 6), "unit": "Mtok/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} full passes of main_prefill (B1 H8 N4096), float64 recurrent form, "
                      f"{el:.1f} s"}


def run_reference(args, world, rank):
    if rank != 0:
        return
    from oracle import c_oracle as C
    from recurrent_states_b200 import synth

    w = MAIN
    q, k, v = synth.qkv(w["B"], w["H"], w["N"], w["d_k"], w["d_v"], seed=0, dtype="bf16")
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    cores = C.default_threads()
    # one step = one head of the workload (a bounded sample), float64 recurrent form
    def step(i):
        h = i % w["H"]
        C.recurrent(qd[:, h:h + 1], kd[:, h:h + 1], vd[:, h:h + 1], w["n"], w["tau"], threads=cores)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    # tokens of the whole workload per head-sample: B*N tokens carry H heads
    tokens = args.steps * w["B"] * w["N"] / w["H"]
    val = tokens / el / 1e6
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(val, 6), "unit": "Mtok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded normal q,k unit-normalised, v normal; bf16 values in float64)",
        "config": {"workload": "main_prefill: causal prefill B=1 H=8 N=4096 d_k=16 d_v=64 n=3 (F=153) tau=2; "
                               "each step is one head of it on the host cores",
                   "B": w["B"], "H": w["H"], "N": w["N"], "d_k": w["d_k"], "d_v": w["d_v"], "n": w["n"],
                   "tau": w["tau"], "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": {"value": round(val, 6), "unit": "Mtok/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} steps of one head x 4096 tokens, float64 recurrent form"},
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
