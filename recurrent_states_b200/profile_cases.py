"""Small launches of the library's hot kernels at the benchmark's shapes, for
profilers (ncu captures of one kernel): four calls of one entry point, so that
a capture can skip the first (cold) launches.

    python -m recurrent_states_b200.profile_cases <case>

prefill  the main prefill, B1 H8 N4096 d_k 16 d_v 64 n 3 (tc_fused_prefill_kernel)
cprefill the order-2 mean-centred prefill of the same inputs (tc_chunk_state_kernel,
         scan_kernel, tc_centred_chunk_out_kernel)
decode   one decode step on 1,024 random states, B64 H16 (decode_ws_kernel)
centred  the same with the order-2 mean-centred read-out (decode_ws_kernel<.., 1>)
multi4   4 new tokens per head on those states (decode_multi_ws_kernel)
multi16  16 new tokens per head (decode_multi_tc_kernel)
large    1/8 of the large head, B1 H8 N32768 d_k 64 n 3 (tcf_state_kernel, tcf_out_kernel)
"""
import sys

import torch

from . import synth
from . import taylor_attn as TA

CASES = ("prefill", "cprefill", "decode", "centred", "multi4", "multi16", "large")


def run(case: str, calls: int = 4) -> float:
    if case not in CASES:
        raise ValueError(f"case must be one of {CASES}")
    dev = torch.device("cuda:0")
    d, dv, n, tau = 16, 64, 3, 2.0
    stride = TA.taylor_attn_state_stride(d, dv, n)
    g = torch.Generator(device="cpu").manual_seed(1)
    if case.startswith("multi"):
        T = int(case[5:])
        q, k, v = (t.to(dev) for t in synth.qkv(64, 16, T, d, dv, seed=1))
        st = (torch.randn((64, 16, stride), generator=g) * 0.01).to(dev)
        out = torch.empty((64, 16, T, dv), device=dev)
        for _ in range(calls):
            TA.taylor_attn_prefill_from_state(q, k, v, st, n, tau, out=out, state_out=st)
    elif case in ("prefill", "cprefill"):
        q, k, v = (t.to(dev) for t in synth.qkv(1, 8, 4096, d, dv, seed=0))
        out = torch.empty((1, 8, 4096, dv), device=dev)
        st = torch.empty((1, 8, stride), device=dev)
        for _ in range(calls):
            if case == "prefill":
                TA.taylor_attn_prefill(q, k, v, n, tau, out=out, state_out=st)
            else:
                TA.taylor_attn_centred_prefill(q, k, v, 2, tau, out=out, state_out=st)
    elif case == "large":
        dl = 64
        q, k, v = (t.to(dev) for t in synth.qkv(1, 8, 32768, dl, dv, seed=3))
        out = torch.empty((1, 8, 32768, dv), device=dev)
        st = torch.empty((1, 8, TA.taylor_attn_state_stride(dl, dv, n)), device=dev)
        for _ in range(calls):
            TA.taylor_attn_prefill(q, k, v, n, tau, out=out, state_out=st)
    else:
        q, k, v = (t[:, :, 0].contiguous().to(dev) for t in synth.qkv(64, 16, 1, d, dv, seed=2))
        st = (torch.randn((64, 16, stride), generator=g) * 0.01).to(dev)
        out = torch.empty((64, 16, dv), device=dev)
        for _ in range(calls):
            if case == "decode":
                TA.taylor_attn_decode(q, k, v, st, n, tau, out=out)
            else:
                TA.taylor_attn_centred_decode(q, k, v, st, 2, tau, out=out)
    torch.cuda.synchronize()
    return float(out.abs().sum())


if __name__ == "__main__":
    case = sys.argv[1] if len(sys.argv) > 1 else "prefill"
    print(case, "ok", run(case))
