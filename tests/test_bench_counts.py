"""The algorithmic work bench.py divides by, against counts fixed independently
of it: the paper's per-head state size at d_k 16, d_v 64, n 3 (9,945 values,
arXiv 2610.20637 abstract), its recurrent work of 4 F (d_v + 1) flops per
head-token, and the byte volume of each workload's inputs and outputs.
CPU only: bench.py's device code is not reached."""
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from recurrent_states_b200 import synth  # noqa: E402


def _F(d, n):
    return sum(math.comb(d + m - 1, m) for m in range(n))


def test_bench_workloads_are_the_named_workloads():
    for key, name in (("MAIN", "main_prefill"), ("DECODE", "decode"), ("LARGE", "large_head"),
                      ("SWEEP", "order_sweep")):
        w, ref = getattr(bench, key), synth.WORKLOADS[name]
        for f in w:
            assert w[f] == ref[f], (key, f)


def test_decode_bytes_are_the_state_read_and_written_plus_the_token():
    w = bench.DECODE
    byts, flops = bench.kernel_algorithmic("decode", w, 1)
    assert _F(16, 3) * 65 == 9945
    per_head = 2 * 9945 * 4 + (2 * 16 + 64) * 2 + 64 * 4   # state r+w, bf16 q k v, fp32 out
    assert per_head == 80_008
    assert byts == 1024 * per_head == 81_928_192
    assert flops == 1024 * 4 * 9945


def test_main_prefill_volume_and_work():
    w = bench.MAIN
    byts, flops = bench.kernel_algorithmic("prefill", w, 1)
    T = 8 * 4096
    stride = math.ceil(9945 / 32) * 32
    assert byts == T * ((2 * 16 + 64) * 2 + 64 * 4) + 8 * stride * 4
    assert 14.9e6 < byts < 15.1e6            # "15.0 MB per step"
    assert flops == T * 4 * 9945
    assert abs(flops / 1e9 - 1.30) < 0.01     # "1.30 GFLOP"


def test_large_head_work():
    w = bench.LARGE
    _, flops = bench.kernel_algorithmic("prefill", w, 1)
    assert _F(64, 3) == 2145
    assert flops == 4 * 16 * 32768 * 4 * 2145 * 65
    assert abs(flops / 1e9 - 1169.6) < 0.1    # "1,169.6 GFLOP"


@pytest.mark.parametrize("key", ["DECODE_WS_DRAM_BYTES"])
def test_recorded_decode_traffic_is_below_the_algorithmic_bytes(key):
    """The ncu-recorded DRAM bytes of one decode launch: the states are read
    once (41 MB) and their updates stay in L2, so traffic is about half the
    algorithmic read + write volume."""
    byts, _ = bench.kernel_algorithmic("decode", bench.DECODE, 1)
    t = getattr(bench, key)
    assert 0.45 * byts < t < 0.55 * byts
