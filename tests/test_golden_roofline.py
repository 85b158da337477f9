"""The roofline arithmetic of the bench, pinned by the worked example the pages print (CPU only), and
the flop/byte ratio of the bench workloads that makes every one of them bandwidth-bound on a B200."""
import json
import os

import pytest

import bench
from paged_kv_cache_tree_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "a100_decode_roofline.json")


def test_pages_worked_decode_example():
    g = json.load(open(GOLDEN))
    io_s, comp_s = bench.time_at_roofline(g["io_bytes"], g["flops"], g["hbm_gbs"], g["fp16_tflops"])
    # printed as "10 ms" and "0.07 ms" (rounded); the exact quotients are 9.81 ms and 0.064 ms
    assert io_s * 1e3 == pytest.approx(g["io_ms_printed"], rel=0.05)
    assert comp_s * 1e3 == pytest.approx(g["compute_ms_printed"], rel=0.10)
    assert io_s > 100 * comp_s           # "bandwidth-bound"


@pytest.mark.parametrize("name,flop_per_byte", [("decode", 4.0), ("chain", 63.0), ("tree", 126.0), ("long", 32.0)])
def test_bench_workloads_are_bandwidth_bound_on_b200(name, flop_per_byte):
    w = wl.make_workload(dict(wl.WORKLOADS[name], B=4), fill="zero")
    L = w.context_lens.double()
    flops = float((4 * w.D * w.num_candidates.double() * w.Hq * L).sum())
    byts = w.kv_bytes() + w.qo_bytes()
    assert flops / byts == pytest.approx(flop_per_byte, rel=0.02)
    # ridge of the B200 at its dense bf16 peak over its copy bandwidth (2.25 PF / 8 TB/s = 281 flop/B)
    assert flops / byts < 2.25e15 / 8e12
