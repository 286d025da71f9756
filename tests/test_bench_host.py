"""Host-side pieces of bench.py that need no GPU: workload selection, the per-kernel source
hashes that tie recorded DRAM traffic to the sources it was measured on, and the rate
arithmetic."""
import os
import re
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from random_access_kv_fq_b200 import workloads as wl  # noqa: E402


def test_tokens_override_shrinks_the_named_workload():
    full = bench.pick_workload(types.SimpleNamespace(workload="large", tokens=None))
    small = bench.pick_workload(types.SimpleNamespace(workload="large", tokens=1024))
    assert full is wl.LARGE
    assert small.cache.n * 32 == full.cache.n            # 32768 -> 1024 tokens
    assert small.cache.d == full.cache.d and small.rates == full.rates
    assert small.name.endswith("_tokens1024") and small.name != full.name


def test_source_hashes_are_per_kernel_and_stable():
    enc = bench.source_sha("encode_k3N64_exactL20c8")
    assert enc == bench.source_sha("encode_k4N8")           # same kernel sources
    assert enc != bench.source_sha("decode_k4N8")
    assert enc != bench.source_sha("attn_B16")
    assert re.fullmatch(r"[0-9a-f]{16}", enc)


def test_recorded_traffic_applies_only_to_its_sources():
    lines = []
    for f in os.listdir(os.path.join(ROOT, "profiles")):
        if f.endswith(".md"):
            lines += [l for l in open(os.path.join(ROOT, "profiles", f)) if l.startswith("traffic ")]
    for line in lines:
        _, label, b, sha = line.split()
        got = bench.profiled_traffic(label)
        if sha.split("=")[1] == bench.source_sha(label):
            assert got == int(b.split("=")[1])
        else:
            assert got is None
    assert bench.profiled_traffic("encode_no_such_label") is None


def test_whole_job_rate_and_single_process_max():
    assert bench.whole_job_rate(4, 2.5e9, 10, 1000.0) == 4 * 2.5e9 * 10 / 1.0 / 1e9
    assert bench.max_over_ranks(None, None, 12.5, None) == 12.5
