"""Host-side pieces of bench.py that need no GPU: workload selection, the per-kernel source
hashes that tie recorded DRAM traffic to the sources it was measured on, and the rate
arithmetic."""
import json
import os
import re
import sys
import types

import numpy as np

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
    enc = bench.source_sha("encode_k3N64_exactL20c8", 64)
    assert enc == bench.source_sha("encode_k4N8", 64)          # same kernel sources
    assert enc != bench.source_sha("decode_k4N8", 64)
    assert enc != bench.source_sha("encode_k4N4096_topL16c8", 128)
    assert enc != bench.source_sha("attn_B16", 64)
    assert re.fullmatch(r"[0-9a-f]{16}", enc)


def test_recorded_traffic_applies_only_to_its_sources(tmp_path, monkeypatch):
    rec = {"large_32Lx8Hx32768T_d128/encode_k4N4096_topL16c8":
           {"bytes_per_vector": 300.5, "source_sha": bench.source_sha("encode_k4", 128)},
           "large_32Lx8Hx32768T_d128/decode_k4N4096_topL16c8":
           {"bytes_per_vector": 310.0, "source_sha": "0" * 16}}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    name = "large_32Lx8Hx32768T_d128_tokens1024"   # a reduced case reads the same record
    assert bench.profiled_traffic(name, "encode_k4N4096_topL16c8", 128, 1000) == 300500
    assert bench.profiled_traffic(name, "decode_k4N4096_topL16c8", 128, 1000) is None  # stale
    assert bench.profiled_traffic(name, "encode_no_such_label", 128, 10) is None
    # the committed record file parses and every entry names a known kernel kind
    committed = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, v in committed.items():
        if key.startswith("_"):
            continue
        assert key.split("/")[1].split("_")[0] in ("encode", "decode", "attn")
        assert v["bytes_per_vector"] > 0 and re.fullmatch(r"[0-9a-f]{16}", v["source_sha"])


def test_step_and_extra_rates_and_cpu_sample():
    step, extra = bench.step_and_extra_rates(wl.LARGE)
    assert [r.search for r in step] == ["top"] and [r.search for r in extra] == ["brute"]
    step, extra = bench.step_and_extra_rates(wl.GPT2)
    assert step == wl.GPT2.rates and extra == ()
    rows = bench.cpu_sample_rows(wl.LARGE.cache, 1000)
    per = wl.LARGE.cache.slab_vectors
    half = wl.LARGE.cache.n // 2
    assert rows.size == 1000 and np.all(np.diff(rows) > 0)
    assert np.all((rows < per) | ((rows >= half) & (rows < half + per)))


def test_whole_job_rate_and_single_process_max():
    assert bench.whole_job_rate(4, 2.5e9, 10, 1000.0) == 4 * 2.5e9 * 10 / 1.0 / 1e9
    assert bench.max_over_ranks(None, None, 12.5, None) == 12.5


def test_e2e_chunks_split_both_halves_evenly():
    """The end-to-end step's row chunks split K and V evenly for every workload (and shrunken
    sequence lengths), up to 32 chunks."""
    from random_access_kv_fq_b200 import workloads as wl
    sizes = [w.cache.n for w in wl.CODEC_WORKLOADS.values()] + [524288, 4096, 6, 2]
    for n in sizes:
        c = bench.e2e_chunks(n)
        half = n // 2
        assert c in (32, 16, 8, 4, 2) and half % (c // 2) == 0
        assert (half // (c // 2)) * c == n
    assert bench.e2e_chunks(wl.LARGE.cache.n) == 32
