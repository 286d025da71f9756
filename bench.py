"""Benchmark of the FibQuant KV codec hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fibquant|reference]
                    [--workload gpt2|tinyllama|large|toy]

One step = one pass of the whole hot path over the workload's synthetic GPT-2-small-shaped
KV cache (12 layers x 12 heads x 1024 tokens, K and V, d = 64, fp16): for each of its two
rates (k=3 N=64 with the exact grid search, k=4 N=8 with brute force) encode K and V
(separate rotations) and decode K and V to fp16.  The metric is fp16-equivalent GB/s:
(encode input + decode output) bytes as an fp16 cache, divided by the step time.  The fused
decode-attention step (B16, Hq32/Hkv4, T32768, d64) is timed in the same run and reported
under "attn".  Inputs rotate over enough copies that every kernel reads data that has left
the 126 MB L2 (the whole-step footprint between reuses is >= 2x L2).

With --gpus N > 1 (launched by torch.distributed.run), every rank processes its own cache of
the same shape (weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import glob
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from random_access_kv_fq_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
WORKLOADS = {"gpt2": wl.GPT2, "tinyllama": wl.TINYLLAMA, "large": wl.LARGE, "toy": wl.TOY}


# ----------------------------------------------------------------------------- helpers

def rank_cache(w, rank: int):
    """Rank `rank`'s cache: the workload's shape with its own seed (weak scaling: every rank
    encodes and decodes a different cache of the same size)."""
    return dataclasses.replace(w.cache, seed=w.cache.seed + 7919 * rank)


def max_over_ranks(torch, dist, ms: float, device) -> float:
    """The slowest rank's time (the job's time); `ms` itself without a process group."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, bytes_per_rank: float, reps: int, ms: float) -> float:
    """GB/s of the whole job: every rank moved bytes_per_rank per rep, in ms for all reps."""
    return world * bytes_per_rank * reps / (ms * 1e-3) / 1e9


def pick_workload(args):
    """The named workload; --tokens shrinks its sequences (small cases for profiling only: the
    bench line then names the reduced workload)."""
    w = WORKLOADS[args.workload]
    if args.tokens:
        w = dataclasses.replace(w, name=f"{w.name}_tokens{args.tokens}",
                                cache=dataclasses.replace(w.cache, tokens=args.tokens))
    return w


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# The sources each timed kernel is built from (its .cu, the headers it includes and the host
# launcher that picks it): a recorded DRAM traffic figure only applies while these are unchanged.
KERNEL_SOURCES = {
    "encode": ["encode_sm100.cu", "codec_sm100.h", "fq_device.cuh", "sm100_ptx.cuh",
               "fq_internal.h", "fq_api.cu"],
    "decode": ["decode_sm100.cu", "codec_sm100.h", "fq_device.cuh", "sm100_ptx.cuh",
               "fq_internal.h", "fq_api.cu"],
    "attn": ["attn_sm100.cu", "attn.cu", "fq_device.cuh", "sm100_ptx.cuh", "fq_internal.h",
             "fq_api.cu"],
}


def source_sha(kernel_label: str) -> str:
    """Hash of the sources of the kernel a bench label names ("encode_k3N64..." -> encode)."""
    kind = kernel_label.split("_")[0]
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind] + ["../../include/fq.h"]:
        h.update(open(os.path.join(ROOT, "random_access_kv_fq_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_label: str):
    """Per-launch DRAM bytes recorded from an ncu capture of this exact source, else None."""
    for f in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(f):
            m = re.match(r"traffic\s+(\S+)\s+bytes_per_launch=(\d+)\s+source_sha=(\w+)", line)
            if m and m.group(1) == kernel_label and m.group(3) == source_sha(kernel_label):
                return int(m.group(2))
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []   # (arrival time, line)
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            deadline = time.time() + 5.0  # the sampler is running before the region starts
            while not self.lines and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *a):
        self.t1 = time.time()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if self.t0 is not None and not (self.t0 <= ts <= self.t1 + 0.1):
                continue  # only samples taken while the timed region ran
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- workload setup

@dataclasses.dataclass
class RateState:
    rate: wl.Rate
    rot: dict        # tensor -> device rotation
    cb: object
    index: object
    P: int
    codes: list      # per copy: [n, P] uint8
    norms: list      # per copy: [n] int16


def build_codec_state(torch, fq, w, rank, copies, device):
    shape = rank_cache(w, rank)
    n, d = shape.n, shape.d
    half = n // 2
    host = wl.cache(shape)
    tdtype = torch.float16 if shape.dtype == "f16" else torch.float32
    xs = [torch.from_numpy(host).to(device) for _ in range(copies)]
    from random_access_kv_fq_b200 import tables
    states = []
    for rate in w.rates:
        dp = fq.fq_padded_dim(d, rate.k)
        rot = {"K": torch.from_numpy(tables.rotation(dp, wl.ROT_SEED_K)).to(device),
               "V": torch.from_numpy(tables.rotation(dp, wl.ROT_SEED_V)).to(device)}
        cb_np = tables.codebook(dp, rate.k, rate.N)
        cb = torch.from_numpy(cb_np).to(device)
        index = None
        if rate.search != "brute":
            kind = fq.FQ_INDEX_EXACT if rate.search == "exact" else fq.FQ_INDEX_TOPC
            index = torch.from_numpy(fq.fq_build_search_index(cb_np, d, rate.k, rate.N, kind,
                                                              rate.grid_L, rate.grid_c)).to(device)
        P = fq.fq_payload_bytes(d, rate.k, rate.N)
        codes = [torch.empty((n, P), dtype=torch.uint8, device=device) for _ in range(copies)]
        norms = [torch.empty((n,), dtype=torch.int16, device=device) for _ in range(copies)]
        st = RateState(rate, rot, cb, index, P, codes, norms)
        for c in range(copies):  # valid records everywhere before timing
            for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
                fq.fq_encode(xs[c][sl], rot[t], cb, rate.k, rate.N, codes=codes[c][sl],
                             norms=norms[c][sl], search_index=index)
        states.append(st)
    ys = [torch.empty((n, d), dtype=torch.float16, device=device) for _ in range(copies)]
    torch.cuda.synchronize()
    return shape, host, xs, ys, states


def codec_launches(fq, shape, xs, ys, states, c, prev):
    """The launches of one step on copy c (decode reads the records of copy `prev`).  Yields
    (label, kind, algorithmic bytes, fp16-equivalent bytes, launch thunk)."""
    n, d = shape.n, shape.d
    half = n // 2
    for st in states:
        r = st.rate
        for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
            nv = sl.stop - sl.start
            xb = xs[c].element_size() * d
            yield (f"encode_{r.label}", "encode", nv * (xb + st.P + 2), nv * 2 * d,
                   lambda st=st, t=t, sl=sl: fq.fq_encode(
                       xs[c][sl], st.rot[t], st.cb, st.rate.k, st.rate.N, codes=st.codes[c][sl],
                       norms=st.norms[c][sl], search_index=st.index))
            yield (f"decode_{r.label}", "decode", nv * (st.P + 2 + 2 * d), nv * 2 * d,
                   lambda st=st, t=t, sl=sl: fq.fq_decode(
                       st.codes[prev][sl], st.norms[prev][sl], st.rot[t], st.cb, d, st.rate.k,
                       st.rate.N, y=ys[c][sl]))


def attn_state(torch, fq, device, copies, rank):
    w = wl.ATTN
    from random_access_kv_fq_b200 import tables
    dpk, dpv = fq.fq_padded_dim(w.d, w.k_rate.k), fq.fq_padded_dim(w.d, w.v_rate.k)
    rk = torch.from_numpy(tables.rotation(dpk, wl.ROT_SEED_K)).to(device)
    rv = torch.from_numpy(tables.rotation(dpv, wl.ROT_SEED_V)).to(device)
    ck = torch.from_numpy(tables.codebook(dpk, w.k_rate.k, w.k_rate.N)).to(device)
    cv = torch.from_numpy(tables.codebook(dpv, w.v_rate.k, w.v_rate.N)).to(device)
    q = torch.from_numpy(wl.attn_queries(w)).to(device)
    kx = torch.from_numpy(wl.attn_kv(w, "K").reshape(-1, w.d)).to(device)
    vx = torch.from_numpy(wl.attn_kv(w, "V").reshape(-1, w.d)).to(device)
    kc, kn = fq.fq_encode(kx, rk, ck, w.k_rate.k, w.k_rate.N)
    vc, vn = fq.fq_encode(vx, rv, cv, w.v_rate.k, w.v_rate.N)
    del kx, vx
    shp = (w.batch, w.hkv, w.tokens)
    kcs = [kc.reshape(*shp, -1).clone() for _ in range(copies)]
    kns = [kn.reshape(shp).clone() for _ in range(copies)]
    vcs = [vc.reshape(*shp, -1).clone() for _ in range(copies)]
    vns = [vn.reshape(shp).clone() for _ in range(copies)]
    ws = torch.empty((fq.fq_attn_workspace_bytes(w.batch, w.hq, w.hkv, w.tokens, w.d,
                                                 w.v_rate.k),), dtype=torch.uint8, device=device)
    out = torch.empty((w.batch, w.hq, w.d), dtype=torch.float32, device=device)
    step_bytes = w.batch * w.hkv * w.tokens * (kcs[0].shape[-1] + 2 + vcs[0].shape[-1] + 2)

    def launch(c):
        fq.fq_attn_decode(q, kcs[c], kns[c], w.k_rate.k, w.k_rate.N, rk, ck, vcs[c], vns[c],
                          w.v_rate.k, w.v_rate.N, rv, cv, scale=1 / math.sqrt(w.d), out=out,
                          workspace=ws)
    return launch, step_bytes


# ----------------------------------------------------------------------------- arms

def run_gpu(args):
    import torch
    import random_access_kv_fq_b200 as fq
    fq.lib()  # fail loudly when the CUDA library is missing
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = pick_workload(args)
    shape0 = w.cache
    step_bytes_est = shape0.n * (shape0.d * 2) * 3 * len(w.rates)
    copies = max(2, math.ceil(2 * L2_BYTES / max(step_bytes_est, 1)) + 1)
    copies = min(copies, 8)
    shape, host, xs, ys, states = build_codec_state(torch, fq, w, rank, copies, device)
    attn_launch, attn_bytes = attn_state(torch, fq, device, 4, rank) if not args.no_attn else (None, 0)
    n_launch = sum(1 for _ in codec_launches(fq, shape, xs, ys, states, 0, 0))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    stream = torch.cuda.current_stream()
    # The timed region replays CUDA graphs of the step's C-ABI calls (one graph per input copy):
    # the kernels, arguments and order are those of the eager calls, without the host-side
    # launch latency between them.
    side = torch.cuda.Stream(device)
    side.wait_stream(stream)

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for fn in fns:
                    fn()
        return g

    for c in range(copies):  # one eager pass (tables, attributes) before capture
        for *_, fn in codec_launches(fq, shape, xs, ys, states, c, (c - 1) % copies):
            fn()
    torch.cuda.synchronize()
    step_graphs = [capture([fn for *_, fn in codec_launches(fq, shape, xs, ys, states, c,
                                                             (c - 1) % copies)])
                   for c in range(copies)]
    meta = [(lab, kind, ab, eb) for lab, kind, ab, eb, _ in
            codec_launches(fq, shape, xs, ys, states, 0, copies - 1)]
    torch.cuda.synchronize()
    for i in range(args.warmup):
        step_graphs[i % copies].replay()
    barrier()
    with ClockSampler(local) as clk:
        barrier()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step_graphs[i % copies].replay()
        t_end.record(stream)
        barrier()
    total_ms = max_over_ranks(torch, dist, t_start.elapsed_time(t_end), device)
    # per-kernel device time: a graph of every launch of one kind over all copies, replayed
    per = {}
    reps = max(5, min(50, args.steps // copies))
    for lab in dict.fromkeys(m[0] for m in meta):
        fns = [fn for c in range(copies) for l, *_, fn in
               codec_launches(fq, shape, xs, ys, states, c, (c - 1) % copies) if l == lab]
        g = capture(fns)
        g.replay()
        barrier()
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for _ in range(reps):
            g.replay()
        k1.record(stream)
        barrier()
        ms = k0.elapsed_time(k1) / (reps * len(fns))
        ab, kind = next((m[2], m[1]) for m in meta if m[0] == lab)
        per_step = sum(1 for m in meta if m[0] == lab)
        per[lab] = {"ms": ms, "per_step": per_step, "alg_bytes": ab, "kind": kind}
        del g
    step_eq = sum(eb for _, _, _, eb in meta)
    value = whole_job_rate(world, step_eq, args.steps, total_ms)
    hbm, hbm_src = peaks()
    dom_lab = max(per, key=lambda k: per[k]["ms"] * per[k]["per_step"])
    dom = per[dom_lab]
    achieved = dom["alg_bytes"] / (dom["ms"] * 1e-3) / 1e9
    tot_share = sum(v["ms"] * v["per_step"] for v in per.values())
    kernels = {lab: {"avg_us": round(1e3 * s_["ms"], 2),
                     "GBps_alg": round(s_["alg_bytes"] / (s_["ms"] * 1e-3) / 1e9, 1),
                     "share": round(s_["ms"] * s_["per_step"] / tot_share, 3)}
               for lab, s_ in per.items()}
    result = {
        "metric": "KV encode/decode GB/s (fp16-equiv) & % of roofline; fused attn us/step",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16->u8/fp32",
        "data": "synthetic (seeded; GPT-2-small-shaped KV cache recipe, no weights)",
        "config": {"workload": w.name, "vectors_per_gpu": shape.n, "d": shape.d,
                   "rates": [r.label for r in w.rates], "decode_out": "fp16",
                   "l2": f"inputs rotate over {copies} copies (>= 2x L2 between reuses)",
                   "step": "encode K,V + decode K,V per rate",
                   "launch": "CUDA graph replay of the step's C-ABI calls"},
        "roofline": {"bound": "hbm", "kernel": dom_lab, "achieved": round(achieved, 1),
                     "peak": hbm, "peak_source": hbm_src, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": profiled_traffic(dom_lab),
                     "alg_bytes_per_launch": dom["alg_bytes"]},
        "kernels": kernels,
        "gpu_launches": None,
        "clocks": clk.summary(),
    }
    launches_per_step = len(meta)
    gpu_launches = launches_per_step * args.steps
    # fused attention step
    if attn_launch:
        for c in range(4):
            attn_launch(c)
        torch.cuda.synchronize()
        agraphs = [capture([lambda c=c: attn_launch(c)]) for c in range(4)]
        areps = max(20, args.steps // 10)
        for i in range(4):
            agraphs[i].replay()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for i in range(areps):
            agraphs[i % 4].replay()
        a1.record(stream)
        barrier()
        us = max_over_ranks(torch, dist, a0.elapsed_time(a1), device) * 1e3 / areps
        result["attn"] = {"workload": wl.ATTN.name, "us_per_step": round(us, 2),
                          "bytes_per_step": attn_bytes,
                          "roofline": {"bound": "hbm", "achieved": round(attn_bytes / (us * 1e-6) / 1e9, 1),
                                       "peak": hbm, "unit": "GB/s",
                                       "frac": round(attn_bytes / (us * 1e-6) / 1e9 / hbm, 4)},
                          "launches_per_step": 2}
        del agraphs
    del step_graphs
    result["gpu_launches"] = gpu_launches
    # end to end through the public API with pinned host buffers
    if not args.no_e2e:
        result["e2e"] = e2e(torch, fq, shape, host, states, args, device, world, dist)
    if rank == 0:
        result["cpu_baseline"] = cpu_baseline(w, args) if not args.no_cpu else None
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def e2e(torch, fq, shape, host, states, args, device, world, dist, chunks=8):
    """Same metric through the public API with host buffers.  Every step copies the pinned host
    cache in, encodes, copies the records out, copies them back in, decodes and copies the fp16
    result out, for each rate.  The step runs in row chunks (each entirely K or V) over three
    CUDA streams (upload, kernels, download) so that uploads, downloads and kernels overlap.  The step's calls are captured once as a CUDA graph and replayed, as in
    the device-resident measurement; every byte still crosses the host link in every step."""
    n, d = shape.n, shape.d
    half = n // 2
    per = half // (chunks // 2)
    assert per * chunks == n, "chunks must split the K and V halves evenly"
    xh = torch.from_numpy(host).pin_memory()
    xd = torch.empty_like(xh, device=device)
    rec_h = [(torch.empty((n, st.P), dtype=torch.uint8).pin_memory(),
              torch.empty((n,), dtype=torch.int16).pin_memory()) for st in states]
    yh = [torch.empty((n, d), dtype=torch.float16).pin_memory() for _ in states]
    yd = [torch.empty((n, d), dtype=torch.float16, device=device) for _ in states]
    cs, su, sc, sd = (torch.cuda.Stream(device) for _ in range(4))

    def rows(j):
        return slice(j * per, (j + 1) * per), ("K" if j < chunks // 2 else "V")

    def mark(stream):
        e = torch.cuda.Event()
        e.record(stream)
        return e

    def step():
        # Enqueued from cs (fork and join).  One stream per copy direction, each in data-flow
        # order with a lag of one chunk, so that no copy waits behind a later chunk's copies:
        #   su (upload):   x0 x1 r0 x2 r1 ...    (r = records back in)
        #   sc (kernels):  e0 e1 d0 e2 d1 ...    (e = encode, d = decode; both rates)
        #   sd (download): o0 o1 y0 o2 y1 ...    (o = records out, y = fp16 result)
        e0 = mark(cs)
        for s_ in (su, sc, sd):
            s_.wait_event(e0)
        ev_x, ev_enc, ev_out, ev_in, ev_dec = {}, {}, {}, {}, {}
        for j in range(chunks + 1):
            if j < chunks:
                sl, _ = rows(j)
                with torch.cuda.stream(su):
                    xd[sl].copy_(xh[sl], non_blocking=True)
                ev_x[j] = mark(su)
            if j >= 1:
                sl, _ = rows(j - 1)
                su.wait_event(ev_out[j - 1])
                with torch.cuda.stream(su):
                    for r, st in enumerate(states):
                        ch, nh = rec_h[r]
                        st.codes[1][sl].copy_(ch[sl], non_blocking=True)
                        st.norms[1][sl].copy_(nh[sl], non_blocking=True)
                ev_in[j - 1] = mark(su)
            if j < chunks:
                sl, t = rows(j)
                sc.wait_event(ev_x[j])
                for st in states:
                    fq.fq_encode(xd[sl], st.rot[t], st.cb, st.rate.k, st.rate.N,
                                 codes=st.codes[0][sl], norms=st.norms[0][sl],
                                 search_index=st.index, stream=sc)
                ev_enc[j] = mark(sc)
                sd.wait_event(ev_enc[j])
                with torch.cuda.stream(sd):
                    for r, st in enumerate(states):
                        ch, nh = rec_h[r]
                        ch[sl].copy_(st.codes[0][sl], non_blocking=True)
                        nh[sl].copy_(st.norms[0][sl], non_blocking=True)
                ev_out[j] = mark(sd)
            if j >= 1:
                sl, t = rows(j - 1)
                sc.wait_event(ev_in[j - 1])
                for r, st in enumerate(states):
                    fq.fq_decode(st.codes[1][sl], st.norms[1][sl], st.rot[t], st.cb, d,
                                 st.rate.k, st.rate.N, y=yd[r][sl], stream=sc)
                ev_dec[j - 1] = mark(sc)
                sd.wait_event(ev_dec[j - 1])
                with torch.cuda.stream(sd):
                    for r in range(len(states)):
                        yh[r][sl].copy_(yd[r][sl], non_blocking=True)
        for s_ in (su, sc, sd):
            cs.wait_event(mark(s_))

    h2d = xh.numel() * xh.element_size() + sum(n * st.P + 2 * n for st in states)
    d2h = sum(n * st.P + 2 * n + n * d * 2 for st in states)
    main = torch.cuda.current_stream()
    cs.wait_stream(main)
    step()  # eager once (library set-up), then capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        step()
    torch.cuda.synchronize()
    for _ in range(max(3, args.warmup // 10)):
        graph.replay()
    torch.cuda.synchronize()
    # the overlapped step must deliver exactly what a plain decode of its records gives
    for r, st in enumerate(states):
        ref = torch.empty((n, d), dtype=torch.float16, device=device)
        for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
            fq.fq_decode(st.codes[1][sl], st.norms[1][sl], st.rot[t], st.cb, d, st.rate.k,
                         st.rate.N, y=ref[sl])
        if not torch.equal(ref.cpu(), yh[r]):
            raise RuntimeError(f"overlapped end-to-end step disagrees with a plain decode "
                               f"({st.rate.label})")
    torch.cuda.synchronize()
    reps = max(5, min(50, args.steps // 20))
    if dist is not None:
        dist.barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(main)
    for _ in range(reps):
        graph.replay()
    s1.record(main)
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dist, s0.elapsed_time(s1), device)
    del graph
    eq = 2 * n * 2 * d * len(states)
    return {"value": round(whole_job_rate(world, eq, reps, ms), 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": reps,
            "overlap": f"{chunks} row chunks over three CUDA streams (upload, kernels, download) "
                       "in data-flow order, one CUDA graph per step"}


def cpu_baseline(w, args, budget_s: float = 12.0):
    """The CPU oracle, as it stands, timed on this host on a bounded sample of the workload
    (single BLAS thread)."""
    from threadpoolctl import threadpool_limits
    from oracle import fq_oracle as fo
    from random_access_kv_fq_b200 import tables
    shape = w.cache
    rng = np.random.default_rng(0)
    sample = np.sort(rng.choice(shape.n, size=min(2048, shape.n), replace=False))
    x = wl.rows_of(shape, sample)
    done_eq = 0
    t0 = time.perf_counter()
    with threadpool_limits(1):
        while time.perf_counter() - t0 < budget_s:
            for rate in w.rates:
                dp = fo.padded_dim(shape.d, rate.k)
                rot = tables.rotation(dp, wl.ROT_SEED_K)
                cb = tables.codebook(dp, rate.k, rate.N)
                enc = fo.encode(x, rot, cb, rate.k)
                codes = fo.pack(enc.idx, rate.N)
                fo.decode(codes, enc.norms, rot, cb, shape.d, rate.k, rate.N)
                done_eq += 2 * x.shape[0] * 2 * shape.d
    el = time.perf_counter() - t0
    return {"value": round(done_eq / el / 1e9, 6), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{x.shape[0]} sampled vectors of {w.name}, encode+pack+decode at every "
                      f"rate, repeated for {el:.1f} s (fp64 NumPy, 1 thread)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = pick_workload(args)
    cb = cpu_baseline(w, args, budget_s=max(3.0, min(20.0, 2.0 * args.steps)))
    line = {"impl": "reference", "metric": "KV encode/decode GB/s (fp16-equiv) & % of roofline; "
            "fused attn us/step", "value": cb["value"], "unit": "GB/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "rates": [r.label for r in w.rates]},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="fibquant", choices=["fibquant", "reference"])
    ap.add_argument("--workload", default="gpt2", choices=list(WORKLOADS))
    ap.add_argument("--no-attn", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="shrink the workload's sequence length (small profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
