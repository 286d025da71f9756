"""Benchmark of the FibQuant KV codec hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fibquant|reference]
                    [--workload large|gpt2|tinyllama|toy] [--tokens T]
                    [--no-configs] [--no-attn] [--no-e2e] [--no-cpu]

Headline (the line's "value"): the large-codebook KV cache, 32 layers x 8 kv heads x 32768
tokens, d = 128, K and V (16,777,216 vectors, 4.3 GB of fp16), at k = 4, N = 4096 with the top-8
grid search (L = 16 cells per axis).  One step encodes K and V (separate rotations) and decodes
both back to fp16; the metric is fp16-equivalent GB/s: (encode input + decode output) bytes as an
fp16 cache, divided by the step time.  The same cache's exact brute-force encode (tensor-core
distance contraction with fp32 re-ranking) is timed as a second labelled kernel under
"extra_kernels".  In the same run: the GPT-2-small-shaped, TinyLlama-shaped and toy caches under
"configs" (their own steps: every rate, encode + decode of K and V), the fused decode-attention
step (B16, Hq32/Hkv4, T32768, d64) under "attn", the end-to-end figure through the C ABI with
host buffers under "e2e", and the CPU oracle on the host's cores under "cpu_baseline".

Inputs larger than 2x the 126 MB L2 stream from HBM; the smaller caches rotate over enough
copies that every kernel reads data that has left L2.  Device times are CUDA events on the
launching stream, around CUDA-graph replays of the step's C-ABI calls.

With --gpus N > 1 (launched by torch.distributed.run), every rank processes its own cache of
the same shape (weak scaling, no data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
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
WORKLOADS = {"large": wl.LARGE, "gpt2": wl.GPT2, "tinyllama": wl.TINYLLAMA, "toy": wl.TOY}
METRIC = "KV encode/decode GB/s (fp16-equiv) & % of roofline; fused attn us/step"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


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


def pick_workload(args, key=None):
    """The named workload; --tokens shrinks its sequences (small cases for profiling only: the
    bench line then names the reduced workload)."""
    w = WORKLOADS[key or args.workload]
    if getattr(args, "tokens", None):
        w = dataclasses.replace(w, name=f"{w.name}_tokens{args.tokens}",
                                cache=dataclasses.replace(w.cache, tokens=args.tokens))
    return w


def step_and_extra_rates(w):
    """(rates in the timed step, rates timed only as extra encode kernels).  For the large
    codebook the exact brute-force encode is a second labelled kernel, not part of the step."""
    if w.cache.d == 128:
        return (tuple(r for r in w.rates if r.search != "brute"),
                tuple(r for r in w.rates if r.search == "brute"))
    return tuple(w.rates), ()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s: the measured burst figure (a kernel timed alone), else the
    fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# The sources a timed kernel is built from (its .cu files, the headers they include and the host
# code that picks them): a recorded DRAM traffic figure only applies while these are unchanged.
_COMMON = ["fq_device.cuh", "sm100_ptx.cuh", "fq_internal.h", "fq_api.cu", "codec_sm100.h"]
KERNEL_SOURCES = {
    ("encode", 64): ["encode_sm100.cu"],
    ("decode", 64): ["decode_sm100.cu"],
    ("encode", 128): ["encode_grid_sm100.cu", "encode_large_sm100.cu"],
    ("decode", 128): ["decode_large_sm100.cu"],
    ("attn", 64): ["attn_sm100.cu", "attn.cu"],
}


def source_sha(kernel_label: str, d: int = 64) -> str:
    """Hash of the sources of the kernel a bench label names ("encode_k3N64..." -> encode)."""
    kind = kernel_label.split("_")[0]
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[(kind, d)] + _COMMON:
        h.update(open(os.path.join(ROOT, "random_access_kv_fq_b200", "csrc", f), "rb").read())
    h.update(open(os.path.join(ROOT, "include", "fq.h"), "rb").read())
    return h.hexdigest()[:16]


def traffic_key(workload_name: str, label: str) -> str:
    base = workload_name.split("_tokens")[0]
    return f"{base}/{label}"


def profiled_traffic(workload_name: str, label: str, d: int, vectors: int):
    """Per-launch DRAM bytes (read + write) from an ncu capture of this exact source, scaled to
    `vectors` per launch, else None.  The record under profiles/traffic.json holds the bytes per
    vector of the captured launch and the source hash it was taken on."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    rec = json.load(open(TRAFFIC_FILE)).get(traffic_key(workload_name, label))
    if not rec or rec.get("source_sha") != source_sha(label, d):
        return None
    return int(round(rec["bytes_per_vector"] * vectors))


class ClockSampler:
    """SM clock and clock-event reasons sampled every 10 ms (NVML) while the timed region runs;
    falls back to `nvidia-smi -lms 100` when NVML is unavailable."""

    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
            "sw_power_cap": 0x4}

    def __init__(self, torch, device_index: int, period_s: float = 0.01):
        self.torch, self.dev, self.period = torch, device_index, period_s
        self.samples = []   # (time, sm_mhz, max_mhz, reasons bitmask)
        self.stop = threading.Event()
        self.thread = None
        self.proc = None
        self.t0 = self.t1 = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = self.torch.cuda.get_device_properties(self.dev)
        uuid = str(props.uuid)
        for u in (uuid, "GPU-" + uuid):
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u)
            except Exception:
                pass
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def run():
                while not self.stop.is_set():
                    try:
                        self.samples.append((time.time(),
                                             float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             mx, int(reasons(h))))
                    except Exception:
                        pass
                    self.stop.wait(self.period)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
        except Exception:
            self._smi()
        deadline = time.time() + 5.0  # the sampler runs before the region starts
        while not self.samples and time.time() < deadline:
            time.sleep(0.005)
        self.t0 = time.time()
        return self

    def _smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={fields}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return

        def read():
            for line in self.proc.stdout:
                p = [x.strip() for x in line.split(",")]
                try:
                    bits = sum(b for (nm, b), v in zip(self.BITS.items(), p[2:6])
                               if v.lower().startswith("active"))
                    self.samples.append((time.time(), float(p[0]), float(p[1]), bits))
                except (ValueError, IndexError):
                    pass
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def __exit__(self, *a):
        self.t1 = time.time()
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        inside = [s for s in self.samples
                  if self.t0 is not None and self.t0 <= s[0] <= self.t1 + 0.02]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({nm for _, _, _, bits in inside for nm, b in self.BITS.items() if bits & b})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": inside[-1][2],
                "reasons": reasons, "samples": len(inside),
                "source": "nvml 10 ms" if self.proc is None else "nvidia-smi 100 ms"}


# ----------------------------------------------------------------------------- codec state

@dataclasses.dataclass
class RateState:
    rate: wl.Rate
    rot: dict        # tensor -> device rotation
    cb: object
    index: object
    P: int
    codes: list      # per copy: [n, P] uint8
    norms: list      # per copy: [n] int16


@dataclasses.dataclass
class CodecRun:
    w: object
    shape: object
    host: object
    xs: list
    ys: list
    step: list       # RateState of the rates in the step
    extra: list      # RateState of the rates timed only as extra encode kernels
    copies: int


def build_codec_run(torch, fq, w, rank, device, with_extra=True):
    from random_access_kv_fq_b200 import tables
    shape = rank_cache(w, rank)
    n, d = shape.n, shape.d
    half = n // 2
    step_rates, extra_rates = step_and_extra_rates(w)
    if not with_extra:
        extra_rates = ()
    in_bytes = n * d * (2 if shape.dtype == "f16" else 4)
    # enough input copies that a kernel never finds its input still in L2 (>= 2x L2 between reuses)
    copies = 1 if in_bytes >= 2 * L2_BYTES else min(8, max(2, math.ceil(2 * L2_BYTES / in_bytes) + 1))
    host = wl.cache(shape, workers=min(32, len(os.sched_getaffinity(0))))
    xs = [torch.from_numpy(host).to(device) for _ in range(copies)]
    tdtype = torch.float16

    def rate_state(rate, ncopies):
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
        codes = [torch.empty((n, P), dtype=torch.uint8, device=device) for _ in range(ncopies)]
        norms = [torch.empty((n,), dtype=torch.int16, device=device) for _ in range(ncopies)]
        return RateState(rate, rot, cb, index, P, codes, norms)

    step = [rate_state(r, copies) for r in step_rates]
    for st in step:
        for c in range(copies):  # valid records everywhere before timing
            for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
                fq.fq_encode(xs[c][sl], st.rot[t], st.cb, st.rate.k, st.rate.N,
                             codes=st.codes[c][sl], norms=st.norms[c][sl], search_index=st.index)
    extra = [rate_state(r, 1) for r in extra_rates]
    ys = [torch.empty((n, d), dtype=tdtype, device=device) for _ in range(copies)]
    torch.cuda.synchronize()
    return CodecRun(w, shape, host, xs, ys, step, extra, copies)


def codec_launches(fq, run, c, prev):
    """The launches of one step on copy c (decode reads the records of copy `prev`).  Yields
    (label, kind, algorithmic bytes, fp16-equivalent bytes, vectors, launch thunk)."""
    n, d = run.shape.n, run.shape.d
    half = n // 2
    xs, ys = run.xs, run.ys
    for st in run.step:
        r = st.rate
        for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
            nv = sl.stop - sl.start
            xb = xs[c].element_size() * d
            yield (f"encode_{r.label}", "encode", nv * (xb + st.P + 2), nv * 2 * d, nv,
                   lambda st=st, t=t, sl=sl: fq.fq_encode(
                       xs[c][sl], st.rot[t], st.cb, st.rate.k, st.rate.N, codes=st.codes[c][sl],
                       norms=st.norms[c][sl], search_index=st.index))
            yield (f"decode_{r.label}", "decode", nv * (st.P + 2 + 2 * d), nv * 2 * d, nv,
                   lambda st=st, t=t, sl=sl: fq.fq_decode(
                       st.codes[prev][sl], st.norms[prev][sl], st.rot[t], st.cb, d, st.rate.k,
                       st.rate.N, y=ys[c][sl]))


def extra_launches(fq, run, c):
    n, d = run.shape.n, run.shape.d
    half = n // 2
    for st in run.extra:
        for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
            nv = sl.stop - sl.start
            yield (f"encode_{st.rate.label}", "encode", nv * (2 * d + st.P + 2), nv * 2 * d, nv,
                   lambda st=st, t=t, sl=sl: fq.fq_encode(
                       run.xs[c][sl], st.rot[t], st.cb, st.rate.k, st.rate.N,
                       codes=st.codes[0][sl], norms=st.norms[0][sl], search_index=st.index))


class GraphTimer:
    """CUDA-graph capture on a side stream and CUDA-event timing on the launching stream."""

    def __init__(self, torch, device, dist):
        self.torch, self.dist, self.device = torch, dist, device
        self.stream = torch.cuda.current_stream()
        self.side = torch.cuda.Stream(device)
        self.side.wait_stream(self.stream)

    def capture(self, fns):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.stream(self.side):
            with self.torch.cuda.graph(g, stream=self.side):
                for fn in fns:
                    fn()
        return g

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()
        self.torch.cuda.synchronize()

    def time(self, graphs, reps):
        """ms for `reps` replays cycling over `graphs` (max over ranks)."""
        self.barrier()
        e0 = self.torch.cuda.Event(enable_timing=True)
        e1 = self.torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for i in range(reps):
            graphs[i % len(graphs)].replay()
        e1.record(self.stream)
        self.barrier()
        return max_over_ranks(self.torch, self.dist, e0.elapsed_time(e1), self.device)

    def adaptive_reps(self, graphs, target_s=0.25, lo=2, hi=50):
        """Replays that fill about target_s (measured on one replay of every graph)."""
        ms = self.time(graphs, len(graphs)) / len(graphs)
        return max(lo, min(hi, int(target_s * 1e3 / max(ms, 1e-3))))


def kernel_table(timer, fq, run, launches_of, hbm):
    """Per-label device time: a graph of every launch of one label over all copies, replayed."""
    per = {}
    meta = [m[:5] for m in launches_of(0)]
    for lab in dict.fromkeys(m[0] for m in meta):
        fns = [fn for c in range(run.copies) for (l, *_, fn) in launches_of(c) if l == lab]
        g = timer.capture(fns)
        reps = timer.adaptive_reps([g])
        ms = timer.time([g], reps) / (reps * len(fns))
        _, kind, ab, _, nv = next(m for m in meta if m[0] == lab)
        per_step = sum(1 for m in meta if m[0] == lab)
        gbs = ab / (ms * 1e-3) / 1e9
        per[lab] = {"ms": ms, "per_step": per_step, "alg_bytes": ab, "kind": kind, "vectors": nv,
                    "GBps": gbs, "frac": gbs / hbm}
        del g
    return per


def kernels_json(per, with_share=True):
    tot = sum(v["ms"] * v["per_step"] for v in per.values())
    out = {}
    for lab, s in per.items():
        o = {"avg_us": round(1e3 * s["ms"], 2), "vectors_per_launch": s["vectors"],
             "Gvec_s": round(s["vectors"] / (s["ms"] * 1e-3) / 1e9, 3),
             "GBps_alg": round(s["GBps"], 1), "frac": round(s["frac"], 4)}
        if with_share:
            o["share"] = round(s["ms"] * s["per_step"] / tot, 3)
        out[lab] = o
    return out


def time_codec_step(timer, fq, run, steps, warmup, clocks=None):
    """(total ms over `steps` step replays, step graphs' metadata).  The step graphs cycle over
    the input copies; decode of copy c reads the records of copy c - 1."""
    copies = run.copies
    for c in range(copies):  # one eager pass (tables, attributes) before capture
        for *_, fn in codec_launches(fq, run, c, (c - 1) % copies):
            fn()
    timer.torch.cuda.synchronize()
    graphs = [timer.capture([fn for *_, fn in codec_launches(fq, run, c, (c - 1) % copies)])
              for c in range(copies)]
    meta = [m[:5] for m in codec_launches(fq, run, 0, copies - 1)]
    for i in range(warmup):
        graphs[i % copies].replay()
    timer.barrier()
    if clocks is None:
        ms = timer.time(graphs, steps)
    else:
        with clocks:
            ms = timer.time(graphs, steps)
    del graphs
    return ms, meta


# ----------------------------------------------------------------------------- attention

def attn_state(torch, fq, device, copies, rank):
    w = wl.ATTN
    from random_access_kv_fq_b200 import tables
    dpk, dpv = fq.fq_padded_dim(w.d, w.k_rate.k), fq.fq_padded_dim(w.d, w.v_rate.k)
    rk = torch.from_numpy(tables.rotation(dpk, wl.ROT_SEED_K)).to(device)
    rv = torch.from_numpy(tables.rotation(dpv, wl.ROT_SEED_V)).to(device)
    ck = torch.from_numpy(tables.codebook(dpk, w.k_rate.k, w.k_rate.N)).to(device)
    cv = torch.from_numpy(tables.codebook(dpv, w.v_rate.k, w.v_rate.N)).to(device)
    q = torch.from_numpy(wl.attn_queries(w)).to(device)
    kx = torch.from_numpy(wl.attn_kv(w, "K")).to(device)
    vx = torch.from_numpy(wl.attn_kv(w, "V")).to(device)
    kc, kn = fq.fq_encode(kx.reshape(-1, w.d), rk, ck, w.k_rate.k, w.k_rate.N)
    vc, vn = fq.fq_encode(vx.reshape(-1, w.d), rv, cv, w.v_rate.k, w.v_rate.N)
    # sanity metric: exact softmax attention over the uncompressed fp16 cache (plain PyTorch,
    # fp32), to compare the compressed step's output with by cosine similarity
    G = w.hq // w.hkv
    qf = q.float().reshape(w.batch, w.hkv, G, w.d)
    s = torch.einsum("bhgd,bhtd->bhgt", qf, kx.float()) / math.sqrt(w.d)
    exact = torch.einsum("bhgt,bhtd->bhgd", torch.softmax(s, dim=-1), vx.float())
    exact = exact.reshape(w.batch, w.hq, w.d)
    del kx, vx, s
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

    def cosine():
        launch(0)
        torch.cuda.synchronize()
        cs = torch.nn.functional.cosine_similarity(out, exact, dim=-1)
        return float(cs.mean()), float(cs.min())

    g = torch.Generator(device=device)
    g.manual_seed(7)
    lengths = torch.randint(1, w.tokens + 1, (w.batch,), dtype=torch.int32, device=device,
                            generator=g)
    lengths_app = torch.empty_like(lengths)
    k_new = torch.randn((w.batch, w.hkv, w.d), generator=g, device=device).half()
    v_new = torch.randn((w.batch, w.hkv, w.d), generator=g, device=device).half()

    def launch_lengths():
        fq.fq_attn_decode_lengths(q, lengths, kcs[0], kns[0], w.k_rate.k, w.k_rate.N, rk, ck,
                                  vcs[0], vns[0], w.v_rate.k, w.v_rate.N, rv, cv,
                                  scale=1 / math.sqrt(w.d), out=out, workspace=ws)

    def launch_append():
        fq.fq_attn_decode_append(q, k_new, v_new, lengths_app, kcs[1], kns[1], w.k_rate.k,
                                 w.k_rate.N, rk, ck, vcs[1], vns[1], w.v_rate.k, w.v_rate.N, rv,
                                 cv, scale=1 / math.sqrt(w.d), out=out, workspace=ws)

    def reset_append(start):
        lengths_app.fill_(start)
    extra = {"lengths": lengths, "launch_lengths": launch_lengths,
             "launch_append": launch_append, "reset_append": reset_append}
    return launch, step_bytes, cosine, extra


def attn_bench(torch, fq, timer, device, rank, hbm):
    launch, attn_bytes, cosine, extra = attn_state(torch, fq, device, 4, rank)
    for c in range(4):
        launch(c)
    torch.cuda.synchronize()
    graphs = [timer.capture([lambda c=c: launch(c)]) for c in range(4)]
    for g in graphs:
        g.replay()
    reps = timer.adaptive_reps(graphs, target_s=0.25, lo=20, hi=2000)
    us = timer.time(graphs, reps) * 1e3 / reps
    del graphs
    cmean, cmin = cosine()
    gbs = attn_bytes / (us * 1e-6) / 1e9
    # random access: per-sequence lengths (random in [1, T]) and the step that appends its token
    # (CUDA-graph replay like the full step: device time, no host launch overhead)
    w = wl.ATTN
    per_tok = attn_bytes / (w.batch * w.hkv * w.tokens)
    extra["reset_append"](w.tokens // 2)
    extra["launch_lengths"]()   # eager once before capture (library set-up of each entry point)
    extra["launch_append"]()
    torch.cuda.synchronize()
    g_len = timer.capture([extra["launch_lengths"]])
    g_len.replay()
    reps_len = timer.adaptive_reps([g_len], target_s=0.1, lo=20, hi=1000)
    us_len = timer.time([g_len], reps_len) * 1e3 / reps_len
    len_bytes = float(extra["lengths"].sum().item()) * w.hkv * per_tok
    g_app = timer.capture([extra["launch_append"]])  # capture records the step, runs nothing
    extra["reset_append"](w.tokens // 2)
    torch.cuda.synchronize()
    us_app = timer.time([g_app], 50) * 1e3 / 50
    del g_len, g_app
    app_tokens = w.tokens // 2 + 26   # lengths advance by one per call: mean over the calls
    app_bytes = w.batch * w.hkv * app_tokens * per_tok
    return {"workload": wl.ATTN.name, "us_per_step": round(us, 2), "bytes_per_step": attn_bytes,
            "reps": reps,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4)},
            "launches_per_step": 2,
            "cosine_vs_exact_fp16_attention": {"mean": round(cmean, 5), "min": round(cmin, 5)},
            "lengths": {"us_per_step": round(us_len, 2), "bytes_per_step": int(len_bytes),
                        "hbm_frac": round(len_bytes / (us_len * 1e-6) / 1e9 / hbm, 4),
                        "lengths": "uniform random in [1, T] per sequence"},
            "append": {"us_per_step": round(us_app, 2), "bytes_per_step": int(app_bytes),
                       "hbm_frac": round(app_bytes / (us_app * 1e-6) / 1e9 / hbm, 4),
                       "launches_per_step": 4,
                       "step": "encode K, V of the new token into slot lengths[b], attend over "
                               "lengths[b] + 1 tokens, advance lengths (from T/2)"}}


# ----------------------------------------------------------------------------- the other rows

def _time_ms(torch, fn, reps=None, target_s=0.2):
    """Mean device ms of fn() (eager C-ABI calls on the current stream, CUDA events)."""
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if reps is None:
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        reps = max(3, min(200, int(target_s * 1e3 / max(e0.elapsed_time(e1), 1e-3))))
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def rows_bench(torch, fq, device, hbm, tflops):
    """Throughput lines of the rows beyond the main codec step, each on a synthetic input of the
    pages' workload shapes: half- and full-vector codes (the 34x end of the frontier), scalar
    TurboQuant (k = 1) as the same-box baseline codec, the variants (BlockQuant rescale with a
    stored rho, TurboQuant_prod), and random access (gather-decode of a token list, attention
    over per-sequence lengths, the decode step that appends its own token)."""
    from random_access_kv_fq_b200 import tables
    out = {}
    shape = wl.GPT2.cache
    n, d = shape.n, shape.d
    x = torch.from_numpy(wl.cache(shape, workers=min(32, len(os.sched_getaffinity(0))))).to(device)
    rot64 = {dp: torch.from_numpy(tables.rotation(dp, wl.ROT_SEED_K)).to(device) for dp in (64, 66)}

    def line(ms, vecs, alg_bytes, **extra):
        gbs = alg_bytes / (ms * 1e-3) / 1e9
        o = {"avg_us": round(ms * 1e3, 2), "vectors": vecs,
             "Gvec_s": round(vecs / (ms * 1e-3) / 1e9, 4), "GBps_alg": round(gbs, 1),
             "hbm_frac": round(gbs / hbm, 4)}
        o.update(extra)
        return o

    # half- and full-vector codes on the GPT-2-shaped cache: tensor-core GEMM search
    hk = {}
    for k in (32, 64):
        N = 32768
        cbn = tables.codebook(64, k, N)
        cb = torch.from_numpy(cbn).to(device)
        ix = torch.from_numpy(fq.fq_build_search_index(cbn, 64, k, N, fq.FQ_INDEX_TENSOR, 0, 0)).to(device)
        P = fq.fq_payload_bytes(64, k, N)
        codes = torch.empty((n, P), dtype=torch.uint8, device=device)
        norms = torch.empty((n,), dtype=torch.int16, device=device)
        y = torch.empty((n, d), dtype=torch.float16, device=device)
        me = _time_ms(torch, lambda: fq.fq_encode(x, rot64[64], cb, k, N, codes=codes, norms=norms,
                                                  search_index=ix), reps=3)
        md = _time_ms(torch, lambda: fq.fq_decode(codes, norms, rot64[64], cb, 64, k, N, y=y))
        m = 64 // k
        issued = 2.0 * n * m * N * (3 * k + 16)
        search = 2.0 * n * m * N * k
        hk[f"k{k}N{N}"] = {
            "encode": line(me, n, n * (2 * d + P + 2), bound="tensor",
                           tflops_issued=round(issued / (me * 1e-3) / 1e12, 1),
                           tensor_frac=round(issued / (me * 1e-3) / 1e12 / tflops, 4),
                           tflops_search=round(search / (me * 1e-3) / 1e12, 1)),
            "decode": line(md, n, n * (P + 2 + 2 * d)),
            "compression": {"pages_16_over_b": round(16 / (15 / k), 2),
                            "true_fp16_over_record": round(2 * d / (P + 2), 2)}}
        del codes, norms, y, ix
    out["high_k"] = {"workload": wl.GPT2.name, "codebook": "Lloyd tables N = 2^15", **hk}

    # scalar TurboQuant (k = 1, b = 2) on the same cache: the baseline codec of Thm 2
    c1 = torch.from_numpy(tables.codebook(64, 1, 4)).to(device)
    P1 = fq.fq_payload_bytes(64, 1, 4)
    codes = torch.empty((n, P1), dtype=torch.uint8, device=device)
    norms = torch.empty((n,), dtype=torch.int16, device=device)
    y = torch.empty((n, d), dtype=torch.float16, device=device)
    me = _time_ms(torch, lambda: fq.fq_encode(x, rot64[64], c1, 1, 4, codes=codes, norms=norms))
    md = _time_ms(torch, lambda: fq.fq_decode(codes, norms, rot64[64], c1, 64, 1, 4, y=y))
    out["scalar_turboquant_k1N4"] = {"encode": line(me, n, n * (2 * d + P1 + 2)),
                                     "decode": line(md, n, n * (P1 + 2 + 2 * d)),
                                     "path": "generic kernels (tiled FFMA rotation)"}

    # variants on the same cache: BlockQuant rescale (k = 3, N = 64) and TurboQuant_prod (b = 2)
    cb3n = tables.codebook(66, 3, 64)
    cb3 = torch.from_numpy(cb3n).to(device)
    ix3 = torch.from_numpy(fq.fq_build_search_index(cb3n, 64, 3, 64, fq.FQ_INDEX_EXACT, 20,
                                                    8)).to(device)  # the GPT-2 k3N64 search
    P3 = fq.fq_payload_bytes(64, 3, 64)
    st = {}
    me = _time_ms(torch, lambda: st.__setitem__("r", fq.fq_encode_rho(x, rot64[66], cb3, 3, 64,
                                                                       search_index=ix3)))
    codes3, norms3, rho = st["r"]
    md = _time_ms(torch, lambda: fq.fq_decode_rescaled(codes3, norms3, rho, rot64[66], cb3, 64, 3,
                                                       64, fq.FQ_RESCALE_MSE,
                                                       out_dtype=torch.float16))
    var = {"rescale_k3N64": {"encode_rho": line(me, n, n * (2 * d + P3 + 4)),
                             "decode_mse_rule": line(md, n, n * (P3 + 4 + 2 * d)),
                             "path": "the d = 64 tensor-core kernels: encode with the exact grid "
                                     "index (L20 c8) and rho, decode with S(rho) in the norm "
                                     "scale"}}
    c12 = torch.from_numpy(tables.codebook(64, 1, 2).ravel().copy()).to(device)
    S = torch.from_numpy(np.random.default_rng(1234).standard_normal((64, 64)).astype(np.float32)).to(device)
    me = _time_ms(torch, lambda: st.__setitem__("p", fq.fq_encode_prod(x, rot64[64], c12, S)))
    pc, ps, pn, pg = st["p"]
    md = _time_ms(torch, lambda: fq.fq_decode_prod(pc, ps, pn, pg, rot64[64], c12, S, 64,
                                                   out_dtype=torch.float16))
    rec = pc.shape[1] + ps.shape[1] + 4
    var["turboquant_prod_b2"] = {"encode": line(me, n, n * (2 * d + rec)),
                                 "decode": line(md, n, n * (rec + 2 * d))}
    out["variants"] = var
    del codes, norms, y, codes3, norms3, rho, pc, ps, pn, pg, x, st
    torch.cuda.empty_cache()

    # random access: gather-decode of a random eighth of a 4 M-record plane (d = 128, k = 4,
    # N = 4096; the decode's cost does not depend on the record values, so they are random)
    nr = 1 << 22
    cb128 = torch.from_numpy(tables.codebook(128, 4, 4096)).to(device)
    rot128 = torch.from_numpy(tables.rotation(128, wl.ROT_SEED_K)).to(device)
    g = torch.Generator(device=device)
    g.manual_seed(5)
    rcodes = torch.randint(0, 256, (nr, 48), dtype=torch.uint8, device=device, generator=g)
    rnorms = torch.full((nr,), 0x3C00, dtype=torch.int16, device=device)   # fp16 1.0
    ids = torch.randint(0, nr, (nr // 8,), dtype=torch.int64, device=device, generator=g)
    yg = torch.empty((nr // 8, 128), dtype=torch.float16, device=device)
    mg = _time_ms(torch, lambda: fq.fq_decode_gather(rcodes, rnorms, ids, rot128, cb128, 128, 4,
                                                     4096, y=yg))
    ra = {"gather_decode_d128_k4N4096": line(mg, nr // 8, (nr // 8) * (48 + 2 + 8 + 256),
                                             ids=nr // 8, plane=nr)}
    del rcodes, rnorms, ids, yg
    out["random_access"] = ra
    return out


# ----------------------------------------------------------------------------- arms

def compression(w, fq):
    out = {}
    d = w.cache.d
    for r in w.rates:
        P = fq.fq_payload_bytes(d, r.k, r.N)
        b = math.log2(r.N) / r.k
        out[r.label] = {"bits_per_coord": round(b, 4), "pages_16_over_b": round(16 / b, 2),
                        "true_fp16_over_record": round(2 * d / (P + 2), 2)}
    return out


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
    hbm, hbm_src = peaks()
    timer = GraphTimer(torch, device, dist)
    w = pick_workload(args)

    # ---- headline: the step over the named workload, with clocks sampled during the region
    run = build_codec_run(torch, fq, w, rank, device)
    clk = ClockSampler(torch, local)
    total_ms, meta = time_codec_step(timer, fq, run, args.steps, args.warmup, clocks=clk)
    step_eq = sum(m[3] for m in meta)
    value = whole_job_rate(world, step_eq, args.steps, total_ms)
    per = kernel_table(timer, fq, run, lambda c: codec_launches(fq, run, c, (c - 1) % run.copies),
                       hbm)
    extra = kernel_table(timer, fq, run, lambda c: extra_launches(fq, run, c), hbm) \
        if run.extra else {}
    dom_lab = max(per, key=lambda k: per[k]["ms"] * per[k]["per_step"])
    dom = per[dom_lab]
    traffic = profiled_traffic(w.name, dom_lab, run.shape.d, dom["vectors"])
    step_rates, extra_rates = step_and_extra_rates(w)
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp16->u8->fp16",
        "data": "synthetic (seeded KV-cache recipe of the pages' workloads, no model weights)",
        "config": {"workload": w.name, "vectors_per_gpu": run.shape.n, "d": run.shape.d,
                   "step_rates": [r.label for r in step_rates],
                   "extra_kernels": [f"encode_{r.label}" for r in extra_rates],
                   "io": "fp16 in -> u8 records + fp16 norms -> fp16 out",
                   "math": "fp32 (tensor-core operands split into fp16 hi + lo)",
                   "l2": (f"inputs {run.copies} copies, >= 2x L2 between reuses" if run.copies > 1
                          else "inputs larger than 2x L2 (no reuse within a step)"),
                   "step": "encode K,V + decode K,V (fp16 out) per step rate",
                   "launch": "CUDA graph replay of the step's C-ABI calls"},
        "roofline": {"bound": "hbm", "kernel": dom_lab,
                     "achieved": round(dom["GBps"], 1), "peak": hbm, "peak_source": hbm_src,
                     "unit": "GB/s", "frac": round(dom["frac"], 4), "traffic": traffic,
                     "alg_bytes_per_launch": dom["alg_bytes"],
                     "alg_bytes_per_vector": dom["alg_bytes"] // dom["vectors"]},
        "kernels": kernels_json(per),
        "extra_kernels": kernels_json(extra, with_share=False),
        "gpu_launches": len(meta) * args.steps,
        "clocks": clk.summary(),
        "compression": compression(w, fq),
    }
    # ---- end to end through the public API with pinned host buffers (headline workload)
    if not args.no_e2e:
        result["e2e"] = e2e(torch, fq, run, args, device, world, dist)
    host_sample = None
    if rank == 0 and not args.no_cpu:
        host_sample = cpu_sample_rows(run.shape)
        host_sample = (host_sample, run.host[host_sample])
    del run
    torch.cuda.empty_cache()

    # ---- the other workloads (their own steps), reported under "configs"
    if not args.no_configs and not args.tokens:
        result["configs"] = {}
        for key, cw in WORKLOADS.items():
            if cw is WORKLOADS[args.workload]:
                continue
            r2 = build_codec_run(torch, fq, cw, rank, device)
            steps2 = max(20, args.steps)
            ms2, meta2 = time_codec_step(timer, fq, r2, steps2, max(3, args.warmup))
            per2 = kernel_table(timer, fq, r2,
                                lambda c: codec_launches(fq, r2, c, (c - 1) % r2.copies), hbm)
            v2 = whole_job_rate(world, sum(m[3] for m in meta2), steps2, ms2)
            result["configs"][cw.name] = {
                "value": round(v2, 2), "unit": "GB/s", "steps": steps2,
                "ms_per_step": round(ms2 / steps2, 4), "vectors_per_gpu": r2.shape.n,
                "rates": [r.label for r in cw.rates], "kernels": kernels_json(per2),
                "compression": compression(cw, fq)}
            del r2
            torch.cuda.empty_cache()

    # ---- fused attention step
    if not args.no_attn:
        result["attn"] = attn_bench(torch, fq, timer, device, rank, hbm)
    # ---- the rows beyond the main step (high-k, scalar baseline, variants, random access)
    if not args.no_configs and not args.tokens:
        result["rows"] = rows_bench(torch, fq, device, hbm, tensor_peak()[0])
    bad = fq.fq_wait_status(clear=True)
    if bad:
        raise RuntimeError(f"{bad} CTAs gave up a bounded wait during the bench")
    if rank == 0:
        if host_sample is not None:
            result["cpu_baseline"] = cpu_baseline(w, args, sample=host_sample)
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def e2e_chunks(n: int) -> int:
    """Row chunks of the end-to-end step over n rows (K then V halves): as many as split both
    halves evenly, up to 32 (the first upload and the last download are the only copies nothing
    overlaps, about 1/chunks of the step each)."""
    half = n // 2
    return next(c for c in (32, 16, 8, 4, 2) if half % (c // 2) == 0)


def e2e(torch, fq, run, args, device, world, dist, chunks=None):
    """Same metric through the public API with host buffers.  Every step copies the pinned host
    cache in, encodes, copies the records out, copies them back in, decodes and copies the fp16
    result out, for each step rate.  The step runs in row chunks (each entirely K or V) over three
    CUDA streams (upload, kernels, download) so that uploads, downloads and kernels overlap.  The
    step's calls are captured once as a CUDA graph and replayed, as in the device-resident
    measurement; every byte still crosses the host link in every step."""
    shape, states = run.shape, run.step
    n, d = shape.n, shape.d
    half = n // 2
    if chunks is None:
        chunks = e2e_chunks(n)
    per = half // (chunks // 2)
    assert per * chunks == n, "chunks must split the K and V halves evenly"
    xh = torch.from_numpy(run.host).pin_memory()
    xd = run.xs[0]
    rec_h = [(torch.empty((n, st.P), dtype=torch.uint8).pin_memory(),
              torch.empty((n,), dtype=torch.int16).pin_memory()) for st in states]
    rec_out = [(torch.empty((n, st.P), dtype=torch.uint8, device=device),
                torch.empty((n,), dtype=torch.int16, device=device)) for st in states]
    rec_in = [(torch.empty((n, st.P), dtype=torch.uint8, device=device),
               torch.empty((n,), dtype=torch.int16, device=device)) for st in states]
    yh = [torch.empty((n, d), dtype=torch.float16).pin_memory() for _ in states]
    yd = [run.ys[0]] + [torch.empty((n, d), dtype=torch.float16, device=device)
                        for _ in states[1:]]
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
        #   sc (kernels):  e0 e1 d0 e2 d1 ...    (e = encode, d = decode; every step rate)
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
                    for r in range(len(states)):
                        rec_in[r][0][sl].copy_(rec_h[r][0][sl], non_blocking=True)
                        rec_in[r][1][sl].copy_(rec_h[r][1][sl], non_blocking=True)
                ev_in[j - 1] = mark(su)
            if j < chunks:
                sl, t = rows(j)
                sc.wait_event(ev_x[j])
                for r, st in enumerate(states):
                    fq.fq_encode(xd[sl], st.rot[t], st.cb, st.rate.k, st.rate.N,
                                 codes=rec_out[r][0][sl], norms=rec_out[r][1][sl],
                                 search_index=st.index, stream=sc)
                ev_enc[j] = mark(sc)
                sd.wait_event(ev_enc[j])
                with torch.cuda.stream(sd):
                    for r in range(len(states)):
                        rec_h[r][0][sl].copy_(rec_out[r][0][sl], non_blocking=True)
                        rec_h[r][1][sl].copy_(rec_out[r][1][sl], non_blocking=True)
                ev_out[j] = mark(sd)
            if j >= 1:
                sl, t = rows(j - 1)
                sc.wait_event(ev_in[j - 1])
                for r, st in enumerate(states):
                    fq.fq_decode(rec_in[r][0][sl], rec_in[r][1][sl], st.rot[t], st.cb, d,
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
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    # the overlapped step must deliver exactly what a plain decode of its records gives
    for r, st in enumerate(states):
        ref = torch.empty((n, d), dtype=torch.float16, device=device)
        for t, sl in (("K", slice(0, half)), ("V", slice(half, n))):
            fq.fq_decode(rec_in[r][0][sl], rec_in[r][1][sl], st.rot[t], st.cb, d, st.rate.k,
                         st.rate.N, y=ref[sl])
        if not torch.equal(ref.cpu(), yh[r]):
            raise RuntimeError(f"overlapped end-to-end step disagrees with a plain decode "
                               f"({st.rate.label})")
        del ref
    torch.cuda.synchronize()
    g1 = time.perf_counter()
    graph.replay()
    torch.cuda.synchronize()
    one = time.perf_counter() - g1
    reps = max(3, min(20, int(1.0 / max(one, 1e-4))))
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


# ----------------------------------------------------------------------------- CPU oracle

def cpu_sample_rows(shape, count=4096):
    """The CPU baseline's sample: rows drawn from the first key slab and the first value slab (so
    that the reference arm regenerates two slabs only, not the whole cache)."""
    per = shape.slab_vectors
    first_v = shape.batch * shape.layers * per
    rng = np.random.default_rng(0)
    k = rng.choice(per, size=min(count // 2, per), replace=False)
    v = first_v + rng.choice(per, size=min(count // 2, per), replace=False)
    return np.sort(np.concatenate([k, v]))


def _oracle_warm(_):
    """Imports the oracle in a pool process before the timed window opens."""
    from oracle import fq_oracle  # noqa: F401
    from random_access_kv_fq_b200 import tables  # noqa: F401
    return 0


def _oracle_worker(job):
    """One host process: encode + pack + decode of its rows with the oracle, repeated until the
    deadline (wall-clock time.time()).  Returns (fp16-equivalent bytes done, seconds)."""
    x, rates, d, deadline, call_rows = job
    from threadpoolctl import threadpool_limits
    from oracle import fq_oracle as fo
    from random_access_kv_fq_b200 import tables
    done = 0
    t0 = time.time()
    with threadpool_limits(1):
        while time.time() < deadline:
            for (k, N) in rates:
                dp = fo.padded_dim(d, k)
                rot, cb = tables.rotation(dp, wl.ROT_SEED_K), tables.codebook(dp, k, N)
                for s in range(0, x.shape[0], call_rows):
                    xc = x[s:s + call_rows]
                    enc = fo.encode(xc, rot, cb, k)
                    fo.decode(fo.pack(enc.idx, N), enc.norms, rot, cb, d, k, N)
                    done += 2 * xc.shape[0] * 2 * d
                    if time.time() >= deadline:
                        break
    return done, time.time() - t0


def cpu_baseline(w, args, budget_s: float = 12.0, sample=None):
    """The CPU oracle, as it stands, on a bounded sample of the workload, one process per host
    core (spawned), each with one BLAS thread: fp16-equivalent GB/s of encode + pack + decode at
    the step's rates (the exact brute-force search: the oracle's definition of the encoder)."""
    import multiprocessing as mp
    shape = w.cache
    if sample is None:
        rows = cpu_sample_rows(shape)
        sample = (rows, wl.rows_of(shape, rows))
    rows, x = sample
    step_rates, _ = step_and_extra_rates(w)
    rates = [(r.k, r.N) for r in step_rates]
    cores = len(os.sched_getaffinity(0))
    call_rows = 16 if shape.d == 128 else 256
    parts = [x[i::cores] for i in range(cores)]
    parts = [p for p in parts if p.shape[0]]
    ctx = mp.get_context("spawn")
    with ctx.Pool(len(parts)) as pool:
        # workers start and import the oracle before the clock: all share one deadline
        pool.map(_oracle_warm, range(len(parts)), chunksize=1)
        deadline = time.time() + budget_s
        res = pool.map(_oracle_worker, [(p, rates, shape.d, deadline, call_rows) for p in parts])
    done = sum(r[0] for r in res)
    el = max(r[1] for r in res)
    return {"value": round(done / el / 1e9, 6), "unit": "GB/s", "cores": len(parts),
            "kind": "oracle",
            "sample": f"{x.shape[0]} vectors of {w.name} (first key and value slabs), "
                      f"encode+pack+decode at {[r.label for r in step_rates]} with the oracle's "
                      f"brute-force encoder, repeated for {el:.1f} s in {len(parts)} spawned "
                      f"processes (fp64 NumPy, 1 BLAS thread each)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = pick_workload(args)
    cb = cpu_baseline(w, args, budget_s=max(3.0, min(20.0, 2.0 * args.steps)))
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "GB/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name,
                       "step_rates": [r.label for r in step_and_extra_rates(w)[0]]},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fibquant", choices=["fibquant", "reference"])
    ap.add_argument("--workload", default="large", choices=list(WORKLOADS))
    ap.add_argument("--no-configs", action="store_true")
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
