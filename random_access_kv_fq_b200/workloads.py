"""Seeded synthetic KV-cache workloads shared by the tests, the oracle checks and the bench.

This module holds random-number recipes and shapes only: none of FibQuant's arithmetic
(no rotation, codebook, search, packing or attention) lives here, so both the CUDA path
and the CPU oracle can take their inputs from it without sharing any method code.

Value recipe (a stand-in for the GPT-2-small / TinyLlama-1.1B caches the FibQuant summary
measures on in its sections 4.2 and 4.3; those weights are not available):

* every element is N(0, 1) times a per-(layer, kv-head, channel) scale exp(sigma * g),
  g ~ N(0, 1), i.e. a log-normal channel scale with log-std sigma;
* with outliers on, one channel per (layer, head) (max(1, round(0.01 d)) = 1 for d = 64)
  is further multiplied by 10;
* the product is rounded to fp16 (round to nearest even) unless the config is fp32.

Layout: a cache is [B, L, H, T, d] (batch, layer, head, token, channel), flattened to
n x d with K first and V second.  Every (tensor, batch, layer) slab has its own seed, so any
slab can be regenerated alone (the oracle checks sampled slabs of the large configs).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator

import numpy as np

_TENSOR_ID = {"K": 0, "V": 1, "Q": 2}


@dataclasses.dataclass(frozen=True)
class CacheShape:
    batch: int
    layers: int
    heads: int
    tokens: int
    d: int
    sigma: float
    outliers: bool
    dtype: str  # "f16" or "f32"
    seed: int

    @property
    def vectors_per_tensor(self) -> int:
        return self.batch * self.layers * self.heads * self.tokens

    @property
    def n(self) -> int:
        """Vectors in the K+V cache."""
        return 2 * self.vectors_per_tensor

    @property
    def slab_vectors(self) -> int:
        return self.heads * self.tokens


@dataclasses.dataclass(frozen=True)
class Rate:
    """A (k, N) operating point and how the encoder searches the codebook: "brute" (all N
    codewords), "exact" (grid candidate lists, L cells per axis, c inline slots per cell) or
    "top" (the approximate grid with the c codewords nearest each cell centre)."""
    k: int
    N: int
    search: str = "brute"
    grid_L: int = 0
    grid_c: int = 0

    @property
    def label(self) -> str:
        s = f"k{self.k}N{self.N}"
        if self.search != "brute":
            s += f"_{self.search}L{self.grid_L}c{self.grid_c}"
        return s


@dataclasses.dataclass(frozen=True)
class CodecWorkload:
    name: str
    cache: CacheShape
    rates: tuple


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    name: str
    batch: int
    hq: int
    hkv: int
    tokens: int
    d: int
    k_rate: Rate
    v_rate: Rate
    cache_sigma: float
    outliers: bool
    seed: int


# The five workloads.  Rotation seeds: 17 for keys, 18 for values; codebook seed 101.
TOY = CodecWorkload(
    "toy_d64_k2N16_f32",
    CacheShape(batch=1, layers=1, heads=1, tokens=2048, d=64, sigma=0.5, outliers=False,
               dtype="f32", seed=1001),
    (Rate(2, 16, "brute"),),
)
GPT2 = CodecWorkload(
    "gpt2small_12Lx12Hx1024T_d64",
    CacheShape(batch=1, layers=12, heads=12, tokens=1024, d=64, sigma=1.0, outliers=True,
               dtype="f16", seed=1002),
    (Rate(3, 64, "exact", grid_L=20, grid_c=8), Rate(4, 8, "brute")),
)
TINYLLAMA = CodecWorkload(
    "tinyllama_22Lx4Hx2048Tx8B_d64",
    CacheShape(batch=8, layers=22, heads=4, tokens=2048, d=64, sigma=1.0, outliers=True,
               dtype="f16", seed=1003),
    (Rate(2, 256, "exact", grid_L=128, grid_c=4), Rate(2, 16, "exact", grid_L=64, grid_c=3),
     Rate(2, 8, "exact", grid_L=32, grid_c=3)),
)
LARGE = CodecWorkload(
    "large_32Lx8Hx32768T_d128",
    CacheShape(batch=1, layers=32, heads=8, tokens=32768, d=128, sigma=1.0, outliers=False,
               dtype="f16", seed=1004),
    (Rate(4, 4096, "brute"), Rate(4, 4096, "top", grid_L=16, grid_c=8)),
)
ATTN = AttnWorkload(
    "attn_B16_Hq32_Hkv4_T32768_d64", batch=16, hq=32, hkv=4, tokens=32768, d=64,
    k_rate=Rate(2, 16), v_rate=Rate(3, 64), cache_sigma=1.0, outliers=True, seed=1005,
)

CODEC_WORKLOADS = {w.name: w for w in (TOY, GPT2, TINYLLAMA, LARGE)}

ROT_SEED_K = 17
ROT_SEED_V = 18
CODEBOOK_SEED = 101


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def channel_scales(shape: CacheShape, tensor: str, layer: int) -> np.ndarray:
    """[H, d] float32 multiplicative channel scales for one layer of one tensor."""
    rng = _rng(shape.seed, _TENSOR_ID[tensor], 1_000_000 + layer)
    s = np.exp(shape.sigma * rng.standard_normal((shape.heads, shape.d))).astype(np.float32)
    if shape.outliers:
        n_out = max(1, int(round(0.01 * shape.d)))
        for h in range(shape.heads):
            ch = rng.choice(shape.d, size=n_out, replace=False)
            s[h, ch] *= np.float32(10.0)
    return s


def slab(shape: CacheShape, tensor: str, b: int, layer: int) -> np.ndarray:
    """One (batch, layer) slab of a tensor: [H*T, d] in the cache dtype."""
    scales = channel_scales(shape, tensor, layer)
    rng = _rng(shape.seed, _TENSOR_ID[tensor], b, layer)
    v = rng.standard_normal((shape.heads, shape.tokens, shape.d), dtype=np.float32)
    v *= scales[:, None, :]
    v = v.reshape(-1, shape.d)
    return v.astype(np.float16) if shape.dtype == "f16" else v


def slabs(shape: CacheShape) -> Iterator[tuple[int, np.ndarray]]:
    """Yield (first flat row, slab) over the whole K+V cache in flat order."""
    row = 0
    for tensor in ("K", "V"):
        for b in range(shape.batch):
            for layer in range(shape.layers):
                s = slab(shape, tensor, b, layer)
                yield row, s
                row += s.shape[0]


def cache(shape: CacheShape, workers: int = 1) -> np.ndarray:
    """The whole flat [n, d] K+V cache (host memory).  Slabs are independent, so `workers`
    threads may draw them at once (NumPy's generators release the GIL); the result does not
    depend on `workers`."""
    dt = np.float16 if shape.dtype == "f16" else np.float32
    out = np.empty((shape.n, shape.d), dtype=dt)
    jobs = [(tensor, b, layer) for tensor in ("K", "V") for b in range(shape.batch)
            for layer in range(shape.layers)]

    def fill(i):
        s = slab(shape, *jobs[i])
        out[i * s.shape[0]:(i + 1) * s.shape[0]] = s

    if workers <= 1:
        for i in range(len(jobs)):
            fill(i)
    else:
        import concurrent.futures as cf
        with cf.ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(fill, range(len(jobs))))
    return out


def rows_of(shape: CacheShape, rows: np.ndarray) -> np.ndarray:
    """Regenerate selected flat rows without building the whole cache."""
    rows = np.asarray(rows, dtype=np.int64)
    dt = np.float16 if shape.dtype == "f16" else np.float32
    out = np.empty((rows.size, shape.d), dtype=dt)
    per = shape.slab_vectors
    slab_id = rows // per
    for sid in np.unique(slab_id):
        sel = np.nonzero(slab_id == sid)[0]
        tensor = "K" if sid < shape.batch * shape.layers else "V"
        rem = sid % (shape.batch * shape.layers)
        b, layer = divmod(int(rem), shape.layers)
        s = slab(shape, tensor, b, layer)
        out[sel] = s[rows[sel] - sid * per]
    return out


def attn_cache_shape(w: AttnWorkload) -> CacheShape:
    """K/V of the attention workload, drawn like the TinyLlama cache: one layer, [B, Hkv, T, d]."""
    return CacheShape(batch=w.batch, layers=1, heads=w.hkv, tokens=w.tokens, d=w.d,
                      sigma=w.cache_sigma, outliers=w.outliers, dtype="f16", seed=w.seed)


def attn_queries(w: AttnWorkload) -> np.ndarray:
    """[B, Hq, d] fp16 queries, N(0, 1)."""
    rng = _rng(w.seed, _TENSOR_ID["Q"])
    return rng.standard_normal((w.batch, w.hq, w.d), dtype=np.float32).astype(np.float16)


def attn_kv(w: AttnWorkload, tensor: str) -> np.ndarray:
    """[B, Hkv, T, d] fp16 keys or values of the attention workload."""
    shape = attn_cache_shape(w)
    out = np.empty((w.batch, w.hkv, w.tokens, w.d), dtype=np.float16)
    for b in range(w.batch):
        out[b] = slab(shape, tensor, b, 0).reshape(w.hkv, w.tokens, w.d)
    return out


def small_attn(batch=2, hq=8, hkv=2, tokens=300, d=64, seed=77) -> AttnWorkload:
    """A reduced attention workload with the same recipe (for oracle-sized parity)."""
    return AttnWorkload(f"attn_small_B{batch}_Hq{hq}_Hkv{hkv}_T{tokens}", batch, hq, hkv, tokens,
                        d, Rate(2, 16), Rate(3, 64), 1.0, True, seed)


def gaussian_rows(n: int, d: int, seed: int, dtype=np.float16, sigma: float = 1.0) -> np.ndarray:
    """Plain iid N(0,1) rows with per-channel log-normal scales (parity edge cases)."""
    rng = _rng(seed, 9)
    s = np.exp(sigma * rng.standard_normal(d)).astype(np.float32)
    v = rng.standard_normal((n, d), dtype=np.float32) * s
    return v.astype(dtype)


def fp16_equiv_bytes(n: int, d: int) -> int:
    """Bytes the same vectors occupy as an fp16 cache (the metric's unit)."""
    return 2 * n * d


def human(nbytes: float) -> str:
    units = ["B", "KB", "MB", "GB", "TB"]
    i = int(min(len(units) - 1, max(0, math.floor(math.log(max(nbytes, 1), 1000)))))
    return f"{nbytes / 1000 ** i:.2f} {units[i]}"
