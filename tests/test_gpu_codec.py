"""GPU parity of fq_encode / fq_decode (through the C ABI) against the CPU oracle."""
import numpy as np
import pytest
import torch

import random_access_kv_fq_b200 as fq
from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import tables, workloads as wl
from tests import parity as par

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _index(cb, d, rate):
    if rate.search == "brute":
        return None
    kind = fq.FQ_INDEX_EXACT if rate.search == "exact" else fq.FQ_INDEX_TOPC
    return _dev(fq.fq_build_search_index(cb, d, rate.k, rate.N, kind, rate.grid_L, rate.grid_c))


def _oracle_encode(x, rot, cb, rate):
    if rate.search == "top":
        enc, bd = fo.encode_grid_topc(x, rot, cb, rate.k, rate.grid_L, rate.grid_c)
        return enc, bd[:, :, None] if bd.ndim == 2 else bd
    return fo.encode(x, rot, cb, rate.k), None


def run_codec(x, rot, cb, rate, d, check_decode=True, out16=False):
    """Encode + decode x on the GPU and check both against the oracle.  Returns the GPU
    indices."""
    k, N = rate.k, rate.N
    m = fo.padded_dim(d, k) // k
    xt, rt, ct = _dev(x), _dev(rot), _dev(cb)
    ix = _index(cb, d, rate)
    codes, norms = fq.fq_encode(xt, rt, ct, k, N, search_index=ix)
    torch.cuda.synchronize()
    gcodes, gnorms = par.to_np(codes), par.to_np(norms)
    enc, bd = _oracle_encode(x, rot, cb, rate)
    exempt = None
    if bd is not None:
        exempt = (bd.reshape(enc.idx.shape) < 1e-6)
    gidx = par.check_records_and_indices(gcodes, enc, N, m, exempt)
    par.check_norms(gnorms, enc)
    if check_decode:
        y = fq.fq_decode(codes, norms, rt, ct, d, k, N)
        torch.cuda.synchronize()
        ref = par.check_recon(par.to_np(y), gidx, gnorms, rot, cb, d)
        if out16:
            y16 = fq.fq_decode(codes, norms, rt, ct, d, k, N, out_dtype=torch.float16)
            par.check_recon_f16(par.to_np(y16).astype(np.float64), ref)
    return gidx


def _table_inputs(dp, k, N, seed=wl.ROT_SEED_K):
    return tables.rotation(dp, seed), tables.codebook(dp, k, N)


CASES = [(w, r) for w in (wl.TOY, wl.GPT2, wl.TINYLLAMA, wl.LARGE) for r in w.rates]


@pytest.mark.parametrize("w,rate", CASES, ids=[f"{w.name}-{r.label}" for w, r in CASES])
def test_codec_small_slice(w, rate):
    """Rows from every layer/head of the workload, several tiles plus a ragged tail."""
    shape = w.cache
    rng = np.random.default_rng(7)
    n = 2048 + 1000 + 77 if shape.d == 64 else 1024 + 77
    rows = np.sort(rng.choice(shape.n, size=min(n, shape.n), replace=False))
    x = wl.rows_of(shape, rows)
    dp = fo.padded_dim(shape.d, rate.k)
    rot, cb = _table_inputs(dp, rate.k, rate.N)
    run_codec(x, rot, cb, rate, shape.d, out16=True)


@pytest.mark.parametrize("w,rate", CASES, ids=[f"{w.name}-{r.label}" for w, r in CASES])
def test_codec_full_size_sampled(w, rate):
    """The whole workload encoded/decoded in one call each (the launch the bench times);
    sampled rows checked against the oracle one by one."""
    shape = w.cache
    dp = fo.padded_dim(shape.d, rate.k)
    rot, cb = _table_inputs(dp, rate.k, rate.N)
    k, N = rate.k, rate.N
    m = dp // k
    x = torch.empty((shape.n, shape.d), dtype=torch.float16 if shape.dtype == "f16" else torch.float32,
                    device="cuda")
    for row, s in wl.slabs(shape):
        x[row:row + s.shape[0]].copy_(torch.from_numpy(s))
    rt, ct = _dev(rot), _dev(cb)
    ix = _index(cb, shape.d, rate)
    codes, norms = fq.fq_encode(x, rt, ct, k, N, search_index=ix)
    y = fq.fq_decode(codes, norms, rt, ct, shape.d, k, N)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    sample = np.sort(rng.choice(shape.n, size=min(4096, shape.n), replace=False))
    sample = np.unique(np.concatenate([sample, [0, shape.n - 1]]))
    st = torch.from_numpy(sample).cuda()
    xs = wl.rows_of(shape, sample)
    np.testing.assert_array_equal(par.to_np(x[st]), xs)
    gcodes = par.to_np(codes[st])
    gnorms = par.to_np(norms[st])
    enc, bd = _oracle_encode(xs, rot, cb, rate)
    exempt = None if bd is None else (bd.reshape(enc.idx.shape) < 1e-6)
    gidx = par.check_records_and_indices(gcodes, enc, N, m, exempt)
    par.check_norms(gnorms, enc)
    par.check_recon(par.to_np(y[st]), gidx, gnorms, rot, cb, shape.d)


# ------------------------------------------------------------------ edge cases

def test_empty_and_single():
    rot, cb = _table_inputs(64, 2, 16)
    x = torch.empty((0, 64), dtype=torch.float16, device="cuda")
    codes, norms = fq.fq_encode(x, _dev(rot), _dev(cb), 2, 16)
    assert codes.shape[0] == 0
    x1 = wl.gaussian_rows(1, 64, 3)
    run_codec(x1, rot, cb, wl.Rate(2, 16), 64)


def test_zero_vectors_and_extremes():
    rot, cb = _table_inputs(64, 2, 16)
    x = wl.gaussian_rows(300, 64, 4)
    x[5] = 0
    x[17] = 0
    x[40] = np.float16(65504.0)       # largest fp16: norm overflows fp16 -> inf
    x[41] = np.float16(6e-8)          # subnormal inputs
    x[42, 3] = np.float16(-1.0)
    x[42, :3] = 0
    x[42, 4:] = 0                     # a one-hot vector
    run_codec(x, rot, cb, wl.Rate(2, 16), 64, check_decode=False)
    xs = np.delete(x, [40], axis=0)   # decode check without the inf-norm row
    run_codec(xs, rot, cb, wl.Rate(2, 16), 64)


def test_codeword_aligned_inputs_reproduce_indices():
    """'Shell' codebooks c_n = u_n / sqrt(m) make every concatenation of codewords a unit
    vector, so x = nu Pi^T zhat has every block exactly on a codeword: the GPU must return
    exactly the constructed indices and decode x back to fp32 accuracy."""
    import math
    for d, k, N in ((64, 2, 16), (64, 4, 8), (64, 2, 256), (128, 4, 64)):
        m = d // k
        rot = tables.rotation(d, 17)
        cb = (fo.init_directions(k, N) / math.sqrt(m)).astype(np.float32)
        rng = np.random.default_rng(d + k + N)
        idx = rng.integers(0, N, size=(500, m))
        zhat = cb.astype(np.float64)[idx].reshape(500, d)
        x = (8.0 * (zhat @ rot.astype(np.float64))).astype(np.float32)
        gidx = run_codec(x, rot, cb, wl.Rate(k, N), d)
        np.testing.assert_array_equal(gidx, idx)


@pytest.mark.parametrize("d,k,N,dtype", [(64, 1, 4, np.float16), (64, 1, 16, np.float32),
                                         (256, 2, 16, np.float16), (128, 2, 16, np.float16),
                                         (96, 5, 32, np.float32), (17, 3, 8, np.float32),
                                         (32, 4, 65536, np.float16), (128, 8, 256, np.float16),
                                         (64, 2, 2, np.float16)])
def test_other_shapes(d, k, N, dtype):
    """Shapes outside the workloads (scalar k = 1, k not dividing d, d = 256, N = 65536)."""
    dp = fo.padded_dim(d, k)
    rot = fo.haar_rotation(dp, 99).astype(np.float32)
    cb = fo.init_codebook(dp, k, N).astype(np.float32) if k > 1 else \
        np.sort(fo.scalar_lloyd(dp, N)).astype(np.float32)[:, None]
    n = 200 if N < 65536 else 40
    x = wl.gaussian_rows(n, d, d * 7 + k, dtype=dtype)
    run_codec(x, rot, cb, wl.Rate(k, N), d, out16=True)


def test_random_access_decode_at_unaligned_offsets():
    """Any token range decodes alone from codes + t0 * P (P = 17: odd byte offsets).  Each
    sub-range decode meets oracle parity on its own records; a range whose start keeps the
    16-byte alignment runs the same kernel as the full decode and matches it bit for bit."""
    rot, cb = _table_inputs(66, 3, 64)
    x = wl.gaussian_rows(1000, 64, 8)
    rt, ct = _dev(rot), _dev(cb)
    codes, norms = fq.fq_encode(_dev(x), rt, ct, 3, 64)
    full = fq.fq_decode(codes, norms, rt, ct, 64, 3, 64)
    torch.cuda.synchronize()
    gcodes, gnorms = par.to_np(codes), par.to_np(norms)
    gidx = fo.unpack(gcodes, 22, 64)
    flat = codes.reshape(-1)
    for t0, cnt in ((1, 5), (333, 100), (999, 1), (7, 993), (16, 500)):
        sub = flat[t0 * 17:(t0 + cnt) * 17].reshape(cnt, 17)
        y = fq.fq_decode(sub, norms[t0:t0 + cnt], rt, ct, 64, 3, 64)
        torch.cuda.synchronize()
        par.check_recon(par.to_np(y), gidx[t0:t0 + cnt], gnorms[t0:t0 + cnt], rot, cb, 64)
        if (t0 * 17) % 16 == 0:
            torch.testing.assert_close(y, full[t0:t0 + cnt], rtol=0, atol=0)


def test_index_with_wrong_codebook_falls_back_to_exact_search():
    """An index built for another (k, N) is ignored (the result is the brute-force one)."""
    rot, cb = _table_inputs(64, 2, 16)
    _, cb8 = _table_inputs(64, 2, 8)
    ix = _dev(fq.fq_build_search_index(cb8, 64, 2, 8, fq.FQ_INDEX_EXACT, 32, 2))
    x = wl.gaussian_rows(500, 64, 9)
    rt, ct = _dev(rot), _dev(cb)
    c1, n1 = fq.fq_encode(_dev(x), rt, ct, 2, 16, search_index=ix)
    c2, n2 = fq.fq_encode(_dev(x), rt, ct, 2, 16)
    assert torch.equal(c1, c2) and torch.equal(n1, n2)


def test_large_grid_index_for_another_codebook_falls_back_to_brute_force():
    """d = 128, N = 4096 with an index built for a 2048-codeword codebook: the grid kernel ignores
    it and searches all 4096 codewords exactly, matching the oracle's brute force."""
    d, k, N = 128, 4, 4096
    rot, cb = tables.rotation(d, wl.ROT_SEED_K), tables.codebook(d, k, N)
    ix = _dev(fq.fq_build_search_index(cb[:2048], d, k, 2048, fq.FQ_INDEX_TOPC, 8, 4))
    x = wl.gaussian_rows(300, d, 11)
    x[3] = 0
    codes, norms = fq.fq_encode(_dev(x), _dev(rot), _dev(cb), k, N, search_index=ix)
    torch.cuda.synchronize()
    enc, _ = _oracle_encode(x, rot, cb, wl.Rate(k, N, "brute"))
    par.check_records_and_indices(par.to_np(codes), enc, N, d // k)
    par.check_norms(par.to_np(norms), enc)


@pytest.mark.parametrize("L,c", [(8, 4), (12, 6), (16, 5)])
def test_large_grid_index_of_other_shapes(L, c):
    """d = 128, N = 4096 with top-c indexes other than 16 cells per axis x 8 candidates: the grid
    kernel's general candidate loop, against the oracle's own top-c search."""
    d = 128
    rate = wl.Rate(4, 4096, "top", L, c)
    rot, cb = tables.rotation(d, wl.ROT_SEED_K), tables.codebook(d, 4, 4096)
    x = wl.rows_of(wl.LARGE.cache, np.arange(0, wl.LARGE.cache.n, wl.LARGE.cache.n // 1100)[:1100])
    x = np.array(x)
    x[5] = 0
    run_codec(x, rot, cb, rate, d)


@pytest.mark.parametrize("dp,k,N", [(64, 2, 16), (66, 3, 64), (64, 4, 8), (64, 2, 256)])
def test_fast_and_generic_paths_meet_parity_on_the_same_rows(dp, k, N):
    """A 16-byte-aligned fp16 input takes the tensor-core kernel; the same rows behind a
    2-byte-offset view take the generic kernel.  Both must meet oracle parity and agree
    everywhere except at oracle near-ties."""
    rot, cb = _table_inputs(dp, k, N)
    x = wl.rows_of(wl.TINYLLAMA.cache, np.arange(0, 2883584, 997)[:1500])
    rt, ct = _dev(rot), _dev(cb)
    m = dp // k
    buf = torch.zeros(x.size + 8, dtype=torch.float16, device="cuda")
    fast_in = buf[:x.size].view(x.shape)
    slow_in = buf[1:1 + x.size].view(x.shape)  # 2-byte offset: not 16-byte aligned
    enc = fo.encode(x, rot, cb, k)
    results = []
    for t in (fast_in, slow_in):
        t.copy_(torch.from_numpy(x))
        codes, norms = fq.fq_encode(t, rt, ct, k, N)
        torch.cuda.synchronize()
        gidx = par.check_records_and_indices(par.to_np(codes), enc, N, m)
        par.check_norms(par.to_np(norms), enc)
        results.append(gidx)
    diff = results[0] != results[1]
    assert not (diff & (enc.gap > par.NEAR_TIE_GAP)).any()


@pytest.mark.parametrize("N", [512, 1024, 2048, 4096])
def test_large_codebook_tensor_core_search(N):
    """d = 128, k = 4, N = 512 .. 4096 without an index runs the tensor-core brute-force search
    with fp32 re-ranking of near ties; indices must match the oracle's brute force (ties to the
    lowest index).  N < 4096 uses unit-ball random codebooks (the search does not depend on
    the codebook being Lloyd-optimal)."""
    d, k = 128, 4
    rot = tables.rotation(d, wl.ROT_SEED_K)
    if N == 4096:
        cb = tables.codebook(d, k, N)
    else:
        rng = np.random.default_rng(N)
        u = rng.standard_normal((N, k))
        u /= np.linalg.norm(u, axis=1, keepdims=True)
        r = rng.beta(k / 2, (d - k) / 2, size=(N, 1)) ** 0.5
        cb = (u * r).astype(np.float32)
    x = wl.gaussian_rows(1000, d, seed=N, sigma=1.0)
    x[7] = 0  # zero vector
    x[8] = x[9]  # duplicate rows
    run_codec(x, rot, cb, wl.Rate(k, N, "brute"), d, out16=True)


@pytest.mark.parametrize("B", [2, 5, 8, 9, 12])
def test_large_decode_tensor_core(B):
    """d = 128, k = 4: the tensor-core decode of arbitrary records (random indices, random
    fp16 norms, a zero norm, a ragged last tile) against the oracle decoder, fp32 and fp16 out;
    several tiles per pipeline."""
    d, k, N = 128, 4, 1 << B
    rng = np.random.default_rng(100 + B)
    rot = tables.rotation(d, wl.ROT_SEED_V)
    u = rng.standard_normal((N, k))
    cb = (u / np.linalg.norm(u, axis=1, keepdims=True) *
          rng.uniform(0.0, 1.0, size=(N, 1))).astype(np.float32)
    n = 3 * 148 * 2 * 128 + 77
    idx = rng.integers(0, N, size=(n, d // k))
    codes = fo.pack(idx, N)
    norms = rng.uniform(0.0, 40.0, size=n).astype(np.float16)
    norms[5] = 0
    ct, nt = torch.from_numpy(codes).cuda(), torch.from_numpy(norms.view(np.int16)).cuda()
    y = fq.fq_decode(ct, nt, _dev(rot), _dev(cb), d, k, N)
    y16 = fq.fq_decode(ct, nt, _dev(rot), _dev(cb), d, k, N, out_dtype=torch.float16)
    torch.cuda.synchronize()
    ref = par.check_recon(par.to_np(y), idx, norms.view(np.int16), rot, cb, d)
    par.check_recon_f16(par.to_np(y16).astype(np.float64), ref)
