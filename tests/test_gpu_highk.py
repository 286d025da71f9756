"""GPU parity of half-vector (k = d/2) and full-vector (k = d) codes through the C ABI: the
tensor-core GEMM search (with an FQ_INDEX_TENSOR index) and the CUDA-core brute force (without
one) against the oracle's brute-force encoder, records, norms and decode."""
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


def _codebook(d, k, N):
    if tables.have(f"cb_d{d}_k{k}_N{N}"):
        return tables.codebook(d, k, N)
    return fo.init_codebook(d, k, N).astype(np.float32)


def _encode_check(x, rot, cb, d, k, N, index):
    m = d // k
    xt = _dev(x)
    codes, norms = fq.fq_encode(xt, _dev(rot), _dev(cb), k, N, search_index=index)
    torch.cuda.synchronize()
    enc = fo.encode(x, rot, cb, k)
    gidx = par.check_records_and_indices(par.to_np(codes), enc, N, m)
    par.check_norms(par.to_np(norms), enc)
    y = fq.fq_decode(codes, norms, _dev(rot), _dev(cb), d, k, N)
    torch.cuda.synchronize()
    par.check_recon(par.to_np(y), gidx, par.to_np(norms), rot, cb, d)
    return codes, norms


@pytest.mark.parametrize("d,k,N,n", [(64, 32, 32768, 700), (64, 64, 32768, 500),
                                     (128, 64, 8192, 500), (64, 32, 256, 3000)])
def test_tensor_core_search_matches_the_oracle(d, k, N, n):
    rot = tables.rotation(d, wl.ROT_SEED_K)
    cb = _codebook(d, k, N)
    ix = _dev(fq.fq_build_search_index(cb, d, k, N, fq.FQ_INDEX_TENSOR, 0, 0))
    x = wl.rows_of(wl.GPT2.cache, np.arange(0, 294912, 294912 // n)[:n]) if d == 64 else \
        wl.gaussian_rows(n, d, seed=k + N)
    x = np.array(x)
    x[3] = 0                 # zero vector
    x[4] = x[5]              # duplicate rows
    _encode_check(x, rot, cb, d, k, N, ix)


def test_without_an_index_the_cuda_core_brute_force_matches():
    d, k, N = 64, 32, 4096
    rot, cb = tables.rotation(d, wl.ROT_SEED_V), _codebook(d, k, N)
    x = wl.gaussian_rows(200, d, seed=3)
    _encode_check(x, rot, cb, d, k, N, None)


def test_index_of_another_codebook_is_ignored():
    """An FQ_INDEX_TENSOR index built for a different N: the kernel ignores it and searches all
    codewords exactly on the CUDA cores (same result as without an index)."""
    d, k, N = 64, 32, 1024
    rot = tables.rotation(d, wl.ROT_SEED_K)
    cb = _codebook(d, k, N)
    other = _dev(fq.fq_build_search_index(cb[:512], d, k, 512, fq.FQ_INDEX_TENSOR, 0, 0))
    x = wl.gaussian_rows(300, d, seed=4)
    c1, n1 = _encode_check(x, rot, cb, d, k, N, other)
    c2, n2 = fq.fq_encode(_dev(x), _dev(rot), _dev(cb), k, N)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(n1, n2)


def test_full_workload_sampled_at_the_34x_point():
    """The whole GPT-2-shaped cache (294,912 vectors) at k = 32, N = 2^15 in one launch (the
    bench's launch); sampled rows checked against the oracle one by one."""
    d, k, N = 64, 32, 32768
    shape = wl.GPT2.cache
    rot, cb = tables.rotation(d, wl.ROT_SEED_K), _codebook(d, k, N)
    ix = _dev(fq.fq_build_search_index(cb, d, k, N, fq.FQ_INDEX_TENSOR, 0, 0))
    x = torch.empty((shape.n, d), dtype=torch.float16, device="cuda")
    for row, s in wl.slabs(shape):
        x[row:row + s.shape[0]].copy_(torch.from_numpy(s))
    codes, norms = fq.fq_encode(x, _dev(rot), _dev(cb), k, N, search_index=ix)
    torch.cuda.synchronize()
    rng = np.random.default_rng(13)
    sample = np.unique(np.concatenate([rng.choice(shape.n, 400, replace=False), [0, shape.n - 1]]))
    xs = wl.rows_of(shape, sample)
    enc = fo.encode(xs, rot, cb, k)
    st = torch.from_numpy(sample).cuda()
    par.check_records_and_indices(par.to_np(codes[st]), enc, N, d // k)
    par.check_norms(par.to_np(norms[st]), enc)
