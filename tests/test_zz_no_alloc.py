"""The allocation-free attention entry point (fq_attn_decode_noalloc), called through the C ABI.

Some callers cannot allocate device memory (a host application whose allocator owns all GPU
memory, or a decode loop that must not call cudaMalloc).  fq_attn_decode_noalloc serves them
with the library's fixed per-GPU scratch instead of a caller workspace.  This file is named to
be collected last so that a stop-at-first-failure run has already run every other test; it
also passes on its own in a fresh process.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import random_access_kv_fq_b200 as fq
from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import _lib, tables, workloads as wl
from tests import parity as par

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _inputs(w):
    dpk, dpv = fo.padded_dim(w.d, w.k_rate.k), fo.padded_dim(w.d, w.v_rate.k)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, w.k_rate.k, w.k_rate.N)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, w.v_rate.k, w.v_rate.N)
    dev = {}
    for name, rot, cb, rate in (("K", rk, ck, w.k_rate), ("V", rv, cv, w.v_rate)):
        x = _dev(wl.attn_kv(w, name).reshape(-1, w.d))
        codes, norms = fq.fq_encode(x, _dev(rot), _dev(cb), rate.k, rate.N)
        dev[name] = (codes.reshape(w.batch, w.hkv, w.tokens, -1),
                     norms.reshape(w.batch, w.hkv, w.tokens), _dev(rot), _dev(cb), rate)
    return _dev(wl.attn_queries(w)), dev


def _call_noalloc(q, dev, scale, out):
    """Raw C-ABI call: pointers, sizes, stream; no workspace argument."""
    kc, kn, rk, ck, kr = dev["K"]
    vc, vn, rv, cv, vr = dev["V"]
    B, Hq, d = q.shape
    _, Hkv, T, _ = kc.shape
    st = _lib.lib().fq_attn_decode_noalloc(
        q.data_ptr(), B, Hq, Hkv, T, d, kc.data_ptr(), kn.data_ptr(), kr.k, kr.N,
        rk.data_ptr(), ck.data_ptr(), vc.data_ptr(), vn.data_ptr(), vr.k, vr.N, rv.data_ptr(),
        cv.data_ptr(), ctypes.c_float(scale), out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == 0, fq.status_string(st)


@pytest.mark.parametrize("w", [wl.small_attn(tokens=4097, seed=31), wl.ATTN],
                         ids=["small", "full"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(w):
    q, dev = _inputs(w)
    scale = 1 / math.sqrt(w.d)
    kc, kn, rk, ck, kr = dev["K"]
    vc, vn, rv, cv, vr = dev["V"]
    ref = fq.fq_attn_decode(q, kc, kn, kr.k, kr.N, rk, ck, vc, vn, vr.k, vr.N, rv, cv, scale=scale)
    torch.cuda.synchronize()
    ref = par.to_np(ref).astype(np.float64)
    for _ in range(2):  # the second call reuses the scratch the first one left behind
        out = torch.full(ref.shape, float("nan"), dtype=torch.float32, device="cuda")
        _call_noalloc(q, dev, scale, out)
        torch.cuda.synchronize()
        par.check_attention(par.to_np(out), ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """Partials larger than the fixed scratch are refused on the host before any launch (the
    pointers below are never dereferenced)."""
    B, Hq, Hkv, T = 64, 256, 16, 1024
    assert fq.fq_attn_workspace_bytes(B, Hq, Hkv, T, 64, 3) > fq.FQ_ATTN_NOALLOC_SCRATCH_BYTES
    st = _lib.lib().fq_attn_decode_noalloc(16, B, Hq, Hkv, T, 64, 16, 16, 2, 16, 16, 16, 16, 16,
                                           3, 64, 16, 16, ctypes.c_float(0.125), 16,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == 4  # FQ_ERR_WORKSPACE
