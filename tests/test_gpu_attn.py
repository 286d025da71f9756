"""GPU parity of fq_attn_decode (through the C ABI) against oracle attention over the decoded
cache, plus the rotated-domain identity and degenerate cases."""
import math

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


def _compress_oracle(kv, rot, cb, k, N):
    """Oracle encode of a [B, Hkv, T, d] cache -> CompressedKV."""
    Bn, H, T, d = kv.shape
    enc = fo.encode(kv.reshape(-1, d), rot, cb, k)
    codes = fo.pack(enc.idx, N).reshape(Bn, H, T, -1)
    return fo.CompressedKV(codes, enc.norms.reshape(Bn, H, T), rot, cb, k, N)


def _gpu_attn(q, Kc, Vc, scale):
    out = fq.fq_attn_decode(_dev(q), _dev(Kc.codes), _dev(Kc.norms.view(np.int16)), Kc.k, Kc.N,
                            _dev(Kc.rot), _dev(Kc.codebook), _dev(Vc.codes),
                            _dev(Vc.norms.view(np.int16)), Vc.k, Vc.N, _dev(Vc.rot),
                            _dev(Vc.codebook), scale=scale)
    torch.cuda.synchronize()
    return par.to_np(out)


def _setup(w):
    kv_k = wl.attn_kv(w, "K")
    kv_v = wl.attn_kv(w, "V")
    dpk, dpv = fo.padded_dim(w.d, w.k_rate.k), fo.padded_dim(w.d, w.v_rate.k)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, w.k_rate.k, w.k_rate.N)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, w.v_rate.k, w.v_rate.N)
    Kc = _compress_oracle(kv_k, rk, ck, w.k_rate.k, w.k_rate.N)
    Vc = _compress_oracle(kv_v, rv, cv, w.v_rate.k, w.v_rate.N)
    return wl.attn_queries(w), Kc, Vc, kv_k, kv_v


@pytest.mark.parametrize("T", [1, 63, 300, 4097])
def test_attention_small(T):
    w = wl.small_attn(tokens=T)
    q, Kc, Vc, _, _ = _setup(w)
    scale = 1 / math.sqrt(w.d)
    ref = fo.attention_decoded(q, Kc, Vc, w.d, scale)
    out = _gpu_attn(q, Kc, Vc, scale)
    par.check_attention(out, ref)


def test_attention_gqa_groups_and_scale():
    w = wl.small_attn(batch=3, hq=16, hkv=1, tokens=700, seed=5)
    q, Kc, Vc, _, _ = _setup(w)
    for scale in (0.125, 0.02, 0.5):
        ref = fo.attention_decoded(q, Kc, Vc, w.d, scale)
        par.check_attention(_gpu_attn(q, Kc, Vc, scale), ref)


def test_attention_degenerate_cases():
    """T = 1 gives the decoded value; q = 0 gives the mean of the decoded values."""
    w = wl.small_attn(tokens=1, seed=6)
    q, Kc, Vc, _, _ = _setup(w)
    vdec = fo.decode(Vc.codes.reshape(-1, Vc.codes.shape[-1]), Vc.norms.reshape(-1), Vc.rot,
                     Vc.codebook, w.d, Vc.k, Vc.N).reshape(w.batch, w.hkv, 1, w.d)
    out = _gpu_attn(q, Kc, Vc, 0.125)
    G = w.hq // w.hkv
    for b in range(w.batch):
        for h in range(w.hq):
            np.testing.assert_allclose(out[b, h], vdec[b, h // G, 0], rtol=1e-5,
                                       atol=1e-5 * np.abs(vdec).max())
    w2 = wl.small_attn(tokens=500, seed=8)
    q2, Kc2, Vc2, _, _ = _setup(w2)
    q2 = np.zeros_like(q2)
    out2 = _gpu_attn(q2, Kc2, Vc2, 0.125)
    vdec2 = fo.decode(Vc2.codes.reshape(-1, Vc2.codes.shape[-1]), Vc2.norms.reshape(-1), Vc2.rot,
                      Vc2.codebook, w2.d, Vc2.k, Vc2.N).reshape(w2.batch, w2.hkv, 500, w2.d)
    mean = vdec2.mean(axis=2)
    G2 = w2.hq // w2.hkv
    for h in range(w2.hq):
        par.check_attention(out2[:, h:h + 1], mean[:, h // G2][:, None])


def test_attention_empty_context_is_zero():
    w = wl.small_attn(tokens=4, seed=9)
    q, Kc, Vc, _, _ = _setup(w)
    empty = lambda c: c[:, :, :0]
    out = fq.fq_attn_decode(_dev(q), _dev(empty(Kc.codes)), _dev(empty(Kc.norms).view(np.int16)),
                            2, 16, _dev(Kc.rot), _dev(Kc.codebook), _dev(empty(Vc.codes)),
                            _dev(empty(Vc.norms).view(np.int16)), 3, 64, _dev(Vc.rot),
                            _dev(Vc.codebook))
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_attention_full_size_all_groups():
    """The full decode step (B16, Hq32/Hkv4, T32768) on a GPU-encoded cache; every (b, kv head)
    group (so every context split of the launch) checked against the oracle over the
    oracle-decoded GPU records."""
    w = wl.ATTN
    shape = wl.attn_cache_shape(w)
    dpk, dpv = fo.padded_dim(w.d, 2), fo.padded_dim(w.d, 3)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, 2, 16)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, 3, 64)
    tensors = {}
    for name, rot, cb, k, N in (("K", rk, ck, 2, 16), ("V", rv, cv, 3, 64)):
        x = torch.from_numpy(wl.attn_kv(w, name).reshape(-1, w.d)).cuda()
        codes, norms = fq.fq_encode(x, _dev(rot), _dev(cb), k, N)
        tensors[name] = (codes.reshape(w.batch, w.hkv, w.tokens, -1),
                         norms.reshape(w.batch, w.hkv, w.tokens))
    q = wl.attn_queries(w)
    out = fq.fq_attn_decode(_dev(q), *tensors["K"], 2, 16, _dev(rk), _dev(ck), *tensors["V"], 3,
                            64, _dev(rv), _dev(cv), scale=1 / math.sqrt(w.d))
    torch.cuda.synchronize()
    out = par.to_np(out)
    G = w.hq // w.hkv
    for b, g in ((b, g) for b in range(w.batch) for g in range(w.hkv)):
        Kc = fo.CompressedKV(par.to_np(tensors["K"][0][b:b + 1, g:g + 1]),
                             par.to_np(tensors["K"][1][b:b + 1, g:g + 1]).view(np.float16),
                             rk, ck, 2, 16)
        Vc = fo.CompressedKV(par.to_np(tensors["V"][0][b:b + 1, g:g + 1]),
                             par.to_np(tensors["V"][1][b:b + 1, g:g + 1]).view(np.float16),
                             rv, cv, 3, 64)
        ref = fo.attention_decoded(q[b:b + 1, g * G:(g + 1) * G], Kc, Vc, w.d, 1 / math.sqrt(w.d))
        par.check_attention(out[b:b + 1, g * G:(g + 1) * G], ref)


@pytest.mark.parametrize("hq,hkv,T", [(16, 2, 1), (16, 2, 129), (16, 2, 1000), (32, 2, 700),
                                      (8, 1, 5000), (16, 1, 256)])
def test_attention_tensor_core_groups(hq, hkv, T):
    """Group sizes 8 and 16 take the tensor-core kernel: ragged tiles, one token, long splits."""
    w = wl.small_attn(batch=2, hq=hq, hkv=hkv, tokens=T, seed=hq + T)
    q, Kc, Vc, _, _ = _setup(w)
    for scale in (1 / math.sqrt(w.d), 0.5):
        ref = fo.attention_decoded(q, Kc, Vc, w.d, scale)
        par.check_attention(_gpu_attn(q, Kc, Vc, scale), ref)


def test_attention_tensor_core_degenerate():
    """T = 1 returns the decoded value; q = 0 returns the mean of the decoded values (G = 8)."""
    w = wl.small_attn(batch=2, hq=16, hkv=2, tokens=1, seed=12)
    q, Kc, Vc, _, _ = _setup(w)
    vdec = fo.decode(Vc.codes.reshape(-1, Vc.codes.shape[-1]), Vc.norms.reshape(-1), Vc.rot,
                     Vc.codebook, w.d, Vc.k, Vc.N).reshape(w.batch, w.hkv, 1, w.d)
    out = _gpu_attn(q, Kc, Vc, 0.125)
    for b in range(w.batch):
        for h in range(w.hq):
            np.testing.assert_allclose(out[b, h], vdec[b, h // 8, 0], rtol=1e-5,
                                       atol=1e-5 * np.abs(vdec).max())
    w2 = wl.small_attn(batch=2, hq=16, hkv=2, tokens=777, seed=13)
    q2, Kc2, Vc2, _, _ = _setup(w2)
    out2 = _gpu_attn(np.zeros_like(q2), Kc2, Vc2, 0.125)
    vdec2 = fo.decode(Vc2.codes.reshape(-1, Vc2.codes.shape[-1]), Vc2.norms.reshape(-1), Vc2.rot,
                      Vc2.codebook, w2.d, Vc2.k, Vc2.N).reshape(w2.batch, w2.hkv, 777, w2.d)
    mean = vdec2.mean(axis=2)
    for h in range(w2.hq):
        par.check_attention(out2[:, h:h + 1], mean[:, h // 8][:, None])


def _misaligned(a, shift_elems):
    """A device copy of `a` whose data pointer sits `shift_elems` elements past an aligned
    allocation (odd byte offsets for records, 2-byte offsets for norms)."""
    t = torch.from_numpy(np.ascontiguousarray(a))
    buf = torch.empty(t.numel() + shift_elems, dtype=t.dtype, device="cuda")
    view = buf[shift_elems:].view(t.shape)
    view.copy_(t.cuda())
    return view


@pytest.mark.parametrize("hq,hkv,T,shift", [(16, 2, 1040, 1), (16, 2, 333, 3), (32, 2, 4112, 5),
                                            (8, 1, 700, 7)])
def test_attention_misaligned_caches(hq, hkv, T, shift):
    """Records and norms at arbitrary (byte / element) offsets: tiles whose aligned bulk-copy
    window would leave the buffer are read from global memory directly."""
    w = wl.small_attn(batch=2, hq=hq, hkv=hkv, tokens=T, seed=3 * T + shift)
    q, Kc, Vc, _, _ = _setup(w)
    scale = 1 / math.sqrt(w.d)
    out = fq.fq_attn_decode(_dev(q), _misaligned(Kc.codes, shift),
                            _misaligned(Kc.norms.view(np.int16), 1), Kc.k, Kc.N, _dev(Kc.rot),
                            _dev(Kc.codebook), _misaligned(Vc.codes, shift + 2),
                            _misaligned(Vc.norms.view(np.int16), 3), Vc.k, Vc.N, _dev(Vc.rot),
                            _dev(Vc.codebook), scale=scale)
    torch.cuda.synchronize()
    ref = fo.attention_decoded(q, Kc, Vc, w.d, scale)
    par.check_attention(par.to_np(out), ref)
