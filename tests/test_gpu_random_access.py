"""GPU parity of the random-access entry points (through the C ABI) against the oracle:
gather-decode of a token list, attention over per-sequence context lengths, and the decode step
that encodes its own token into the cache.  Records outside a list or past a length are
scrambled with random bytes, which must not change any result (fixed-address independence)."""
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


# ------------------------------------------------------------------ gather-decode

@pytest.mark.parametrize("d,k,N", [(128, 4, 4096), (64, 3, 64), (64, 2, 16)])
def test_gather_decode_matches_the_oracle_and_ignores_other_records(d, k, N):
    dp = fo.padded_dim(d, k)
    rot, cb = tables.rotation(dp, wl.ROT_SEED_V), tables.codebook(dp, k, N)
    n = 5000
    x = wl.gaussian_rows(n, d, seed=d + k + N)
    rt, ct = _dev(rot), _dev(cb)
    codes, norms = fq.fq_encode(_dev(x), rt, ct, k, N)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    ids = np.concatenate([[n - 1, 0, 17, 17], rng.integers(0, n, size=700)]).astype(np.int64)
    idt = _dev(ids)
    y = fq.fq_decode_gather(codes, norms, idt, rt, ct, d, k, N)
    y16 = fq.fq_decode_gather(codes, norms, idt, rt, ct, d, k, N, out_dtype=torch.float16)
    torch.cuda.synchronize()
    gcodes, gnorms = par.to_np(codes), par.to_np(norms)
    m = dp // k
    ref = fo.decode_tokens(gcodes, gnorms.view(np.float16), ids, rot, cb, d, k, N)
    par.check_recon(par.to_np(y), fo.unpack(gcodes[ids], m, N), gnorms[ids], rot, cb, d)
    par.check_recon_f16(par.to_np(y16).astype(np.float64), ref)
    # records not in the list hold random bytes: the result is unchanged, bit for bit
    keep = np.zeros(n, dtype=bool)
    keep[ids] = True
    sc, sn = gcodes.copy(), gnorms.copy()
    sc[~keep] = rng.integers(0, 256, size=sc[~keep].shape, dtype=np.uint8)
    sn[~keep] = rng.integers(0, 1 << 15, size=int((~keep).sum())).astype(np.int16)
    y2 = fq.fq_decode_gather(_dev(sc), _dev(sn), idt, rt, ct, d, k, N)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    # the listed rows equal a plain decode of the whole plane (same kernel for d = 128)
    full = fq.fq_decode(codes, norms, rt, ct, d, k, N)
    torch.cuda.synchronize()
    if d == 128:
        assert torch.equal(y, full[idt])
    else:
        par.check_recon(par.to_np(full[idt]), fo.unpack(gcodes[ids], m, N), gnorms[ids], rot, cb, d)


def test_gather_decode_out_of_range_ids_give_nan_rows_and_empty_lists():
    d, k, N = 128, 4, 4096
    rot, cb = tables.rotation(d, 17), tables.codebook(d, k, N)
    x = wl.gaussian_rows(300, d, seed=1)
    rt, ct = _dev(rot), _dev(cb)
    codes, norms = fq.fq_encode(_dev(x), rt, ct, k, N)
    ids = _dev(np.array([5, -1, 300, 299, 1 << 40], dtype=np.int64))
    for dd, kk, NN, c, nm, r_, cb_ in ((d, k, N, codes, norms, rt, ct),):
        y = fq.fq_decode_gather(c, nm, ids, r_, cb_, dd, kk, NN)
        torch.cuda.synchronize()
        bad = torch.isnan(y).all(dim=1).cpu().numpy()
        assert bad.tolist() == [False, True, True, False, True]
    # d = 64 through the generic kernel
    rot64, cb64 = tables.rotation(66, 18), tables.codebook(66, 3, 64)
    c64, n64 = fq.fq_encode(_dev(wl.gaussian_rows(40, 64, seed=2)), _dev(rot64), _dev(cb64), 3, 64)
    y = fq.fq_decode_gather(c64, n64, _dev(np.array([39, 40, -5], dtype=np.int64)), _dev(rot64),
                            _dev(cb64), 64, 3, 64)
    torch.cuda.synchronize()
    assert torch.isnan(y).all(dim=1).cpu().tolist() == [False, True, True]
    empty = fq.fq_decode_gather(c64, n64, torch.empty(0, dtype=torch.int64, device="cuda"),
                                _dev(rot64), _dev(cb64), 64, 3, 64)
    assert empty.shape == (0, 64)


# ------------------------------------------------------------------ per-sequence lengths

def _caches(w):
    dpk, dpv = fo.padded_dim(w.d, w.k_rate.k), fo.padded_dim(w.d, w.v_rate.k)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, w.k_rate.k, w.k_rate.N)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, w.v_rate.k, w.v_rate.N)
    out = {}
    for name, rot, cb, rate in (("K", rk, ck, w.k_rate), ("V", rv, cv, w.v_rate)):
        kv = wl.attn_kv(w, name)
        codes, norms = fq.fq_encode(_dev(kv.reshape(-1, w.d)), _dev(rot), _dev(cb), rate.k, rate.N)
        torch.cuda.synchronize()
        out[name] = fo.CompressedKV(par.to_np(codes).reshape(w.batch, w.hkv, w.tokens, -1),
                                    par.to_np(norms).view(np.float16).reshape(w.batch, w.hkv, w.tokens),
                                    rot, cb, rate.k, rate.N)
    return wl.attn_queries(w), out["K"], out["V"]


def _scramble_past(c, lengths, rng):
    codes, norms = c.codes.copy(), c.norms.copy()
    for b, L in enumerate(lengths):
        L = max(0, int(L))
        codes[b, :, L:] = rng.integers(0, 256, size=codes[b, :, L:].shape, dtype=np.uint8)
        norms[b, :, L:] = rng.uniform(0.5, 60.0, size=norms[b, :, L:].shape).astype(np.float16)
    return fo.CompressedKV(codes, norms, c.rot, c.codebook, c.k, c.N)


def _gpu_lengths(q, Kc, Vc, lengths, scale):
    t = _dev
    out = fq.fq_attn_decode_lengths(t(q), t(np.asarray(lengths, np.int32)), t(Kc.codes),
                                    t(Kc.norms.view(np.int16)), Kc.k, Kc.N, t(Kc.rot),
                                    t(Kc.codebook), t(Vc.codes), t(Vc.norms.view(np.int16)),
                                    Vc.k, Vc.N, t(Vc.rot), t(Vc.codebook), scale=scale)
    torch.cuda.synchronize()
    return par.to_np(out)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (16, 2)], ids=["generic-G4", "tensor-core-G8"])
def test_attention_with_lengths_matches_the_oracle(hq, hkv):
    w = wl.small_attn(batch=4, hq=hq, hkv=hkv, tokens=1100, seed=41)
    q, Kc, Vc = _caches(w)
    lengths = [1, 129, 1100, 640]
    rng = np.random.default_rng(5)
    Ks, Vs = _scramble_past(Kc, lengths, rng), _scramble_past(Vc, lengths, rng)
    out = _gpu_lengths(q, Ks, Vs, lengths, 1 / 8)
    ref = fo.attention_decoded_lengths(q, Kc, Vc, w.d, 1 / 8, lengths)
    par.check_attention(out, ref)
    # one token of context returns that token's decoded value
    v0 = fo.decode(Vc.codes[0, :, 0], Vc.norms[0, :, 0], Vc.rot, Vc.codebook, w.d, Vc.k, Vc.N)
    G = hq // hkv
    np.testing.assert_allclose(out[0], v0[np.arange(hq) // G], rtol=0,
                               atol=2e-3 * np.abs(v0).max())


def test_attention_with_length_zero_outputs_zero_and_full_lengths_equal_plain_attention():
    w = wl.small_attn(batch=3, hq=16, hkv=2, tokens=700, seed=42)
    q, Kc, Vc = _caches(w)
    out = _gpu_lengths(q, Kc, Vc, [0, 700, 3], 1 / 8)
    assert np.all(out[0] == 0)
    t = _dev
    plain = fq.fq_attn_decode(t(q), t(Kc.codes), t(Kc.norms.view(np.int16)), Kc.k, Kc.N, t(Kc.rot),
                              t(Kc.codebook), t(Vc.codes), t(Vc.norms.view(np.int16)), Vc.k, Vc.N,
                              t(Vc.rot), t(Vc.codebook), scale=1 / 8)
    torch.cuda.synchronize()
    assert np.array_equal(out[1], par.to_np(plain)[1])
    ref = fo.attention_decoded_lengths(q, Kc, Vc, w.d, 1 / 8, [1, 700, 3])
    par.check_attention(out[1:], ref[1:])


def test_attention_with_lengths_at_full_size_sampled():
    """The full attention workload's shape (B16, Hq32/Hkv4, T32768) with random lengths: the
    tensor-core kernel's launch; a sample of (batch) rows checked against the oracle."""
    w = wl.ATTN
    dpk, dpv = fo.padded_dim(w.d, w.k_rate.k), fo.padded_dim(w.d, w.v_rate.k)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, w.k_rate.k, w.k_rate.N)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, w.v_rate.k, w.v_rate.N)
    dev = {}
    for name, rot, cb, rate in (("K", rk, ck, w.k_rate), ("V", rv, cv, w.v_rate)):
        x = _dev(wl.attn_kv(w, name).reshape(-1, w.d))
        c, n = fq.fq_encode(x, _dev(rot), _dev(cb), rate.k, rate.N)
        dev[name] = (c.reshape(w.batch, w.hkv, w.tokens, -1), n.reshape(w.batch, w.hkv, w.tokens))
    rng = np.random.default_rng(9)
    lengths = rng.integers(1, w.tokens + 1, size=w.batch).astype(np.int32)
    lengths[:3] = [1, 32768, 300]
    q = _dev(wl.attn_queries(w))
    out = fq.fq_attn_decode_lengths(q, _dev(lengths), dev["K"][0], dev["K"][1], 2, 16, _dev(rk),
                                    _dev(ck), dev["V"][0], dev["V"][1], 3, 64, _dev(rv), _dev(cv),
                                    scale=1 / math.sqrt(w.d))
    torch.cuda.synchronize()
    out = par.to_np(out)
    for b in (0, 1, 2, 7, 15):
        L = int(lengths[b])
        sl = lambda c, nn, rot, cb, k, N: fo.CompressedKV(
            par.to_np(c[b:b + 1, :, :L]), par.to_np(nn[b:b + 1, :, :L]).view(np.float16), rot, cb, k, N)
        Kc = sl(*dev["K"], rk, ck, 2, 16)
        Vc = sl(*dev["V"], rv, cv, 3, 64)
        ref = fo.attention_decoded(wl.attn_queries(w)[b:b + 1], Kc, Vc, w.d, 1 / math.sqrt(w.d))
        par.check_attention(out[b:b + 1], ref)


# ------------------------------------------------------------------ the step that appends its token

def _gpu_append(q, k_new, v_new, lengths_t, dKc, dKn, dVc, dVn, Kc, Vc, scale):
    t = _dev
    out = fq.fq_attn_decode_append(t(q), t(k_new), t(v_new), lengths_t, dKc, dKn, Kc.k, Kc.N,
                                   t(Kc.rot), t(Kc.codebook), dVc, dVn, Vc.k, Vc.N, t(Vc.rot),
                                   t(Vc.codebook), scale=scale)
    torch.cuda.synchronize()
    return par.to_np(out)


@pytest.mark.parametrize("hq,hkv", [(8, 2), (16, 2)], ids=["generic-G4", "tensor-core-G8"])
def test_append_step_writes_the_encoder_records_and_attends_over_them(hq, hkv):
    w = wl.small_attn(batch=3, hq=hq, hkv=hkv, tokens=300, seed=43)
    q, Kc, Vc = _caches(w)
    rng = np.random.default_rng(11)
    lengths = np.array([0, 150, 299], dtype=np.int32)
    dKc, dKn = _dev(Kc.codes), _dev(Kc.norms.view(np.int16))
    dVc, dVn = _dev(Vc.codes), _dev(Vc.norms.view(np.int16))
    lt = _dev(lengths)
    Kcur, Vcur, Lcur = Kc, Vc, lengths.astype(np.int64)
    for step in range(3):   # a short decode loop: every step appends at the next slot
        k_new = rng.standard_normal((w.batch, hkv, w.d)).astype(np.float16)
        v_new = (3 * rng.standard_normal((w.batch, hkv, w.d))).astype(np.float16)
        qs = rng.standard_normal((w.batch, hq, w.d)).astype(np.float16)
        out = _gpu_append(qs, k_new, v_new, lt, dKc, dKn, dVc, dVn, Kc, Vc, 1 / 8)
        # capacity T = 300: the sequence already full is neither written nor advanced
        writable = Lcur < w.tokens
        ref_out, K2, V2, L2 = fo.append_and_attend(qs, k_new, v_new, Kcur, Vcur, w.d, 1 / 8,
                                                   np.minimum(Lcur, w.tokens - 1))
        # the records the GPU wrote are the oracle packing of its own indices, and the indices
        # match the oracle encoder except at near-ties
        gK, gV = par.to_np(dKc), par.to_np(dVc)
        gKn, gVn = par.to_np(dKn).view(np.float16), par.to_np(dVn).view(np.float16)
        ek = fo.encode(k_new.reshape(-1, w.d), Kc.rot, Kc.codebook, Kc.k)
        ev = fo.encode(v_new.reshape(-1, w.d), Vc.rot, Vc.codebook, Vc.k)
        mk, mv = Kc.codes.shape[-1], Vc.codes.shape[-1]
        for b in range(w.batch):
            if not writable[b]:
                continue
            L = int(Lcur[b])
            rows = slice(b * hkv, (b + 1) * hkv)
            ek_b = fo.Encoded(ek.idx[rows], ek.norms[rows], ek.gap[rows], ek.z[rows], ek.nu[rows])
            ev_b = fo.Encoded(ev.idx[rows], ev.norms[rows], ev.gap[rows], ev.z[rows], ev.nu[rows])
            par.check_records_and_indices(gK[b, :, L], ek_b, Kc.N, fo.padded_dim(w.d, Kc.k) // Kc.k)
            par.check_records_and_indices(gV[b, :, L], ev_b, Vc.N, fo.padded_dim(w.d, Vc.k) // Vc.k)
            par.check_norms(gKn[b, :, L].view(np.int16), ek_b)
            par.check_norms(gVn[b, :, L].view(np.int16), ev_b)
        Kg = fo.CompressedKV(gK, gKn, Kc.rot, Kc.codebook, Kc.k, Kc.N)
        Vg = fo.CompressedKV(gV, gVn, Vc.rot, Vc.codebook, Vc.k, Vc.N)
        want_len = np.where(writable, Lcur + 1, Lcur)
        assert par.to_np(lt).tolist() == want_len.tolist()
        # attention over the GPU's own cache (its records) matches the oracle over it
        par.check_attention(out, fo.attention_decoded_lengths(qs, Kg, Vg, w.d, 1 / 8, want_len))
        # and, where a slot was written, over the oracle's own appended records
        par.check_attention(out[writable], ref_out[writable])
        Kcur, Vcur, Lcur = Kg, Vg, want_len
        Kc, Vc = Kg, Vg
