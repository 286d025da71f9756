"""GPU parity of the variants through the C ABI: BlockQuant's target-aware rescale (the stored
rho and the three S rules of the decoder) and TurboQuant_prod (scalar MSE code plus the QJL sign
sketch of its residual), against the oracle on the same seeded inputs."""
import types

import numpy as np
import pytest
import torch

import random_access_kv_fq_b200 as fq
from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import tables, workloads as wl
from tests import parity as par

pytestmark = pytest.mark.gpu

RULES = {"plain": fq.FQ_RESCALE_PLAIN, "mse": fq.FQ_RESCALE_MSE, "unbiased": fq.FQ_RESCALE_UNBIASED}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _rows(n):
    x = wl.rows_of(wl.GPT2.cache, np.arange(0, 294912, 294912 // n)[:n]).copy()
    x[7] = 0   # zero vector: rho = 1, decodes to 0
    return x


@pytest.mark.parametrize("dp,k,N,grid", [(66, 3, 64, None), (64, 2, 16, None), (64, 4, 8, None),
                                         (66, 3, 64, (20, 8)), (64, 2, 256, (128, 4))])
def test_rescale_rho_and_rules_match_the_oracle(dp, k, N, grid):
    """rho and the decoder's S rules; fp16 rows of d = 64 take the tensor-core encode (with an
    exact grid index: the grid search), others the generic kernels."""
    d = 64
    rot, cb = tables.rotation(dp, wl.ROT_SEED_V), tables.codebook(dp, k, N)
    x = _rows(1500)
    rt, ct = _dev(rot), _dev(cb)
    ix = None if grid is None else \
        _dev(fq.fq_build_search_index(cb, d, k, N, fq.FQ_INDEX_EXACT, grid[0], grid[1]))
    codes, norms, rho = fq.fq_encode_rho(_dev(x), rt, ct, k, N, search_index=ix)
    torch.cuda.synchronize()
    enc, _ = fo.encode_rescaled(x, rot, cb, k)
    gidx = par.check_records_and_indices(par.to_np(codes), enc, N, dp // k)
    par.check_norms(par.to_np(norms), enc)
    # rho of the GPU's own indices, rounded to fp16 like the norm (+-1 ulp at rounding midpoints)
    zbar = np.asarray(cb, np.float64)[gidx].reshape(len(x), dp)
    rho_ref = np.where(enc.nu > 0, np.sum(enc.z * zbar, axis=1), 1.0)
    par.check_norms(par.to_np(rho), types.SimpleNamespace(norms=rho_ref.astype(np.float16),
                                                          nu=rho_ref))
    grho = par.to_np(rho).view(np.float16).astype(np.float64)
    for name, rule in RULES.items():
        y = fq.fq_decode_rescaled(codes, norms, rho, rt, ct, d, k, N, rule)
        torch.cuda.synchronize()
        ref = fo.decode_rescaled(gidx, par.to_np(norms).view(np.float16), grho, rot, cb, d, name)
        y = par.to_np(y).astype(np.float64)
        num = np.linalg.norm(y - ref, axis=1)
        den = np.linalg.norm(ref, axis=1)
        assert np.all(num[den == 0] == 0)
        assert (num[den > 0] / den[den > 0]).max() <= par.RECON_RTOL, name
    # the plain rule is the plain decoder
    y_plain = fq.fq_decode_rescaled(codes, norms, rho, rt, ct, d, k, N, fq.FQ_RESCALE_PLAIN)
    y_dec = fq.fq_decode(codes, norms, rt, ct, d, k, N)
    torch.cuda.synchronize()
    par.check_recon(par.to_np(y_plain), gidx, par.to_np(norms), rot, cb, d)
    par.check_recon(par.to_np(y_dec), gidx, par.to_np(norms), rot, cb, d)


@pytest.mark.parametrize("N1", [2, 4, 8])
def test_turboquant_prod_matches_the_oracle(N1):
    d = 64
    rot = tables.rotation(d, wl.ROT_SEED_K)
    c1 = np.sort(fo.scalar_lloyd(d, N1)).astype(np.float32)
    S = fo.qjl_matrix(d, 1234).astype(np.float32)
    x = _rows(1200)
    codes, signs, norms, gamma = fq.fq_encode_prod(_dev(x), _dev(rot), _dev(c1), _dev(S))
    torch.cuda.synchronize()
    xs = x.astype(np.float64)
    nu = np.linalg.norm(xs, axis=1)
    u = np.where(nu[:, None] > 0, xs / np.where(nu > 0, nu, 1)[:, None], 0.0)
    R, C1, S64 = rot.astype(np.float64), c1.astype(np.float64), S.astype(np.float64)
    # norms
    par.check_norms(par.to_np(norms), types.SimpleNamespace(norms=nu.astype(np.float16), nu=nu))
    # indices: the oracle's scalar MSE quantizer, except where two levels are (nearly) equidistant
    gidx = fo.unpack(par.to_np(codes), d, N1)
    oidx = fo.turboquant_mse_quantize(u, R, C1)
    y = u @ R.T
    dist = np.sort(np.abs(y[:, :, None] - C1[None, None, :]), axis=2)
    near = (dist[:, :, 1] - dist[:, :, 0]) <= 1e-5
    assert not np.any((gidx != oidx) & ~near)
    # signs: QJL of the residual of the GPU's own indices, except where S r is ~0
    r = u - fo.turboquant_mse_dequantize(gidx, R, C1)
    sr = r @ S64.T
    q = np.unpackbits(par.to_np(signs), axis=1, bitorder="little")[:, :d].astype(bool)
    tiny = np.abs(sr) <= 1e-5 * (np.linalg.norm(r, axis=1, keepdims=True) + 1e-30) * np.sqrt(d)
    assert not np.any((q != (sr >= 0)) & ~tiny)
    # gamma = |r| in fp16
    g = np.linalg.norm(r, axis=1)
    par.check_norms(par.to_np(gamma), types.SimpleNamespace(norms=g.astype(np.float16), nu=g))
    # decode: nu (Pi^T c1[idx] + gamma sqrt(pi/2)/d S^T q) with the GPU's own records
    yd = fq.fq_decode_prod(codes, signs, norms, gamma, _dev(rot), _dev(c1), _dev(S), d)
    torch.cuda.synchronize()
    gnu = par.to_np(norms).view(np.float16).astype(np.float64)
    gg = par.to_np(gamma).view(np.float16).astype(np.float64)
    ref = gnu[:, None] * fo.turboquant_prod_dequantize(gidx, np.where(q, 1.0, -1.0), gg, R, C1, S64)
    yd = par.to_np(yd).astype(np.float64)
    num = np.linalg.norm(yd - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    assert np.all(num[den == 0] == 0)
    assert (num[den > 0] / den[den > 0]).max() <= par.RECON_RTOL


def test_turboquant_prod_inner_products_are_unbiased_on_the_gpu():
    """TurboQuant notes sec. 3.2: over random rotations and QJL matrices the decoded inner
    product <y, x_hat> is unbiased (within 5 sigma), while the MSE part alone shrinks it."""
    d, T = 64, 300
    c1 = np.sort(fo.scalar_lloyd(d, 2)).astype(np.float32)
    rng = np.random.default_rng(3)
    x = rng.standard_normal((1, d))
    x /= np.linalg.norm(x)
    yv = 1.3 * x[0] + 0.3 * rng.standard_normal(d)
    xt = _dev(x.astype(np.float32))
    est, mse = np.empty(T), np.empty(T)
    for t in range(T):
        rot = fo.haar_rotation(d, 7000 + t).astype(np.float32)
        S = fo.qjl_matrix(d, 8000 + t).astype(np.float32)
        codes, signs, norms, gamma = fq.fq_encode_prod(xt, _dev(rot), _dev(c1), _dev(S))
        xh = fq.fq_decode_prod(codes, signs, norms, gamma, _dev(rot), _dev(c1), _dev(S), d)
        est[t] = par.to_np(xh)[0].astype(np.float64) @ yv
        idx = fo.unpack(par.to_np(codes), d, 2)
        mse[t] = fo.turboquant_mse_dequantize(idx, rot.astype(np.float64), c1.astype(np.float64))[0] @ yv
    target = float(x[0] @ yv)
    assert abs(est.mean() - target) <= 5 * est.std() / np.sqrt(T)
    assert abs(mse.mean() - target) > 5 * mse.std() / np.sqrt(T)
