"""Pins of the oracle's variants (BlockQuant's target-aware rescale, QJL and TurboQuant_prod)
against what the pages state and the mathematics fixes: closed forms, invariants and the
expectations the pages prove (checked over seeded random draws, 5 sigma)."""
import math

import numpy as np
from scipy import special

from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import tables


def _pair(d, seed, cos=0.6):
    """A unit x and a y with <x, y> = cos * |y|-ish, fixed by the seed."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(d)
    x /= np.linalg.norm(x)
    w = rng.standard_normal(d)
    w -= (w @ x) * x
    w /= np.linalg.norm(w)
    return x, 1.3 * (cos * x + math.sqrt(1 - cos * cos) * w)


def _mean_close(samples, target):
    return abs(samples.mean() - target) <= 5 * samples.std() / math.sqrt(samples.size)


def test_qjl_is_unbiased_with_variance_within_the_bound():
    """TurboQuant notes sec. 2.2 (QJL lemma): for unit x, E <y, Q^-1(Q(x))> = <y, x> and
    Var <= pi / (2 d) |y|^2."""
    d, T = 64, 4000
    x, y = _pair(d, 5)
    est = np.empty(T)
    for t in range(T):
        S = fo.qjl_matrix(d, 1000 + t)
        est[t] = fo.qjl_dequantize(fo.qjl_quantize(x, S), S)[0] @ y
    bound = math.pi / (2 * d) * (y @ y)
    assert est.var() <= 1.1 * bound
    assert _mean_close(est, y @ x)


def _mean_abs_coord(d):
    """E|u_1| for u uniform on the unit sphere of R^d."""
    return math.exp(special.gammaln(d / 2) - special.gammaln((d + 1) / 2)) / math.sqrt(math.pi)


def test_one_bit_turboquant_mse_has_the_two_over_pi_bias():
    """TurboQuant notes sec. 3.2: the 1-bit MSE quantizer's inner products are biased by 2/pi
    (large d).  At finite d the 1-bit Lloyd centroid is E|u_1| and the bias is exactly
    d E|u_1|^2 (rotation symmetry), which tends to 2/pi."""
    d, T = 128, 1500
    c1 = fo.scalar_lloyd(d, 2)
    m1 = _mean_abs_coord(d)
    np.testing.assert_allclose(c1, [-m1, m1], rtol=1e-9)
    ratio = d * m1 * m1
    assert abs(4096 * _mean_abs_coord(4096) ** 2 - 2 / math.pi) < 2e-4
    x, y = _pair(d, 6)
    est = np.empty(T)
    for t in range(T):
        rot = fo.haar_rotation(d, 2000 + t)
        est[t] = fo.turboquant_mse_dequantize(fo.turboquant_mse_quantize(x, rot, c1), rot, c1)[0] @ y
    assert _mean_close(est, ratio * (x @ y))
    assert not _mean_close(est, x @ y)


def test_turboquant_prod_is_unbiased_where_the_mse_part_is_not():
    """TurboQuant notes sec. 3.2: 1-bit MSE code plus the QJL sketch of its residual and the
    residual norm gives unbiased inner products; the MSE part alone is biased low."""
    d, T = 64, 2000
    c1 = fo.scalar_lloyd(d, 2)
    x, y = _pair(d, 7)
    prod, mse = np.empty(T), np.empty(T)
    for t in range(T):
        rot, S = fo.haar_rotation(d, 3000 + t), fo.qjl_matrix(d, 9000 + t)
        idx, q, g = fo.turboquant_prod_quantize(x, rot, c1, S)
        prod[t] = fo.turboquant_prod_dequantize(idx, q, g, rot, c1, S)[0] @ y
        mse[t] = fo.turboquant_mse_dequantize(idx, rot, c1)[0] @ y
    assert _mean_close(prod, x @ y)
    assert mse.mean() < x @ y - 5 * mse.std() / math.sqrt(T)


def test_rescale_mse_rule_is_the_least_squares_factor():
    """Block Sphere VQ notes, key design 3: S = rho / |zbar|^2 minimises |z - S zbar|^2, so the
    residual is orthogonal to zbar and the error is never above the plain rule's."""
    rot, cb = tables.rotation(64, 17).astype(np.float64), tables.codebook(64, 2, 16)
    x = np.random.default_rng(8).standard_normal((300, 64))
    enc, rho = fo.encode_rescaled(x, rot, cb, 2)
    zbar = np.asarray(cb, dtype=np.float64)[enc.idx].reshape(300, 64)
    S = fo.rescale_factor(rho, np.sum(zbar * zbar, axis=1), "mse")
    resid = enc.z - S[:, None] * zbar
    assert np.max(np.abs(np.sum(resid * zbar, axis=1))) < 1e-12
    err_mse = np.sum(resid ** 2, axis=1)
    err_plain = np.sum((enc.z - zbar) ** 2, axis=1)
    assert np.all(err_mse <= err_plain + 1e-15)
    # the decoder applies it: x_hat = nu S Pi^T zbar
    y = fo.decode_rescaled(enc.idx, enc.norms, rho, rot, cb, 64, "mse")
    ref = (enc.norms.astype(np.float64) * S)[:, None] * (zbar @ rot)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)


def test_rescale_unbiased_rule_removes_the_shrinkage():
    """Block Sphere VQ notes, key design 3: with S = 1 / rho the component of x_hat along x is
    exact, so inner products are unbiased over random rotations, while the plain rule (S = 1)
    shrinks them by E[rho] < 1."""
    d, T = 64, 400
    cb = tables.codebook(64, 2, 16)
    x, y = _pair(d, 9)
    ub, pl = np.empty(T), np.empty(T)
    for t in range(T):
        rot = fo.haar_rotation(d, 5000 + t)
        enc, rho = fo.encode_rescaled(x[None], rot, cb, 2)
        ub[t] = fo.decode_rescaled(enc.idx, enc.norms, rho, rot, cb, d, "unbiased")[0] @ y
        pl[t] = fo.decode_rescaled(enc.idx, enc.norms, rho, rot, cb, d, "plain")[0] @ y
    assert _mean_close(ub, x @ y)
    assert pl.mean() < x @ y - 5 * pl.std() / math.sqrt(T)
