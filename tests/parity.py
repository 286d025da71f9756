"""Parity rules shared by the GPU tests (CUDA path vs the CPU oracle, same inputs).

  * records: the CUDA record must equal the oracle packing of its own indices (bit-exact);
  * indices: equal to the oracle's except at near-ties, where the oracle's best-two squared
    distance gap on the unit-scale block is <= 1e-4; such blocks may differ but must be at
    most 0.01 % of all blocks;
  * norms: fp16 bit-exact, except +-1 ulp where the exact norm lies within 2^-20 (relative) of
    an fp16 rounding midpoint (the kernel's fp32 norm may land on either side);
  * reconstructions: per vector, |y - y*|_2 / |y*|_2 <= 1e-5 with y* the oracle decoding of
    the CUDA indices and stored norm;
  * attention: per (batch, head), |o - o*|_inf / |o*|_inf <= 2e-3 with o* the oracle
    attention over the decoded cache.
"""
import numpy as np

from oracle import fq_oracle as fo

NEAR_TIE_GAP = 1e-4
NEAR_TIE_FRACTION = 1e-4
RECON_RTOL = 1e-5
ATTN_RTOL = 2e-3


def to_np(t):
    return t.detach().cpu().numpy()


def check_records_and_indices(codes, enc, N, m, extra_exempt=None):
    """codes: CUDA record bytes [n, P]; enc: oracle Encoded.  Returns the CUDA indices."""
    gidx = fo.unpack(codes, m, N)
    np.testing.assert_array_equal(fo.pack(gidx, N), codes, err_msg="record is not the packing "
                                  "of its own indices (tail bits or layout)")
    diff = gidx != enc.idx
    n_diff = int(diff.sum())
    if n_diff:
        allowed = enc.gap <= NEAR_TIE_GAP
        if extra_exempt is not None:
            allowed = allowed | extra_exempt
        bad = diff & ~allowed
        assert not bad.any(), (
            f"{int(bad.sum())} index mismatches outside near-ties; first at "
            f"{np.argwhere(bad)[:5].tolist()} gap={enc.gap[bad][:5]}")
        assert n_diff <= max(1, NEAR_TIE_FRACTION * diff.size), \
            f"{n_diff} near-tie mismatches of {diff.size} blocks"
    return gidx


def fp16_midpoint_near(nu):
    """True where nu (fp64) is within 2^-20 relative of a midpoint between fp16 neighbours."""
    nu = np.asarray(nu, dtype=np.float64)
    h = nu.astype(np.float16).astype(np.float64)
    up = np.nextafter(nu.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(nu.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    mid = np.where(nu >= h, (h + up) / 2, (h + dn) / 2)
    return np.abs(nu - mid) <= 2.0 ** -20 * np.abs(nu)


def check_norms(gpu_bits, enc):
    gb = np.asarray(gpu_bits).view(np.uint16).astype(np.int64)
    ob = enc.norms.view(np.uint16).astype(np.int64)
    diff = gb != ob
    if diff.any():
        ok = (np.abs(gb - ob) == 1) & fp16_midpoint_near(enc.nu)
        bad = diff & ~ok
        assert not bad.any(), f"{int(bad.sum())} norm mismatches, e.g. rows {np.argwhere(bad)[:5].ravel()}"


def check_recon(y, gidx, gnorm_bits, rot, cb, d):
    ref = fo.decode_idx(gidx, np.asarray(gnorm_bits).view(np.float16), rot, cb, d)
    y = np.asarray(y, dtype=np.float64)
    num = np.linalg.norm(y - ref, axis=1)
    den = np.linalg.norm(ref, axis=1)
    zero = den == 0
    assert np.all(num[zero] == 0), "zero vectors must decode to zero"
    rel = num[~zero] / den[~zero]
    assert rel.size == 0 or rel.max() <= RECON_RTOL, f"max relative error {rel.max():.3e}"
    return ref


def check_recon_f16(y16, ref):
    """fp16 output: round-to-nearest-even of the fp32 result, so within one fp16 rounding of
    the fp64 reference (2^-11 relative per element, and at most 2^-25 absolute below 2^-14,
    half the subnormal spacing), plus the fp32 error."""
    y = np.asarray(y16, dtype=np.float64)
    tol = (np.maximum(2.0 ** -11 * np.abs(ref), 2.0 ** -25) +
           1e-5 * np.linalg.norm(ref, axis=1, keepdims=True))
    assert np.all(np.abs(y - ref) <= tol)


def check_attention(out, ref):
    out = np.asarray(out, dtype=np.float64)
    num = np.abs(out - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    rel = num / den
    assert rel.max() <= ATTN_RTOL, f"attention max relative error {rel.max():.3e}"
    return rel.max()
