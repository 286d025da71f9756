"""CPU pins of the oracle's attention and of the Roberts-Kronecker direction sequence.

Every attention parity test on the GPU is judged by ``attention_decoded`` (and its rotated-domain
twin ``attention_lut``), so these pins check them against values fixed by hand or by the
mathematics, not against themselves:

  * two tokens with dyadic codewords, an identity rotation and k not dividing d: the softmax weight
    of token 1 is 1 / (1 + e^(s2 - s1)) with s computed by hand, and the output is the hand-mixed
    value vector;
  * q = 0 gives the plain mean of the decoded values;
  * a very large scale saturates the softmax onto the arg-max token's value;
  * grouped-query mapping: query head h reads kv head h // (Hq / Hkv);
  * the decoded form and the rotated-domain LUT form agree to 1e-12 (an algebraic identity).

The k >= 4 direction sequence (FibQuant summary sec. 2.2, Roberts-Kronecker points) is pinned by
its first two points computed by hand from g^5 = g + 1.

Each pin is also run against planted mistakes (patched into the oracle module for the duration of
one test) and must fail on every one of them.
"""
import math

import numpy as np
import pytest
from scipy import special

from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import tables, workloads as wl

# ------------------------------------------------------------------ a hand-made 2-token cache
# d = 3 with k = 2 (so d' = 4 and the decoder must drop coordinate 3); identity rotation.
D = 3
ROT = np.eye(4)
CB_K = np.array([[0.5, 0.0], [0.0, 0.25]])        # N = 2 codewords
CB_V = np.array([[1.0, -0.5], [0.25, 0.75]])


def _kv(idx, norms, cb):
    """[1, 1, T, P] records of the given per-token block indices and fp16 norms."""
    idx = np.asarray(idx)
    codes = fo.pack(idx, 2)
    return fo.CompressedKV(codes[None, None], np.asarray(norms, np.float16)[None, None], ROT, cb,
                           2, 2)


# token 1: key blocks (0, 1) -> zhat = (0.5, 0, 0, 0.25), norm 2 -> k1 = (1, 0, 0)
# token 2: key blocks (1, 0) -> zhat = (0, 0.25, 0.5, 0), norm 4 -> k2 = (0, 1, 2)
# token 1: value blocks (0, 0) -> (1, -0.5, 1, -0.5), norm 1 -> v1 = (1, -0.5, 1)
# token 2: value blocks (1, 1) -> (0.25, 0.75, 0.25, 0.75), norm 2 -> v2 = (0.5, 1.5, 0.5)
KC = _kv([[0, 1], [1, 0]], [2.0, 4.0], CB_K)
VC = _kv([[0, 0], [1, 1]], [1.0, 2.0], CB_V)
K_HAND = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 2.0]])
V_HAND = np.array([[1.0, -0.5, 1.0], [0.5, 1.5, 0.5]])


def pin_two_token_closed_form():
    q = np.array([[[2.0, 1.0, 1.0], [0.0, 0.5, -1.0]]])   # B = 1, Hq = 2, Hkv = 1
    scale = 1.0 / math.sqrt(D)
    # head 0: q.k1 = 2, q.k2 = 1 + 2 = 3; head 1: q.k1 = 0, q.k2 = 0.5 - 2 = -1.5
    for h, (d1, d2) in enumerate(((2.0, 3.0), (0.0, -1.5))):
        p1 = 1.0 / (1.0 + math.exp((d2 - d1) * scale))
        want = p1 * V_HAND[0] + (1.0 - p1) * V_HAND[1]
        for fn in (fo.attention_decoded, fo.attention_lut):
            got = fn(q, KC, VC, D, scale)
            np.testing.assert_allclose(got[0, h], want, rtol=0, atol=1e-14)


def pin_zero_query_is_the_mean():
    w = wl.small_attn(batch=1, hq=4, hkv=2, tokens=37, seed=21)
    q, Kc, Vc = _real_caches(w)
    vdec = fo.decode(Vc.codes.reshape(-1, Vc.codes.shape[-1]), Vc.norms.reshape(-1), Vc.rot,
                     Vc.codebook, w.d, Vc.k, Vc.N).reshape(w.batch, w.hkv, w.tokens, w.d)
    zero = np.zeros_like(q, dtype=np.float64)
    for fn in (fo.attention_decoded, fo.attention_lut):
        got = fn(zero, Kc, Vc, w.d, 0.125)
        for h in range(w.hq):
            want = vdec[0, h // 2].sum(axis=0) / w.tokens
            np.testing.assert_allclose(got[0, h], want, rtol=0, atol=1e-12 * np.abs(want).max())


def pin_large_scale_picks_the_argmax_token():
    w = wl.small_attn(batch=1, hq=4, hkv=2, tokens=29, seed=22)
    q, Kc, Vc = _real_caches(w)
    kdec = fo.decode(Kc.codes.reshape(-1, Kc.codes.shape[-1]), Kc.norms.reshape(-1), Kc.rot,
                     Kc.codebook, w.d, Kc.k, Kc.N).reshape(w.batch, w.hkv, w.tokens, w.d)
    vdec = fo.decode(Vc.codes.reshape(-1, Vc.codes.shape[-1]), Vc.norms.reshape(-1), Vc.rot,
                     Vc.codebook, w.d, Vc.k, Vc.N).reshape(w.batch, w.hkv, w.tokens, w.d)
    qq = q.astype(np.float64)
    for fn in (fo.attention_decoded, fo.attention_lut):
        got = fn(qq, Kc, Vc, w.d, 1e4)
        for h in range(w.hq):
            s = kdec[0, h // 2] @ qq[0, h]
            top2 = np.sort(s)[-2:]
            assert top2[1] - top2[0] > 1e-2   # a clear winner: the others weigh < e^-100
            want = vdec[0, h // 2][int(np.argmax(s))]
            np.testing.assert_allclose(got[0, h], want, rtol=0, atol=1e-12 * np.abs(want).max())


def pin_gqa_mapping():
    """Hq = 4 over Hkv = 2: heads 0, 1 read kv head 0 and heads 2, 3 read kv head 1.  With two
    different one-token caches the output of a head is exactly its kv head's decoded value."""
    Kc = fo.CompressedKV(np.concatenate([KC.codes[:, :, :1], KC.codes[:, :, 1:]], axis=1),
                         np.concatenate([KC.norms[:, :, :1], KC.norms[:, :, 1:]], axis=1),
                         ROT, CB_K, 2, 2)
    Vc = fo.CompressedKV(np.concatenate([VC.codes[:, :, :1], VC.codes[:, :, 1:]], axis=1),
                         np.concatenate([VC.norms[:, :, :1], VC.norms[:, :, 1:]], axis=1),
                         ROT, CB_V, 2, 2)
    q = np.arange(12, dtype=np.float64).reshape(1, 4, 3) / 7.0
    for fn in (fo.attention_decoded, fo.attention_lut):
        got = fn(q, Kc, Vc, D, 0.5)
        for h in range(4):
            np.testing.assert_allclose(got[0, h], V_HAND[h // 2], rtol=0, atol=1e-14)


def pin_lut_equals_decoded():
    w = wl.small_attn(batch=2, hq=8, hkv=2, tokens=53, seed=23)
    q, Kc, Vc = _real_caches(w)
    ref = fo.attention_decoded(q, Kc, Vc, w.d, 1 / 8)
    lut = fo.attention_lut(q, Kc, Vc, w.d, 1 / 8)
    np.testing.assert_allclose(lut, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def _real_caches(w):
    dpk, dpv = fo.padded_dim(w.d, w.k_rate.k), fo.padded_dim(w.d, w.v_rate.k)
    rk, ck = tables.rotation(dpk, wl.ROT_SEED_K), tables.codebook(dpk, w.k_rate.k, w.k_rate.N)
    rv, cv = tables.rotation(dpv, wl.ROT_SEED_V), tables.codebook(dpv, w.v_rate.k, w.v_rate.N)

    def comp(x, rot, cb, k, N):
        B, H, T, d = x.shape
        enc = fo.encode(x.reshape(-1, d), rot, cb, k)
        return fo.CompressedKV(fo.pack(enc.idx, N).reshape(B, H, T, -1),
                               enc.norms.reshape(B, H, T), rot, cb, k, N)
    return (wl.attn_queries(w), comp(wl.attn_kv(w, "K"), rk, ck, w.k_rate.k, w.k_rate.N),
            comp(wl.attn_kv(w, "V"), rv, cv, w.v_rate.k, w.v_rate.N))


# ------------------------------------------------------------------ Roberts-Kronecker points

def _root_by_bisection(k):
    """g > 1 with g^(k+1) = g + 1, by plain bisection (independent of the oracle's Newton)."""
    lo, hi = 1.0, 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if mid ** (k + 1) - mid - 1.0 > 0:
            hi = mid
        else:
            lo = mid
    return 0.5 * (lo + hi)


def pin_roberts_first_points():
    g = _root_by_bisection(4)
    assert abs(g - 1.1673039782614187) < 1e-13    # the plastic-number analogue for R_4
    alpha = [g ** -1, g ** -2, g ** -3, g ** -4]
    u = fo.init_directions(4, 8)
    for n in (0, 1, 5):
        t = [math.fmod(0.5 + (n + 1) * a, 1.0) for a in alpha]
        v = np.array([special.ndtri(ti) for ti in t])
        np.testing.assert_allclose(u[n], v / np.linalg.norm(v), rtol=0, atol=1e-12)
    # k = 5 as well: g^6 = g + 1
    g5 = _root_by_bisection(5)
    t = [math.fmod(0.5 + 1 * g5 ** -(i + 1), 1.0) for i in range(5)]
    v = np.array([special.ndtri(ti) for ti in t])
    np.testing.assert_allclose(fo.init_directions(5, 4)[0], v / np.linalg.norm(v), atol=1e-12)


PINS = {
    "two_token": pin_two_token_closed_form,
    "zero_query": pin_zero_query_is_the_mean,
    "large_scale": pin_large_scale_picks_the_argmax_token,
    "gqa": pin_gqa_mapping,
    "lut_identity": pin_lut_equals_decoded,
    "roberts": pin_roberts_first_points,
}


@pytest.mark.parametrize("name", list(PINS))
def test_pin_holds_on_the_oracle(name):
    PINS[name]()


# ------------------------------------------------------------------ planted mistakes
# Each mutant is a plausible slip in the oracle; the listed pins must catch it.

def _attention_exact_mutant(kind):
    def f(q, K, V, scale):
        q = np.asarray(q, dtype=np.float64)
        K = np.asarray(K, dtype=np.float64)
        V = np.asarray(V, dtype=np.float64)
        Bn, Hq, d = q.shape
        Hkv = K.shape[1]
        G = Hq // Hkv
        out = np.empty((Bn, Hq, V.shape[-1]))
        for b in range(Bn):
            for h in range(Hq):
                g = h % Hkv if kind == "gqa_modulo" else h // G
                sc = 1.0 / math.sqrt(d + 1) if kind == "scale_padded_dim" else scale
                s = K[b, g] @ q[b, h] * sc
                if kind == "softmax_of_negative":
                    s = -s
                p = np.exp(s - s.max())
                p = p / p.sum() if kind != "unnormalised" else p
                out[b, h] = p @ V[b, g]
        return out
    return f


def _softmax_mutant(kind):
    def f(s):
        if kind == "no_normalisation":
            return np.exp(s - np.max(s, axis=-1, keepdims=True))
        if kind == "temperature_two":
            e = np.exp((s - np.max(s, axis=-1, keepdims=True)) / 2)
            return e / np.sum(e, axis=-1, keepdims=True)
        raise ValueError(kind)
    return f


def _directions_mutant(kind):
    real = fo.init_directions

    def f(k, N):
        if k < 4:
            return real(k, N)
        g = fo.roberts_root(k)
        alpha = g ** (-np.arange(1, k + 1, dtype=np.float64))
        n = np.arange(N, dtype=np.float64)
        if kind == "n_alpha":
            t = np.mod(0.5 + n[:, None] * alpha[None, :], 1.0)
        elif kind == "no_half":
            t = np.mod((n[:, None] + 1.0) * alpha[None, :], 1.0)
        elif kind == "alpha_from_zero":
            alpha = g ** (-np.arange(0, k, dtype=np.float64))
            t = np.mod(0.5 + (n[:, None] + 1.0) * alpha[None, :], 1.0)
        v = special.ndtri(t)
        return v / np.linalg.norm(v, axis=1, keepdims=True)
    return f


MUTANTS = [
    ("attention_exact", _attention_exact_mutant, "gqa_modulo", ["gqa"]),
    ("attention_exact", _attention_exact_mutant, "scale_padded_dim", ["two_token"]),
    ("attention_exact", _attention_exact_mutant, "softmax_of_negative",
     ["two_token", "large_scale"]),
    ("attention_exact", _attention_exact_mutant, "unnormalised", ["two_token", "zero_query"]),
    ("_softmax", _softmax_mutant, "no_normalisation", ["two_token", "zero_query"]),
    ("_softmax", _softmax_mutant, "temperature_two", ["two_token"]),
    ("init_directions", _directions_mutant, "n_alpha", ["roberts"]),
    ("init_directions", _directions_mutant, "no_half", ["roberts"]),
    ("init_directions", _directions_mutant, "alpha_from_zero", ["roberts"]),
]


@pytest.mark.parametrize("target,make,kind,pins", MUTANTS,
                         ids=[f"{m[0]}-{m[2]}" for m in MUTANTS])
def test_pins_catch_planted_mistakes(monkeypatch, target, make, kind, pins):
    monkeypatch.setattr(fo, target, make(kind))
    for name in pins:
        with pytest.raises(AssertionError):
            PINS[name]()
