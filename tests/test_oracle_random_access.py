"""Pins of the oracle's random-access pieces (gather-decode of a token list, per-sequence
context lengths, the decode step that appends its own token): fixed-address independence
(records outside the list or past a length may hold anything), the one-token closed form of
attention, and the written records being the encoder's."""
import numpy as np

from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import tables

D = 64
ROT_K, CB_K = tables.rotation(64, 17), tables.codebook(64, 2, 16)
ROT_V, CB_V = tables.rotation(66, 18), tables.codebook(66, 3, 64)


def _compress(X, rot, cb, k, N):
    B, H, T, d = X.shape
    enc = fo.encode(X.reshape(-1, d), rot, cb, k)
    return fo.CompressedKV(fo.pack(enc.idx, N).reshape(B, H, T, -1), enc.norms.reshape(B, H, T),
                           rot, cb, k, N)


def _caches(B, H, T, seed):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((B, H, T, D))
    V = rng.standard_normal((B, H, T, D))
    return _compress(K, ROT_K, CB_K, 2, 16), _compress(V, ROT_V, CB_V, 3, 64)


def _scramble(c, keep, rng):
    """Random bytes and random finite norms everywhere keep[b, t] is False."""
    codes, norms = c.codes.copy(), c.norms.copy()
    B, H, T, P = codes.shape
    for b in range(B):
        for t in range(T):
            if not keep[b, t]:
                codes[b, :, t] = rng.integers(0, 256, size=(H, P), dtype=np.uint8)
                norms[b, :, t] = rng.uniform(0.1, 50.0, size=H).astype(np.float16)
    return fo.CompressedKV(codes, norms, c.rot, c.codebook, c.k, c.N)


def test_gather_decode_reads_only_the_listed_records():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((300, D))
    enc = fo.encode(x, ROT_V, CB_V, 3)
    codes, norms = fo.pack(enc.idx, 64), enc.norms
    ids = [299, 0, 17, 17, 150]
    full = fo.decode(codes, norms, ROT_V, CB_V, D, 3, 64)
    keep = np.zeros((1, 300), dtype=bool)
    keep[0, ids] = True
    c = _scramble(fo.CompressedKV(codes[None, None], norms[None, None], ROT_V, CB_V, 3, 64),
                  keep, rng)
    got = fo.decode_tokens(c.codes[0, 0], c.norms[0, 0], ids, ROT_V, CB_V, D, 3, 64)
    np.testing.assert_allclose(got, full[ids], rtol=1e-12, atol=1e-12)


def test_lengths_one_token_is_its_value_and_records_past_a_length_are_never_read():
    B, H, T, Hq = 2, 2, 50, 8
    Kc, Vc = _caches(B, H, T, 4)
    q = np.random.default_rng(5).standard_normal((B, Hq, D))
    lengths = [1, 37]
    keep = np.arange(T)[None, :] < np.asarray(lengths)[:, None]
    rng = np.random.default_rng(6)
    out = fo.attention_decoded_lengths(q, _scramble(Kc, keep, rng), _scramble(Vc, keep, rng),
                                       D, 1 / 8, lengths)
    v0 = fo.decode(Vc.codes[0, :, 0], Vc.norms[0, :, 0], ROT_V, CB_V, D, 3, 64)  # [H, D]
    np.testing.assert_allclose(out[0], v0[np.arange(Hq) // (Hq // H)], rtol=1e-12, atol=1e-12)
    sl = lambda c: fo.CompressedKV(c.codes[1:2, :, :37], c.norms[1:2, :, :37], c.rot, c.codebook,
                                   c.k, c.N)
    ref = fo.attention_decoded(q[1:2], sl(Kc), sl(Vc), D, 1 / 8)
    np.testing.assert_allclose(out[1:2], ref, rtol=1e-12, atol=1e-12)


def test_append_and_attend_writes_the_encoder_records_and_attends_over_them():
    B, H, T, Hq = 2, 2, 32, 4
    Kc, Vc = _caches(B, H, T, 7)
    rng = np.random.default_rng(8)
    q = rng.standard_normal((B, Hq, D))
    k_new, v_new = rng.standard_normal((B, H, D)), rng.standard_normal((B, H, D))
    lengths = np.array([0, 20])
    out, K2, V2, L2 = fo.append_and_attend(q, k_new, v_new, Kc, Vc, D, 1 / 8, lengths)
    assert L2.tolist() == [1, 21]
    ek, ev = fo.encode(k_new.reshape(-1, D), ROT_K, CB_K, 2), fo.encode(v_new.reshape(-1, D), ROT_V, CB_V, 3)
    rk, rv = fo.pack(ek.idx, 16).reshape(B, H, -1), fo.pack(ev.idx, 64).reshape(B, H, -1)
    for b in range(B):
        np.testing.assert_array_equal(K2.codes[b, :, lengths[b]], rk[b])
        np.testing.assert_array_equal(V2.codes[b, :, lengths[b]], rv[b])
        others = np.arange(T) != lengths[b]
        np.testing.assert_array_equal(K2.codes[b][:, others], Kc.codes[b][:, others])
        np.testing.assert_array_equal(V2.norms[b][:, others], Vc.norms[b][:, others])
    # empty context: the step's output is its own decoded value
    vhat = fo.decode(fo.pack(ev.idx, 64), ev.norms, ROT_V, CB_V, D, 3, 64).reshape(B, H, D)
    np.testing.assert_allclose(out[0], vhat[0][np.arange(Hq) // (Hq // H)], rtol=1e-12, atol=1e-12)
