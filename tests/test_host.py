"""CPU tests of the record packer (oracle), the C ABI surface and the host-side index builder."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import random_access_kv_fq_b200 as fq
from oracle import fq_oracle as fo
from random_access_kv_fq_b200 import _lib, tables
from tests.conftest import ROOT


# ---------------------------------------------------------------- packer (oracle) pins

def _python_int_pack(row, B):
    """Independent packer: the record as one little-endian integer, index j at bit j*B."""
    v = 0
    for j, i in enumerate(row):
        v |= int(i) << (j * B)
    P = (len(row) * B + 7) // 8
    return list(v.to_bytes(P, "little"))


@pytest.mark.parametrize("m,N", [(32, 16), (22, 64), (16, 8), (32, 256), (32, 8), (32, 4096),
                                 (3, 2), (5, 65536), (1, 1024)])
def test_pack_matches_integer_packer_and_unpacks(m, N):
    B = fo.index_bits(N)
    rng = np.random.default_rng(m * 1000 + N)
    idx = rng.integers(0, N, size=(50, m))
    idx[0] = N - 1  # all ones
    idx[1] = 0
    codes = fo.pack(idx, N)
    assert codes.shape == (50, (m * B + 7) // 8)
    for r in range(50):
        assert codes[r].tolist() == _python_int_pack(idx[r], B)
    np.testing.assert_array_equal(fo.unpack(codes, m, N), idx)


def test_pack_tail_bits_zero():
    idx = np.full((1, 22), 63)
    codes = fo.pack(idx, 64)  # 132 bits in 17 bytes: top 4 bits of the last byte unused
    assert codes[0, -1] == 0x0F


# ---------------------------------------------------------------- C ABI surface

def _header_functions():
    src = open(os.path.join(ROOT, "include", "fq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fq_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = _lib.lib()
    declared = _header_functions()
    assert declared, "no declarations parsed"
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(_lib.exported_symbols())


def test_host_functions():
    assert fq.lib().fq_abi_version() == 1
    for d, k, N in [(64, 2, 16), (64, 3, 64), (64, 4, 8), (64, 2, 256), (64, 2, 8), (128, 4, 4096),
                    (256, 1, 65536), (1, 1, 2), (17, 5, 32)]:
        assert fq.fq_payload_bytes(d, k, N) == fo.payload_bytes(d, k, N)
        assert fq.fq_padded_dim(d, k) == fo.padded_dim(d, k)
    for bad in [(64, 2, 3), (64, 2, 1), (64, 2, 131072), (0, 1, 2), (257, 1, 2), (64, 65, 16),
                (4, 5, 16)]:
        assert fq.fq_payload_bytes(*bad) == 0
    for s in range(7):
        assert fq.status_string(s)


def test_entry_points_validate_before_touching_the_device():
    L = _lib.lib()
    # n = 0 is an OK no-op; unsupported sizes and null pointers are rejected on the host
    assert L.fq_encode(None, 0, 0, 64, 2, 16, None, None, None, None, None, None) == 0
    assert L.fq_encode(None, 0, 10, 64, 2, 15, None, None, None, None, None, None) == 2
    assert L.fq_encode(None, 0, 10, 64, 2, 16, None, None, None, None, None, None) == 1
    assert L.fq_encode(None, 7, 10, 64, 2, 16, None, None, None, None, None, None) == 1
    assert L.fq_encode(None, 0, -1, 64, 2, 16, None, None, None, None, None, None) == 1
    assert L.fq_decode(None, None, 0, 64, 2, 16, None, None, None, 0, None) == 0
    assert L.fq_decode(None, None, 5, 300, 2, 16, None, None, None, 0, None) == 2
    # misaligned fp16 input pointer
    assert L.fq_encode(1, 0, 10, 64, 2, 16, 4, 4, 4, 2, None, None) == 3
    # attention: Hq not a multiple of Hkv; group too large; missing workspace
    args = [16, 1, 6, 4, 100, 64, 16, 16, 2, 16, 16, 16, 16, 16, 3, 64, 16, 16,
            ctypes.c_float(0.125), 16, None, 0, None]
    assert L.fq_attn_decode(*args) == 1
    args2 = list(args); args2[2] = 34; args2[3] = 2
    assert L.fq_attn_decode(*args2) == 2
    args3 = list(args); args3[2] = 32
    assert L.fq_attn_decode(*args3) == 4
    assert fq.fq_attn_workspace_bytes(16, 32, 4, 32768, 64, 3) > 0
    assert fq.fq_attn_workspace_bytes(1, 3, 2, 10, 64, 3) == 0


def test_noalloc_attention_validates_like_the_workspace_entry_point():
    """The allocation-free attention entry point refuses a bad call with the same status as
    fq_attn_decode, on the host, before it looks up its scratch array (no CUDA call is made, so
    this runs without a GPU)."""
    L = _lib.lib()
    base = [16, 1, 32, 4, 100, 64, 16, 16, 2, 16, 16, 16, 16, 16, 3, 64, 16, 16,
            ctypes.c_float(0.125), 16, None]
    bad = {
        "Hq not a multiple of Hkv": ({2: 6}, 1),
        "group too large": ({2: 34, 3: 2}, 2),
        "d above 128": ({5: 200}, 2),
        "N not a power of two": ({9: 15}, 2),
        "non-finite scale": ({18: ctypes.c_float(float("nan"))}, 1),
        "null query": ({0: None}, 1),
        "null key records": ({6: None}, 1),
        "misaligned norms": ({7: 17}, 3),
        "scratch too small": ({1: 64, 2: 256, 3: 16, 4: 1024}, 4),
    }
    for why, (edits, status) in bad.items():
        ws_args = list(base[:20]) + [None, 0, None]
        na_args = list(base)
        for i, v in edits.items():
            na_args[i] = v
            ws_args[i] = v
        assert L.fq_attn_decode_noalloc(*na_args) == status, why
        if status != 4:
            assert L.fq_attn_decode(*ws_args) == status, why


# ---------------------------------------------------------------- host index builder

def _cell_of(z, hdr):
    t = (z.astype(np.float32) - np.float32(hdr["lo"])) * np.float32(hdr["inv_h"])
    c = np.clip(np.floor(t).astype(np.int64), 0, hdr["L"] - 1)
    return np.sum(c * hdr["L"] ** np.arange(z.shape[-1]), axis=-1)


def _parse_index(buf):
    h = np.frombuffer(buf[:64].tobytes(), dtype=np.int32)
    f = np.frombuffer(buf[:64].tobytes(), dtype=np.float32)
    u = np.frombuffer(buf[:64].tobytes(), dtype=np.uint32)
    u16 = np.frombuffer(buf[:64].tobytes(), dtype=np.uint16)
    hdr = dict(kind=h[2], k=h[3], N=h[4], L=h[5], dp=h[6], slots=h[7], lo=f[8], inv_h=f[9],
               n_cells=h[10], entry_bytes=h[11], cells_offset=u[12], overflow_offset=u[13],
               max_candidates=int(u16[30]), id_bytes=int(u16[31]))
    assert u[0] == 0x58495146 and u[1] == 2
    return hdr


def _cell_ids(buf, hdr, cell):
    e = buf[hdr["cells_offset"] + cell * hdr["entry_bytes"]:][:hdr["entry_bytes"]]
    dt = np.uint8 if hdr["id_bytes"] == 1 else np.uint16
    ids = [int(i) for i in np.frombuffer(e[:hdr["slots"] * hdr["id_bytes"]].tobytes(), dtype=dt)]
    if hdr["kind"] == 0 and hdr["max_candidates"] > hdr["slots"]:
        w = int(np.frombuffer(e[-4:].tobytes(), dtype=np.uint32)[0])
        if w != 0xFFFFFFFF:
            ov = np.frombuffer(buf[hdr["overflow_offset"]:].tobytes(), dtype=np.uint16)
            ids += [int(i) for i in ov[w + 1:w + 1 + ov[w]]]
    return ids


def _cell_list(buf, hdr, cell):
    return set(_cell_ids(buf, hdr, cell))


@pytest.mark.parametrize("dp,k,N,L,slots", [(64, 2, 16, 64, 2), (64, 2, 256, 128, 4),
                                            (66, 3, 64, 16, 4), (64, 4, 8, 8, 4), (64, 2, 8, 32, 2)])
def test_exact_index_lists_contain_the_brute_force_nearest(dp, k, N, L, slots):
    C = tables.codebook(dp, k, N)
    d = 64
    buf = fq.fq_build_search_index(C, d, k, N, fq.FQ_INDEX_EXACT, L, slots)
    hdr = _parse_index(buf)
    assert (hdr["k"], hdr["N"], hdr["L"], hdr["dp"]) == (k, N, L, dp)
    rng = np.random.default_rng(1)
    # source-distributed blocks plus points spread over the whole ball (edge cells)
    z = np.concatenate([fo.sample_source_blocks(3000, dp, k, rng),
                        fo.sample_source_blocks(500, k + 2, k, rng)])
    nn, _ = fo.nearest_codeword(z, C.astype(np.float64))
    cells = _cell_of(z, hdr)
    for zi, ci, ni in zip(z, cells, nn):
        assert int(ni) in _cell_list(buf, hdr, int(ci))
    # lists are sorted by index (padding repeats the last id), so a strict-less scan keeps
    # the lowest index on exact ties
    for cell in range(0, hdr["n_cells"], max(1, hdr["n_cells"] // 500)):
        ids = _cell_ids(buf, hdr, cell)
        assert ids == sorted(ids)


def test_topc_index_equals_oracle_table():
    C = tables.codebook(64, 4, 8)
    L, c = 6, 3
    buf = fq.fq_build_search_index(C, 64, 4, 8, fq.FQ_INDEX_TOPC, L, c)
    hdr = _parse_index(buf)
    R = fo.grid_range(C.astype(np.float64), 64)
    ref = fo.grid_topc_table(C.astype(np.float64), R, L, c)
    for cell in range(L ** 4):
        assert _cell_ids(buf, hdr, cell) == sorted(int(i) for i in ref[cell])
    assert abs(hdr["lo"] + R) < 1e-6 and abs(hdr["inv_h"] - L / (2 * R)) < 1e-3


def test_index_builder_rejects_bad_arguments():
    C = tables.codebook(64, 2, 16)
    with pytest.raises(fq.FQError):
        fq.fq_build_search_index(C, 64, 2, 16, 0, 1, 2)      # L too small
    with pytest.raises(fq.FQError):
        fq.fq_build_search_index(C, 64, 2, 16, 1, 8, 17)     # c > N
    with pytest.raises(fq.FQError):
        fq.fq_build_search_index(C, 64, 2, 16, 5, 8, 2)      # bad kind
