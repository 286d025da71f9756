"""ctypes binding of libfq (the C ABI in include/fq.h): argument marshalling only.

Every function here checks tensor shapes/dtypes/devices, passes ``data_ptr()`` values and the
current CUDA stream to the C entry point of the same name, and raises FQError on a non-OK
status.  All computation happens in the CUDA kernels of libfq.so; there is no fallback: if the
library is missing, importing a compute function raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfq.so")

FQ_F16 = 0
FQ_F32 = 1
FQ_INDEX_EXACT = 0
FQ_INDEX_TOPC = 1
FQ_INDEX_TENSOR = 2
FQ_RESCALE_PLAIN = 0
FQ_RESCALE_MSE = 1
FQ_RESCALE_UNBIASED = 2

_c_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i = ctypes.c_int

_SIGS = {
    "fq_abi_version": (_i, []),
    "fq_status_string": (ctypes.c_char_p, [_i]),
    "fq_padded_dim": (_i, [_i, _i]),
    "fq_payload_bytes": (_sz, [_i, _i, _i]),
    "fq_encode": (_i, [_vp, _i, _c_i64, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fq_decode": (_i, [_vp, _vp, _c_i64, _i, _i, _i, _vp, _vp, _vp, _i, _vp]),
    "fq_attn_workspace_bytes": (_sz, [_i, _i, _i, _c_i64, _i, _i]),
    "fq_attn_decode": (_i, [_vp, _i, _i, _i, _c_i64, _i,
                            _vp, _vp, _i, _i, _vp, _vp,
                            _vp, _vp, _i, _i, _vp, _vp,
                            ctypes.c_float, _vp, _vp, _sz, _vp]),
    "fq_build_search_index": (_i, [_vp, _i, _i, _i, _i, _i, _i, _vp, _sz,
                                   ctypes.POINTER(_sz)]),
    "fq_decode_gather": (_i, [_vp, _vp, _c_i64, _vp, _c_i64, _i, _i, _i, _vp, _vp, _vp, _i,
                              _vp]),
    "fq_attn_decode_lengths": (_i, [_vp, _i, _i, _i, _c_i64, _i, _vp,
                                    _vp, _vp, _i, _i, _vp, _vp,
                                    _vp, _vp, _i, _i, _vp, _vp,
                                    ctypes.c_float, _vp, _vp, _sz, _vp]),
    "fq_attn_decode_append": (_i, [_vp, _vp, _vp, _i, _i, _i, _c_i64, _i, _vp,
                                   _vp, _vp, _i, _i, _vp, _vp,
                                   _vp, _vp, _i, _i, _vp, _vp,
                                   ctypes.c_float, _vp, _vp, _sz, _vp]),
    "fq_encode_rho": (_i, [_vp, _i, _c_i64, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fq_decode_rescaled": (_i, [_vp, _vp, _vp, _c_i64, _i, _i, _i, _vp, _vp, _i, _vp, _i, _vp]),
    "fq_encode_prod": (_i, [_vp, _i, _c_i64, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fq_decode_prod": (_i, [_vp, _vp, _vp, _vp, _c_i64, _i, _i, _vp, _vp, _vp, _vp, _i, _vp]),
    "fq_wait_status": (_i, [ctypes.POINTER(ctypes.c_uint), _i]),
    "fq_selftest_wait_timeout": (_i, [ctypes.c_uint32, _vp]),
    "fq_attn_decode_noalloc": (_i, [_vp, _i, _i, _i, _c_i64, _i,
                                    _vp, _vp, _i, _i, _vp, _vp,
                                    _vp, _vp, _i, _i, _vp, _vp,
                                    ctypes.c_float, _vp, _vp]),
}

FQ_ATTN_NOALLOC_SCRATCH_BYTES = 4 << 20

_lib = None


class FQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: status {status} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """The loaded libfq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m random_access_kv_fq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def status_string(status: int) -> str:
    return lib().fq_status_string(int(status)).decode()


def _check(fn: str, st: int) -> None:
    if st != 0:
        raise FQError(fn, st)


def fq_padded_dim(d: int, k: int) -> int:
    return int(lib().fq_padded_dim(d, k))


def fq_payload_bytes(d: int, k: int, N: int) -> int:
    return int(lib().fq_payload_bytes(d, k, N))


def fq_attn_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, d: int, kV: int) -> int:
    return int(lib().fq_attn_workspace_bytes(B, Hq, Hkv, T, d, kV))


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return FQ_F16
    if t.dtype == torch.float32:
        return FQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def fq_encode(x, rot, codebook, k: int, N: int, codes=None, norms=None, search_index=None,
              stream=None):
    """Encode rows of x [n, d] (fp16/fp32, CUDA).  Returns (codes uint8 [n, P], norms int16
    [n] holding fp16 bit patterns; view them with .view(torch.float16))."""
    import torch
    assert x.dim() == 2 and x.is_cuda and x.is_contiguous()
    n, d = x.shape
    P = fq_payload_bytes(d, k, N)
    if codes is None:
        codes = torch.empty((n, max(P, 1)), dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty((n,), dtype=torch.int16, device=x.device)
    st = lib().fq_encode(_ptr(x), _dtype_code(x), n, d, k, N, _ptr(rot), _ptr(codebook),
                         _ptr(codes), _ptr(norms), _ptr(search_index), _stream(stream))
    _check("fq_encode", st)
    return codes, norms


def fq_decode(codes, norms, rot, codebook, d: int, k: int, N: int, out_dtype=None, y=None,
              stream=None):
    """Decode n records into y [n, d] (fp32 by default, or fp16)."""
    import torch
    n = codes.shape[0]
    if y is None:
        y = torch.empty((n, d), dtype=out_dtype or torch.float32, device=codes.device)
    st = lib().fq_decode(_ptr(codes), _ptr(norms), n, d, k, N, _ptr(rot), _ptr(codebook),
                         _ptr(y), _dtype_code(y), _stream(stream))
    _check("fq_decode", st)
    return y


def fq_attn_decode(q, k_codes, k_norms, kK: int, NK: int, rotK, cbK, v_codes, v_norms,
                   kV: int, NV: int, rotV, cbV, scale: Optional[float] = None, out=None,
                   workspace=None, stream=None):
    """One decode-attention step.  q [B, Hq, d] fp16; k/v codes [B, Hkv, T, P]; norms
    [B, Hkv, T] (fp16 bits).  Returns out [B, Hq, d] fp32."""
    import torch
    B, Hq, d = q.shape
    _, Hkv, T, _ = k_codes.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    need = fq_attn_workspace_bytes(B, Hq, Hkv, T, d, kV)
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().fq_attn_decode(_ptr(q), B, Hq, Hkv, T, d,
                              _ptr(k_codes), _ptr(k_norms), kK, NK, _ptr(rotK), _ptr(cbK),
                              _ptr(v_codes), _ptr(v_norms), kV, NV, _ptr(rotV), _ptr(cbV),
                              float(scale), _ptr(out), _ptr(workspace), ws_bytes,
                              _stream(stream))
    _check("fq_attn_decode", st)
    return out


def fq_decode_gather(codes, norms, token_ids, rot, codebook, d: int, k: int, N: int,
                     out_dtype=None, y=None, stream=None):
    """Decode the records at token_ids (int64 CUDA tensor, any order, repeats allowed) of the
    plane (codes [n, P], norms [n]) into y [len(token_ids), d]."""
    import torch
    n_ids = token_ids.numel()
    if y is None:
        y = torch.empty((n_ids, d), dtype=out_dtype or torch.float32, device=token_ids.device)
    assert token_ids.dtype == torch.int64 and token_ids.is_contiguous()
    st = lib().fq_decode_gather(_ptr(codes), _ptr(norms), codes.shape[0], _ptr(token_ids), n_ids,
                                d, k, N, _ptr(rot), _ptr(codebook), _ptr(y), _dtype_code(y),
                                _stream(stream))
    _check("fq_decode_gather", st)
    return y


def _attn_ws(q, B, Hq, Hkv, T, d, kV, workspace):
    import torch
    need = fq_attn_workspace_bytes(B, Hq, Hkv, T, d, kV)
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return workspace, ws_bytes


def fq_attn_decode_lengths(q, lengths, k_codes, k_norms, kK: int, NK: int, rotK, cbK, v_codes,
                           v_norms, kV: int, NV: int, rotV, cbV, scale: Optional[float] = None,
                           out=None, workspace=None, stream=None):
    """fq_attn_decode with per-sequence context lengths (int32 CUDA tensor [B])."""
    import torch
    B, Hq, d = q.shape
    _, Hkv, T, _ = k_codes.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    assert lengths.dtype == torch.int32 and lengths.numel() == B
    workspace, ws_bytes = _attn_ws(q, B, Hq, Hkv, T, d, kV, workspace)
    st = lib().fq_attn_decode_lengths(_ptr(q), B, Hq, Hkv, T, d, _ptr(lengths),
                                      _ptr(k_codes), _ptr(k_norms), kK, NK, _ptr(rotK), _ptr(cbK),
                                      _ptr(v_codes), _ptr(v_norms), kV, NV, _ptr(rotV), _ptr(cbV),
                                      float(scale), _ptr(out), _ptr(workspace), ws_bytes,
                                      _stream(stream))
    _check("fq_attn_decode_lengths", st)
    return out


def fq_attn_decode_append(q, k_new, v_new, lengths, k_codes, k_norms, kK: int, NK: int, rotK,
                          cbK, v_codes, v_norms, kV: int, NV: int, rotV, cbV,
                          scale: Optional[float] = None, out=None, workspace=None, stream=None):
    """One decode step that encodes its own key/value (fp16 [B, Hkv, d]) into slot lengths[b]
    of the caches (in place), attends over lengths[b] + 1 tokens and advances lengths."""
    import torch
    B, Hq, d = q.shape
    _, Hkv, T, _ = k_codes.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    assert lengths.dtype == torch.int32 and lengths.numel() == B
    assert k_new.shape == (B, Hkv, d) and v_new.shape == (B, Hkv, d)
    workspace, ws_bytes = _attn_ws(q, B, Hq, Hkv, T, d, kV, workspace)
    st = lib().fq_attn_decode_append(_ptr(q), _ptr(k_new), _ptr(v_new), B, Hq, Hkv, T, d,
                                     _ptr(lengths), _ptr(k_codes), _ptr(k_norms), kK, NK,
                                     _ptr(rotK), _ptr(cbK), _ptr(v_codes), _ptr(v_norms), kV, NV,
                                     _ptr(rotV), _ptr(cbV), float(scale), _ptr(out),
                                     _ptr(workspace), ws_bytes, _stream(stream))
    _check("fq_attn_decode_append", st)
    return out


def fq_attn_decode_noalloc(q, k_codes, k_norms, kK: int, NK: int, rotK, cbK, v_codes, v_norms,
                           kV: int, NV: int, rotV, cbV, scale: Optional[float] = None, out=None,
                           stream=None):
    """fq_attn_decode without a workspace argument: the library's fixed per-GPU scratch holds
    the partials (for callers that cannot allocate device memory)."""
    import torch
    B, Hq, d = q.shape
    _, Hkv, T, _ = k_codes.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    st = lib().fq_attn_decode_noalloc(_ptr(q), B, Hq, Hkv, T, d,
                                      _ptr(k_codes), _ptr(k_norms), kK, NK, _ptr(rotK), _ptr(cbK),
                                      _ptr(v_codes), _ptr(v_norms), kV, NV, _ptr(rotV), _ptr(cbV),
                                      float(scale), _ptr(out), _stream(stream))
    _check("fq_attn_decode_noalloc", st)
    return out


def fq_encode_rho(x, rot, codebook, k: int, N: int, search_index=None, stream=None):
    """fq_encode plus the rho plane of the target-aware rescale.  Returns (codes, norms, rho);
    norms and rho hold fp16 bit patterns."""
    import torch
    assert x.dim() == 2 and x.is_cuda and x.is_contiguous()
    n, d = x.shape
    P = fq_payload_bytes(d, k, N)
    codes = torch.empty((n, max(P, 1)), dtype=torch.uint8, device=x.device)
    norms = torch.empty((n,), dtype=torch.int16, device=x.device)
    rho = torch.empty((n,), dtype=torch.int16, device=x.device)
    st = lib().fq_encode_rho(_ptr(x), _dtype_code(x), n, d, k, N, _ptr(rot), _ptr(codebook),
                             _ptr(codes), _ptr(norms), _ptr(rho), _ptr(search_index),
                             _stream(stream))
    _check("fq_encode_rho", st)
    return codes, norms, rho


def fq_decode_rescaled(codes, norms, rho, rot, codebook, d: int, k: int, N: int, rule: int,
                       out_dtype=None, stream=None):
    import torch
    n = codes.shape[0]
    y = torch.empty((n, d), dtype=out_dtype or torch.float32, device=codes.device)
    st = lib().fq_decode_rescaled(_ptr(codes), _ptr(norms), _ptr(rho), n, d, k, N, _ptr(rot),
                                  _ptr(codebook), rule, _ptr(y), _dtype_code(y), _stream(stream))
    _check("fq_decode_rescaled", st)
    return y


def fq_encode_prod(x, rot, c1, qjl, stream=None):
    """TurboQuant_prod encode.  Returns (codes, signs, norms, gamma)."""
    import torch
    assert x.dim() == 2 and x.is_cuda and x.is_contiguous()
    n, d = x.shape
    N1 = c1.numel()
    P1 = fq_payload_bytes(d, 1, N1)
    codes = torch.empty((n, max(P1, 1)), dtype=torch.uint8, device=x.device)
    signs = torch.empty((n, (d + 7) // 8), dtype=torch.uint8, device=x.device)
    norms = torch.empty((n,), dtype=torch.int16, device=x.device)
    gamma = torch.empty((n,), dtype=torch.int16, device=x.device)
    st = lib().fq_encode_prod(_ptr(x), _dtype_code(x), n, d, N1, _ptr(rot), _ptr(c1), _ptr(qjl),
                              _ptr(codes), _ptr(signs), _ptr(norms), _ptr(gamma), _stream(stream))
    _check("fq_encode_prod", st)
    return codes, signs, norms, gamma


def fq_decode_prod(codes, signs, norms, gamma, rot, c1, qjl, d: int, out_dtype=None,
                   stream=None):
    import torch
    n = codes.shape[0]
    y = torch.empty((n, d), dtype=out_dtype or torch.float32, device=codes.device)
    st = lib().fq_decode_prod(_ptr(codes), _ptr(signs), _ptr(norms), _ptr(gamma), n, d,
                              c1.numel(), _ptr(rot), _ptr(c1), _ptr(qjl), _ptr(y), _dtype_code(y),
                              _stream(stream))
    _check("fq_decode_prod", st)
    return y


def fq_wait_status(clear: bool = False) -> int:
    """Number of CTAs whose bounded device-side waits gave up on the current device (waits for
    the device first).  0 means no launch since the last clear lost a wait."""
    n = ctypes.c_uint(0)
    st = lib().fq_wait_status(ctypes.byref(n), 1 if clear else 0)
    if st not in (0, 6):
        _check("fq_wait_status", st)
    return int(n.value)


def fq_build_search_index(codebook, d: int, k: int, N: int, kind: int, L: int,
                          c: int) -> np.ndarray:
    """Build the grid candidate index on the host; returns a uint8 numpy buffer to upload."""
    cb = np.ascontiguousarray(np.asarray(codebook, dtype=np.float32))
    need = _sz(0)
    st = lib().fq_build_search_index(cb.ctypes.data, d, k, N, kind, L, c, None, 0,
                                     ctypes.byref(need))
    if st not in (0, 4):
        _check("fq_build_search_index", st)
    buf = np.zeros(int(need.value), dtype=np.uint8)
    st = lib().fq_build_search_index(cb.ctypes.data, d, k, N, kind, L, c, buf.ctypes.data,
                                     buf.size, ctypes.byref(need))
    _check("fq_build_search_index", st)
    return buf
