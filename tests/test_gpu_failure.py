"""Failure detection on the GPU without a fault: a kernel whose bounded wait runs out (on an
mbarrier phase that nothing completes) must be reported by fq_wait_status as FQ_ERR_TIMEOUT,
and the context must stay usable afterwards."""
import ctypes

import numpy as np
import pytest
import torch

import random_access_kv_fq_b200 as fq
from random_access_kv_fq_b200 import _lib, tables, workloads as wl

pytestmark = pytest.mark.gpu

FQ_ERR_TIMEOUT = 6


def test_a_wait_that_runs_out_is_reported_and_the_context_survives():
    L = _lib.lib()
    n = ctypes.c_uint(0)
    L.fq_wait_status(ctypes.byref(n), 1)          # start from a clear count
    assert L.fq_wait_status(ctypes.byref(n), 0) == 0 and n.value == 0
    stream = torch.cuda.current_stream().cuda_stream
    assert L.fq_selftest_wait_timeout(2000, stream) == 0
    assert L.fq_wait_status(ctypes.byref(n), 0) == FQ_ERR_TIMEOUT and n.value == 1
    assert L.fq_selftest_wait_timeout(500, stream) == 0
    assert L.fq_wait_status(ctypes.byref(n), 1) == FQ_ERR_TIMEOUT and n.value == 2
    assert L.fq_wait_status(ctypes.byref(n), 0) == 0 and n.value == 0   # cleared
    assert L.fq_selftest_wait_timeout(0, stream) == 1                  # invalid poll count
    # the context still runs the codec, and a healthy launch counts nothing
    rot, cb = tables.rotation(64, 17), tables.codebook(64, 2, 16)
    x = torch.from_numpy(wl.gaussian_rows(4096, 64, 5)).cuda()
    codes, norms = fq.fq_encode(x, torch.from_numpy(rot).cuda(), torch.from_numpy(cb).cuda(), 2, 16)
    y = fq.fq_decode(codes, norms, torch.from_numpy(rot).cuda(), torch.from_numpy(cb).cuda(), 64, 2, 16)
    torch.cuda.synchronize()
    assert torch.isfinite(y).all()
    assert fq.fq_wait_status() == 0
