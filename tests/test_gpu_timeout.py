"""The tensor-core pipeline's bounded waits, exercised without a fault or a
hang (needs a B200): a diagnostic kernel waits on an mbarrier that nothing
completes; its wait gives up well under a second, counts itself and raises
the host-visible flag; the next tensor-core ecco_decode_gemv returns
ECCO_ERR_TIMEOUT and enqueues nothing until ecco_device_timeouts reads the
count and clears the flag; after that the call works again."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import entropy_coded_kv_b200 as ecco
from entropy_coded_kv_b200 import _lib
from test_gpu_parity import inputs, table_set, gemv_check, to_dev_bf16, bits

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def test_a_wait_that_gives_up_is_reported_and_cleared():
    lib = _lib.load()
    blob = table_set("learned_w")
    t = ecco.Tables(blob, DEV)
    rows, cols = 300, 256
    blk_np = oracle.encode(blob, inputs("t5", rows * cols // 128, seed=8), nthreads=8)[0]
    blocks = torch.from_numpy(blk_np).to(DEV)
    x = W.activations(cols, 8, device=DEV)
    n0 = ctypes.c_uint(0)
    assert lib.ecco_device_timeouts(ctypes.byref(n0)) == 0  # also clears the flag

    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    assert lib.ecco_selftest_wait_timeout(stream) == 0
    torch.cuda.synchronize()  # the wait gave up: the context is still usable
    y = torch.full((8, rows), 7.0, dtype=torch.float32, device=DEV)
    rc = lib.ecco_decode_gemv(t.handle, ctypes.c_void_p(blocks.data_ptr()), rows, cols,
                              ctypes.c_void_p(x.data_ptr()), 8, ctypes.c_void_p(y.data_ptr()), stream)
    assert rc == _lib.ECCO_ERR_TIMEOUT and "gave up" in _lib.strerror(rc)
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())  # nothing was enqueued
    # CUDA-core batches do not use the tensor-core pipeline and still run
    y1 = ecco.decode_gemv(blocks, t, rows, cols, x[:2])
    gemv_check(blob, blk_np, rows, cols, bits(x[:2]), y1.cpu().numpy())

    n1 = ctypes.c_uint(0)
    assert lib.ecco_device_timeouts(ctypes.byref(n1)) == 0
    assert n1.value == n0.value + 1
    y8 = ecco.decode_gemv(blocks, t, rows, cols, x)  # flag cleared: works again
    gemv_check(blob, blk_np, rows, cols, bits(x), y8.cpu().numpy())
