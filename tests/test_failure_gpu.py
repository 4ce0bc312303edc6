"""Failure detection on the GPU without a fault: every wait in the kernels is bounded and
reports through the device error word. Here a wait that can never complete (an mbarrier
nothing arrives at) is given a 20 ms limit: the kernel gives up, records its code, returns
normally, the host reads NVFP4_ERR_TIMEOUT, and the same CUDA context then runs a GEMM that
matches the oracle with the error word clear."""
import time

import numpy as np
import pytest

import nvfp4_block_scaled_08_b200 as nv
from nvfp4_block_scaled_08_b200 import workloads
import oracle
from helpers import check_within_tolerance, gpu_quantize

pytestmark = pytest.mark.gpu

TIMEOUT = 6            # NVFP4_ERR_TIMEOUT
CHECK_CODE = 0x1FF     # recorded by the bounded-wait check


def test_bounded_wait_gives_up_and_context_stays_usable(cuda_device):
    d = cuda_device
    assert nv.last_device_error()[0] == 0            # clear before
    t0 = time.perf_counter()
    nv.check_bounded_wait(20000)
    status, code = nv.last_device_error()            # synchronises
    dt = time.perf_counter() - t0
    assert status == TIMEOUT and code == CHECK_CODE
    assert 0.015 < dt < 1.0, dt
    assert nv.last_device_error() == (0, 0)          # reading cleared it

    case = workloads.single_case()
    a, b = case.a(), case.b()
    Aq, sfA, gsA = gpu_quantize(a, d)
    Bq, sfB, gsB = gpu_quantize(b, d)
    out = nv.gemm(Aq, sfA, Bq, sfB, nv.alpha(gsA, gsB))
    ga, gb = oracle.global_scale(a.numpy()), oracle.global_scale(b.numpy())
    qa, sa = oracle.quantize(a.numpy(), ga)
    qb, sb = oracle.quantize(b.numpy(), gb)
    alo = oracle.alpha(ga, gb)
    v, S, _ = oracle.gemm(qa, sa, qb, sb, alo)
    check_within_tolerance(out, v, S, alo, "GEMM after a timed-out wait")
    assert nv.last_device_error() == (0, 0)
