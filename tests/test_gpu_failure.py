"""Failure detection on the GPU without a fault: an in-kernel wait that never
completes must give up after its wall-clock limit, raise MSA_DEV_PIPE_TIMEOUT
in the device status word and let the kernel finish; the context must stay
usable for the next call.  Nothing here traps, faults or hangs: the waited-on
barrier simply never receives an arrival, and every wait is bounded."""
import time

import numpy as np
import pytest
import torch

import oracle
import routed_sparse_attention_b200 as msa
from gpu_cases import Case
from workloads import TINY_F32

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_expired_wait_flags_the_status_and_the_context_stays_usable():
    assert msa.device_status() == 0
    t0 = time.perf_counter()
    assert msa.debug_expire_wait(2000) == 64          # 2 ms limit: every thread gives up
    assert time.perf_counter() - t0 < 1.0
    assert msa.device_status() & msa.DEV_PIPE_TIMEOUT
    assert msa.device_status() == 0                   # read-and-clear
    case = Case(TINY_F32.replace(per_token=False))    # the next calls run normally
    idx, sc = case.route()
    ref_idx, ref_sc, _ = case.oracle_route()
    assert np.array_equal(idx, ref_idx) and np.array_equal(sc, ref_sc)
    assert msa.device_status() == 0


def test_the_kernels_own_wait_limit_is_about_a_second():
    t0 = time.perf_counter()
    assert msa.debug_expire_wait(0) == 64
    dt = time.perf_counter() - t0
    assert 0.9 <= dt <= 5.0, dt
    assert msa.device_status() & msa.DEV_PIPE_TIMEOUT
