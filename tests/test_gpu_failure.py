"""Failure detection on the GPU without a fault (B200 only).

A device wait that nothing satisfies must give up after its limit, report
the timeout in the status word and return normally; the CUDA context must
stay usable.  The wait here is on an mbarrier no thread arrives at, bounded
to 20 ms; nothing traps, faults or hangs.
"""
import time

import pytest
import torch

from tests.gpu_util import ensure_lib, ptr, stream
from tests.test_gpu_kernels import test_block_attention_matches_oracle as _attention_case

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    abi = ensure_lib()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    abi.check(abi.dllm_selftest_wait_timeout(ptr(status), 20000, stream()), "selftest")
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert int(status.item()) & abi.DLLM_DEVICE_TIMEOUT
    assert 0.015 <= waited < 5.0
    # the context is intact: kernels launched afterwards still agree with the oracle
    _attention_case(4, 4, 32, 1, 8, 96, [[(0, 72), (0, 0)]], 0)


def test_selftest_rejects_a_null_status():
    abi = ensure_lib()
    assert abi.dllm_selftest_wait_timeout(None, 100, stream()) == abi.DLLM_ERR_INVALID
