"""Failure detection on the GPU without a fault: a kernel waits on a barrier
that nothing completes, gives up after a short limit through the same bounded
wait every prefill kernel uses, and the host reads LA_ERR_TIMEOUT from the
device error word.  The context stays usable: a prefill right after is still
correct."""
import numpy as np
import pytest
import torch

import recurrent_decode_la_b200 as la
from gpu_util import BF16_TOL, gpu_prefill, nerr
from oracle import la_oracle as ora
from recurrent_decode_la_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    la.load_library()


def test_bounded_wait_times_out_and_reports():
    assert la.la_device_status() == la.LA_OK
    la.la_selftest_wait_timeout(50.0)
    assert la.la_device_status() == la.LA_ERR_TIMEOUT
    assert "0xf00" in la.binding.last_cuda_error()
    assert la.la_device_status() == la.LA_OK          # reported once, then cleared


def test_context_usable_after_timeout():
    la.la_selftest_wait_timeout(20.0)
    assert la.la_device_status() == la.LA_ERR_TIMEOUT
    q, k, v = inputs.random_qkv(77, 1, 2, 300, 128, 128, dtype=torch.bfloat16)
    O_ref, S_ref = ora.recurrent(q, k, v)
    o, S = gpu_prefill(q, k, v, chunk=128)
    assert nerr(o, O_ref) <= BF16_TOL
    assert nerr(S.reshape(S_ref.shape), S_ref) <= BF16_TOL


def test_selftest_rejects_bad_limits():
    lib = la.load_library()
    assert lib.la_selftest_wait_timeout(0.0, None) == la.LA_ERR_INVALID_ARG
    assert lib.la_selftest_wait_timeout(1e6, None) == la.LA_ERR_INVALID_ARG
