"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported through
hbl_device_status, the flag clears on reading, and the context keeps computing exact results."""
import numpy as np
import pytest

import oracle
import hadamard_bit_quant_hbl_b200 as hbl
from test_gpu_parity import run_gemm_with_oracle_codes

pytestmark = pytest.mark.gpu


def test_bounded_wait_time_out_is_reported_and_the_context_survives():
    import torch

    torch.cuda.set_device(0)
    assert hbl.hbl_device_status() == hbl.HBL_OK  # nothing pending
    hbl.hbl_selftest_timeout(50)  # a wait on a barrier nothing completes, 50 ms limit
    assert hbl.hbl_device_status() == hbl.HBL_ETIMEOUT
    assert hbl.hbl_device_status() == hbl.HBL_OK  # the flag was cleared by the read

    rng = np.random.default_rng(11)
    q = rng.integers(-8, 8, size=(3, 1024)).astype(np.int8)
    t = rng.integers(-1, 2, size=(1024, 136)).astype(np.int8)
    s = rng.uniform(0.01, 0.1, size=3)
    acc, _ = run_gemm_with_oracle_codes(q, t, s, 0.02, hbl.HBL_CODES_I8, 4)
    np.testing.assert_array_equal(acc.astype(np.int64), oracle.ternary_matmul(q, t))
    assert hbl.hbl_device_status() == hbl.HBL_OK
