"""Failure reporting without a GPU fault: a kernel whose bounded pipeline wait is
never satisfied gives up after its limit, records FP4_ERR_TIMEOUT in the device
status word and returns; the context stays usable."""
import numpy as np
import pytest
import torch

import fp4_block_scaled_deterministic_b200 as fp4
from fp4_block_scaled_deterministic_b200 import synthetic
from gpu_util import gpu_quantize_raw, need_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def test_bounded_wait_reports_timeout_and_context_survives(orc):
    assert fp4.fp4_check_status() == 0
    assert fp4.fp4_selftest_timeout(20_000_000) == 0  # 20 ms limit
    assert fp4.fp4_check_status() == 6                 # FP4_ERR_TIMEOUT
    assert fp4.fp4_check_status() == 0                 # cleared by the read
    x = synthetic.normal(128, 256, seed=4)
    got = gpu_quantize_raw(x, 0, 16, 0)
    want = orc.quantize(x, 0, 16, 0)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])


def test_non_sm100_device_check_is_host_side():
    major, _ = torch.cuda.get_device_capability()
    assert major == 10, "these tests target B200 (sm_100)"
