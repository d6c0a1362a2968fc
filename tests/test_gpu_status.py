"""Device status word: a bounded wait that runs out reports a timeout without
faulting, and the context stays usable afterwards."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as O
from nvfp4_block_scaled_15_b200 import inputs
from parity import dev_bf16, host_u8

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(lib):
    assert lib.nvfp4_check_device_status() == lib.OK
    lib.nvfp4_selftest_wait_timeout(50_000_000)            # 50 ms on a barrier nothing arrives on
    assert lib.nvfp4_check_device_status() == lib.ERR_TIMEOUT
    assert lib.nvfp4_check_device_status() == lib.OK       # read clears it
    x = inputs.gaussian_bf16((4, 64), seed=9)
    q = lib.quantize(dev_bf16(x), lib.SF_ROWMAJOR)
    assert lib.nvfp4_check_device_status() == lib.OK
    assert np.array_equal(host_u8(q.codes), O.quantize(x)[0])


def test_arch_is_sm100(lib):
    assert torch.cuda.get_device_capability() == (10, 0)
