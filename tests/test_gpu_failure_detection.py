"""Failure detection without a GPU fault: a kernel's bounded wait on a barrier that nothing
arrives on must expire, the host must read KREA2_ERR_TIMEOUT, and the context must stay usable."""
import ctypes

import numpy as np
import pytest
import torch

import krea2_inputs as KI
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K2(cuda_device):
    import flow_matching_stream_b200 as K2
    return K2


def test_bounded_wait_expires_and_is_reported(K2):
    lib = K2.lib()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.krea2_check_device_error(stream) == 0          # clean before
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.krea2_selftest_wait_timeout(200, ctypes.c_void_p(waited.data_ptr()), stream) == 0
    rc = lib.krea2_check_device_error(stream)
    assert rc == -4, lib.krea2_last_error_string()             # KREA2_ERR_TIMEOUT
    assert b"wait expired" in lib.krea2_last_error_string()
    assert int(waited.item()) == 1
    assert lib.krea2_check_device_error(stream) == 0          # the word was cleared
    # the context still runs real work
    d = KI.FULL
    pos = dev(KI.position_ids(16, 4, 4), torch.float32)
    cs = torch.empty(32, 64, device="cuda")
    sn = torch.empty_like(cs)
    K2.rope_tables(d, pos, cs, sn)
    K2.check_device_error()
    assert np.all(np.isfinite(host(cs)))


def test_selftest_rejects_bad_limits_on_the_host(K2):
    lib = K2.lib()
    assert lib.krea2_selftest_wait_timeout(0, None, None) == -1
    assert lib.krea2_selftest_wait_timeout(10000, None, None) == -1
