"""Failure detection on the GPU without any fault: a kernel waits on an mbarrier that nothing
arrives on, gives up after a 1 ms limit, records DSA_ERR_TIMEOUT in the device status word and
returns; the next normal call on the same context succeeds."""
import time

import numpy as np
import pytest
import torch

import dsa_inputs
from oracle import oracle as ref
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import sparse_attention_tcgen05_b200 as m
    m.load()
    return m


def test_bounded_wait_expires_and_the_context_stays_usable(dsa):
    assert dsa.dsa_last_device_status() == 0
    dsa.dsa_set_wait_limit_ns(1_000_000)  # 1 ms
    try:
        t0 = time.perf_counter()
        dsa.dsa_selftest_wait()
        code = dsa.dsa_last_device_status()  # synchronises
        elapsed = time.perf_counter() - t0
    finally:
        dsa.dsa_set_wait_limit_ns(0)  # back to the default
    assert code == 5, dsa.dsa_status_str(code)  # DSA_ERR_TIMEOUT
    assert elapsed < 1.0
    assert dsa.dsa_last_device_status() == 0  # reading cleared it
    # a normal call afterwards: status OK and a bit-exact result
    wl = dsa_inputs.custom("after_timeout", 4321, 1, 3, 300, 64, 128, 16, 8, 1, 16, 16)
    dw = parity.DeviceWorkload(wl, with_attention=False)
    scores = torch.empty(1, 3, 300, device="cuda")
    dsa.dsa_indexer(dw.qI, dw.kI, dw.w, scores)
    assert dsa.dsa_last_device_status() == 0
    got = scores.cpu().numpy()
    for i in range(3):
        exp = ref.indexer_row(dw.qI_np[i], dw.kI_np[0], dw.w_np[i], wl.t_of(i)).astype(np.float32)
        np.testing.assert_array_equal(got[0, i], exp)
