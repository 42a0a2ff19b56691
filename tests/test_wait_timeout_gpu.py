"""The bounded pipeline wait, made to run out on purpose.

Every pipelined kernel of the library waits on mbarriers with a bounded
wait: after the device's wait limit it sets MIMO_ATTN_DEVERR_TIMEOUT in the
device error word and tears down instead of hanging. Here the limit is
shortened to ~1 ms through the test hook and a probe kernel waits on an
mbarrier that nothing ever arrives on (no copy or tensor-core operation in
flight). The wait must end, the timeout bit must reach the host, and the
context must stay usable: after the default limit is restored, a normal
prefill of each layer kind still passes parity against the fp64 oracle.
"""
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
from tests.parity_util import check_prefill

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mimo.load()
    mimo.mimo_attn_get_device_error()  # clear


def test_wait_timeout_sets_error_bit_and_context_survives():
    assert mimo.mimo_attn_get_device_error() == 0
    try:
        assert mimo.mimo_attn_debug_set_wait_limit(2_000_000) == mimo.OK  # ~1 ms of SM cycles
        for _ in range(2):
            assert mimo.mimo_attn_debug_wait_probe() == mimo.OK
            torch.cuda.synchronize()  # the probe ended by itself
            bits = mimo.mimo_attn_get_device_error()
            assert bits & mimo.DEVERR_TIMEOUT
            assert mimo.mimo_attn_get_device_error() == 0  # read clears it
    finally:
        assert mimo.mimo_attn_debug_set_wait_limit(0) == mimo.OK  # default limit again
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        c, _, _ = check_prefill(spec, 1, 300, torch.bfloat16, seed=21)
        assert c.ok(torch.bfloat16), f"type {lt} after a timeout: {c.max_abs:.3e} {c.mean_abs:.3e}"
    assert mimo.mimo_attn_get_device_error() == 0
