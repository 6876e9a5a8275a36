"""Failure detection without a GPU fault: a kernel whose bounded mbarrier wait
runs out (a barrier that nothing completes, no copy or product in flight)
returns, the library counts it, intlora_device_status() reports
INTLORA_ERR_TIMEOUT once, and the context stays usable for the next call."""
import pytest
import torch

from quantized_lora_merge_b200 import binding as B

from .parity import gpu_merge, spec_for
from .test_parity_gpu import _check_mul, _oracle_prepared

pytestmark = pytest.mark.gpu

INTLORA_OK, INTLORA_ERR_TIMEOUT = 0, 5


def test_bounded_wait_gives_up_and_is_reported_once():
    torch.cuda.set_device(0)
    assert B.intlora_device_status() == INTLORA_OK           # nothing pending from earlier tests
    before = B.intlora_device_timeouts()
    B.intlora_selftest_bounded_wait(1000)                    # 1 ms, then give up
    assert B.intlora_device_status() == INTLORA_ERR_TIMEOUT
    assert "1 bounded device wait" in B.lib().intlora_last_error().decode()
    assert B.intlora_device_timeouts() == before + 1
    assert B.intlora_device_status() == INTLORA_OK           # reported once
    # the context is still usable: a merge right after matches the oracle
    spec = spec_for(64, 2048, 16, 8, "mul", 8, sid=91)
    inp = _oracle_prepared(spec)
    _check_mul(spec, inp, gpu_merge([spec], [inp])[0])
    assert B.intlora_device_status() == INTLORA_OK

