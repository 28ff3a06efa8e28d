"""The failure path of the kernels' bounded waits, on the GPU without a fault.

Every mbarrier wait in the library gives up after a wall-clock limit, sets
MOE_ERR_TIMEOUT in the device status word and lets its kernel return.  Here a
wait runs out for real: moe_selftest_bounded_wait waits, through the kernels'
own bounded-wait routine, on a barrier nothing arrives at, with a 1 ms limit.
The kernel must end by itself, report the timeout, and leave the GPU usable:
the tiny layer is then run and checked against the oracle.
"""
import time

import pytest
import torch

import mixture_experts_lora_b200 as ml
from moe_inputs import CONFIGS

from gpu_common import check_full_parity, ensure_built, inputs_on, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    ensure_built()


def test_expired_wait_reports_timeout_and_gpu_stays_usable():
    assert ml.moe_get_device_error() == ml.MOE_OK          # nothing pending
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    ml.moe_selftest_bounded_wait(1_000_000, done)          # 1 ms limit
    assert ml.moe_get_device_error() == ml.MOE_ERR_TIMEOUT  # synchronises, then clears
    elapsed = time.perf_counter() - t0
    assert done.item() == 1                                 # the kernel ran to its end
    assert elapsed < 5.0
    assert ml.moe_get_device_error() == ml.MOE_OK           # cleared by the read
    # the context is intact: a whole layer still runs and matches the oracle
    cfg = CONFIGS["tiny"]
    inp, cpu = inputs_on(cfg)
    buf = run_layer(inp, cfg)
    check_full_parity(buf, cpu, cfg)


def test_timeout_limit_is_honoured_from_1ms_to_50ms():
    # a longer limit takes at least that long on the device (globaltimer), each run
    # ending by itself with the status set
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    for limit_ms in (1, 50):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        ml.moe_selftest_bounded_wait(limit_ms * 1_000_000, done)
        e.record()
        assert ml.moe_get_device_error() == ml.MOE_ERR_TIMEOUT
        assert done.item() == 1
        assert s.elapsed_time(e) >= 0.9 * limit_ms
