"""Failure detection on the GPU without a fault: a bounded wait that nothing completes gives
up after its limit, reports QLORA_DEV_TIMEOUT through the status word, and the context stays
usable (a forward right after it still matches the oracle)."""

import time

import pytest
import torch

from bit_quantized_lora_03_b200 import binding as B
from bit_quantized_lora_03_b200 import inputs
from oracle import nf4_oracle as O

from gpu_util import assert_close_rms, f32, require_gpu

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives():
    require_gpu()
    assert B.last_status() == 0                      # clean start
    t0 = time.monotonic()
    B.selftest_wait_timeout(50_000_000)              # 50 ms
    status = B.last_status()
    elapsed = time.monotonic() - t0
    assert status & B.QLORA_DEV_TIMEOUT, status
    assert elapsed >= 0.05
    assert B.last_status() == 0                      # reading the word cleared it

    li = inputs.random_linear(40, 256, 320, 16, 1.0, seed=77, with_grad=False)
    p = B.nf4_quantize(li.Wt.cuda())
    Y, sT = B.qlora_linear_fwd(li.X.cuda(), p, li.L1.cuda(), li.L2.cuda(), li.s)
    assert B.last_status() == 0
    Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
    Y_ref, _ = O.qlora_linear_fwd(f32(li.X), Wdq, f32(li.L1), f32(li.L2), li.s)
    assert_close_rms(f32(Y), Y_ref, "Y after the expired wait")


def test_selftest_limit_is_checked():
    require_gpu()
    with pytest.raises(RuntimeError):
        B.selftest_wait_timeout(10)                  # below 1 us
    with pytest.raises(RuntimeError):
        B.selftest_wait_timeout(3_000_000_000)       # above 2 s
