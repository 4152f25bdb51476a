"""Failure detection on the device, without a GPU fault: every wait in the
kernels is bounded and, when it runs out, records a bit of the device error
word and returns. lg_wait_selftest runs that path on a barrier nothing ever
arrives on (a short limit); the test reads the bit through lg_device_status
and then checks the device still computes correctly.
"""

import math

import pytest
import torch

import oracle
import attention_sink_long_b200 as lg
import synthetic_inputs as si
from parity import assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_is_reported_and_the_device_stays_usable():
    assert lg.lg_device_status(0) == 0
    lg.lg_wait_selftest(2_000_000)  # about a millisecond of SM cycles
    assert lg.lg_device_status(0) == 32
    assert lg.lg_device_status(0) == 0  # reading clears it
    pat = (64, 1, 4, 0)
    q, k, v = si.prefill_inputs(1, 256, 2, 2, 64)
    o = torch.empty(1, 256, 2, 64, dtype=torch.float32, device="cuda")
    lg.lg_sparse_attn_fwd(pat, q.cuda(), k.cuda(), v.cuda(), o, None, 0.125)
    torch.cuda.synchronize()
    ro, _ = oracle.attention_forward(q, k, v, oracle.Pattern(*pat), 0.125)
    assert_close("O after the self-test", o.cpu().numpy(), ro)
    assert lg.lg_device_status(0) == 0
