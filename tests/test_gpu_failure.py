"""Failure detection without a GPU fault: every wait inside the library's
kernels is bounded.  The self-test kernel waits on a barrier that nothing
completes; the wait must give up by itself, raise the timeout flag that the host
reads, and leave the context usable for the next call."""
import time

import numpy as np
import pytest
import torch

import mixture_experts_layer_31_b200 as moe
import synth
from gpu_util import gpu_logits, judge, run

pytestmark = pytest.mark.gpu

MOE_FLAG_TIMEOUT = 0x8


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    moe.moe_device_flags(clear=True)
    t0 = time.monotonic()
    moe.moe_selftest_bounded_wait()
    flags = moe.moe_device_flags(clear=True)  # synchronises
    elapsed = time.monotonic() - t0
    assert flags & MOE_FLAG_TIMEOUT
    assert 1.0 < elapsed < 30.0
    prob = synth.make_problem(3, T=40, H=256, E=16, I=128)
    layer, x, y, idx, w = run(prob)
    judge(prob, y, idx, w, logits=gpu_logits(layer, x))
    assert moe.moe_device_flags(clear=True) == 0
