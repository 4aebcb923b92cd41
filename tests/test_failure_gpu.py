"""Failure reporting on the GPU without a fault: the library's bounded waits
run out on purpose (an mbarrier nothing completes, a grid barrier nothing
reaches), report PB_DEV_TIMEOUT through the status word, and leave the
context usable."""
import time

import pytest
import torch

from part_pair_bias_b200 import configs, ops, synth
from tests import parity as pt

pytestmark = pytest.mark.gpu


def test_bounded_waits_run_out_report_and_leave_the_context_usable(oracle_lib):
    assert torch.cuda.is_available(), "the gpu tests need a CUDA device"
    torch.cuda.set_device(0)
    assert ops.get_device_status() == 0
    t0 = time.time()
    ops.selftest_wait_timeouts()
    bits = ops.get_device_status()                 # synchronises
    elapsed = time.time() - t0
    assert bits & ops.PB_DEV_TIMEOUT
    assert 3.0 <= elapsed < 60.0, f"two 2 s waits took {elapsed:.1f} s"
    assert ops.get_device_status() == 0            # reading cleared the word
    b = synth.make_jets(**configs.workload("pr1_n8_p32", seed=0))
    d = pt.Device(b)
    pt.check_attention(pt.to_np(d.fused()), oracle_lib.forward(b), b)
    pt.check_attention(pt.to_np(d.fused(balanced=True)), oracle_lib.forward(b), b)   # grid barrier reset
    assert ops.get_device_status() == 0
