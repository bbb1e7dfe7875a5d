"""Failure detection on the GPU, without a GPU fault.

A test-only knob (moda_test_set_device_fault) shortens every bounded kernel wait to 1 ms
and makes the forward kernel's TMA producer issue no loads.  Every wait for that data then
runs out: each CTA records the timeout in the device error word, waits (bounded) for the
operations it has in flight, releases its tensor memory and exits.
moda_check_device_errors() must return MODA_ERR_TIMEOUT with the timeout bit set and clear
the word, and the context must stay usable: with the knob cleared, the next forward
matches the oracle.  Nothing here traps, faults or hangs the GPU: every wait involved is
bounded, and the kernel leaves through its normal exit.
"""
import ctypes
import math

import pytest
import torch

import depth_aware_attention_b200 as moda
import workloads
from parity_util import compare_forward, gpu_inputs, oracle_forward_window

pytestmark = pytest.mark.gpu

FAULT_FORWARD_NO_LOADS = 1
WAIT_LIMIT_NS = 1_000_000  # 1 ms


@pytest.mark.parametrize("path", [1, 2], ids=["fold", "dense"])
def test_forward_wait_timeout_is_reported_and_the_context_recovers(cuda_device, path):
    cfg = workloads.CONFIGS["tiny"]
    x = gpu_inputs(cfg, seed_base=410 + path)
    scale = 1.0 / math.sqrt(cfg["d"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    moda.check_device_errors()  # the word starts clear
    try:
        assert moda.moda_test_set_device_fault(FAULT_FORWARD_NO_LOADS, WAIT_LIMIT_NS) == \
            moda.MODA_OK, moda.moda_last_error_message()
        moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True, depth_path=path)
        st, flags = moda.moda_check_device_errors(stream)
    finally:
        assert moda.moda_test_set_device_fault(0, 0) == moda.MODA_OK
    assert st == moda.MODA_ERR_TIMEOUT, moda.moda_status_string(st)
    assert flags & 1
    assert moda.moda_check_device_errors(stream) == (moda.MODA_OK, 0)  # read clears it
    # the context is intact: the same call, without the fault, is correct
    out, lse = moda.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], scale, True,
                            depth_path=path)
    moda.check_device_errors()
    ref_out, ref_lse = oracle_forward_window(x, 0, cfg["T"], scale, True)
    compare_forward(out, lse, ref_out, ref_lse, f"after the timeout, path {path}")
