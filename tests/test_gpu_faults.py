"""Failure detection on the GPU, without a GPU fault.

The kernels' pipeline waits are bounded: a wait that runs out sets a bit of a
device fault word and the kernel finishes without its result instead of
hanging. These tests make a wait run out on purpose (a weight stage that the
producer never issues, so its barrier is never completed, with a wait limit
of 2 ms), and make a kernel refuse a ring depth it cannot use. They check that
the call returns, that moeffn_device_faults reports the right bit, and that
the next ordinary call matches the oracle. Nothing here traps, faults or hangs
a GPU: every wait ends.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from devutil import DeviceLayer, assert_bf16_close

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("moe_expert_layer_dequant_b200")


@pytest.fixture
def layer():
    c = synth.scaled_config(2, H=512, I=1280)     # INT4, weight-streaming GEMV path at M = 1, 2
    w = synth.make_weights(c, 9)
    dl = DeviceLayer(synth.make_inputs(c, 1, 9, weights=w))
    lib.device_faults(True)                        # start from a clear fault word
    yield c, w, dl
    lib.test_inject_gemv_fault(0)


def _ordinary_call_matches(c, w, dl, M, seed):
    inp = synth.make_inputs(c, M, seed, weights=w)
    assert_bf16_close(dl.run(inp.x, inp.residual), oracle.layer(inp), f"after the fault M={M}")


# The gate/up GEMV of this shape gives each CTA 16 rows (two stages of 8):
# stop 0 starves every stage, stop 1 the second stage of each CTA.
@pytest.mark.parametrize("stop", [0, 1])
def test_timed_out_wait_sets_bit0_and_next_call_is_correct(layer, stop):
    c, w, dl = layer
    _ordinary_call_matches(c, w, dl, 2, 1)
    assert lib.device_faults(True) == 0
    # The producer of the next gate/up GEMV issues no stage from `stop` on:
    # consumers wait 2 ms for a barrier nothing completes, then give up.
    lib.test_inject_gemv_fault(1, stop, 2000)
    inp = synth.make_inputs(c, 2, 2, weights=w)
    dl.run(inp.x, inp.residual)                   # returns; its output is garbage
    torch.cuda.synchronize()                       # the context is still usable
    assert lib.device_faults(True) & 1 == 1
    assert lib.device_faults(True) == 0            # cleared by the read above
    _ordinary_call_matches(c, w, dl, 2, 3)
    _ordinary_call_matches(c, w, dl, 1, 4)
    assert lib.device_faults(True) == 0


def test_invalid_ring_depth_is_refused_with_bit1(layer):
    c, w, dl = layer
    lib.test_inject_gemv_fault(2, 3, 2000)         # 3 is not a multiple of the two consumer groups
    inp = synth.make_inputs(c, 1, 5, weights=w)
    dl.run(inp.x, inp.residual)
    torch.cuda.synchronize()
    assert lib.device_faults(True) & 2 == 2
    _ordinary_call_matches(c, w, dl, 1, 6)
    assert lib.device_faults(True) == 0
