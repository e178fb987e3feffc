"""The allocation-free dense FFN entry point (ffn_dense_noalloc).

It serves callers that cannot allocate device memory at call time; its
scratch is a fixed array inside the library. Checked through the C ABI against
ffn_dense (the workspace entry point) on the same inputs, for two calls in a
row with different inputs (the array keeps the previous call's contents).
This file is collected last so that a failure here leaves every other test run.
"""
import numpy as np
import pytest

import synth
from devutil import DeviceLayer, dev_bf16, host_bf16

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("moe_expert_layer_dequant_b200")


# Token counts 3 and 5 run the weight-streaming GEMVs, 16 and 64 the tcgen05
# GEMMs (their tensor maps then point into the library's array).
@pytest.mark.parametrize("cfg,shape,Ms", [(2, dict(H=512, I=1280), (3, 5)), (1, dict(H=512, I=1408), (3, 5)),
                                          (2, dict(H=256, I=4352), (3, 5)), (2, dict(H=512, I=1280), (16, 64))])
def test_noalloc_matches_workspace_entry_twice(cfg, shape, Ms):
    c = synth.scaled_config(cfg, **shape)
    w = synth.make_weights(c, 3)
    dl = DeviceLayer(synth.make_inputs(c, 1, 3, weights=w))
    assert lib.workspace_bytes(lib.KIND_DENSE, max(Ms), c.H, c.I) <= lib.NOALLOC_SCRATCH_BYTES
    for M, seed in zip(Ms, (11, 12)):           # two calls in a row, different inputs
        inp = synth.make_inputs(c, M, seed, weights=w)
        want = dev_bf16(inp.residual)
        lib.ffn_dense(dl.ffn, dev_bf16(inp.x), want, c.act)
        got = dev_bf16(inp.residual)
        lib.ffn_dense_noalloc(dl.ffn, dev_bf16(inp.x), got, c.act)
        assert np.array_equal(host_bf16(got), host_bf16(want)), f"noalloc M={M}"   # same kernels, same inputs


def test_noalloc_refuses_calls_above_its_array():
    c = synth.scaled_config(2, H=512, I=1280)
    dl = DeviceLayer(synth.make_inputs(c, 1, 0))
    M = 2048                                     # scratch need far above 4 MiB
    assert lib.workspace_bytes(lib.KIND_DENSE, M, 512, 1280) > lib.NOALLOC_SCRATCH_BYTES
    x = dev_bf16(np.zeros((M, 512), np.uint16))
    res = dev_bf16(np.zeros((M, 512), np.uint16))
    with pytest.raises(lib.MoeffnError) as e:
        lib.ffn_dense_noalloc(dl.ffn, x, res, "silu")
    assert e.value.status == -3
