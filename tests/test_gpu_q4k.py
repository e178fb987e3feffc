"""GPU parity of the Q4_K block type (the K-quant format of Q4_K_M files)
against the CPU oracle: dequantization bit for bit, and dense layers through
the bulk-copy GEMV (decode token counts) and the tcgen05 GEMM (from 6 token
rows), alone and mixed per tensor with the other block types.

Shapes span several CTA row tiles, K ranges of several super-blocks, a down
projection split along K with a ragged last split, and ragged token tiles.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden
from devutil import DeviceLayer, assert_bf16_close, dev_bf16, host_bf16
from synth import FMT_INT4_G32, FMT_INT8_ROW, FMT_Q4_K

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("moe_expert_layer_dequant_b200")


@pytest.mark.parametrize("N,K", [(37, 512), (256, 4096), (8, 256)])
def test_q4_k_dequant_bit_exact(N, K):
    w = synth.random_qweight(FMT_Q4_K, N, K, np.random.default_rng(21))
    f32, b16 = lib.test_dequant(lib.upload_qweight(w))
    torch.cuda.synchronize()
    ref = oracle.dequant(w)
    assert np.array_equal(f32.cpu().numpy().astype(np.float64), ref)
    assert np.array_equal(b16.cpu().numpy().view(np.uint16), oracle.bf16_bits(ref))


def test_q4_k_golden_block_on_gpu():
    kv, _ = read_golden("q4_k_block.txt")
    blk = np.concatenate([np.array([int(t, 16) for t in kv["header_hex"]], np.uint8),
                          np.arange(128, dtype=np.uint8)])[None, :]
    f32, _ = lib.test_dequant(lib.upload_qweight(synth.QWeight(FMT_Q4_K, 1, 256, blk, None)))
    got = f32.cpu().numpy()[0]
    for t in kv["expected"]:
        k, v = t.split(":")
        assert float(got[int(k)]) == float(v)


Q4K_DENSE = [
    dict(H=512, I=1536),     # 2 and 6 blocks per row
    dict(H=1024, I=4352),    # down split along K (2 splits, the last one ragged)
]


def _q4k_config(shape, cfg=2):
    return synth.scaled_config(cfg, fmt=FMT_Q4_K, **shape)


@pytest.mark.parametrize("shape", Q4K_DENSE)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 16, 40, 150])
def test_q4_k_dense(shape, M):
    """Decode GEMV for M <= 5, tensor-core GEMM from M = 6."""
    c = _q4k_config(shape)
    inp = synth.make_inputs(c, M, 5)
    dl = DeviceLayer(inp)
    assert_bf16_close(dl.run(inp.x, inp.residual), oracle.layer(inp), "out")
    inp.residual = np.zeros_like(inp.residual)
    assert_bf16_close(dl.run(inp.x, inp.residual), oracle.layer(inp), "h")


# An INT8 down projection after 4-bit gate/up weights is checked on the GEMV
# path only (M <= 5): on the tensor-core path the 4-bit gate/up weights enter
# the MMA rounded to bf16, and with this INT8 weight mix (zero-mean codes, so
# the down sums cancel) that rounding alone moves a few outputs past 2e-2 * RMS
# (7 of 8192 at M = 16; a CPU model of the same arithmetic moves more), as
# for INT4 gate/up with an INT8 down.
MIXED = [(FMT_Q4_K, FMT_INT4_G32, M) for M in (1, 3, 16)] + \
        [(FMT_INT4_G32, FMT_Q4_K, M) for M in (1, 3, 16)] + \
        [(FMT_Q4_K, FMT_INT8_ROW, M) for M in (1, 3)]


@pytest.mark.parametrize("gu_fmt,down_fmt,M", MIXED)
def test_q4_k_mixed_per_tensor(gu_fmt, down_fmt, M):
    """A Q4_K_M-style file: gate/up and down in different block types."""
    c = synth.scaled_config(2, fmt=gu_fmt, H=512, I=1536)
    inp = synth.with_down_format(synth.make_inputs(c, M, 6), down_fmt, 6, int8_scale=(0.0002, 0.002))
    dl = DeviceLayer(inp)
    assert_bf16_close(dl.run(inp.x, inp.residual), oracle.layer(inp), "out")


@pytest.mark.parametrize("M", [1, 8])
def test_q4_k_shared_expert_rmsnorm_tail(M):
    c = synth.scaled_config(3, fmt=FMT_Q4_K, H=768, I=2304)
    inp = synth.make_inputs(c, M, 2)
    dl = DeviceLayer(inp)
    assert_bf16_close(dl.run(inp.x, inp.residual), oracle.layer(inp), "h1")


@pytest.mark.parametrize("M", [1, 16])
def test_q4_k_dense_prenorm(M):
    c = _q4k_config(dict(H=512, I=1536))
    inp = synth.make_inputs(c, M, 3)
    w = synth.to_bf16_bits(1.0 + np.random.default_rng(3).normal(0, 0.1, c.H))
    dl = DeviceLayer(inp)
    res = dev_bf16(inp.residual)
    lib.ffn_dense_prenorm(dl.ffn, dev_bf16(w), res, c.act, 1e-6)
    assert_bf16_close(host_bf16(res), oracle.layer_prenorm(inp, w, 1e-6), "out")
