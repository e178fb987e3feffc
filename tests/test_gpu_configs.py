"""GPU parity at the five measured configurations' full sizes.

Every configuration and token count the library is measured on runs through
the C ABI on its full-size seeded inputs; the oracle computes a sample of the
output rows (all rows where it is cheap) and the GPU rows must agree within
max |err| <= 2e-2 * RMS. The selected experts must equal the oracle's wherever
the oracle's top-k margin is not within rounding noise.
"""
import numpy as np
import pytest

import oracle
import synth
from devutil import DeviceLayer, assert_bf16_close, dev_bf16, host_bf16

pytestmark = pytest.mark.gpu

lib = pytest.importorskip("moe_expert_layer_dequant_b200")

ALL_ROWS = 16   # up to this many token rows the oracle checks every row


def _rows(M):
    """Token rows the oracle checks: all of them for small M; else the first and
    last row, the rows on each side of every multiple of 64 (tile edges of the
    GEMMs' token tiles, which hold 16 to 192 rows), and two seeded random rows
    of every 64-row block."""
    if M <= ALL_ROWS:
        return list(range(M))
    rng = np.random.default_rng(M)
    rows = {0, M - 1}
    for b in range(64, M, 64):
        rows |= {b - 1, b}
    for b in range(0, M, 64):
        rows |= set(rng.integers(b, min(M, b + 64), size=2).tolist())
    return sorted(rows)


@pytest.fixture(scope="module", params=[1, 2, 3, 4, 5])
def layer(request):
    c = synth.CONFIGS[request.param]
    w = synth.make_weights(c, 0)
    dl = DeviceLayer(synth.make_inputs(c, 1, 0, weights=w))
    yield c, w, dl
    dl.close()


def test_full_size_parity(layer):
    c, w, dl = layer
    for M in c.Ms:
        inp = synth.make_inputs(c, M, 0, weights=w)
        dl.inp = inp
        if c.kind == "moe":
            out, idx = dl.run(inp.x, inp.residual, topk_out=True)
        else:
            out = dl.run(inp.x, inp.residual)
        rows = _rows(M)
        if c.kind == "moe":
            ref, it = oracle.moe_layer(inp, return_internals=True, tokens=rows)
            lg = it["logits"]
            srt = np.sort(lg, axis=1)[:, ::-1]
            margin = srt[:, c.k - 1] - srt[:, c.k]
            ok = margin > 1e-4 * np.sqrt(np.mean(lg ** 2))
            assert np.array_equal(idx[rows][ok], it["idx"][ok]), f"cfg{c.cfg} M={M}: top-k differs"
        else:
            ref = oracle.layer(inp, tokens=rows)
        assert_bf16_close(out[rows], ref, f"cfg{c.cfg} M={M}")


@pytest.mark.parametrize("cfg,Ms", [(2, (1, 16)), (5, (1, 512))])
def test_full_size_prenorm_parity(cfg, Ms):
    """The input norm folded into the layer at full size (decode and prefill)."""
    c = synth.CONFIGS[cfg]
    w = synth.make_weights(c, 0)
    dl = DeviceLayer(synth.make_inputs(c, 1, 0, weights=w))
    nw = synth.to_bf16_bits(1.0 + np.random.default_rng(cfg).normal(0.0, 0.1, c.H))
    for M in Ms:
        inp = synth.make_inputs(c, M, 0, weights=w)
        res = dev_bf16(inp.residual)
        if c.kind == "moe":
            lib.moe_layer_prenorm(dl.plan, dev_bf16(nw), res, 1e-6)
        else:
            lib.ffn_dense_prenorm(dl.ffn, dev_bf16(nw), res, c.act, 1e-6)
        rows = _rows(M)
        ref = oracle.layer_prenorm(inp, nw, 1e-6, tokens=rows)
        assert_bf16_close(host_bf16(res)[rows], ref, f"cfg{cfg} prenorm M={M}")
    dl.close()
