"""Helpers of the GPU tests: upload seeded inputs, run the library, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import moe_expert_layer_dequant_b200 as lib

RTOL_RMS = 2e-2   # max |err| <= 2e-2 * RMS(oracle output), bf16 outputs
WTOL_REL = 1e-3   # routing weights, relative

# (what, elements compared, rounding flips accepted, worst |err| / RMS among the
# rest) of every comparison in this session; printed at the end of the run.
FLIP_LOG = []


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def rms(v: np.ndarray) -> float:
    return float(np.sqrt(np.mean(np.asarray(v, np.float64) ** 2)))


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_bf16_close(got_bits: np.ndarray, want_bits: np.ndarray, what: str = "", rtol: float = RTOL_RMS):
    """max |got - want| <= rtol * RMS(want) on bf16 outputs, up to rounding flips.

    For final bf16 outputs of the layer only (never for intermediate values,
    which are compared bit-exactly or at the plain tolerance). Both sides round
    their own pre-rounding values (fp32 here, float64 in the oracle) to bf16
    wherever the layer stores a 2-byte value, the output being the last. Where the two straddle a rounding boundary the stored values
    differ by one bf16 ulp, and a flip in a stored intermediate (h1 before the
    norm, the activation) can add one more. For |v| >= 2.56 * RMS one ulp
    already exceeds 2e-2 * RMS, so an element may instead differ by at most
    two bf16 ulps of its magnitude; such elements must be rare (< 1%).
    """
    g = oracle.bf16_to_f64(got_bits)
    w = oracle.bf16_to_f64(want_bits)
    assert g.shape == w.shape, (g.shape, w.shape)
    scale = rms(w)
    if g.size == 0:
        return 0.0
    err = np.abs(g - w)
    tol = rtol * max(scale, 1e-30)
    flip = (err > tol) & (err <= 2 * bf16_ulp(np.maximum(np.abs(g), np.abs(w))))
    bad = (err > tol) & ~flip
    worst = float(np.max(np.where(flip, 0.0, err)))
    FLIP_LOG.append((what, int(g.size), int(flip.sum()), worst / max(scale, 1e-30)))
    assert not np.any(bad), f"{what}: max|err| {float(err[bad].max()):.3e} > {rtol} * RMS {scale:.3e} ({int(bad.sum())} elements)"
    assert flip.mean() < 1e-2, f"{what}: {int(flip.sum())} rounding flips of {g.size}"
    return worst / max(scale, 1e-30)


class DeviceLayer:
    """A synth.LayerInputs uploaded to the GPU, callable through the C ABI."""

    def __init__(self, inp):
        self.inp = inp
        c = self.c = inp.config
        if c.kind in ("dense", "shared"):
            self.ffn = lib.upload_ffn(inp.ffn)
        if c.kind == "shared":
            self.norm_w = dev_bf16(inp.norm_w)
        if c.kind == "moe":
            r = inp.router
            rt = torch.from_numpy(r).cuda() if r.dtype == np.float32 else dev_bf16(r)
            self.router = lib.plain_weight(rt)
            self.experts = [lib.upload_ffn(e) for e in inp.experts]
            self.shared = lib.upload_ffn(inp.shared) if inp.shared is not None else None
            self.w_sg = lib.plain_weight(dev_bf16(inp.w_sg)) if inp.w_sg is not None else None
            es = getattr(inp, "expert_scale", None)
            sn = getattr(inp, "shared_norm_w", None)
            self.expert_scale = torch.from_numpy(np.asarray(es, np.float32)).cuda() if es is not None else None
            self.shared_norm = dev_bf16(sn) if sn is not None else None
            self.plan = lib.MoePlan(self.router, self.experts, c.k, c.act, self.shared,
                                    None if sn is not None else self.w_sg, self.expert_scale, self.shared_norm,
                                    getattr(inp, "shared_norm_eps", 1e-6))

    def run(self, x_bits: np.ndarray, res_bits: np.ndarray, topk_out: bool = False):
        x = dev_bf16(x_bits)
        res = dev_bf16(res_bits)
        idx = None
        if self.c.kind == "dense":
            lib.ffn_dense(self.ffn, x, res, self.c.act)
            out = res
        elif self.c.kind == "shared":
            out = torch.empty_like(x)
            lib.ffn_shared_expert(self.ffn, x, self.norm_w, out, self.c.act, self.c.eps)
        else:
            idx = torch.empty((x.shape[0], self.c.k), dtype=torch.int32, device="cuda") if topk_out else None
            lib.moe_layer(self.plan, x, res, idx)
            out = res
        torch.cuda.synchronize()
        o = host_bf16(out)
        if topk_out:
            return o, idx.cpu().numpy()
        return o

    def close(self):
        if self.c.kind == "moe":
            self.plan.close()
