"""Seeded synthetic inputs for the quantized gated FFN / MoE layer.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It holds no arithmetic of the method: it only draws random numbers and stores
them in the documented storage formats.

Storage formats (the pages name only "INT8" for the Gemma shared expert and
"INT4-affine" for the routed blobs; the layouts below are this library's choice):

* bf16 tensors are ``numpy.uint16`` arrays of raw bf16 bits.
* INT8-row: ``q`` int8 [N][K] and ``scale`` fp16 [N]; weight = q * scale.
* INT4-affine, groups of 32 along K: ``packed`` uint8 [N][K/2] where element 2j
  is the low nibble of byte j and element 2j+1 the high nibble, ``scale`` fp16
  [N][K/32] and ``min`` fp16 [N][K/32]; weight = q * scale + min.

Random streams: every tensor draws from its own
``numpy.random.default_rng(SeedSequence([config, seed, tensor_id]))``; the
per-call activations (x, residual) add the token count M to the key, so that
weights are the same for every M of a configuration.

Value recipes follow the five configurations the library is measured on:
x, residual ~ N(0,1) (bf16); INT8 q ~ U{-127..127}, per-row scale ~ U(0.001,
0.01); INT4 q ~ U{0..15}, scale ~ U(0.002, 0.02), min ~ N(0, 0.05); RMSNorm
weight ~ 1 + N(0, 0.1) (bf16); router weights ~ N(0, 0.02) in fp32 (Qwen-shaped)
or bf16 (Mixtral-shaped); shared-expert gate vector ~ N(0, 0.02) bf16.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np
import torch

FMT_INT8_ROW = "int8_row"
FMT_INT4_G32 = "int4_g32"
FMT_Q4_K = "q4_k"      # GGUF K-quant super-blocks: 256 weights in 144 bytes

# Tensor ids of the random streams.
_T_X, _T_RES, _T_NORM_W, _T_ROUTER, _T_WSG = 0, 1, 2, 3, 4
_T_DENSE = 10          # gate/up/down -> 10, 11, 12
_T_SHARED = 20         # shared expert gate/up/down -> 20, 21, 22
_T_EXPERT = 1000       # expert e matrix j -> 1000 + 3e + j


@dataclass(frozen=True)
class LayerConfig:
    """Shape and format of one measured layer configuration."""
    cfg: int
    name: str
    kind: str              # "dense" | "shared" | "moe"
    H: int                 # hidden size (model width)
    I: int                 # intermediate width (dense) or per-expert width
    fmt: str               # weight format of the FFN matrices
    act: str               # "silu" | "gelu_tanh"
    Ms: tuple              # token counts measured
    E: int = 0             # experts (moe)
    k: int = 0             # top-k (moe)
    I_s: int = 0           # shared-expert width (moe, 0 = none)
    router: str = ""       # "f32" | "bf16" (moe)
    eps: float = 1e-6      # RMSNorm epsilon (shared)


CONFIGS: Dict[int, LayerConfig] = {
    1: LayerConfig(1, "dense-h512-i1408-int8row", "dense", 512, 1408, FMT_INT8_ROW, "silu", (1,)),
    2: LayerConfig(2, "llama3-8b-ffn-h4096-i14336-int4g32", "dense", 4096, 14336, FMT_INT4_G32,
                   "silu", (1, 4, 16)),
    3: LayerConfig(3, "gemma-shared-expert-h3072-i12288-int8row-rmsnorm", "shared", 3072, 12288,
                   FMT_INT8_ROW, "gelu_tanh", (1, 8, 32)),
    4: LayerConfig(4, "qwen-moe-h2048-e128-i768-top8-shared512", "moe", 2048, 768, FMT_INT4_G32,
                   "silu", (1, 2, 4), E=128, k=8, I_s=512, router="f32"),
    5: LayerConfig(5, "mixtral-moe-h4096-e8-i14336-top2", "moe", 4096, 14336, FMT_INT4_G32,
                   "silu", (1, 16, 64, 256, 512), E=8, k=2, I_s=0, router="bf16"),
}


def scaled_config(cfg: int, **overrides) -> LayerConfig:
    """A configuration with the same formats and recipe but other shapes."""
    return replace(CONFIGS[cfg], **overrides)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) for k in key]))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Store float values as bf16 bits (round to nearest even, via torch)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


@dataclass
class QWeight:
    """One quantized matrix W[N][K] in a storage format."""
    fmt: str
    N: int
    K: int
    q: np.ndarray                    # int8 [N][K], uint8 packed [N][K/2] or Q4_K blocks [N][K/256*144]
    scale: Optional[np.ndarray]      # fp16 [N] or [N][K/32]; None for Q4_K (in the blocks)
    min: Optional[np.ndarray] = None  # fp16 [N][K/32] (INT4 only)

    @property
    def nbytes(self) -> int:
        return int(self.q.nbytes + (0 if self.scale is None else self.scale.nbytes)
                   + (0 if self.min is None else self.min.nbytes))


@dataclass
class FFNWeights:
    gate: QWeight
    up: QWeight
    down: QWeight

    @property
    def nbytes(self) -> int:
        return self.gate.nbytes + self.up.nbytes + self.down.nbytes


def random_qweight(fmt: str, N: int, K: int, rng: np.random.Generator,
                   int8_scale=(0.001, 0.01), int4_scale=(0.002, 0.02), int4_min_sd=0.05) -> QWeight:
    if fmt == FMT_INT8_ROW:
        q = rng.integers(-127, 128, size=(N, K), dtype=np.int16).astype(np.int8)
        scale = rng.uniform(*int8_scale, size=N).astype(np.float16)
        return QWeight(fmt, N, K, q, scale)
    if fmt == FMT_INT4_G32:
        if K % 32:
            raise ValueError("INT4-affine needs K % 32 == 0")
        # A uniform byte is two independent uniform nibbles.
        packed = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
        scale = rng.uniform(*int4_scale, size=(N, K // 32)).astype(np.float16)
        mn = rng.normal(0.0, int4_min_sd, size=(N, K // 32)).astype(np.float16)
        return QWeight(fmt, N, K, packed, scale, mn)
    if fmt == FMT_Q4_K:
        if K % 256:
            raise ValueError("Q4_K needs K % 256 == 0")
        nb = K // 256
        # Effective step d * scale in [0, 0.04) and offset dmin * min in
        # [0, 0.13), the ranges of the INT4-affine weights; the packed scale
        # bytes and the codes are uniform bytes (every 6-bit field uniform).
        blocks = rng.integers(0, 256, size=(N, nb, 144), dtype=np.uint8)
        d = rng.uniform(int4_scale[0] / 32, int4_scale[1] / 32, size=(N, nb)).astype(np.float16)
        dmin = rng.uniform(0.0005, 0.002, size=(N, nb)).astype(np.float16)
        blocks[..., 0:2] = d.view(np.uint8).reshape(N, nb, 2)
        blocks[..., 2:4] = dmin.view(np.uint8).reshape(N, nb, 2)
        return QWeight(fmt, N, K, blocks.reshape(N, nb * 144), None)
    raise ValueError(f"unknown format {fmt}")


def random_ffn(fmt: str, H: int, I: int, cfg: int, seed: int, base_id: int, down_fmt: Optional[str] = None) -> FFNWeights:
    """gate, up [I][H] in `fmt`; down [H][I] in `down_fmt` (default: the same)."""
    return FFNWeights(
        gate=random_qweight(fmt, I, H, _rng(cfg, seed, base_id + 0)),
        up=random_qweight(fmt, I, H, _rng(cfg, seed, base_id + 1)),
        down=random_qweight(down_fmt or fmt, H, I, _rng(cfg, seed, base_id + 2)),
    )


@dataclass
class LayerInputs:
    """Everything one layer call reads, in storage formats."""
    config: LayerConfig
    M: int
    seed: int
    x: np.ndarray                          # bf16 bits [M][H]
    residual: np.ndarray                   # bf16 bits [M][H]
    ffn: Optional[FFNWeights] = None       # dense / shared configs
    norm_w: Optional[np.ndarray] = None    # bf16 bits [H]
    router: Optional[np.ndarray] = None    # f32 [E][H] or bf16 bits [E][H]
    experts: List[FFNWeights] = field(default_factory=list)
    shared: Optional[FFNWeights] = None
    w_sg: Optional[np.ndarray] = None      # bf16 bits [H]
    # Gemma-style routed layer: learned per-expert scale of the routing
    # weights (fp32 [E]; None = ones) and the shared branch's post-FFN norm
    # weight (bf16 bits [H]; None = the shared expert is gated and seeds the sum)
    expert_scale: Optional[np.ndarray] = None
    shared_norm_w: Optional[np.ndarray] = None
    shared_norm_eps: float = 1e-6

    def weight_bytes_total(self) -> int:
        n = 0
        if self.ffn is not None:
            n += self.ffn.nbytes
        n += sum(e.nbytes for e in self.experts)
        if self.shared is not None:
            n += self.shared.nbytes
        for a in (self.norm_w, self.router, self.w_sg, self.expert_scale, self.shared_norm_w):
            if a is not None:
                n += a.nbytes
        return n


def make_activations(c: LayerConfig, M: int, seed: int):
    x = to_bf16_bits(_rng(c.cfg, seed, _T_X, M).standard_normal((M, c.H)))
    res = to_bf16_bits(_rng(c.cfg, seed, _T_RES, M).standard_normal((M, c.H)))
    return x, res


def make_weights(c: LayerConfig, seed: int) -> LayerInputs:
    """Weights of a configuration (independent of M); x/residual left empty."""
    li = LayerInputs(c, 0, seed, np.zeros((0, c.H), np.uint16), np.zeros((0, c.H), np.uint16))
    if c.kind in ("dense", "shared"):
        li.ffn = random_ffn(c.fmt, c.H, c.I, c.cfg, seed, _T_DENSE)
    if c.kind == "shared":
        li.norm_w = to_bf16_bits(1.0 + _rng(c.cfg, seed, _T_NORM_W).normal(0.0, 0.1, c.H))
    if c.kind == "moe":
        r = _rng(c.cfg, seed, _T_ROUTER).normal(0.0, 0.02, (c.E, c.H))
        li.router = r.astype(np.float32) if c.router == "f32" else to_bf16_bits(r)
        li.experts = [random_ffn(c.fmt, c.H, c.I, c.cfg, seed, _T_EXPERT + 3 * e) for e in range(c.E)]
        if c.I_s:
            li.shared = random_ffn(c.fmt, c.H, c.I_s, c.cfg, seed, _T_SHARED)
            li.w_sg = to_bf16_bits(_rng(c.cfg, seed, _T_WSG).normal(0.0, 0.02, c.H))
    return li


def make_inputs(c: LayerConfig, M: int, seed: int, weights: Optional[LayerInputs] = None) -> LayerInputs:
    """Full inputs of one call: the configuration's weights plus M token rows."""
    li = make_weights(c, seed) if weights is None else replace(weights)
    li.M = M
    li.x, li.residual = make_activations(c, M, seed)
    return li


def zero_like_qweight(fmt: str, N: int, K: int) -> QWeight:
    """An all-zero matrix (q = 0, scale = 0, min = 0) for hand-built cases."""
    if fmt == FMT_INT8_ROW:
        return QWeight(fmt, N, K, np.zeros((N, K), np.int8), np.zeros(N, np.float16))
    if fmt == FMT_Q4_K:
        return QWeight(fmt, N, K, np.zeros((N, K // 256 * 144), np.uint8), None)
    return QWeight(fmt, N, K, np.zeros((N, K // 2), np.uint8), np.zeros((N, K // 32), np.float16),
                   np.zeros((N, K // 32), np.float16))


_T_EXPERT_SCALE, _T_SHARED_NORM = 5, 6


def with_down_format(li: LayerInputs, down_fmt: str, seed: int, int8_scale=(0.001, 0.01)) -> LayerInputs:
    """A dense layer whose down projection is stored in another block format
    (per-tensor block types, as in a mixed quantized file)."""
    c = li.config
    out = replace(li)
    out.ffn = FFNWeights(li.ffn.gate, li.ffn.up,
                         random_qweight(down_fmt, c.H, c.I, _rng(c.cfg, seed, _T_DENSE + 2), int8_scale=int8_scale))
    return out


def make_gemma_form(li: LayerInputs, seed: int) -> LayerInputs:
    """The same routed layer in the Gemma form: a per-expert routing scale
    ~ U(0.5, 2) (fp32) and a post-FFN norm weight of the shared branch
    ~ 1 + N(0, 0.1) (bf16); the shared gate vector is dropped."""
    c = li.config
    out = replace(li)
    out.expert_scale = _rng(c.cfg, seed, _T_EXPERT_SCALE).uniform(0.5, 2.0, c.E).astype(np.float32)
    out.shared_norm_w = to_bf16_bits(1.0 + _rng(c.cfg, seed, _T_SHARED_NORM).normal(0.0, 0.1, c.H))
    out.w_sg = None
    return out
