"""Hand-built MoE layers whose outputs are derived by hand (tests/golden).

Input construction only (no arithmetic of the method): each builder places a
few quantized weights so that every intermediate value is exact, and the
derivations in the golden files give the outputs. Shared by the oracle pins
(tests/test_oracle.py) and the GPU checks of the same layers
(tests/test_gpu_kernels.py). ``H`` sets the hidden and intermediate width (256
and up reach the bulk-copy GEMV; several token replicas reach the grouped
tensor-core GEMMs) and ``reps`` repeats the token rows.
"""
from __future__ import annotations

import math

import numpy as np

import synth
from synth import FFNWeights, FMT_INT4_G32


def _zero(N, K):
    return synth.zero_like_qweight(FMT_INT4_G32, N, K)


def _set(w, row, col, q, scale, mn):
    """Code q at W[row][col] (INT4-affine) with the scale and min of its group."""
    byte, hi = col // 2, col % 2
    cur = int(w.q[row, byte])
    w.q[row, byte] = (cur & 0x0F) | (q << 4) if hi else (cur & 0xF0) | q
    w.scale[row, col // 32] = scale
    w.min[row, col // 32] = mn


def _ffn(H, I, cols, down_q, down_scale, down_min):
    """Gate row 0 = 64 and up row 0 = 2^-6 at the given input columns, so the
    activation a_0 = bf16(silu(64) * 1) = 1 for a token e_c, c in cols (silu(64)
    is 64 to fp32 precision); down column 0 of output row 0 is q*scale + min."""
    g, u, d = _zero(I, H), _zero(I, H), _zero(H, I)
    for c in cols:
        _set(g, 0, c, 15, 4.0, 4.0)          # 15 * 4 + 4 = 64
        _set(u, 0, c, 1, 2.0 ** -6, 0.0)     # 2^-6
    _set(d, 0, 0, down_q, down_scale, down_min)
    return FFNWeights(g, u, d)


def _one_hot_rows(H, cols, reps):
    x = np.zeros((len(cols) * reps, H), np.uint16)
    for r in range(reps):
        for i, c in enumerate(cols):
            x[r * len(cols) + i, c] = 0x3F80                # 1.0
    return x


def seed_counterexample(H=32, reps=1):
    """Seeding decides the result (exact in fp32): E = 2, k = 2, zero router
    (equal logits: experts 0, 1, weights 1/2, 1/2), token e_0, shared output 2
    with w_sg = 0 (sigmoid 1/2, seed 1), expert 0 gives d = 2^-23 and expert 1
    gives -2 at feature 0, residual 0. Seed then ranks: (1 + 2^-24) rounds to 1,
    then -1: y = 0. Routed sum then the seed: 2^-24."""
    c = synth.scaled_config(4, H=H, I=H, E=2, k=2, I_s=H)
    shared = _ffn(H, H, [0], 1, 2.0, 0.0)                  # s_0 = 2
    e0 = _ffn(H, H, [0], 2, 2.0 ** -24, 0.0)               # d_0 = 2^-23
    e1 = _ffn(H, H, [0], 0, 0.0, -2.0)                     # d_1 = -2
    x = _one_hot_rows(H, [0], reps)
    return synth.LayerInputs(c, x.shape[0], 0, x, np.zeros_like(x), router=np.zeros((2, H), np.float32),
                             experts=[e0, e1], shared=shared, w_sg=np.zeros(H, np.uint16))


def shared_gate_layer(H=32, reps=1):
    """The sign and operand of the shared-expert gate logit (golden
    shared_gate_seed.txt): w_sg = +141/128 at column 0 and -141/128 at column 1;
    tokens e_0, e_1; the shared expert gives 2 at feature 0 for both; routed
    experts all zero; residual 0. Output feature 0 = bf16(2 * sigmoid(+-141/128))."""
    c = synth.scaled_config(4, H=H, I=H, E=2, k=2, I_s=H)
    shared = _ffn(H, H, [0, 1], 1, 2.0, 0.0)
    zero = FFNWeights(_zero(H, H), _zero(H, H), _zero(H, H))
    w_sg = np.zeros(H, np.uint16)
    w_sg[0] = synth.to_bf16_bits(np.array([141 / 128]))[0]
    w_sg[1] = synth.to_bf16_bits(np.array([-141 / 128]))[0]
    x = _one_hot_rows(H, [0, 1], reps)
    return synth.LayerInputs(c, x.shape[0], 0, x, np.zeros_like(x), router=np.zeros((2, H), np.float32),
                             experts=[zero, zero], shared=shared, w_sg=w_sg)


def rank_pairing_layer(H=32, reps=1):
    """Which routing weight meets which expert output (golden
    rank_weight_pairing.txt): fp32 router rows with ln 3 at columns 0 and 1,
    tokens e_0, e_1 (logits (ln 3, 0) and (0, ln 3): weights 0.75, 0.25),
    expert outputs 4 and -8 at feature 0, no shared expert, residual 0."""
    c = synth.scaled_config(5, H=H, I=H, E=2, k=2, I_s=0, router="f32")
    e0 = _ffn(H, H, [0, 1], 1, 4.0, 0.0)                   # d = 4
    e1 = _ffn(H, H, [0, 1], 0, 0.0, -8.0)                  # d = -8
    router = np.zeros((2, H), np.float32)
    router[0, 0] = np.float32(math.log(3.0))
    router[1, 1] = np.float32(math.log(3.0))
    x = _one_hot_rows(H, [0, 1], reps)
    return synth.LayerInputs(c, x.shape[0], 0, x, np.zeros_like(x), router=router, experts=[e0, e1])


def gemma_routed_layer(H=256, reps=1):
    """The Gemma-style routed layer (golden gemma_routed_layer.txt): the routed
    part of rank_pairing_layer with per-expert scale (2, 0.5), and a shared
    expert with output 2 at feature 0, post-norm weight ones, residual 0."""
    li = rank_pairing_layer(H, reps)
    c = synth.scaled_config(5, H=H, I=H, E=2, k=2, I_s=H, router="f32")
    li.config = c
    li.shared = _ffn(H, H, [0, 1], 1, 2.0, 0.0)             # s_0 = 2 for tokens e_0, e_1
    li.expert_scale = np.array([2.0, 0.5], np.float32)
    li.shared_norm_w = synth.to_bf16_bits(np.ones(H))
    li.shared_norm_eps = 1e-6
    return li
