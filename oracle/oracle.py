"""CPU oracle for the quantized gated FFN / MoE expert layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or load
this module: only the tests, the smoke check of the package entry file and the
benchmark's CPU-baseline leg use it. It shares no code with the CUDA library.

It is a plain, slow, step-by-step restatement of what the layer computes, in
float64 (numpy), with values rounded to bf16 / fp16 / fp32 exactly where the
method stores them in that precision. The step order follows the pages:

* [gemma]  turbospark-runtime 0.1.0, ``src/families/gemma4/shared_expert.rs``:
  ``encode_shared_expert_branch`` and its batched sibling (gate and up
  projections, gated activation, down projection, then an in-place RMSNorm with
  ``post_feedforward_layernorm_1`` and ``RMS_EPS = 1e-6``).
* [qwen]   turbospark-runtime 0.3.0, ``src/families/qwen/moe_batch.rs``:
  module doc (seeded accumulator, no sandwich norm, ``per_expert_ones``, pair
  order) and ``encode_qwen_layer_moe_batched`` (host top-k, routes, gated
  shared expert, phase 1, phase 2, raw residual add).
* [llama]  turbospark-runtime 0.3.0, ``src/families/llama/dense.rs``: module
  doc formula box (``h = down_proj(act(gate_proj @ m, up_proj @ m)); x = x + h``)
  and ``encode_llama_layer_dense``.

Readings taken where the pages are silent (each is listed with its reason in the
design notes of the repository):

1. Weight formats and layouts come from the measured configurations: INT8 with
   a per-row fp16 scale, and INT4-affine with groups of 32 along K, fp16 scale
   and fp16 min, ``w = q * scale + min``; nibble 2j is the low half of byte j.
2. The activation multiplies ``act(gate)`` by ``up`` (argument order gate, up,
   out of ``encode_silu_mul`` / ``encode_gelu_mul`` in [gemma]); GELU is the
   tanh form.
3. RMSNorm multiplies by ``w`` (not ``1 + w``), with eps inside the root and
   the mean taken over the hidden size, on the bf16 value of ``h1``.
4. Top-k orders experts by (logit descending, index ascending); the routing
   weights are the softmax over the k selected logits times the per-expert
   scale (all ones), rounded to fp16 (the routes carry ``routing16``).
5. Phase 2 accumulates in fp32, seed first, then ranks 0..k-1 in order, each
   term rounded as a product then a sum.
6. Values the pages keep in 2-byte buffers are rounded to bf16: the gated
   activation, the FFN output before a tail, the shared-expert output, the
   seed, the routed output ``y`` and the layer output. Router logits and the
   shared-expert gate logit are fp32; gate/up/down dot products are float64.
7. The K-quant block type Q4_K ([llama]: a Q4_K_M file mixes block types per
   tensor, resolved by ``encode_gemv_any``) is not laid out on the pages; its
   layout is the public GGUF one (256-weight super-blocks of 144 bytes: fp16 d
   and dmin, eight 6-bit scales and mins packed in 12 bytes, 128 bytes of
   4-bit codes), with w = d * scale * q - dmin * min rounded once to fp32.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64: the upper half of an fp32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), as bit patterns.

    Written from the definition: bf16 keeps 8 significant bits and fp32's
    exponent range. The value is scaled so that its 8 significant bits form an
    integer, rounded with round-half-even, and scaled back; subnormals keep the
    fixed quantum 2^-133. Finite inputs only.
    """
    v = np.asarray(v, dtype=np.float64)
    out = v.copy()                                # zeros keep their sign
    nz = v != 0
    m, e = np.frexp(v[nz])                        # v = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                       # below 2^-126: fixed quantum 2^-133
    quantum_exp = e - 8
    out[nz] = np.rint(np.ldexp(v[nz], -quantum_exp)) * np.ldexp(1.0, quantum_exp)
    f32 = out.astype(np.float32)                  # exact: out has <= 8 significant bits
    if not np.all(np.isfinite(f32)):
        raise OverflowError("value outside the bf16 range")
    return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16(v: np.ndarray) -> np.ndarray:
    """Round to bf16 and return the rounded value as float64."""
    return bf16_to_f64(bf16_bits(v))


def f32(v: np.ndarray) -> np.ndarray:
    """Round to fp32 (nearest even) and return as float64."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


def f16(v: np.ndarray) -> np.ndarray:
    """Round to fp16 (nearest even) and return as float64."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------
# Dequantization (reading 1)
# ----------------------------------------------------------------------------


def dequant_int8_row(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """W[n][k] = q[n][k] * scale[n]. Exact in fp32 (8-bit times 11-bit)."""
    return np.asarray(q, np.float64) * np.asarray(scale, np.float64)[:, None]


def int4_codes(packed: np.ndarray) -> np.ndarray:
    """Unpack uint8 [N][K/2] into codes [N][K]; element 2j is the low nibble."""
    p = np.asarray(packed, np.uint8)
    q = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.int64)
    q[:, 0::2] = p & 0x0F
    q[:, 1::2] = p >> 4
    return q


def dequant_int4_affine_g32(packed: np.ndarray, scale: np.ndarray, mn: np.ndarray) -> np.ndarray:
    """W[n][k] = q[n][k] * scale[n][k // 32] + min[n][k // 32].

    "INT4-affine" is the only expert blob layout the batched routed pass
    accepts ([qwen], ``encode_qwen_layer_moe_batched`` refusal of
    ``RoutedBlobLayout`` other than ``Affine``).
    """
    q = int4_codes(packed).astype(np.float64)
    g = np.arange(q.shape[1]) // 32
    s = np.asarray(scale, np.float64)[:, g]
    m = np.asarray(mn, np.float64)[:, g]
    return q * s + m


Q4K_BLOCK = 256       # weights per K-quant super-block
Q4K_BYTES = 144       # 2 (d) + 2 (dmin) + 12 (packed 6-bit scales and mins) + 128 (codes)


def q4_k_scales_mins(packed12: np.ndarray):
    """The eight 6-bit (scale, min) pairs of a Q4_K super-block from its 12
    packed bytes [..., 12] (the GGUF K-quant layout, which the pages name as
    the block type of a Q4_K_M file but do not spell out, reading 7):

    * sub-blocks 0..3: scale = low 6 bits of byte j, min = low 6 bits of byte j + 4;
    * sub-blocks 4..7: the low 4 bits of scale and min are the low and high
      nibble of byte j + 4, and their top 2 bits are the top 2 bits of bytes
      j - 4 (scale) and j (min).
    """
    b = np.asarray(packed12, np.int64)
    sc = np.empty(b.shape[:-1] + (8,), np.int64)
    mn = np.empty_like(sc)
    for j in range(4):
        sc[..., j] = b[..., j] & 63
        mn[..., j] = b[..., j + 4] & 63
    for j in range(4, 8):
        sc[..., j] = (b[..., j + 4] & 15) | ((b[..., j - 4] >> 6) << 4)
        mn[..., j] = (b[..., j + 4] >> 4) | ((b[..., j] >> 6) << 4)
    return sc, mn


def q4_k_codes(blocks: np.ndarray) -> np.ndarray:
    """Codes [..., 256] of super-blocks [..., 144]: the 128 code bytes are four
    runs of 32; run c holds elements 64c..64c+31 in its low nibbles and
    64c+32..64c+63 in its high nibbles."""
    qs = np.asarray(blocks, np.int64)[..., 16:Q4K_BYTES]
    q = np.empty(qs.shape[:-1] + (Q4K_BLOCK,), np.int64)
    for c in range(4):
        run = qs[..., 32 * c:32 * c + 32]
        q[..., 64 * c:64 * c + 32] = run & 15
        q[..., 64 * c + 32:64 * c + 64] = run >> 4
    return q


def dequant_q4_k(blocks: np.ndarray, N: int, K: int) -> np.ndarray:
    """W[n][k] of a Q4_K matrix stored as super-blocks [N][K/256][144]:
    w = d * scale_j * q - dmin * min_j for element k of sub-block j = (k % 256) // 32,
    with d and dmin the block's fp16 super-scales (little-endian bytes 0-1, 2-3).

    Both products are exact in fp32 (at most 21 and 17 significant bits), so
    the value is the exact difference rounded once to fp32, which is what the
    format's fp32 dequantization gives with or without a fused multiply-add
    (reading 7). The difference is formed exactly in float64 whenever its
    fp32 rounding depends on it.
    """
    b = np.asarray(blocks, np.uint8).reshape(N, K // Q4K_BLOCK, Q4K_BYTES)
    d = b[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    dmin = b[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    sc, mn = q4_k_scales_mins(b[..., 4:16])
    q = q4_k_codes(b)
    sub = np.arange(Q4K_BLOCK) // 32
    w = d[..., None] * sc[..., sub] * q - dmin[..., None] * mn[..., sub]
    return f32(w).reshape(N, K)


def dequant(w) -> np.ndarray:
    """Dequantize a ``synth.QWeight``-like object (fields fmt, q, scale, min)."""
    if w.fmt == "int8_row":
        return dequant_int8_row(w.q, w.scale)
    if w.fmt == "int4_g32":
        return dequant_int4_affine_g32(w.q, w.scale, w.min)
    if w.fmt == "q4_k":
        return dequant_q4_k(w.q, w.N, w.K)
    raise ValueError(f"unknown format {w.fmt}")


# ----------------------------------------------------------------------------
# FFN steps
# ----------------------------------------------------------------------------


def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g * sigmoid(g) = g / (1 + exp(-g))."""
    g = np.asarray(g, np.float64)
    return g / (1.0 + np.exp(-g))


def gelu_tanh(g: np.ndarray) -> np.ndarray:
    """GELU, tanh form: 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))."""
    g = np.asarray(g, np.float64)
    return 0.5 * g * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (g + 0.044715 * g ** 3)))


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


ACTS = {"silu": silu, "gelu_tanh": gelu_tanh}


def gated_activation(g: np.ndarray, u: np.ndarray, act: str) -> np.ndarray:
    """a = bf16(act(g) * u): ``encode_silu_mul`` / ``encode_gelu_mul`` take
    (gate, up, out) in that order ([gemma] shared branch) and write a 2-byte
    buffer (``ffn_act``)."""
    return bf16(ACTS[act](g) * u)


def gate_up_act(Wg: np.ndarray, Wu: np.ndarray, x: np.ndarray, act: str) -> np.ndarray:
    """Gate and up projections of the token rows x [M][K], then the gated
    activation: ``gate_proj @ m`` and ``up_proj @ m`` ([llama] formula box)."""
    g = x @ Wg.T
    u = x @ Wu.T
    return gated_activation(g, u, act)


def ffn_hidden(weights, x: np.ndarray, act: str) -> np.ndarray:
    """h = down_proj(act(gate_proj @ x, up_proj @ x)) in float64, [M][H]."""
    a = gate_up_act(dequant(weights.gate), dequant(weights.up), x, act)
    return a @ dequant(weights.down).T


def residual_add(res: np.ndarray, y_bf16: np.ndarray) -> np.ndarray:
    """x = x + h: ``encode_residual_add`` of a bf16 row into the bf16 stream.
    The only tail of the llama layer ([llama]: a plain residual add, no norm)."""
    return bf16(res + y_bf16)


def rms_norm(h1: np.ndarray, w: np.ndarray, eps: float) -> np.ndarray:
    """out = bf16(h1 / sqrt(mean(h1^2) + eps) * w), per row, reading 3."""
    ms = np.mean(h1 * h1, axis=-1, keepdims=True)
    return bf16(h1 / np.sqrt(ms + eps) * w)


def rms_norm_prologue(res_bits: np.ndarray, w_bits: np.ndarray, eps: float) -> np.ndarray:
    """The FFN's input m = rms_norm(x, post_attention_layernorm) (bf16 bits).

    [llama] module doc formula box: ``m = rms_norm(x, post_attention_layernorm)``,
    encoded by the caller; ``encode_llama_layer_dense`` reads it from the 2-byte
    ``moe_x`` buffer. The norm is the one the pages encode everywhere
    (``encode_rms_norm_bf16w``, bf16 weight): reading 3, on the bf16 residual
    row ``x``, the result rounded to bf16.
    """
    return bf16_bits(rms_norm(bf16_to_f64(res_bits), bf16_to_f64(w_bits), eps))


def ffn_dense(weights, x_bits: np.ndarray, res_bits: np.ndarray, act: str) -> np.ndarray:
    """Dense llama FFN plus raw residual add; returns the new residual (bf16 bits).

    [llama] ``encode_llama_layer_dense``: gate and up GEMV on the normed input,
    activation, down GEMV into the 2-byte ``h2``, then residual add into ``x``.
    """
    x = bf16_to_f64(x_bits)
    h = bf16(ffn_hidden(weights, x, act))
    return bf16_bits(residual_add(bf16_to_f64(res_bits), h))


def ffn_shared_expert(weights, x_bits: np.ndarray, norm_w_bits: np.ndarray, act: str,
                      eps: float = 1e-6) -> np.ndarray:
    """Gemma shared-expert branch; returns h1 (bf16 bits) after the norm.

    [gemma] ``encode_shared_expert_branch``: the down projection writes the
    2-byte row ``h1_out``, which ``encode_rms_norm_bf16w`` normalizes in place
    with ``post_feedforward_layernorm_1`` and ``RMS_EPS``.
    """
    x = bf16_to_f64(x_bits)
    h1 = bf16(ffn_hidden(weights, x, act))
    return bf16_bits(rms_norm(h1, bf16_to_f64(norm_w_bits), eps))


# ----------------------------------------------------------------------------
# Routing
# ----------------------------------------------------------------------------


def router_logits(router: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """logits[t][e] = Wr[e] . x[t], stored fp32 (``batch_router_logits_f32``).

    ``router`` is fp32 [E][H], or bf16 bits (uint16) [E][H].
    """
    Wr = bf16_to_f64(router) if router.dtype == np.uint16 else np.asarray(router, np.float64)
    return f32(bf16_to_f64(x_bits) @ Wr.T)


def topk_softmax(logits: np.ndarray, k: int, per_expert_scale: Optional[np.ndarray] = None):
    """Per token: the k experts with the largest logits and their weights.

    Order is (logit descending, expert index ascending) (reading 4), so the rank
    order is unique. Weights are exp(l_r - l_0) / sum_j exp(l_j - l_0) over the
    selected ranks, times the per-expert scale (``per_expert_ones`` in [qwen]),
    rounded to fp16 (``routing16``). Returns (idx int32 [M][k], w float64 [M][k]).
    """
    logits = np.asarray(logits, np.float64)
    M, E = logits.shape
    scale = np.ones(E) if per_expert_scale is None else np.asarray(per_expert_scale, np.float64)
    idx = np.zeros((M, k), np.int32)
    w = np.zeros((M, k), np.float64)
    for t in range(M):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        sel = logits[t, order]
        z = np.exp(sel - sel[0])
        idx[t] = order
        w[t] = f16(z / z.sum() * scale[order])
    return idx, w


def expert_permutation(idx: np.ndarray, E: int):
    """Expert-grouped order of the (token, rank) pairs.

    Pairs are numbered p = t*k + r (PAIR order, token-major, rank within: [qwen]
    module doc). ``perm`` lists the pairs sorted by expert, stable in p;
    ``offsets[e]..offsets[e+1]`` is expert e's range of ``perm``; ``union`` is
    the ascending list of experts with at least one pair (the expert UNION the
    sub-batches are bounded by). Returns (perm, offsets, union) as int32.
    """
    experts = np.asarray(idx, np.int64).reshape(-1)
    perm = np.argsort(experts, kind="stable").astype(np.int32)
    counts = np.bincount(experts, minlength=E)
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    union = np.nonzero(counts)[0].astype(np.int32)
    return perm, offsets, union


# ----------------------------------------------------------------------------
# MoE layer
# ----------------------------------------------------------------------------


def shared_seed(shared, w_sg_bits: np.ndarray, x_bits: np.ndarray, act: str) -> np.ndarray:
    """Seed of the routed accumulator: the gated shared-expert output.

    [qwen] ``encode_qwen_layer_moe_batched``, shared-expert loop: the shared
    FFN writes ``batch_h1`` (2-byte), a 1-row GEMV with
    ``mlp.shared_expert_gate.weight`` gives the gate logit, and
    ``encode_sigmoid_scalar_mul`` scales the row by sigmoid(logit) in place.
    Returns float64 [M][H] (bf16 values).
    """
    x = bf16_to_f64(x_bits)
    s = bf16(ffn_hidden(shared, x, act))
    gate = f32(x @ bf16_to_f64(w_sg_bits))
    return bf16(s * sigmoid(gate)[:, None])


def seeded_rank_sum(seed: np.ndarray, w: np.ndarray, d: np.ndarray) -> np.ndarray:
    """y = bf16(((seed + w0 d0) + w1 d1) + ...) with an fp32 accumulator.

    [qwen] phase-2 call: the kernel's accumulator begins at the gated shared
    expert and the ranks are added after it in order -- the seed is the start, not a later
    addend. seed [M][H], w [M][k], d [M][k][H] (d rounded to fp32 here).
    """
    acc = f32(seed)
    for r in range(w.shape[1]):
        acc = f32(acc + f32(w[:, r:r + 1] * f32(d[:, r, :])))
    return bf16(acc)


def gemma_shared_branch(shared, x_bits: np.ndarray, norm_w_bits: np.ndarray, act: str, eps: float) -> np.ndarray:
    """The Gemma shared branch that joins the routed layer's tail: the shared
    FFN, then ``post_feedforward_layernorm_1`` ([gemma]
    ``encode_shared_expert_branch``: h1 = RMSNorm of the 2-byte down output,
    in place). Returns float64 [M][H] (bf16 values)."""
    return bf16_to_f64(ffn_shared_expert(shared, x_bits, norm_w_bits, act, eps))


def gemma_routed_tail(res: np.ndarray, y: np.ndarray, h1: np.ndarray) -> np.ndarray:
    """Tail of the Gemma-style routed layer ([qwen] module doc, contrasting the
    families: Gemma's "routed sum starts from nothing and its shared branch
    joins in the sandwich tail after a norm"): the routed output y (summed from
    zero) and the normed shared branch h1 join as two 2-byte rows, then the
    raw residual add. Reading: the pages name no other norm for this tail.
    Returns float64 (bf16 values)."""
    return bf16(res + bf16(y + h1))


def moe_layer(inp, return_internals: bool = False, tokens: Optional[Sequence[int]] = None):
    """Routed MoE layer with optional gated shared expert, raw residual tail.

    ``inp`` is a ``synth.LayerInputs`` of a "moe" configuration. Steps in the
    order of [qwen] ``encode_qwen_layer_moe_batched``: router logits, top-k,
    pair routes, shared-expert seed, phase 1 (expert gate/up + activation per
    pair), phase 2 (expert down per pair, seeded rank-ordered sum), one raw
    residual add. ``tokens`` restricts the computation to some token rows
    (the result then has only those rows).
    Returns the new residual (bf16 bits [M][H]) or (that, internals dict).
    """
    c = inp.config
    x_bits = inp.x if tokens is None else inp.x[list(tokens)]
    res_bits = inp.residual if tokens is None else inp.residual[list(tokens)]
    M, H, k = x_bits.shape[0], c.H, c.k
    x = bf16_to_f64(x_bits)

    logits = router_logits(inp.router, x_bits)
    gemma = getattr(inp, "shared_norm_w", None) is not None
    idx, w = topk_softmax(logits, k, getattr(inp, "expert_scale", None))
    perm, offsets, union = expert_permutation(idx, c.E)

    if inp.shared is not None and not gemma:
        seed = shared_seed(inp.shared, inp.w_sg, x_bits, c.act)
    else:
        seed = np.zeros((M, H))   # the routed sum starts from nothing

    d = np.zeros((M, k, H))
    for e in union:
        pairs = perm[offsets[e]:offsets[e + 1]]
        t, r = pairs // k, pairs % k
        ex = inp.experts[e]
        a = gate_up_act(dequant(ex.gate), dequant(ex.up), x[t], c.act)   # phase 1
        d[t, r, :] = a @ dequant(ex.down).T                               # phase 2 (down)
    y = seeded_rank_sum(seed, w, d)
    h1 = None
    if gemma:
        h1 = gemma_shared_branch(inp.shared, x_bits, inp.shared_norm_w, c.act, inp.shared_norm_eps)
        out = bf16_bits(gemma_routed_tail(bf16_to_f64(res_bits), y, h1))
    else:
        out = bf16_bits(residual_add(bf16_to_f64(res_bits), y))
    if not return_internals:
        return out
    return out, dict(logits=logits, idx=idx, w=w, perm=perm, offsets=offsets, union=union,
                     seed=seed, y=y, d=d, h1=h1)


def dense_layer(inp) -> np.ndarray:
    """Dispatch for the dense and shared-expert configurations."""
    c = inp.config
    if c.kind == "dense":
        return ffn_dense(inp.ffn, inp.x, inp.residual, c.act)
    if c.kind == "shared":
        return ffn_shared_expert(inp.ffn, inp.x, inp.norm_w, c.act, c.eps)
    raise ValueError(c.kind)


def layer_prenorm(inp, norm_w_bits: np.ndarray, eps: float,
                  tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """The layer with its input norm: m = rms_norm(residual, w), then the layer
    on (m, residual). ``inp.x`` is not read. Dense and MoE configurations."""
    from copy import copy
    sub = copy(inp)
    sub.x = rms_norm_prologue(inp.residual, norm_w_bits, eps)
    return layer(sub, tokens=tokens)


def layer(inp, tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """The whole layer of any configuration (bf16 bits of the output rows)."""
    if inp.config.kind == "moe":
        return moe_layer(inp, tokens=tokens)
    if tokens is not None:
        from copy import copy
        sub = copy(inp)
        sub.x = inp.x[list(tokens)]
        sub.residual = inp.residual[list(tokens)]
        return dense_layer(sub)
    return dense_layer(inp)
