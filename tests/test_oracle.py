"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test checks the oracle against something the pages or mathematics fix: a
hand-derived worked example (tests/golden), a closed form, an invariant, a
library routine, or brute force on tiny inputs. They are chosen so that a
dropped term, a wrong sign or index, a transposed operand, or a swapped
gate/up would fail at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import read_golden
import handbuilt
from synth import FFNWeights, QWeight, FMT_INT4_G32, FMT_INT8_ROW

pytestmark = pytest.mark.cpu


def _hex16(tokens, dtype):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint16).view(dtype)


# --------------------------------------------------------------------------- dequant


def test_dequant_int4_golden_block():
    kv, _ = read_golden("int4_affine_g32_block.txt")
    packed = np.array([int(t, 16) for t in kv["packed_hex"]], np.uint8)[None, :]
    scale = _hex16(kv["scale_fp16_hex"], np.float16)[None, :]
    mn = _hex16(kv["min_fp16_hex"], np.float16)[None, :]
    want = np.array([float(t) for t in kv["expected"]])
    got = oracle.dequant_int4_affine_g32(packed, scale, mn)[0]
    assert np.array_equal(got, want)
    # The fp32 form is exact: rounding to fp32 changes nothing.
    assert np.array_equal(oracle.f32(got), want)


def test_dequant_int4_subnormal_scale_exact():
    kv, _ = read_golden("int4_affine_g32_subnormal.txt")
    packed = np.array([int(t, 16) for t in kv["packed_hex"]], np.uint8)[None, :]
    scale = _hex16(kv["scale_fp16_hex"], np.float16)[None, :]
    mn = _hex16(kv["min_fp16_hex"], np.float16)[None, :]
    want = np.array([float(t) for t in kv["expected"]])
    assert np.array_equal(oracle.dequant_int4_affine_g32(packed, scale, mn)[0], want)


def _q4k_block(header_bytes, codes):
    return np.concatenate([np.asarray(header_bytes, np.uint8), np.asarray(codes, np.uint8)])[None, :]


def test_dequant_q4_k_golden_block():
    """Hand-derived Q4_K super-block (golden q4_k_block.txt): the 6-bit
    scale/min unpacking of all eight sub-blocks and values in each of them."""
    kv, _ = read_golden("q4_k_block.txt")
    header = [int(t, 16) for t in kv["header_hex"]]
    assert kv["codes"] == ["0..127"]
    blk = _q4k_block(header, np.arange(128))
    sc, mn = oracle.q4_k_scales_mins(blk[0, 4:16])
    want = [tuple(int(v) for v in t.split(",")) for t in kv["scales_mins"]]
    assert list(zip(sc.tolist(), mn.tolist())) == want
    w = oracle.dequant_q4_k(blk, 1, 256)[0]
    for t in kv["expected"]:
        k, v = t.split(":")
        assert w[int(k)] == float(v), (k, w[int(k)], v)


@pytest.mark.parametrize("c,r,hi", [(0, 0, False), (0, 31, True), (1, 7, False), (2, 16, True), (3, 31, False),
                                   (3, 31, True)])
def test_q4_k_code_runs(c, r, hi):
    """One code of 1 in byte r of run c (low or high nibble), all scales 1,
    mins 0, d = 1: exactly element 64c + r (+ 32 for the high nibble) is 1."""
    header = [0x00, 0x3C, 0, 0] + [1, 1, 1, 1, 0, 0, 0, 0, 1, 1, 1, 1]   # d = 1, dmin = 0, scale 1, min 0
    codes = np.zeros(128, np.uint8)
    codes[32 * c + r] = 0x10 if hi else 0x01
    w = oracle.dequant_q4_k(_q4k_block(header, codes), 1, 256)[0]
    want = np.zeros(256)
    want[64 * c + r + (32 if hi else 0)] = 1.0
    assert np.array_equal(w, want)


def test_q4_k_rounds_once_to_fp32():
    """d * scale * q is exact; the difference with dmin * min is rounded once
    to fp32, ties to even: 945 - 2^-15 lies halfway between 945 - 2^-14 and 945
    (fp32 spacing 2^-14 there) and rounds to 945 (even significand);
    945 - 3 * 2^-15 lies halfway between 945 - 2^-14 (odd) and 945 - 2^-13
    (even) and rounds to the latter; zero blocks give zeros."""
    def one(dmin_bits, m):
        # d = 1, scale 63 for sub-block 0, min m, codes 15
        s = [63, 0, 0, 0, m, 0, 0, 0, 0, 0, 0, 0]
        header = [0x00, 0x3C, dmin_bits & 0xFF, dmin_bits >> 8] + s
        return oracle.dequant_q4_k(_q4k_block(header, np.full(128, 0xFF, np.uint8)), 1, 256)[0, 0]
    half_ulp = 0x0200   # fp16 subnormal 512 * 2^-24 = 2^-15
    assert one(half_ulp, 1) == 945.0
    assert one(half_ulp, 3) == 945.0 - 2.0 ** -13
    assert np.all(oracle.dequant_q4_k(np.zeros((2, 288), np.uint8), 2, 512) == 0.0)


def test_dequant_int8_golden_block():
    kv, _ = read_golden("int8_row_block.txt")
    q = np.array([[int(t) for t in kv["q_row0"]], [int(t) for t in kv["q_row1"]]], np.int8)
    scale = _hex16(kv["scale_fp16_hex"], np.float16)
    got = oracle.dequant_int8_row(q, scale)
    assert np.array_equal(got[0], [float(t) for t in kv["expected_row0"]])
    assert np.array_equal(got[1], [float(t) for t in kv["expected_row1"]])


def test_dequant_int4_fp32_exact_on_config_ranges():
    """q*scale + min is exact in fp32 for the configurations' value ranges: the
    fp32 evaluation with one fused step equals the float64 one."""
    rng = np.random.default_rng(5)
    w = synth.random_qweight(FMT_INT4_G32, 64, 256, rng)
    ref = oracle.dequant(w)
    q = oracle.int4_codes(w.q).astype(np.float32)
    g = np.arange(256) // 32
    s = w.scale.astype(np.float32)[:, g]
    m = w.min.astype(np.float32)[:, g]
    prod = (q.astype(np.float64) * s.astype(np.float64))
    assert np.array_equal(oracle.f32(prod), prod)            # the product is exact in fp32
    assert np.array_equal((np.float32(1) * (q * s) + m).astype(np.float64), ref)


# --------------------------------------------------------------------------- rounding


def test_bf16_rounding_golden():
    _, rows = read_golden("bf16_rounding.txt")
    vals = np.array([float(r[0]) for r in rows])
    want = np.array([int(r[1], 16) for r in rows], np.uint16)
    assert np.array_equal(oracle.bf16_bits(vals), want)


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_bits(v.astype(np.float64)), ref)


def test_activations_match_torch():
    g = torch.linspace(-12, 12, 4001, dtype=torch.float64)
    assert np.allclose(oracle.silu(g.numpy()), torch.nn.functional.silu(g).numpy(), rtol=1e-14, atol=1e-300)
    assert np.allclose(oracle.gelu_tanh(g.numpy()),
                       torch.nn.functional.gelu(g, approximate="tanh").numpy(), rtol=1e-13, atol=1e-15)
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert oracle.silu(np.array([64.0]))[0] == 64.0


def test_sigmoid_matches_torch_and_gates_the_product():
    z = torch.linspace(-40, 40, 8001, dtype=torch.float64)
    assert np.allclose(oracle.sigmoid(z.numpy()), torch.sigmoid(z).numpy(), rtol=1e-14, atol=1e-300)
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    # bf16(silu(g) * u): act on the gate operand, one rounding to bf16 (torch's own conversion)
    g, u = np.array([1.5, -2.0, 3.0]), np.array([2.0, 0.5, -1.0])
    want = torch.from_numpy(g / (1.0 + np.exp(-g)) * u).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.gated_activation(g, u, "silu"), want)
    swapped = torch.from_numpy(u / (1.0 + np.exp(-u)) * g).to(torch.bfloat16).to(torch.float64).numpy()
    assert not np.array_equal(oracle.gated_activation(g, u, "silu"), swapped)


# --------------------------------------------------------------------------- helpers


def _int8_matrix(values: np.ndarray, scale) -> QWeight:
    """INT8 weights with integer entries and one per-row scale."""
    N, K = values.shape
    sc = np.full(N, scale, np.float16) if np.isscalar(scale) else np.asarray(scale, np.float16)
    return QWeight(FMT_INT8_ROW, N, K, values.astype(np.int8), sc)


def _int4_matrix(codes: np.ndarray, scale, mn) -> QWeight:
    N, K = codes.shape
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    s = np.full((N, K // 32), scale, np.float16)
    m = np.full((N, K // 32), mn, np.float16)
    return QWeight(FMT_INT4_G32, N, K, packed, s, m)


def _perm_matrix(n, shift):
    P = np.zeros((n, n), np.int64)
    P[np.arange(n), (np.arange(n) + shift) % n] = 1      # (P x)[i] = x[i + shift]
    return P


# --------------------------------------------------------------------------- dense FFN


@pytest.mark.parametrize("fmt,down_fmt", [(FMT_INT8_ROW, FMT_INT8_ROW), (FMT_INT4_G32, FMT_INT4_G32),
                                          (FMT_INT4_G32, FMT_INT8_ROW), (FMT_INT8_ROW, FMT_INT4_G32)])
def test_dense_permutation_closed_form(fmt, down_fmt):
    """gate = 2 P1, up = Q/2... with non-symmetric permutations: a transposed
    operand, swapped gate/up or a dropped scale changes which entries meet.
    Mixed block types (down in another format) give the same closed form."""
    n, M = 64, 3
    P1, P2, P3 = _perm_matrix(n, 5), _perm_matrix(n, 0), _perm_matrix(n, 17)
    if fmt == FMT_INT8_ROW:
        gate, up = _int8_matrix(P1, 2.0), _int8_matrix(P2, 0.5)
    else:
        gate, up = _int4_matrix(P1, 2.0, 0.0), _int4_matrix(P2, 0.5, 0.0)
    down = _int8_matrix(P3, 1.0) if down_fmt == FMT_INT8_ROW else _int4_matrix(P3, 1.0, 0.0)
    rng = np.random.default_rng(1)
    x = synth.to_bf16_bits(rng.standard_normal((M, n)))
    res = synth.to_bf16_bits(rng.standard_normal((M, n)))
    out = oracle.ffn_dense(FFNWeights(gate, up, down), x, res, "silu")
    xf = oracle.bf16_to_f64(x)
    i = np.arange(n)
    g = 2.0 * xf[:, (i + 5) % n]
    u = 0.5 * xf
    a = oracle.bf16(g / (1 + np.exp(-g)) * u)
    h = a[:, (i + 17) % n]
    want = oracle.bf16_bits(oracle.bf16_to_f64(res) + h)
    assert np.array_equal(out, want)


def test_int4_min_only_closed_form():
    """All codes 0: W[n][k] = min[n][k//32], so gate . x is min times the group sums."""
    n, K = 8, 96
    codes = np.zeros((n, K), np.int64)
    w = _int4_matrix(codes, 0.25, 0.0)
    mins = (np.arange(n * 3).reshape(n, 3) - 7) * 0.0625
    w.min[:] = mins.astype(np.float16)
    x = np.arange(K, dtype=np.float64) / 16.0
    got = oracle.dequant(w) @ x
    gsum = x.reshape(3, 32).sum(axis=1)
    assert np.allclose(got, mins @ gsum, rtol=0, atol=1e-12)


def test_residual_is_only_tail_on_llama():
    """out - res is the bf16 FFN output: no norm sits between FFN and stream."""
    c = synth.scaled_config(1, H=64, I=96)
    inp = synth.make_inputs(c, 2, 0)
    out = oracle.bf16_to_f64(oracle.layer(inp))
    h = oracle.bf16(oracle.ffn_hidden(inp.ffn, oracle.bf16_to_f64(inp.x), "silu"))
    res = oracle.bf16_to_f64(inp.residual)
    assert np.array_equal(out, oracle.bf16(res + h))
    # A norm on h would change its RMS; the FFN output here is far from unit RMS.
    assert abs(np.sqrt(np.mean(h ** 2)) - 1.0) > 0.1


@pytest.mark.parametrize("cfg", [1, 2, 5])
def test_zero_input_leaves_residual(cfg):
    c = synth.scaled_config(cfg, H=64, I=64) if cfg != 5 else synth.scaled_config(5, H=64, I=64, E=4)
    inp = synth.make_inputs(c, 2, 0)
    inp.x = np.zeros_like(inp.x)
    assert np.array_equal(oracle.layer(inp), inp.residual)


def test_zero_input_shared_expert_gives_zero():
    c = synth.scaled_config(3, H=64, I=64)
    inp = synth.make_inputs(c, 2, 0)
    inp.x = np.zeros_like(inp.x)
    assert not np.any(oracle.bf16_to_f64(oracle.layer(inp)))


def test_zero_input_qwen_moe():
    """x = 0: logits 0, top-k = experts 0..k-1 by the tie rule, w = 1/k, seed 0."""
    c = synth.scaled_config(4, H=64, I=32, E=16, k=8, I_s=32)
    inp = synth.make_inputs(c, 3, 0)
    inp.x = np.zeros_like(inp.x)
    out, it = oracle.moe_layer(inp, return_internals=True)
    assert np.array_equal(it["idx"], np.tile(np.arange(8), (3, 1)))
    assert np.all(it["w"] == 0.125)
    assert not np.any(it["seed"])
    assert np.array_equal(out, inp.residual)


def test_rmsnorm_constant_row_closed_form():
    H = 48
    w = oracle.bf16(1.0 + np.random.default_rng(2).normal(0, 0.1, H))
    for c in (0.5, -3.0, 1e-4):
        h1 = np.full((1, H), oracle.bf16(np.array([c]))[0])
        want = oracle.bf16(h1 / math.sqrt(h1[0, 0] ** 2 + 1e-6) * w)
        assert np.array_equal(oracle.rms_norm(h1, w, 1e-6), want)
    # Scale invariance (eps negligible): 4*h1 normalizes to the same row.
    h1 = oracle.bf16(np.random.default_rng(3).standard_normal((1, H)))
    assert np.allclose(oracle.rms_norm(4 * h1, w, 0.0), oracle.rms_norm(h1, w, 0.0), rtol=0, atol=0)


def test_shared_expert_branch_ends_with_norm():
    """The Gemma branch's output rows have RMS close to RMS(w) (up to bf16)."""
    c = synth.scaled_config(3, H=128, I=64)
    inp = synth.make_inputs(c, 2, 1)
    out = oracle.bf16_to_f64(oracle.layer(inp))
    w = oracle.bf16_to_f64(inp.norm_w)
    x = oracle.bf16_to_f64(inp.x)
    h1 = oracle.bf16(oracle.ffn_hidden(inp.ffn, x, "gelu_tanh"))
    n = h1 / np.sqrt(np.mean(h1 ** 2, axis=1, keepdims=True))
    assert np.allclose(out, n * w, rtol=1e-2, atol=1e-2)


# --------------------------------------------------------------------------- routing


def _is_topk(logits_row, chosen, k):
    """Brute-force definition: chosen beats every other expert under (logit, -index)."""
    E = len(logits_row)
    S = set(chosen)
    if len(S) != k:
        return False
    for e in S:
        for o in range(E):
            if o in S:
                continue
            if not (logits_row[e] > logits_row[o] or (logits_row[e] == logits_row[o] and e < o)):
                return False
    return True


def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(3)
    for E in (2, 3, 5, 8):
        for k in range(1, E + 1):
            for _ in range(20):
                logits = rng.integers(-2, 3, size=(1, E)).astype(np.float64)
                idx, w = oracle.topk_softmax(logits, k)
                sets = [s for s in itertools.combinations(range(E), k) if _is_topk(logits[0], s, k)]
                assert len(sets) == 1                         # exactly one correct answer
                assert set(idx[0]) == set(sets[0])
                # ranks in (logit desc, index asc) order
                keys = [(-logits[0, e], e) for e in idx[0]]
                assert keys == sorted(keys)
                assert abs(w.sum() - 1) < 3e-3


def test_topk_softmax_closed_forms():
    logits = np.array([[0.5, 0.5, 0.5, 0.5, -1.0]])
    idx, w = oracle.topk_softmax(logits, 4)
    assert list(idx[0]) == [0, 1, 2, 3] and np.all(w == 0.25)
    d = 0.75
    idx, w = oracle.topk_softmax(np.array([[0.0, d, -5.0]]), 2)
    assert list(idx[0]) == [1, 0]
    assert w[0, 0] == np.float16(1 / (1 + math.exp(-d)))
    assert w[0, 1] == np.float16(math.exp(-d) / (1 + math.exp(-d)))


def test_router_logits_one_hot_rows():
    H, E = 32, 4
    Wr = np.zeros((E, H), np.float32)
    for e in range(E):
        Wr[e, 3 * e + 1] = 2.0
    x = synth.to_bf16_bits(np.random.default_rng(4).standard_normal((2, H)))
    got = oracle.router_logits(Wr, x)
    xf = oracle.bf16_to_f64(x)
    assert np.array_equal(got, 2.0 * xf[:, [1, 4, 7, 10]])


def test_permutation_invariants():
    rng = np.random.default_rng(7)
    for M, k, E in [(1, 8, 128), (4, 8, 128), (37, 2, 8), (512, 2, 8), (5, 3, 4)]:
        idx = np.stack([rng.choice(E, k, replace=False) for _ in range(M)]).astype(np.int32)
        perm, offsets, union = oracle.expert_permutation(idx, E)
        flat = idx.reshape(-1)
        assert sorted(perm.tolist()) == list(range(M * k))                 # a permutation
        ex = flat[perm]
        assert np.all(np.diff(ex) >= 0)                                    # grouped by expert
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]]
            assert np.all(np.diff(seg) > 0)                                # stable in pair order
            assert np.all(flat[seg] == e)
            assert len(seg) == int(np.sum(flat == e))
        assert offsets[0] == 0 and offsets[-1] == M * k
        assert list(union) == sorted(set(flat.tolist()))


# --------------------------------------------------------------------------- seeded sum


def test_seed_is_accumulator_start_not_addend():
    li = handbuilt.seed_counterexample()
    out, it = oracle.moe_layer(li, return_internals=True)
    assert list(it["idx"][0]) == [0, 1] and np.all(it["w"] == 0.5)
    assert it["seed"][0, 0] == 1.0
    assert it["d"][0, 0, 0] == 2.0 ** -23 and it["d"][0, 1, 0] == -2.0
    assert oracle.bf16_to_f64(out)[0, 0] == 0.0                      # seed, then ranks
    # Adding the shared expert after the routed sum gives another function.
    routed = np.float32(np.float32(0.5) * np.float32(2.0 ** -23)) + np.float32(np.float32(0.5) * np.float32(-2.0))
    add_after = np.float32(routed + np.float32(1.0))
    assert add_after == np.float32(2.0 ** -24)


def test_moe_single_expert_reduces_to_dense():
    """E = 1, k = 1, no shared expert: the routed layer is the dense FFN (w = 1)."""
    c = synth.scaled_config(5, H=64, I=96, E=1, k=1)
    inp = synth.make_inputs(c, 3, 2)
    moe = oracle.bf16_to_f64(oracle.layer(inp))
    dense = oracle.bf16_to_f64(oracle.ffn_dense(inp.experts[0], inp.x, inp.residual, "silu"))
    # identical up to the fp32 rounding of d before the bf16 rounding of y
    assert np.max(np.abs(moe - dense) / np.maximum(np.abs(dense), 1e-3)) <= 2.0 ** -7


def test_moe_token_rows_independent():
    """Rows are independent: M-row output equals the single-row outputs."""
    c = synth.scaled_config(4, H=64, I=32, E=16, k=4, I_s=32)
    inp = synth.make_inputs(c, 4, 1)
    full = oracle.layer(inp)
    for t in range(4):
        assert np.array_equal(oracle.layer(inp, tokens=[t])[0], full[t])


def test_zero_gate_vector_seeds_half_the_shared_expert():
    """w_sg = 0 and routed experts that contribute nothing: sigma(0) = 1/2, so
    the layer output is res + bf16(bf16(shared FFN) / 2), the shared branch
    taken from the dense FFN definition and halved exactly."""
    c = synth.scaled_config(4, H=64, I=32, E=8, k=2, I_s=64)
    inp = synth.make_inputs(c, 3, 4)
    zero = FFNWeights(synth.zero_like_qweight(FMT_INT4_G32, c.I, c.H), synth.zero_like_qweight(FMT_INT4_G32, c.I, c.H),
                      synth.zero_like_qweight(FMT_INT4_G32, c.H, c.I))
    inp.experts = [zero] * c.E
    inp.w_sg = np.zeros(c.H, np.uint16)
    out = oracle.bf16_to_f64(oracle.layer(inp))
    s = oracle.bf16(oracle.ffn_hidden(inp.shared, oracle.bf16_to_f64(inp.x), "silu"))
    want = oracle.bf16(oracle.bf16_to_f64(inp.residual) + oracle.bf16(0.5 * s))
    assert np.any(s != 0)
    assert np.array_equal(out, want)


def test_shared_gate_logit_sign_and_operand():
    """The seed is bf16(s * sigmoid(w_sg . x)) with the gate logit of THIS token
    and its sign as written (golden shared_gate_seed.txt): tokens whose logits are
    +-141/128 get seeds 1.5 and 0.498046875; sigmoid(-logit) swaps them and a
    zero or wrong gate vector gives 1.0 for both."""
    kv, _ = read_golden("shared_gate_seed.txt")
    want_logit = [float(t) for t in kv["gate_logit"]]
    want_seed = [float(t) for t in kv["seed_feature0"]]
    li = handbuilt.shared_gate_layer()
    out, it = oracle.moe_layer(li, return_internals=True)
    x = oracle.bf16_to_f64(li.x)
    assert list(x @ oracle.bf16_to_f64(li.w_sg)) == want_logit
    assert list(it["seed"][:, 0]) == want_seed
    assert not np.any(it["seed"][:, 1:])
    assert list(oracle.bf16_to_f64(out)[:, 0]) == want_seed          # residual 0, routed sum 0


def test_rank_weights_meet_their_own_expert_outputs():
    """Unequal routing weights (0.75, 0.25) on experts with outputs 4 and -8
    (golden rank_weight_pairing.txt): token 0 ranks (0, 1) -> y = 1, token 1
    ranks (1, 0) -> y = -5; weights paired with reversed ranks give -5 and 1."""
    kv, _ = read_golden("rank_weight_pairing.txt")
    li = handbuilt.rank_pairing_layer()
    out, it = oracle.moe_layer(li, return_internals=True)
    assert list(it["idx"][0]) == [int(t) for t in kv["topk_idx_token0"]]
    assert list(it["idx"][1]) == [int(t) for t in kv["topk_idx_token1"]]
    w = [float(t) for t in kv["weights"]]
    assert np.array_equal(it["w"], np.array([w, w]))
    assert it["d"][0, 0, 0] == 4.0 and it["d"][0, 1, 0] == -8.0     # rank 0 of token 0 is expert 0
    assert it["d"][1, 0, 0] == -8.0 and it["d"][1, 1, 0] == 4.0     # rank 0 of token 1 is expert 1
    assert list(oracle.bf16_to_f64(out)[:, 0]) == [float(t) for t in kv["y_feature0"]]


# --------------------------------------------------------------------------- pre-FFN norm


def test_rms_norm_prologue_golden():
    kv, _ = read_golden("rms_norm_prologue.txt")
    x = synth.to_bf16_bits(np.array([[float(t) for t in kv["x"]]]))
    w = synth.to_bf16_bits(np.array([float(t) for t in kv["w"]]))
    got = oracle.bf16_to_f64(oracle.rms_norm_prologue(x, w, float(kv["eps"][0])))[0]
    assert list(got) == [float(t) for t in kv["expected"]]


def test_rms_norm_prologue_closed_forms():
    """Constant row c: m = bf16(c / sqrt(c^2 + eps) * w); eps inside the root
    shows for small c. A row scaled by 2^k gives the same m when eps = 0."""
    H = 64
    w = synth.to_bf16_bits(1.0 + np.random.default_rng(8).normal(0, 0.1, H))
    wf = oracle.bf16_to_f64(w)
    for c, eps in ((0.5, 1e-6), (-3.0, 1e-6), (1e-3, 1e-6), (1e-3, 1e-5)):
        x = synth.to_bf16_bits(np.full((1, H), c))
        cf = oracle.bf16_to_f64(x)[0, 0]
        want = oracle.bf16(cf / math.sqrt(cf * cf + eps) * wf)
        assert np.array_equal(oracle.bf16_to_f64(oracle.rms_norm_prologue(x, w, eps))[0], want)
    x = synth.to_bf16_bits(np.random.default_rng(9).standard_normal((3, H)))
    x8 = synth.to_bf16_bits(oracle.bf16_to_f64(x) * 8.0)
    assert np.array_equal(oracle.rms_norm_prologue(x, w, 0.0), oracle.rms_norm_prologue(x8, w, 0.0))


def test_prenorm_layer_feeds_the_normed_residual():
    """layer_prenorm = the layer on x = rms_norm(residual), residual added raw;
    it reads the residual twice (norm input, then the add) and never inp.x."""
    c = synth.scaled_config(2, H=64, I=96)
    inp = synth.make_inputs(c, 2, 3)
    w = synth.to_bf16_bits(1.0 + np.random.default_rng(1).normal(0, 0.1, c.H))
    got = oracle.layer_prenorm(inp, w, 1e-6)
    inp2 = synth.make_inputs(c, 2, 3)
    inp2.x = np.zeros_like(inp2.x) + np.uint16(0x3F80)        # a different x changes nothing
    assert np.array_equal(oracle.layer_prenorm(inp2, w, 1e-6), got)
    m = oracle.rms_norm_prologue(inp.residual, w, 1e-6)
    want = oracle.ffn_dense(inp.ffn, m, inp.residual, "silu")
    assert np.array_equal(got, want)



# --------------------------------------------------------------------------- Gemma-style routed layer


def test_gemma_routed_layer_golden():
    """Per-expert scale looked up by expert, routed sum from zero, normed shared
    branch joined in the tail (golden gemma_routed_layer.txt)."""
    kv, _ = read_golden("gemma_routed_layer.txt")
    li = handbuilt.gemma_routed_layer()
    out, it = oracle.moe_layer(li, return_internals=True)
    assert list(it["w"][0]) == [float(t) for t in kv["weights_token0"]]
    assert list(it["w"][1]) == [float(t) for t in kv["weights_token1"]]
    assert not np.any(it["seed"])                                     # the routed sum starts from nothing
    assert list(it["y"][:, 0]) == [float(t) for t in kv["y_feature0"]]
    assert list(it["h1"][:, 0]) == [float(t) for t in kv["h1_feature0"]]
    assert list(oracle.bf16_to_f64(out)[:, 0]) == [float(t) for t in kv["out_feature0"]]
    assert not np.any(oracle.bf16_to_f64(out)[:, 1:])


def test_topk_per_expert_scale_follows_the_expert():
    """The scale multiplies the softmax weight of the expert it belongs to and
    does not change which experts are selected."""
    logits = np.array([[0.0, 2.0, 1.0, -1.0]])
    scale = np.array([3.0, 0.5, 2.0, 7.0])
    idx1, w1 = oracle.topk_softmax(logits, 2)
    idx2, w2 = oracle.topk_softmax(logits, 2, scale)
    assert list(idx1[0]) == list(idx2[0]) == [1, 2]
    z = np.exp(np.array([0.0, -1.0]))
    assert np.array_equal(w2[0], oracle.f16(z / z.sum() * np.array([0.5, 2.0])))
