"""Expert-parallel MoE on the GPU through the C ABI (moe_dispatch_rows,
moe_experts_grouped, moe_combine), against the oracle's layer.

One process, one GPU: W virtual ranks each hold a block of E / W experts
(their own plan) and route their own token rows; the two exchanges between
them are device copies made here, in the order an all-to-all delivers (by
source rank), and the ranks' kernels run one after another, never waiting on
each other. W = 1 is the layer without exchange.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import moe_expert_layer_dequant_b200 as lib
from moe_expert_layer_dequant_b200.ep import ExpertParallelMoE, GpuOps
from devutil import assert_bf16_close, dev_bf16, host_bf16

pytestmark = pytest.mark.gpu

SHAPES = [
    dict(cfg=4, H=256, I=256, E=16, k=4, I_s=256),   # Qwen form: gated shared expert seeds the sum
    dict(cfg=5, H=512, I=512, E=8, k=2, I_s=0),      # Mixtral form
]


def _layer(shape, M, seed=6):
    shape = dict(shape)
    c = synth.scaled_config(shape.pop("cfg"), **shape)
    return synth.make_inputs(c, M, seed)


def _ops(inp, rank, world):
    c = inp.config
    r = inp.router
    router = lib.plain_weight(torch.from_numpy(r).cuda() if r.dtype == np.float32 else dev_bf16(r))
    n = c.E // world
    experts = [lib.upload_ffn(e) for e in inp.experts[rank * n:(rank + 1) * n]]
    shared = lib.upload_ffn(inp.shared) if inp.shared is not None else None
    sg = lib.plain_weight(dev_bf16(inp.w_sg)) if inp.w_sg is not None else None
    return GpuOps(router, experts, c.E, c.k, c.act, rank, world, shared, sg)


def _run_virtual_ranks(inp, shards, world):
    """Each virtual rank's new residual rows (bf16 bits), exchanges as copies."""
    ranks = [ExpertParallelMoE(_ops(inp, r, world), inp.config.E, world=world) for r in range(world)]
    xs = [dev_bf16(inp.x[s]) for s in shards]
    res = [dev_bf16(inp.residual[s]) for s in shards]
    pend = [ranks[r].begin(xs[r]) for r in range(world)]
    # rows bound for rank q from each source rank r (contiguous blocks of r's slots)
    starts = [np.concatenate([[0], np.cumsum(p.send)]) for p in pend]
    rows_in = [torch.cat([pend[r].rows[starts[r][q]:starts[r][q + 1]] for r in range(world)]) for q in range(world)]
    exp_in = [torch.cat([pend[r].experts[starts[r][q]:starts[r][q + 1]] for r in range(world)]) for q in range(world)]
    d_in = [ranks[q].expert_work(rows_in[q], exp_in[q]) for q in range(world)]
    # down outputs back to their source, in the order the source sent them
    recv = [[pend[r].send[q] for r in range(world)] for q in range(world)]
    rstarts = [np.concatenate([[0], np.cumsum(recv[q])]) for q in range(world)]
    out = []
    for r in range(world):
        d_back = torch.cat([d_in[q][rstarts[q][r]:rstarts[q][r + 1]] for q in range(world)])
        ranks[r].finish(pend[r], d_back, xs[r], res[r])
        out.append(res[r])
    torch.cuda.synchronize()
    for ep in ranks:
        ep.ops.close()
    return [host_bf16(o) for o in out]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("M", [1, 5, 40, 200])   # GEMV and tensor-core paths of moe_experts_grouped
def test_one_rank_matches_the_oracle(shape, M):
    inp = _layer(shape, M)
    ep = ExpertParallelMoE(_ops(inp, 0, 1), inp.config.E)
    x, res = dev_bf16(inp.x), dev_bf16(inp.residual)
    ep.forward(x, res)
    torch.cuda.synchronize()
    ep.ops.close()
    assert lib.device_faults(True) == 0
    assert_bf16_close(host_bf16(res), oracle.moe_layer(inp), f"ep W=1 M={M}")


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("world,M_per_rank", [(2, [7, 3]), (4, [1, 9, 2, 40]), (2, [64, 100])])
def test_virtual_ranks_match_the_oracle(shape, world, M_per_rank):
    inp = _layer(shape, sum(M_per_rank))
    shards, t = [], 0
    for m in M_per_rank:
        shards.append(list(range(t, t + m)))
        t += m
    got = _run_virtual_ranks(inp, shards, world)
    assert lib.device_faults(True) == 0
    for r, s in enumerate(shards):
        assert_bf16_close(got[r], oracle.moe_layer(inp, tokens=s), f"ep W={world} rank {r}")


def test_experts_grouped_rows_in_any_order_and_foreign_rows_zero():
    """Rows in a scrambled order give the same down outputs as in expert
    order (stable grouping on the device); rows of experts outside the plan
    give zero rows."""
    inp = _layer(SHAPES[1], 24)
    c = inp.config
    ops = _ops(inp, 1, 2)             # experts 4..7
    rng = np.random.default_rng(0)
    exp = rng.integers(0, c.E, 24).astype(np.int32)
    rows = dev_bf16(inp.x)
    d1 = lib.moe_experts_grouped(ops.plan, rows, torch.from_numpy(exp).cuda(), ops.base).cpu().numpy()
    order = rng.permutation(24)
    d2 = lib.moe_experts_grouped(ops.plan, dev_bf16(inp.x[order]), torch.from_numpy(exp[order]).cuda(),
                                 ops.base).cpu().numpy()
    ops.close()
    assert np.array_equal(d1[order], d2)
    foreign = (exp < 4) | (exp >= 8)
    assert np.all(d1[foreign] == 0.0) and np.all(np.any(d1[~foreign] != 0.0, axis=1))
    # Each row went through its own expert. d is the fp32 down output before
    # any bf16 rounding, and the tensor-core path contracts bf16-rounded
    # weights, so its error is compared at 5e-2 x RMS over the rows (a row
    # run through another expert is off by about 1.4 x RMS); the layer
    # outputs built from d meet the 2e-2 x RMS bar in the tests above.
    x = oracle.bf16_to_f64(inp.x)
    mine = np.nonzero(~foreign)[0]
    want = np.zeros((len(mine), c.H))
    for j, i in enumerate(mine):
        ex = inp.experts[exp[i]]
        a = oracle.gate_up_act(oracle.dequant(ex.gate), oracle.dequant(ex.up), x[i:i + 1], c.act)
        want[j] = (a @ oracle.dequant(ex.down).T)[0]
    assert np.max(np.abs(d1[mine] - want)) <= 5e-2 * np.sqrt(np.mean(want ** 2))
