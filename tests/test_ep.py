"""Expert-parallel MoE: the exchange logic on CPU gloo ranks.

Each rank holds a block of E / world experts and routes its own token rows;
the pairs travel to their expert's rank and their down outputs come back
(moe_expert_layer_dequant_b200.ep). The ranks here do their local work with
the oracle's functions (tests/ep_oracle_ops.py), so the result must equal the
oracle's single-process layer on the same rows exactly: token rows are
independent, and every value reaches the seeded sum through the same
arithmetic, only over the wire.
"""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import oracle  # noqa: E402
import synth  # noqa: E402
from moe_expert_layer_dequant_b200.ep import ExpertParallelMoE, owner_blocks, send_counts  # noqa: E402

SHAPES = {
    # Qwen form: shared expert seeding the sum, fp32 router, top-4 of 8
    "qwen": dict(cfg=4, H=128, I=64, E=8, k=4, I_s=64),
    # Mixtral form: no shared expert, bf16 router, top-2 of 8
    "mixtral": dict(cfg=5, H=128, I=96, E=8, k=2, I_s=0),
    # top-1 routing (one pair per token)
    "top1": dict(cfg=5, H=96, I=64, E=4, k=1, I_s=0),
    # 16 experts, top-4, shared expert: four experts per rank at world 4
    "wide": dict(cfg=4, H=64, I=32, E=16, k=4, I_s=32),
}


def _inputs(name, M):
    shape = dict(SHAPES[name])
    c = synth.scaled_config(shape.pop("cfg"), **shape)
    return synth.make_inputs(c, M, 3)


def _shards(M_per_rank):
    out, t = [], 0
    for m in M_per_rank:
        out.append(list(range(t, t + m)))
        t += m
    return out


def _run_rank(inp, tokens, rank, world, group):
    import torch
    from ep_oracle_ops import OracleOps
    x = torch.from_numpy(inp.x[tokens].view(np.int16).copy())
    res = torch.from_numpy(inp.residual[tokens].view(np.int16).copy())
    ExpertParallelMoE(OracleOps(inp, rank, world), inp.config.E, group=group).forward(x, res)
    return res.numpy().view(np.uint16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, name, M_per_rank, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        inp = _inputs(name, sum(M_per_rank))
        tokens = _shards(M_per_rank)[rank]
        got = _run_rank(inp, tokens, rank, world, dist.group.WORLD)
        want = oracle.moe_layer(inp, tokens=tokens)
        out.put((rank, bool(np.array_equal(got, want)), int(np.count_nonzero(got != want))))
    finally:
        dist.destroy_process_group()


def _spawn(world, name, M_per_rank):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, M_per_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
        assert p.exitcode == 0
    res = dict((r, (ok, n)) for r, ok, n in (q.get(timeout=10) for _ in range(world)))
    for r in range(world):
        assert res[r][0], f"rank {r}: {res[r][1]} elements differ from the oracle's layer"


# --------------------------------------------------------------------------- host logic


def test_owner_blocks_need_an_even_split():
    assert owner_blocks(8, 2) == 4 and owner_blocks(128, 8) == 16
    with pytest.raises(ValueError):
        owner_blocks(8, 3)


def test_send_counts_are_the_owners_blocks_of_the_expert_order():
    # 8 experts over 4 ranks (2 each); expert e has e+1 pairs
    counts = np.arange(1, 9)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    assert send_counts(offsets.tolist(), 8, 4) == [1 + 2, 3 + 4, 5 + 6, 7 + 8]
    assert send_counts(offsets.tolist(), 8, 1) == [int(counts.sum())]


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_one_rank_equals_the_oracle_layer(name):
    inp = _inputs(name, 6)
    got = _run_rank(inp, list(range(6)), 0, 1, None)
    assert np.array_equal(got, oracle.moe_layer(inp))


# --------------------------------------------------------------------------- gloo ranks


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_two_ranks_equal_the_oracle_layer(name):
    # unequal token counts per rank
    _spawn(2, name, [5, 3])


def test_four_ranks_two_experts_each():
    _spawn(4, "mixtral", [3, 1, 4, 2])


def test_a_rank_that_receives_no_rows():
    # one token row with top-2 of 8 experts reaches at most 2 of 4 ranks; the
    # others exchange empty blocks and still take every collective step
    _spawn(4, "mixtral", [1, 1, 1, 1])


@pytest.mark.parametrize("name,world,M_per_rank", [("top1", 2, [4, 7]), ("top1", 4, [2, 2, 2, 2]),
                                                   ("wide", 4, [5, 1, 3, 6]), ("wide", 2, [9, 2])])
def test_routing_widths_and_world_sizes(name, world, M_per_rank):
    _spawn(world, name, M_per_rank)


def test_a_rank_without_token_rows():
    # rank 1 routes nothing but holds experts for rank 0's rows
    _spawn(2, "qwen", [6, 0])


# --------------------------------------------------------------------------- hand-derived layers


GOLDEN = {
    # builder, golden fixture, key of the expected output at feature 0 (per token row)
    "rank_pairing": ("rank_pairing_layer", "rank_weight_pairing.txt", "y_feature0"),
    "shared_gate": ("shared_gate_layer", "shared_gate_seed.txt", "seed_feature0"),
    "seed_first": ("seed_counterexample", None, None),          # y = 0 exactly (seed, then the ranks)
}


def _golden_rank_main(rank, world, port, name, out):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import handbuilt
    from ep_oracle_ops import OracleOps
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        li = getattr(handbuilt, GOLDEN[name][0])(32, 1)
        tokens = [t for t in range(li.x.shape[0]) if t % world == rank]
        x = torch.from_numpy(li.x[tokens].view(np.int16).copy())
        res = torch.from_numpy(li.residual[tokens].view(np.int16).copy())
        ExpertParallelMoE(OracleOps(li, rank, world), li.config.E, group=dist.group.WORLD).forward(x, res)
        out.put((rank, tokens, res.numpy().view(np.uint16).copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", sorted(GOLDEN))
def test_hand_derived_layers_with_one_expert_per_rank(name):
    """The worked examples of tests/golden with each of the two experts on
    its own rank and the token rows split between the ranks: the pairs cross
    the exchange and the outputs keep their hand-derived values."""
    import handbuilt
    from conftest import read_golden
    li = getattr(handbuilt, GOLDEN[name][0])(32, 1)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_golden_rank_main, args=(r, 2, port, name, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(240)
        assert p.exitcode == 0
    got = np.zeros_like(li.x)
    for _ in range(2):
        _, tokens, rows = q.get(timeout=10)
        got[tokens] = rows
    _, fixture, key = GOLDEN[name]
    if fixture is None:
        want0 = np.zeros(li.x.shape[0])
    else:
        kv, _ = read_golden(fixture)
        want0 = np.array([float(v) for v in kv[key]])
    assert np.array_equal(oracle.bf16_to_f64(got)[:, 0], want0)
    assert np.array_equal(got, oracle.layer(li))
