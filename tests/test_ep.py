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


def test_a_rank_without_token_rows():
    # rank 1 routes nothing but holds experts for rank 0's rows
    _spawn(2, "qwen", [6, 0])
