"""CPU stand-in for the expert-parallel layer's GPU work (tests only).

The same five steps as ``moe_expert_layer_dequant_b200.ep.GpuOps``, written
with the oracle's functions on CPU tensors, so that the exchange logic of
``ExpertParallelMoE`` (split sizes, the two all-to-alls, the order rows come
back in) can run on gloo ranks without a GPU. A rank only touches the experts
of its own block.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


class OracleOps:
    def __init__(self, inp, rank: int, world: int):
        c = inp.config
        self.inp, self.c, self.k, self.E = inp, c, c.k, c.E
        self.n = c.E // world
        self.base = rank * self.n

    @staticmethod
    def _bits(t: torch.Tensor) -> np.ndarray:
        return t.numpy().view(np.uint16)

    def route(self, x):
        logits = oracle.router_logits(self.inp.router, self._bits(x))
        idx, w = oracle.topk_softmax(logits, self.k)
        perm, offsets, _ = oracle.expert_permutation(idx, self.E)
        return (torch.from_numpy(np.asarray(idx, np.int32)), torch.from_numpy(np.asarray(w, np.float64)),
                torch.from_numpy(perm), torch.from_numpy(offsets))

    def dispatch(self, x, idx, perm):
        p = perm.long()
        return x[p // self.k].contiguous(), idx.reshape(-1)[p].contiguous()

    def experts(self, rows, row_expert):
        x = oracle.bf16_to_f64(self._bits(rows))
        local = row_expert.numpy().astype(np.int64) - self.base
        assert np.all((local >= 0) & (local < self.n)), "a row reached a rank that does not hold its expert"
        d = np.zeros((x.shape[0], self.c.H))
        for e in np.unique(local):
            sel = np.nonzero(local == e)[0]
            ex = self.inp.experts[self.base + int(e)]
            a = oracle.gate_up_act(oracle.dequant(ex.gate), oracle.dequant(ex.up), x[sel], self.c.act)
            d[sel] = a @ oracle.dequant(ex.down).T
        return torch.from_numpy(d)

    def shared(self, x):
        if self.inp.shared is None:
            return None
        return oracle.shared_seed(self.inp.shared, self.inp.w_sg, self._bits(x), self.c.act)

    def combine(self, d, perm, w, residual, seed):
        M, H, k = residual.shape[0], self.c.H, self.k
        pairs = np.zeros((M * k, H))
        pairs[perm.numpy().astype(np.int64)] = d.numpy()
        if seed is None:
            seed = np.zeros((M, H))
        y = oracle.seeded_rank_sum(seed, w.numpy(), pairs.reshape(M, k, H))
        out = oracle.bf16_bits(oracle.residual_add(oracle.bf16_to_f64(self._bits(residual)), y))
        residual.copy_(torch.from_numpy(out.view(np.int16)))
