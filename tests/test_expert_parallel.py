"""Expert parallelism's host logic on CPU: the ranks' expert ranges and shared-expert ownership
partition the layer, and world_size gloo ranks whose partial outputs come from the fp64 oracle
(each over its own experts) sum, through the layer's all-reduce, to the oracle's whole layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_expert_ffn_logits_b200.expert_parallel import (ExpertParallelLayer, expert_range,
                                                           shared_mask)


def test_ranges_and_masks_partition_the_experts():
    for E in range(1, 41):
        for world in range(1, 10):
            seen = []
            sizes = []
            for r in range(world):
                b, e = expert_range(E, world, r)
                assert 0 <= b <= e <= E
                seen += list(range(b, e))
                sizes.append(e - b)
            assert seen == list(range(E))  # contiguous, in rank order, each expert once
            assert max(sizes) - min(sizes) <= 1
    for S in range(0, 9):
        for world in range(1, 6):
            masks = [shared_mask(S, world, r) for r in range(world)]
            assert sum(masks) == (1 << S) - 1
            for a in range(world):
                for b in range(a):
                    assert masks[a] & masks[b] == 0
    with pytest.raises(ValueError):
        expert_range(8, 2, 2)


class OracleBackend:
    """A rank's partial output from the fp64 oracle: the sum over the rank's (token, expert)
    pairs of w * y, with the oracle's own routing, gate, selection and expert output."""

    def __init__(self, shape, rank, world):
        import oracle
        import synth
        self.o, self.shape = oracle, shape
        self.begin, self.end = expert_range(shape.n_routed, world, rank)
        self.mask = shared_mask(shape.n_shared, world, rank)
        self.router = synth.host_tensor(shape, "router")
        self.ex = {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
                       synth.host_tensor(shape, "down", e)) for e in range(shape.n_routed)}
        self.sh = [(synth.host_tensor(shape, "sh_gate", s), synth.host_tensor(shape, "sh_up", s),
                    synth.host_tensor(shape, "sh_down", s)) for s in range(shape.n_shared)]

    def _pair(self, xt, w, rule):
        g, u, d = w
        _, a = self.o.gate(xt, g)
        keep = self.o.select(np.abs(a), rule)
        return self.o.expert(xt, u, d, keep, a)

    def partial(self, x, router, routed_local, shared, rule_r, rule_s, stream=None):
        layer = self.o.Layer(self.shape, self.router, {}, [])
        _, idx, w = layer.route(x)
        out = np.zeros((x.shape[0], self.shape.hidden))
        for t in range(x.shape[0]):
            for j in range(self.shape.top_k):
                e = int(idx[t][j])
                if self.begin <= e < self.end:
                    out[t] += w[t][j] * self._pair(x[t], self.ex[e], rule_r)
            for s in range(self.shape.n_shared):
                if (self.mask >> s) & 1:
                    out[t] += self._pair(x[t], self.sh[s], rule_s)
        return torch.from_numpy(out)

    def cast(self, total, out, stream=None):
        out.copy_(total)
        return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, res):
    import datetime

    import torch.distributed as dist

    import synth
    from tests.helpers import small_shape
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        shape = small_shape(n_routed=7, top_k=3, n_shared=2, inter_shared=24)
        layer = ExpertParallelLayer(OracleBackend(shape, rank, world))
        x = synth.host_tokens(shape, 5, 17)
        out = torch.empty((5, shape.hidden), dtype=torch.float64)
        layer.forward(x, None, None, None, ("topk", 0.5), ("topk", 0.25), out=out)
        res[rank] = out.numpy().copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_sum_to_the_whole_layer(world):
    import synth
    from tests.helpers import host_layer, small_shape
    with mp.Manager() as m:
        res = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), res), nprocs=world, join=True)
        outs = [res[r] for r in range(world)]
    shape = small_shape(n_routed=7, top_k=3, n_shared=2, inter_shared=24)
    x = synth.host_tokens(shape, 5, 17)
    want = host_layer(shape).forward(x, ("topk", 0.5), ("topk", 0.25))["out"]
    for r in range(world):
        assert np.array_equal(outs[r], outs[0])  # every rank holds the same sum
    assert np.max(np.abs(outs[0] - want)) <= 1e-12 * np.max(np.abs(want))
