"""Expert parallelism through the C ABI on one GPU: G handles restricted to the ranks' experts
run one after another (the ranks of one decode step, emulated in turn); the sum of their fp32
partial outputs, the all-reduce's result, is rounded by moe_cast_output.  The combined layer is
checked against the fp64 oracle with the parity rules (every token's routing and kept sets, each
pair taken from the rank that owns its expert), and each handle must read only its own block of
routed weights."""
import numpy as np
import pytest
import torch

import synth
from sparse_expert_ffn_logits_b200 import (expert_weights, moe_cast_output, moe_create,
                                           moe_debug_lists, moe_destroy, moe_forward_partial,
                                           moe_set_expert_range, sparsity)
from sparse_expert_ffn_logits_b200.expert_parallel import expert_range, shared_mask
from sparse_expert_ffn_logits_b200.workload import DeviceLayer
from tests import parity

pytestmark = pytest.mark.gpu


class EmulatedRanks:
    """The G ranks of an expert-parallel layer on one device, with the interface parity.compare
    uses (shape, forward, debug)."""

    def __init__(self, dl, world):
        self.dl, self.shape, self.world = dl, dl.shape, world
        self.ranks = []
        for r in range(world):
            h = moe_create(dl.cfg)
            b, e = expert_range(self.shape.n_routed, world, r)
            moe_set_expert_range(h, b, e, shared_mask(self.shape.n_shared, world, r))
            # only the rank's own block of routed weights is handed over
            routed = expert_weights(dl.gate[b:e], dl.updown[b:e])
            self.ranks.append((h, b, e, routed))

    def forward(self, x, rule_r, rule_s=None):
        n = x.shape[0]
        total = torch.zeros((n, self.shape.hidden), dtype=torch.float32, device=x.device)
        for h, b, e, routed in self.ranks:
            part = torch.full_like(total, float("nan"))
            moe_forward_partial(h, x, n, self.dl.router, routed, self.dl.shared,
                                sparsity(rule_r), sparsity(rule_s) if rule_s else None, part)
            total += part
        out = torch.empty_like(x)
        moe_cast_output(self.ranks[0][0], total, n, out)
        return out

    def debug(self, n):
        s = self.shape
        k, S = s.top_k, s.n_shared
        P = k + S
        imax = max(s.inter, s.inter_shared if S else 0)
        per = []
        for h, *_ in self.ranks:
            r = {"idx": torch.empty((n, k), dtype=torch.int32, device="cuda"),
                 "w": torch.empty((n, k), dtype=torch.float32, device="cuda"),
                 "logits": torch.empty((n, s.n_routed), dtype=torch.float32, device="cuda"),
                 "cnt": torch.empty((n, P), dtype=torch.int32, device="cuda"),
                 "lists": torch.empty((n, P, imax), dtype=torch.int32, device="cuda"),
                 "act": torch.empty((n, P, imax), dtype=torch.float32, device="cuda")}
            moe_debug_lists(h, n, r["idx"], r["w"], r["logits"], r["cnt"], r["lists"], r["act"])
            per.append({key: v.cpu().numpy() for key, v in r.items()})
        torch.cuda.synchronize()
        for d in per[1:]:  # every rank routed every token the same way
            assert np.array_equal(d["idx"], per[0]["idx"])
            assert np.array_equal(d["w"], per[0]["w"])
        out = {key: per[0][key].copy() for key in ("idx", "w", "logits", "cnt", "lists", "act")}
        for t in range(n):
            for j in range(P):
                if j < k:
                    e = int(out["idx"][t][j])
                    owner = next(i for i, (_, b, en, _) in enumerate(self.ranks) if b <= e < en)
                else:
                    owner = (j - k) % self.world
                for key in ("cnt", "lists", "act"):
                    out[key][t][j] = per[owner][key][t][j]
                for i, d in enumerate(per):  # the other ranks report nothing for the pair
                    if i != owner:
                        assert d["cnt"][t][j] == 0 and (d["lists"][t][j] == -1).all()
        return out

    def close(self):
        for h, *_ in self.ranks:
            moe_destroy(h)
        self.ranks = []


@pytest.mark.parametrize("shape,world,B,rules", [
    (synth.OLMOE, 2, 16, (("topk", 0.9), None)),
    (synth.OLMOE, 3, 64, (("topk", 0.5), None)),
    (synth.DSV2L, 2, 8, (("topk", 0.9), ("topk", 0.5))),
    (synth.DSV2L, 3, 16, (("topk", 0.5), ("topk", 0.0))),
], ids=lambda v: getattr(v, "name", str(v)))
def test_ranks_sum_to_the_layer(shape, world, B, rules):
    dl = DeviceLayer(shape, max_tokens=64)
    ep = EmulatedRanks(dl, world)
    try:
        seed = synth.token_seed(shape, 60 + world)
        xh, xd = synth.host_tokens(shape, B, seed), dl.tokens(B, seed)
        rep = parity.compare(ep, xh, xd, rules[0], rules[1],
                             name=f"{shape.name} expert-parallel x{world} B={B}")
        print(rep)
        # against the unrestricted layer: the same kernels, other fp32 summation orders
        whole = dl.forward(xd, rules[0], rules[1]).float()
        got = ep.forward(xd, rules[0], rules[1]).float()
        scale = whole.pow(2).mean().sqrt()
        assert ((got - whole).abs() <= 1e-2 * torch.maximum(whole.abs(), scale)).all()
    finally:
        ep.close()
        dl.close()
