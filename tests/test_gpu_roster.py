"""Roster routing ("Predatory MoE", technical summary, Methodology 2) through the C ABI against
the fp64 oracle, over consecutive decode steps of a batch of sequences.  Each step the oracle
computes every sequence's bias from its own copy of the selection counts, and the layer's
routing, kept sets and output are compared as in the other parity tests; the layer's counts
(updated on the device by the router) must then equal the oracle's exactly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from sparse_expert_ffn_logits_b200 import MoEError, moe_last_launches
from sparse_expert_ffn_logits_b200.workload import DeviceLayer
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,m,delta", [(synth.OLMOE, 12, 0.5), (synth.TINY, 3, 0.25),
                                           (synth.DSV2L, 8, 0.25)],
                         ids=lambda v: getattr(v, "name", str(v)))
def test_roster_steps_match_the_oracle(shape, m, delta):
    B, steps = 16, 14
    delta = float(np.float32(delta))
    dl = DeviceLayer(shape, max_tokens=B)
    try:
        counts_h = np.zeros((B, shape.n_routed), np.int32)
        counts_d = torch.zeros((B, shape.n_routed), dtype=torch.int32, device="cuda")
        pinned_d = torch.zeros(B, dtype=torch.int32, device="cuda")
        dl.roster = (counts_d, pinned_d, m, delta)
        cache = {}
        shared = parity.host_shared(shape)
        after_pin = [set() for _ in range(B)]
        rule_s = ("topk", 0.5) if shape.n_shared else None
        for step in range(steps):
            # even sequences pin their roster from step 5 on; odd ones stay in the barrier phase
            pinned_h = np.array([int(step >= 5 and t % 2 == 0) for t in range(B)], np.int32)
            pinned_d.copy_(torch.from_numpy(pinned_h))
            bias = oracle.roster_bias(counts_h, pinned_h, m, delta)
            seed = synth.token_seed(shape, 300 + step)
            xh, xd = synth.host_tokens(shape, B, seed), dl.tokens(B, seed)
            rep = parity.compare(dl, xh, xd, ("topk", 0.5), rule_s, router_bias=bias,
                                 expert_cache=cache, shared_weights=shared,
                                 name=f"{shape.name} roster step {step}")
            # roster bias, router, gate, selection, up/down, output cast
            assert moe_last_launches(dl.h) == 6
            oracle.roster_update(counts_h, rep.idx)
            assert np.array_equal(counts_d.cpu().numpy(), counts_h), f"counts differ at {step}"
            for t in range(B):
                if pinned_h[t]:
                    after_pin[t].update(int(e) for e in rep.idx[t])
        # a pinned sequence keeps to its m experts
        assert max(len(s) for s in after_pin) <= m
    finally:
        dl.roster = None
        dl.close()


def test_roster_arguments_are_checked():
    shape = synth.TINY
    dl = DeviceLayer(shape, max_tokens=4)
    try:
        counts = torch.zeros((4, shape.n_routed), dtype=torch.int32, device="cuda")
        pinned = torch.zeros(4, dtype=torch.int32, device="cuda")
        x = dl.tokens(4, 1)
        for m, delta in ((shape.top_k - 1, 0.1), (shape.n_routed + 1, 0.1), (3, -1.0),
                         (3, float("inf"))):
            dl.roster = (counts, pinned, m, delta)
            with pytest.raises(MoEError):
                dl.forward(x, ("topk", 0.5))
        assert not counts.any()  # nothing ran
    finally:
        dl.roster = None
        dl.close()
