"""The parity checker (tests/parity.py) on the CPU, against a stand-in for the CUDA layer whose
results come from the oracle with planted disagreements.  It must fail a kept set that differs
far from the cut, take a disagreement inside the 1e-6 band as an allowed exemption, and count a
disagreement outside the band but inside the fp32 bound as the separate kind that fails the
comparison unless the test names an allowance."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity
from tests.helpers import f32, small_shape

SHAPE = small_shape(name="checker", hidden=64, n_routed=6, top_k=2, inter=64, n_shared=1,
                    inter_shared=32, dtype="f32", seed=5)


class FakeLayer:
    """Results of the oracle in the layout of the device layer's debug export, with the fp32
    rounding of the device; ``plant(fake, dbg, None)`` may alter the routing, activations and
    kept sets before they are returned, and the output follows the altered sets."""

    def __init__(self, shape, experts, shared, router, plant=None):
        self.shape = shape
        self.layer = oracle.Layer(shape, router, experts, shared)
        self.plant = plant
        self._dbg = None

    def forward(self, x_dev, rule_r, rule_s=None, out=None):
        x = x_dev.numpy()
        s = self.shape
        B, P = x.shape[0], s.top_k + s.n_shared
        ref = self.layer.forward(x, rule_r, rule_s)
        imax = max(s.inter, s.inter_shared)
        act = ref["a"].astype(np.float32)
        cnt = np.zeros((B, P), np.int32)
        lists = -np.ones((B, P, imax), np.int32)
        for t in range(B):
            for j in range(P):
                In = s.inter if j < s.top_k else s.inter_shared
                rule = rule_r if j < s.top_k else rule_s
                keep = oracle.select(np.abs(act[t][j][:In].astype(np.float64)), rule)
                kept = np.flatnonzero(keep)
                cnt[t][j] = len(kept)
                lists[t][j][: len(kept)] = kept
        dbg = {"idx": ref["idx"].copy(), "w": ref["w"].astype(np.float32),
               "logits": ref["logits"].astype(np.float32), "cnt": cnt, "lists": lists,
               "act": act}
        if self.plant:
            self.plant(self, dbg, None)
        # the output of the (possibly planted) routing and kept sets, as a device would give
        keep = np.zeros((B, P, imax), np.uint8)
        for t in range(B):
            for j in range(P):
                keep[t][j][dbg["lists"][t][j][: dbg["cnt"][t][j]]] = 1
        out_np = self.layer.forward(x, rule_r, rule_s, idx_in=dbg["idx"], keep_in=keep,
                                    keep_flag=np.ones((B, P), np.uint8))["out"]
        self._dbg = dbg
        return torch.from_numpy(out_np.astype(np.float32))

    def debug(self, n_tokens):
        return self._dbg


def _inputs(gate_edit=None):
    s = SHAPE
    router = synth.host_tensor(s, "router")
    experts = parity.host_inputs(s, range(s.n_routed))
    x = synth.host_tokens(s, 6, synth.token_seed(s, 1))
    if gate_edit:
        experts = gate_edit(experts, x, router)
    shared = parity.host_shared(s)
    return router, experts, shared, x


def _compare(plant=None, gate_edit=None, rule=("topk", 0.5), **kw):
    router, experts, shared, x = _inputs(gate_edit)
    fake = FakeLayer(SHAPE, experts, shared, router, plant)
    return parity.compare(fake, x, torch.from_numpy(x), rule, ("topk", 0.5),
                          shared_weights=shared, expert_cache=experts, router_host=router,
                          name="checker self-test on planted results", **kw)


def test_clean_results_pass_without_exemptions():
    rep = _compare()
    assert rep.pairs == 6 * 3 and rep.tokens_routed == 6 and rep.tokens_output == 6
    assert rep.fp32_only == 0 and rep.sel_band_pairs == 0 and rep.route_band == 0


def _swap_at_cut(fake, dbg, t, j, far):
    """Swap one kept neuron of pair (t, j) for a dropped one: the lowest kept and the highest
    dropped score (at the cut), or the highest kept and the lowest dropped (far from it)."""
    s = fake.shape
    In = s.inter if j < s.top_k else s.inter_shared
    a = np.abs(dbg["act"][t][j][:In])
    kept = list(dbg["lists"][t][j][: dbg["cnt"][t][j]])
    dropped = [n for n in range(In) if n not in kept]
    if far:
        out_n, in_n = max(kept, key=lambda n: a[n]), min(dropped, key=lambda n: a[n])
    else:
        out_n, in_n = min(kept, key=lambda n: a[n]), max(dropped, key=lambda n: a[n])
    # the activations move with the set, so the device's own selection stays consistent
    act = dbg["act"][t][j]
    act[out_n], act[in_n] = act[in_n], act[out_n]
    kept = sorted([n for n in kept if n != out_n] + [in_n])
    dbg["lists"][t][j][: len(kept)] = kept


def test_a_swap_far_from_the_cut_fails():
    with pytest.raises(AssertionError, match="neuron"):
        _compare(plant=lambda f, d, o: _swap_at_cut(f, d, 2, 1, far=True))


def test_wrong_expert_fails():
    def plant(f, dbg, out):
        lg = dbg["logits"][3]
        worst = int(np.argmin(lg))
        dbg["idx"][3][1] = worst
        lg[worst] = lg[dbg["idx"][3][0]] + 1.0  # keep the device's own top-k consistent
        dbg["idx"][3] = oracle.topk(lg.astype(np.float64), f.shape.top_k)
    with pytest.raises(AssertionError, match="differs"):
        _compare(plant=plant)


def _near_tie(gap):
    """An edit of the gate of token 0's first expert: the neuron just below that pair's cut
    (rank K + 1) gets the gate row of the neuron at the cut (rank K) plus a change of `gap` in
    the weight that meets token 0's largest |x|, so the two scores lie about `gap` apart and
    straddle the cut.  Returns the edit and, through `rows`, the expert and the two neurons."""
    rows = []

    def edit(experts, x, router):
        s = SHAPE
        _, idx, _ = oracle.Layer(s, router, {}, []).route(x[:1])
        e = int(idx[0][0])
        g = experts[e][0].copy()
        _, a = oracle.gate(x[0], g)
        sig = np.abs(a)
        order = np.lexsort((np.arange(s.inter), -sig))
        K = oracle.keep_count(s.inter, 0.5)
        n_c, n_d = int(order[K - 1]), int(order[K])
        h = int(np.argmax(np.abs(f32(x[0]))))
        g[n_d] = g[n_c]
        g[n_d][h] = np.float32(g[n_c][h] + gap)
        rows[:] = [e, n_c, n_d]
        out = dict(experts)
        out[e] = (g, experts[e][1], experts[e][2])
        return out

    return edit, rows


def _swap_rows(rows):
    """Where exactly one of the two neurons is kept in a pair of the edited expert, keep the
    other one.  The
    device activations are changed to match (the dropped neuron's score below the kept one's,
    by one fp32 step where the two round to the same value), so that the device's own selection
    stays consistent, as a device whose fp32 gate ordered the two differently would report."""
    def plant(fake, dbg, out):
        s = fake.shape
        e, n1, n2 = rows
        for t in range(dbg["idx"].shape[0]):
            for j in range(s.top_k):
                if int(dbg["idx"][t][j]) != e:
                    continue
                kept = set(dbg["lists"][t][j][: dbg["cnt"][t][j]].tolist())
                if (n1 in kept) == (n2 in kept):
                    continue
                n_in, n_out = (n1, n2) if n1 in kept else (n2, n1)
                act = dbg["act"][t][j]
                if abs(act[n_in]) != abs(act[n_out]):
                    act[n_in], act[n_out] = act[n_out], act[n_in]
                else:
                    act[n_in] = np.nextafter(act[n_in], np.float32(0))
                kept ^= {n1, n2}
                dbg["lists"][t][j][: len(kept)] = sorted(kept)
    return plant


def test_a_swap_inside_the_band_is_an_allowed_exemption():
    edit, rows = _near_tie(1e-9)
    rep = _compare(plant=_swap_rows(rows), gate_edit=edit)
    assert rep.sel_band_pairs > 0 and rep.fp32_only == 0


def test_a_swap_outside_the_band_inside_the_fp32_bound_needs_an_allowance():
    # |x| ~ 1 and H = 64: a 2e-6 weight change moves the score by ~1e-6 of a cut of ~0.3,
    # beyond the 1e-6 band (3e-7) and inside the fp32 bound (64 * 2^-24 * sum|w||x| ~ 1e-5)
    edit, rows = _near_tie(4e-6)
    with pytest.raises(AssertionError, match="outside the 1e-6 band"):
        _compare(plant=_swap_rows(rows), gate_edit=edit)
    rep = _compare(plant=_swap_rows(rows), gate_edit=edit, allow_fp32_bound=100)
    assert len(rep.sel_fp32_only) > 0
    assert "inside fp32 bound" in str(rep)
