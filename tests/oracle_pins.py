"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` takes an oracle library handle and raises AssertionError on a mismatch, so the
same pins run against the real oracle (test_oracle_pins.py) and against copies of it with a
planted mistake (test_oracle_mutants.py), which must each fail at least one pin.

What pins what:
  keep count      exact rational ceil((1 - s) I) from the decimal s
  gate / SiLU     numpy matmul and torch.nn.functional.silu (library routines)
  selection       brute force over every K-subset: the kept set is the one of maximal exact
                  score sum, ties broken by the lexicographically smallest index tuple
  threshold       strict comparison on constructed equal scores; t = -inf keeps everything
  routing         numpy logits, brute force over k-subsets (tied router rows included),
                  scipy softmax / expit for the three weight rules
  layer output    s = 0 equals the textbook dense SwiGLU MoE (torch fp64); s > 0 equals the
                  dense layer with an explicit 0/1 mask built by a full stable sort
  invariants      expert relabelling, batch independence, W_up scaling, calibration quantile
  roster routing  the roster by brute force over m-subsets of the counts; the biased top-k by
                  brute force with scipy weights on the unbiased logits; simulated sequences:
                  no bias while exploring, a pinned sequence never leaves its m experts, and
                  the barrier shrinks the experts a sequence uses
"""
import itertools
import sys
from fractions import Fraction

import numpy as np
import scipy.special
import torch

import oracle
import synth
from tests.helpers import f32, host_layer, small_shape

F = torch.nn.functional


def _t(a):
    return torch.from_numpy(np.asarray(f32(a), dtype=np.float64))


def _rel(a, b):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# --------------------------------------------------------------------------------------------
def pin_keep_count(lib):
    for s_str in ["0", "0.1", "0.25", "0.29", "0.3", "0.5", "0.7", "0.9", "0.908", "0.95",
                  "0.98", "0.999", "1"]:
        s = Fraction(s_str)
        for I in [1, 7, 40, 100, 512, 1000, 1024, 1408, 2880, 8192]:
            want = -((-(1 - s) * I).__floor__())  # ceil((1 - s) I), exact
            got = oracle.keep_count(I, float(s_str), lib=lib)
            assert got == want, (s_str, I, got, want)


def pin_gate_matches_library(lib):
    rng = np.random.default_rng(3)
    for dt in (np.float32, np.uint16):
        H, I = 40, 33
        if dt is np.float32:
            x = rng.standard_normal(H).astype(np.float32)
            wg = rng.standard_normal((I, H)).astype(np.float32)
        else:
            x = synth.fill_host(H, 5, 1, 0, 1.0, synth.BF16)
            wg = synth.fill_host(I * H, 5, 3, 0, 0.3, synth.BF16).reshape(I, H)
        g, a = oracle.gate(x, wg, lib=lib)
        g_ref = f32(wg).astype(np.float64) @ f32(x).astype(np.float64)
        assert _rel(g, g_ref) < 1e-12
        a_ref = F.silu(torch.from_numpy(g)).numpy()
        assert _rel(a, a_ref) < 1e-14


def _brute_topk(score, K):
    best = None
    for sub in itertools.combinations(range(len(score)), K):
        key = (sum(Fraction(float(score[i])) for i in sub), tuple(-i for i in sub))
        if best is None or key > best[0]:
            best = (key, sub)
    keep = np.zeros(len(score), np.uint8)
    keep[list(best[1])] = 1
    return keep


def pin_select_bruteforce(lib):
    rng = np.random.default_rng(7)
    for trial in range(60):
        I = int(rng.integers(5, 11))
        if trial % 2:
            score = rng.choice([0.1, 0.5, 0.5, 0.9, 0.0], size=I)  # many ties
        else:
            score = np.abs(rng.standard_normal(I))
        K = int(rng.integers(0, I + 1))
        s = (I - K) / I
        assert oracle.keep_count(I, s, lib=lib) == K
        got = oracle.select(score, ("topk", s), lib=lib)
        want = _brute_topk(score, K)
        assert np.array_equal(got, want), (score, K, got, want)


def pin_threshold_strict(lib):
    t = 0.25
    score = np.array([0.25, np.nextafter(0.25, 1.0), np.nextafter(0.25, 0.0), 3.0, 0.0])
    got = oracle.select(score, ("threshold", t), lib=lib)
    assert list(got) == [0, 1, 0, 1, 0], got
    got = oracle.select(np.array([0.0, 1.0, 5.0]), ("threshold", -np.inf), lib=lib)
    assert list(got) == [1, 1, 1]


def _tied_layer(route, lib):
    shape = small_shape(route=route, n_routed=6, top_k=2, n_shared=0, inter_shared=0)
    layer = host_layer(shape, lib=lib)
    router = synth.host_tensor(shape, "router").copy()
    router[3] = router[1]  # experts 1 and 3 always tie
    router[5] = router[1]  # and 5
    ex = {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
              synth.host_tensor(shape, "down", e)) for e in range(shape.n_routed)}
    return shape, oracle.Layer(shape, router, ex, lib=lib), router, layer


def pin_routing(lib):
    for route in ("softmax_topk", "softmax_all", "sigmoid"):
        shape, layer, router, _ = _tied_layer(route, lib)
        x = synth.host_tokens(shape, 24, 77)
        # push some tokens so that the tied experts lead
        logits, idx, w = layer.route(x)
        lg_ref = f32(x).astype(np.float64) @ f32(router).astype(np.float64).T
        assert _rel(logits, lg_ref) < 1e-12
        for t in range(x.shape[0]):
            want = _brute_topk(logits[t], shape.top_k)
            got = np.zeros(shape.n_routed, np.uint8)
            got[idx[t]] = 1
            assert np.array_equal(got, want), (route, t)
            # ordered by (logit desc, index asc)
            pairs = [(-logits[t][e], e) for e in idx[t]]
            assert pairs == sorted(pairs)
            if route == "softmax_topk":
                w_ref = scipy.special.softmax(logits[t][idx[t]])
            elif route == "softmax_all":
                w_ref = scipy.special.softmax(logits[t])[idx[t]]
            else:
                w_ref = scipy.special.expit(logits[t][idx[t]])
            assert _rel(w[t], w_ref) < 1e-13, (route, w[t], w_ref)
    # a token whose three best experts are the tied 1, 3, 5 must keep 1 and 3
    shape, layer, router, _ = _tied_layer("softmax_topk", lib)
    x = f32(router[1]).astype(np.float32)[None, :] * 50.0
    _, idx, _ = layer.route(x.astype(np.float32))
    assert list(idx[0]) == [1, 3], idx


def _dense_reference(shape, layer_inputs, x, idx, w, masks=None):
    """Textbook SwiGLU MoE in torch fp64; masks[t][j] optionally zeroes neurons of pair j."""
    router, experts, shared = layer_inputs
    X = _t(x)
    out = torch.zeros(X.shape[0], shape.hidden, dtype=torch.float64)
    for t in range(X.shape[0]):
        pairs = [(experts[int(idx[t][j])], float(w[t][j])) for j in range(shape.top_k)]
        pairs += [(sh, 1.0) for sh in shared]
        for j, ((g, u, d), wj) in enumerate(pairs):
            hid = F.silu(_t(g) @ X[t]) * (_t(u) @ X[t])
            if masks is not None:
                hid = hid * torch.from_numpy(masks[t][j][: hid.shape[0]].astype(np.float64))
            out[t] += wj * (_t(d) @ hid)
    return out.numpy()


def _inputs(shape):
    router = synth.host_tensor(shape, "router")
    experts = {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
                   synth.host_tensor(shape, "down", e)) for e in range(shape.n_routed)}
    shared = [(synth.host_tensor(shape, "sh_gate", s), synth.host_tensor(shape, "sh_up", s),
               synth.host_tensor(shape, "sh_down", s)) for s in range(shape.n_shared)]
    return router, experts, shared


def pin_dense_at_zero_sparsity(lib):
    for route, dtype, nsh in (("softmax_topk", "f32", 1), ("softmax_all", "bf16", 2),
                              ("sigmoid", "f32", 1), ("softmax_topk", "bf16", 0)):
        shape = small_shape(route=route, dtype=dtype, n_shared=nsh,
                            inter_shared=24 if nsh else 0)
        ins = _inputs(shape)
        layer = oracle.Layer(shape, *ins, lib=lib)
        x = synth.host_tokens(shape, 5, 21)
        for rule in (("topk", 0.0), ("threshold", -np.inf)):
            r = layer.forward(x, rule, rule)
            ref = _dense_reference(shape, ins, x, r["idx"], r["w"])
            assert _rel(r["out"], ref) < 1e-12, (route, dtype, rule, _rel(r["out"], ref))
            assert r["keep"][:, : shape.top_k, : shape.inter].all()


def _sorted_mask(sigma, K):
    order = np.lexsort((np.arange(len(sigma)), -sigma))  # sigma desc, then index asc
    m = np.zeros(len(sigma), np.uint8)
    m[order[:K]] = 1
    return m


def pin_masked_layer(lib):
    for dtype, s_r, s_sh in (("f32", 0.5, 0.25), ("bf16", 0.9, 0.5), ("f32", 0.29, 0.0)):
        shape = small_shape(dtype=dtype, n_shared=1, inter_shared=24)
        ins = _inputs(shape)
        router, experts, shared = ins
        layer = oracle.Layer(shape, *ins, lib=lib)
        x = synth.host_tokens(shape, 6, 5)
        r = layer.forward(x, ("topk", s_r), ("topk", s_sh))
        masks = np.zeros_like(r["keep"])
        X = _t(x)
        for t in range(x.shape[0]):
            for j in range(shape.top_k + shape.n_shared):
                if j < shape.top_k:
                    g = experts[int(r["idx"][t][j])][0]; I = shape.inter; s = s_r
                else:
                    g = shared[j - shape.top_k][0]; I = shape.inter_shared; s = s_sh
                a = F.silu(_t(g) @ X[t]).numpy()
                assert _rel(r["a"][t][j][:I], a) < 1e-12
                K = -((-(1 - Fraction(str(s))) * I).__floor__())
                # the mask from the oracle's own activations (its scores), full stable sort
                masks[t][j][:I] = _sorted_mask(np.abs(r["a"][t][j][:I]), K)
                assert int(r["keep"][t][j][:I].sum()) == K
        assert np.array_equal(masks, r["keep"]), "kept sets differ from the full-sort mask"
        ref = _dense_reference(shape, ins, x, r["idx"], r["w"], masks)
        assert _rel(r["out"], ref) < 1e-12, _rel(r["out"], ref)


def pin_invariants(lib):
    shape = small_shape(n_shared=1, inter_shared=24)
    router, experts, shared = _inputs(shape)
    layer = oracle.Layer(shape, router, experts, shared, lib=lib)
    x = synth.host_tokens(shape, 5, 9)
    rule = ("topk", 0.5)
    base = layer.forward(x, rule, rule)
    # batch independence
    for t in range(x.shape[0]):
        one = layer.forward(x[t:t + 1], rule, rule)
        assert np.array_equal(one["out"][0], base["out"][t])
    # relabelling the experts together with their router rows
    perm = np.random.default_rng(1).permutation(shape.n_routed)
    router_p = router[perm]
    experts_p = {i: experts[int(perm[i])] for i in range(shape.n_routed)}
    rp = oracle.Layer(shape, router_p, experts_p, shared, lib=lib).forward(x, rule, rule)
    assert _rel(rp["out"], base["out"]) < 1e-14
    assert np.array_equal(np.sort(perm[rp["idx"]], 1), np.sort(base["idx"], 1))
    # scaling W_up by 2 keeps the sets and doubles the output exactly
    experts_2 = {e: (g, (f32(u) * 2).astype(np.float32), d) for e, (g, u, d) in experts.items()}
    shared_2 = [(g, (f32(u) * 2).astype(np.float32), d) for (g, u, d) in shared]
    r2 = oracle.Layer(shape, router, experts_2, shared_2, lib=lib).forward(x, rule, rule)
    assert np.array_equal(r2["keep"], base["keep"])
    assert np.array_equal(r2["out"], 2 * base["out"])
    # s = 1 drops every routed neuron: only the shared expert remains
    r1 = layer.forward(x, ("topk", 1.0), ("topk", 0.0))
    only_sh = oracle.Layer(shape, router, experts, shared, lib=lib).forward(
        x, ("threshold", np.inf), ("topk", 0.0))
    assert np.array_equal(r1["out"], only_sh["out"])
    assert r1["keep"][:, : shape.top_k].sum() == 0


def pin_calibration(lib):
    shape = small_shape(n_shared=1, inter_shared=24)
    router, experts, shared = _inputs(shape)
    layer = oracle.Layer(shape, router, experts, shared, lib=lib)
    x = synth.host_tokens(shape, 64, 1000)
    _, idx, _ = layer.route(x)
    X = _t(x)
    for sh, s in ((False, 0.5), (False, 0.9), (True, 0.3), (False, 0.0)):
        t, N = layer.calibrate(x, s, shared=sh)
        sc = []
        for ti in range(x.shape[0]):
            gs = [shared[0][0]] if sh else [experts[int(e)][0] for e in idx[ti]]
            for g in gs:
                sc.append(np.abs(F.silu(_t(g) @ X[ti]).numpy()))
        sc = np.sort(np.concatenate(sc))
        assert N == sc.size
        m = int(np.floor(s * N))
        if m == 0:
            assert t == -np.inf
            continue
        assert abs(t - sc[m - 1]) <= 1e-12 * abs(sc[m - 1])
        assert int((sc > sc[m - 1]).sum()) == N - m


def pin_roster_bias(lib):
    rng = np.random.default_rng(11)
    for trial in range(80):
        E = int(rng.integers(3, 8))
        m = int(rng.integers(1, E + 1))
        counts = rng.integers(0, 4, size=(1, E)).astype(np.int32)
        if trial % 3 == 0:
            counts[0, rng.integers(0, E)] += 5
        pinned = int(trial % 4 == 1)
        delta = float(rng.choice([0.0, 0.25, 3.0]))
        b = oracle.roster_bias(counts, [pinned], m, delta, lib=lib)[0]
        roster = _brute_topk(counts[0].astype(np.float64), m)  # lower index wins equal counts
        distinct = int((counts[0] > 0).sum())
        for e in range(E):
            if pinned:
                want = 0.0 if roster[e] else -np.inf
            elif distinct < m:
                want = 0.0
            else:
                want = delta if roster[e] else -delta
            assert b[e] == want, (counts, m, pinned, delta, e, b)
    c = np.zeros((2, 5), np.int32)
    oracle.roster_update(c, np.array([[4, 1], [0, 4]]), lib=lib)
    oracle.roster_update(c, np.array([[4, 2], [3, 0]]), lib=lib)
    assert c.tolist() == [[0, 1, 1, 0, 2], [2, 0, 0, 1, 1]]


def pin_route_biased(lib):
    shape = small_shape(route="softmax_topk", n_routed=7, top_k=3, n_shared=0, inter_shared=0)
    router = synth.host_tensor(shape, "router")
    for route in ("softmax_topk", "softmax_all", "sigmoid"):
        sh = shape.with_(route=route)
        layer = oracle.Layer(sh, router, {}, lib=lib)
        x = synth.host_tokens(sh, 12, 31)
        lg_ref = f32(x).astype(np.float64) @ f32(router).astype(np.float64).T
        # no bias is the plain router
        l0, i0, w0 = layer.route(x)
        l1, i1, w1 = layer.route_biased(x, None)
        assert np.array_equal(i0, i1) and np.array_equal(w0, w1)
        rng = np.random.default_rng(5)
        bias = rng.choice([0.0, 0.02, -0.02, 0.5, -np.inf], size=(12, 7))
        bias[:, :3] = rng.choice([0.0, 0.02, -0.02], size=(12, 3))  # >= k finite entries
        lg, idx, w = layer.route_biased(x, bias)
        assert _rel(lg, lg_ref) < 1e-12
        for t in range(12):
            v = lg_ref[t] + bias[t]
            want = _brute_topk(np.where(np.isinf(v), -1e30, v), sh.top_k)  # exact sums
            got = np.zeros(7, np.uint8)
            got[idx[t]] = 1
            assert np.array_equal(got, want), (route, t)
            if route == "softmax_topk":
                w_ref = scipy.special.softmax(lg_ref[t][idx[t]])
            elif route == "softmax_all":
                w_ref = scipy.special.softmax(lg_ref[t])[idx[t]]
            else:
                w_ref = scipy.special.expit(lg_ref[t][idx[t]])
            assert _rel(w[t], w_ref) < 1e-12, (route, w[t], w_ref)


def pin_roster_sequences(lib):
    """Decode steps of 24 sequences with the roster rule, on the oracle's own routing."""
    shape = small_shape(n_routed=16, top_k=2, n_shared=0, inter_shared=0)
    router = synth.host_tensor(shape, "router")
    layer = oracle.Layer(shape, router, {}, lib=lib)
    S, steps, m, pin_at = 24, 40, 4, 8
    used = {}
    for delta in (0.0, 0.05):
        counts = np.zeros((S, 16), np.int32)
        seen_after_pin = [set() for _ in range(S)]
        for step in range(steps):
            x = synth.host_tokens(shape, S, 400 + step)
            pinned = np.full(S, int(delta > 0 and step >= pin_at), np.int32)
            b = oracle.roster_bias(counts, pinned, m, delta, lib=lib)
            _, idx, _ = layer.route_biased(x, b)
            _, idx0, _ = layer.route(x)
            for t in range(S):
                if int((counts[t] > 0).sum()) < m and not pinned[t]:
                    # exploring: the choice is the router's own
                    assert np.array_equal(idx[t], idx0[t])
                if pinned[t]:
                    # the roster (pinned by brute force in pin_roster_bias): a stable sort
                    roster = np.lexsort((np.arange(16), -counts[t]))[:m]
                    assert all(int(e) in roster for e in idx[t])
                    seen_after_pin[t].update(int(e) for e in idx[t])
            oracle.roster_update(counts, idx, lib=lib)
        used[delta] = np.mean([(c > 0).sum() for c in counts])
        if delta > 0:
            assert max(len(v) for v in seen_after_pin) <= m
    # the unbiased router spreads each sequence over many more experts than the budget
    assert used[0.0] > 2 * m and used[0.05] < used[0.0], used


PINS = [pin_keep_count, pin_gate_matches_library, pin_select_bruteforce, pin_threshold_strict,
        pin_routing, pin_dense_at_zero_sparsity, pin_masked_layer, pin_invariants,
        pin_calibration, pin_roster_bias, pin_route_biased, pin_roster_sequences]


def run_all(lib):
    failed = []
    for p in PINS:
        try:
            p(lib)
        except AssertionError:
            failed.append(p.__name__)
        except Exception as e:  # a broken oracle may also raise
            failed.append(f"{p.__name__}:{type(e).__name__}")
    return failed


def main(paths):
    for path in paths:
        failed = run_all(oracle.load(path))
        print(f"FAILED_PINS {path}=" + ",".join(failed), flush=True)


if __name__ == "__main__":
    main(sys.argv[1:])
