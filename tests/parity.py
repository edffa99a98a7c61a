"""Element-by-element comparison of the CUDA layer with the fp64 oracle on the same seeded inputs.

Rules (tolerances from the target the layer is built to; see the design notes):
  * routing: the chosen experts match the oracle's exactly, except a token whose k-th / (k+1)-th
    oracle logits lie within max(1e-6 |l|, fp32 bound) of each other; such a token is re-run in
    the oracle with the GPU's experts.  Feeding the GPU's own fp32 logits to the oracle's top-k
    must give the GPU's experts with no exemption.
  * selection: the kept sets match exactly, except neurons whose oracle score lies within
    max(1e-6 |cut|, fp32 bound of the GPU score) of the cut (K-th largest score, or t); such
    pairs are re-run in the oracle with the GPU's set.  Feeding the GPU's own fp32 activations
    to the oracle's selection must give the GPU's sets with no exemption.
  * output: |gpu - ref| <= tol * max(|ref|, rms(ref)) elementwise; tol 2e-2 for bf16, 1e-5 fp32.
The fp32 bound of a dot product of length H with exact products is H * 2^-24 * sum|w||x|
(recursive-summation worst case), widened by 1.1 for SiLU's slope and 4 ulp for its evaluation.
"""
import numpy as np
import torch

import oracle
import synth
from tests.helpers import f32

U32 = 2.0 ** -24


def tolerance(shape):
    return 2e-2 if shape.dtype == "bf16" else 1e-5


def host_inputs(shape, experts):
    return {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
                synth.host_tensor(shape, "down", e)) for e in experts}


def host_shared(shape):
    return [(synth.host_tensor(shape, "sh_gate", s), synth.host_tensor(shape, "sh_up", s),
             synth.host_tensor(shape, "sh_down", s)) for s in range(shape.n_shared)]


class Report:
    def __init__(self):
        self.route_exempt = 0
        self.sel_exempt_pairs = 0
        self.sel_exempt_neurons = 0
        self.pairs = 0
        self.max_err = 0.0

    def __str__(self):
        return (f"pairs={self.pairs} route_exempt_tokens={self.route_exempt} "
                f"sel_exempt_pairs={self.sel_exempt_pairs} "
                f"sel_exempt_neurons={self.sel_exempt_neurons} max_scaled_err={self.max_err:.3e}")


def _mask_from_list(cnt, lst, I):
    m = np.zeros(I, np.uint8)
    if cnt:
        m[lst[:cnt]] = 1
    return m


def compare(dl, x_host, x_dev, rule_r, rule_s=None, tokens=None, shared_weights=None,
            expert_cache=None, router_host=None):
    """Runs the layer on x_dev and checks it against the oracle on x_host (same values).
    ``tokens`` restricts the oracle comparison to a subset of tokens (sampled check)."""
    shape = dl.shape
    B = x_host.shape[0]
    k, S, I, Ish, H = shape.top_k, shape.n_shared, shape.inter, shape.inter_shared, shape.hidden
    P = k + S
    out = dl.forward(x_dev, rule_r, rule_s)
    torch.cuda.synchronize()
    out_gpu = out.float().cpu().numpy().astype(np.float64)
    dbg = dl.debug(B)
    rep = Report()
    sel_tokens = np.arange(B) if tokens is None else np.asarray(tokens)
    xs = x_host[sel_tokens]
    router = synth.host_tensor(shape, "router") if router_host is None else router_host
    xf = f32(xs).astype(np.float64)
    wr = f32(router).astype(np.float64)

    # ---- routing
    rl = oracle.Layer(shape, router, {}, [])
    logits_o, idx_o, _ = rl.route(xs)
    idx_use = idx_o.copy()
    for i, t in enumerate(sel_tokens):
        g_idx = dbg["idx"][t]
        # second check: the oracle's top-k on the GPU's own logits
        assert np.array_equal(oracle.topk(dbg["logits"][t].astype(np.float64), k), g_idx), \
            f"top-k logic differs on token {t}"
        if np.array_equal(np.sort(g_idx), np.sort(idx_o[i])):
            idx_use[i] = g_idx
            continue
        lo = logits_o[i]
        order = np.lexsort((np.arange(shape.n_routed), -lo))
        cut = lo[order[k - 1]]
        bound = H * U32 * (np.abs(wr) @ np.abs(xf[i]))
        diff = set(g_idx.tolist()) ^ set(idx_o[i].tolist())
        for e in diff:
            tol_e = max(1e-6 * abs(cut), bound[e] + bound[order[k - 1]])
            assert abs(lo[e] - cut) <= tol_e, \
                f"token {t}: expert {e} differs, logit gap {abs(lo[e]-cut):.3e} > {tol_e:.3e}"
        rep.route_exempt += 1
        idx_use[i] = g_idx
    # routing weights of the common choice
    for i, t in enumerate(sel_tokens):
        w_o = rl.route_weights(logits_o[i], dbg["idx"][t])
        assert np.max(np.abs(w_o - dbg["w"][t])) <= (1e-5 if shape.dtype == "f32" else 2e-4) * max(
            1.0, np.max(np.abs(w_o))), f"routing weights differ on token {t}"

    # ---- oracle layer with the experts it needs
    need = sorted(set(int(e) for e in idx_use.ravel()))
    cache = expert_cache if expert_cache is not None else {}
    missing = [e for e in need if e not in cache]
    cache.update(host_inputs(shape, missing))
    experts = {e: cache[e] for e in need}
    shared = shared_weights if shared_weights is not None else host_shared(shape)
    layer = oracle.Layer(shape, router, experts, shared)
    ref = layer.forward(xs, rule_r, rule_s, idx_in=idx_use)

    # ---- selection
    imax = max(I, Ish if S else 0)
    keep_in = np.zeros((len(sel_tokens), P, imax), np.uint8)
    flag = np.zeros((len(sel_tokens), P), np.uint8)
    for i, t in enumerate(sel_tokens):
        # the oracle's pairs follow idx_use order, which equals the GPU's idx order
        for j in range(P):
            In = I if j < k else Ish
            rule = rule_r if j < k else rule_s
            rep.pairs += 1
            gm = _mask_from_list(int(dbg["cnt"][t][j]), dbg["lists"][t][j], In)
            lst = dbg["lists"][t][j][: int(dbg["cnt"][t][j])]
            assert np.all(np.diff(lst) > 0), "kept list not ascending"
            if rule[0] == "topk":
                assert gm.sum() == oracle.keep_count(In, rule[1]), "kept count != K"
            # second check: the oracle's selection on the GPU's own activations
            ga = dbg["act"][t][j][:In].astype(np.float64)
            assert np.array_equal(oracle.select(np.abs(ga), rule), gm), \
                f"selection logic differs (token {t}, pair {j})"
            om = ref["keep"][i][j][:In]
            if np.array_equal(gm, om):
                continue
            sig = np.abs(ref["a"][i][j][:In])
            if rule[0] == "topk":
                K = oracle.keep_count(In, rule[1])
                cut = np.sort(sig)[::-1][K - 1]
            else:
                cut = float(np.float32(rule[1]))
            if j < k:
                wg = f32(experts[int(idx_use[i][j])][0]).astype(np.float64)
            else:
                wg = f32(shared[j - k][0]).astype(np.float64)
            gb = H * U32 * (np.abs(wg) @ np.abs(xf[i]))
            bound = 1.1 * gb + 4 * 2.0 ** -23 * sig
            bad = np.flatnonzero(gm != om)
            for n in bad:
                tol_n = max(1e-6 * abs(cut), bound[n] + (bound[np.argmin(np.abs(sig - cut))]))
                assert abs(sig[n] - cut) <= tol_n, (
                    f"token {t} pair {j} neuron {n}: score {sig[n]:.9g} vs cut {cut:.9g} "
                    f"(gap {abs(sig[n]-cut):.3e} > {tol_n:.3e})")
            rep.sel_exempt_pairs += 1
            rep.sel_exempt_neurons += len(bad)
            keep_in[i][j][:In] = gm
            flag[i][j] = 1
    if flag.any():
        ref = layer.forward(xs, rule_r, rule_s, idx_in=idx_use, keep_in=keep_in, keep_flag=flag)

    # ---- output
    r = ref["out"]
    g = out_gpu[sel_tokens]
    scale = np.maximum(np.abs(r), np.sqrt(np.mean(r * r)) if r.size else 1.0)
    err = np.abs(g - r) / np.maximum(scale, 1e-30)
    rep.max_err = float(err.max()) if err.size else 0.0
    tol = tolerance(shape)
    assert rep.max_err <= tol, f"output error {rep.max_err:.3e} > {tol} ({rep})"
    return rep
