"""Element-by-element comparison of the CUDA layer with the fp64 oracle on the same seeded inputs.

Rules (tolerances of the target the layer is built to):
  * routing, checked for EVERY token of the batch: the chosen experts match the oracle's exactly,
    except an expert whose oracle logit lies within 1e-6 |l_k| of the k-th logit l_k (the
    allowed band).  A mismatch outside that band but inside the fp32 accumulation bound of the
    GPU logits is a separate kind, counted and listed in the report, and it fails the check
    unless the test names an allowance for it.  Feeding the GPU's own fp32 logits to the
    oracle's top-k must give the GPU's experts with no exemption at all.
  * selection, checked for EVERY (token, expert) pair of the batch: the kept sets match exactly,
    except neurons whose oracle score lies within 1e-6 |cut| of the cut (the K-th largest score,
    or t).  Mismatches beyond that band but inside the fp32 bound of the GPU's gate are the
    separate kind above.  Feeding the GPU's own fp32 activations to the oracle's selection must
    give the GPU's sets with no exemption.  In top-K mode every pair keeps exactly K neurons.
  * output, on every token or on the sampled ``tokens``:
    |gpu - ref| <= tol * max(|ref|, rms(ref)) elementwise, an rms-floored relative error (a pure
    relative error is undefined where an output element is near zero); tol 2e-2 for bf16 layers,
    1e-5 for fp32 ones.  Pairs with an exempted selection are re-run in the oracle with the GPU's
    set first.
The fp32 bound of a dot product of length H with exact products is H * 2^-24 * sum|w||x|
(recursive-summation worst case), widened by 1.1 for SiLU's slope and 4 ulp for its evaluation.
"""
import numpy as np
import torch

import oracle
import synth
from tests.helpers import f32

U32 = 2.0 ** -24
BAND = 1e-6  # the allowed relative band around a cut

# every comparison of the session, for the terminal summary (tests/conftest.py)
RECORDS = []


def tolerance(shape):
    return 2e-2 if shape.dtype == "bf16" else 1e-5


def host_inputs(shape, experts):
    return {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
                synth.host_tensor(shape, "down", e)) for e in experts}


def host_shared(shape):
    return [(synth.host_tensor(shape, "sh_gate", s), synth.host_tensor(shape, "sh_up", s),
             synth.host_tensor(shape, "sh_down", s)) for s in range(shape.n_shared)]


class Report:
    """What one comparison checked and which exemptions it took, by kind."""

    def __init__(self, name=""):
        self.name = name
        self.tokens_routed = 0        # tokens whose routing was checked
        self.pairs = 0                # (token, expert) pairs whose kept set was checked
        self.tokens_output = 0        # tokens whose output was checked
        self.route_band = 0           # experts exempted inside the 1e-6 band
        self.route_fp32_only = []     # (token, expert, gap, bound) outside the band
        self.sel_band_pairs = 0       # pairs with neurons exempted inside the 1e-6 band
        self.sel_band_neurons = 0
        self.sel_fp32_only = []       # (token, pair, neuron, gap, bound) outside the band
        self.max_err = 0.0

    @property
    def fp32_only(self):
        return len(self.route_fp32_only) + len(self.sel_fp32_only)

    def __str__(self):
        s = (f"tokens_routed={self.tokens_routed} pairs={self.pairs} "
             f"tokens_output={self.tokens_output} route_within_1e-6={self.route_band} "
             f"route_fp32_bound_only={len(self.route_fp32_only)} "
             f"sel_within_1e-6_pairs={self.sel_band_pairs} "
             f"sel_within_1e-6_neurons={self.sel_band_neurons} "
             f"sel_fp32_bound_only={len(self.sel_fp32_only)} max_scaled_err={self.max_err:.3e}")
        for t, e, gap, b in self.route_fp32_only:
            s += f"\n  routing token {t} expert {e}: gap {gap:.3e} inside fp32 bound {b:.3e}"
        for t, j, n, gap, b in self.sel_fp32_only:
            s += (f"\n  selection token {t} pair {j} neuron {n}: gap {gap:.3e} inside fp32 "
                  f"bound {b:.3e}")
        return s


def _mask_from_list(cnt, lst, I):
    m = np.zeros(I, np.uint8)
    if cnt:
        m[lst[:cnt]] = 1
    return m


def _classify(gap, cut, bound):
    """'band' (inside 1e-6 |cut|), 'fp32' (outside it, inside the fp32 bound) or None."""
    if gap <= BAND * abs(cut):
        return "band"
    if gap <= bound:
        return "fp32"
    return None


def compare(dl, x_host, x_dev, rule_r, rule_s=None, tokens=None, shared_weights=None,
            expert_cache=None, router_host=None, allow_fp32_bound=0, name=None,
            router_bias=None):
    """Runs the layer on x_dev and checks it against the oracle on x_host (same values).
    Routing and selection are checked for every token; ``tokens`` restricts only the output
    comparison to a subset of tokens (sampled check).  ``allow_fp32_bound`` is the number of
    fp32-bound-only exemptions this comparison may take (0: any fails it).  ``router_bias``
    ([B][E], the oracle's roster bias of this call, exact in fp32) makes the oracle choose the
    top-k of logits + bias, as the layer does under roster routing.  The report's ``idx`` is the
    routing the comparison adopted (the layer's)."""
    shape = dl.shape
    B = x_host.shape[0]
    k, S, I, Ish, H = shape.top_k, shape.n_shared, shape.inter, shape.inter_shared, shape.hidden
    P = k + S
    out = dl.forward(x_dev, rule_r, rule_s)
    if out.is_cuda:
        torch.cuda.synchronize()
    out_gpu = out.float().cpu().numpy().astype(np.float64)
    dbg = dl.debug(B)
    rep = Report(name or f"{shape.name} B={B} {rule_r} {rule_s}")
    router = synth.host_tensor(shape, "router") if router_host is None else router_host
    xf = f32(x_host).astype(np.float64)
    wr = f32(router).astype(np.float64)
    cache = expert_cache if expert_cache is not None else {}
    shared = shared_weights if shared_weights is not None else host_shared(shape)

    # ---- routing, every token
    rl = oracle.Layer(shape, router, {}, [])
    logits_o, idx_o, _ = rl.route_biased(x_host, router_bias)
    bias32 = None if router_bias is None else np.asarray(router_bias, np.float32)
    idx_use = idx_o.copy()
    for t in range(B):
        rep.tokens_routed += 1
        g_idx = dbg["idx"][t]
        # second check: the oracle's top-k on the GPU's own logits (plus the bias, added in fp32
        # as the layer adds it)
        g_sel = dbg["logits"][t].astype(np.float32)
        if bias32 is not None:
            g_sel = g_sel + bias32[t]
        assert np.array_equal(oracle.topk(g_sel.astype(np.float64), k), g_idx), \
            f"top-k logic differs on token {t}"
        idx_use[t] = g_idx
        if np.array_equal(np.sort(g_idx), np.sort(idx_o[t])):
            continue
        lo = logits_o[t] + (0.0 if router_bias is None else np.asarray(router_bias)[t])
        order = np.lexsort((np.arange(shape.n_routed), -lo))
        cut = lo[order[k - 1]]
        # the fp32 logits, then the fp32 addition of the bias (one more rounding)
        bound = H * U32 * (np.abs(wr) @ np.abs(xf[t])) + U32 * np.abs(lo)
        for e in set(g_idx.tolist()) ^ set(idx_o[t].tolist()):
            gap = abs(lo[e] - cut)
            b = bound[e] + bound[order[k - 1]]
            kind = _classify(gap, cut, b)
            assert kind is not None, \
                f"token {t}: expert {e} differs, logit gap {gap:.3e} > fp32 bound {b:.3e}"
            if kind == "band":
                rep.route_band += 1
            else:
                rep.route_fp32_only.append((t, int(e), gap, b))
    for t in range(B):
        w_o = rl.route_weights(logits_o[t], dbg["idx"][t])
        assert np.max(np.abs(w_o - dbg["w"][t])) <= (1e-5 if shape.dtype == "f32" else 2e-4) * max(
            1.0, np.max(np.abs(w_o))), f"routing weights differ on token {t}"

    # ---- selection, every pair: the oracle's gate of each expert over that expert's tokens
    imax = max(I, Ish if S else 0)
    keep_in = np.zeros((B, P, imax), np.uint8)
    flag = np.zeros((B, P), np.uint8)
    jobs = {}  # ("r", e) or ("s", j) -> [(token, pair)]
    for t in range(B):
        for j in range(k):
            jobs.setdefault(("r", int(idx_use[t][j])), []).append((t, j))
        for j in range(S):
            jobs.setdefault(("s", j), []).append((t, k + j))
    for (kind, e), pairs in sorted(jobs.items()):
        if kind == "r":
            wg = cache[e][0] if e in cache else synth.host_tensor(shape, "gate", e)
            In, rule = I, rule_r
        else:
            wg = shared[e][0]
            In, rule = Ish, rule_s
        toks = np.array([t for t, _ in pairs])
        a_o = oracle.gate_tokens(x_host[toks], wg)
        wgd = None
        for (t, j), a_row in zip(pairs, a_o):
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
            sig = np.abs(a_row)
            om = oracle.select(sig, rule)
            if np.array_equal(gm, om):
                continue
            if rule[0] == "topk":
                K = oracle.keep_count(In, rule[1])
                cut = np.sort(sig)[::-1][K - 1]
            else:
                cut = float(np.float32(rule[1]))
            if wgd is None:
                wgd = np.abs(f32(wg).astype(np.float64))
            gb = H * U32 * (wgd @ np.abs(xf[t]))
            bound = 1.1 * gb + 4 * 2.0 ** -23 * sig
            near = bound[np.argmin(np.abs(sig - cut))]
            bad = np.flatnonzero(gm != om)
            band = True
            for n in bad:
                gap = abs(sig[n] - cut)
                kind_n = _classify(gap, cut, bound[n] + near)
                assert kind_n is not None, (
                    f"token {t} pair {j} neuron {n}: score {sig[n]:.9g} vs cut {cut:.9g} "
                    f"(gap {gap:.3e} > fp32 bound {bound[n] + near:.3e})")
                if kind_n == "fp32":
                    band = False
                    rep.sel_fp32_only.append((t, j, int(n), gap, bound[n] + near))
            if band:
                rep.sel_band_pairs += 1
                rep.sel_band_neurons += len(bad)
            keep_in[t][j][:In] = gm
            flag[t][j] = 1

    # ---- output, every token or the sampled ones; the oracle layer with the experts it needs
    sel_tokens = np.arange(B) if tokens is None else np.asarray(tokens)
    need = sorted(set(int(e) for e in idx_use[sel_tokens].ravel()))
    missing = [e for e in need if e not in cache]
    cache.update(host_inputs(shape, missing))
    layer = oracle.Layer(shape, router, {e: cache[e] for e in need}, shared)
    fl = flag[sel_tokens]
    ref = layer.forward(x_host[sel_tokens], rule_r, rule_s, idx_in=idx_use[sel_tokens],
                        keep_in=keep_in[sel_tokens] if fl.any() else None,
                        keep_flag=fl if fl.any() else None)
    rep.tokens_output = len(sel_tokens)
    r = ref["out"]
    g = out_gpu[sel_tokens]
    scale = np.maximum(np.abs(r), np.sqrt(np.mean(r * r)) if r.size else 1.0)
    err = np.abs(g - r) / np.maximum(scale, 1e-30)
    rep.max_err = float(err.max()) if err.size else 0.0
    rep.idx = idx_use
    RECORDS.append(rep)
    tol = tolerance(shape)
    assert rep.max_err <= tol, f"output error {rep.max_err:.3e} > {tol} ({rep})"
    assert rep.fp32_only <= allow_fp32_bound, (
        f"{rep.fp32_only} mismatches outside the 1e-6 band (inside the fp32 bound), "
        f"{allow_fp32_bound} allowed: {rep}")
    return rep
