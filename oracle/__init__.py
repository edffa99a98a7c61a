"""fp64 CPU oracle of the intra-expert activation-sparse MoE FFN layer.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg are
the only callers.  The oracle shares no code with the CUDA library (see ``oracle.cpp`` for the
definition it implements and the readings it takes).  This module only marshals numpy arrays
into the C entry points.

Inputs are numpy arrays exactly as stored for the device: uint16 bf16 bit patterns or float32.
A selection rule is ``("topk", s)`` (keep K = I - floor(s I + 1e-9) neurons) or
``("threshold", t)`` (keep |SiLU(g)| > t).
"""
import ctypes
import os

import numpy as np

from . import build as _build

ROUTE = {"softmax_topk": 0, "softmax_all": 1, "sigmoid": 2}


class _Layer(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_routed", ctypes.c_int), ("top_k", ctypes.c_int),
                ("inter", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("inter_shared", ctypes.c_int), ("route", ctypes.c_int), ("elt", ctypes.c_int),
                ("router", ctypes.c_void_p),
                ("gate", ctypes.POINTER(ctypes.c_void_p)), ("up", ctypes.POINTER(ctypes.c_void_p)),
                ("down", ctypes.POINTER(ctypes.c_void_p)),
                ("sh_gate", ctypes.POINTER(ctypes.c_void_p)),
                ("sh_up", ctypes.POINTER(ctypes.c_void_p)),
                ("sh_down", ctypes.POINTER(ctypes.c_void_p))]


class _Sel(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("sparsity", ctypes.c_double),
                ("threshold", ctypes.c_double)]


_lib = None


def load(path=None):
    """Loads (building if needed) the oracle library; ``path`` selects another build of it."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(lib):
    P = ctypes.c_void_p
    lib.oracle_keep_count.restype = ctypes.c_int
    lib.oracle_keep_count.argtypes = [ctypes.c_int, ctypes.c_double]
    lib.oracle_threads.restype = ctypes.c_int
    lib.oracle_route.argtypes = [ctypes.POINTER(_Layer), P, ctypes.c_int, P, P, P]
    lib.oracle_route_weights.argtypes = [ctypes.POINTER(_Layer), P, P, P]
    lib.oracle_route_biased.argtypes = [ctypes.POINTER(_Layer), P, ctypes.c_int, P, P, P, P]
    lib.oracle_roster_bias.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_double, P]
    lib.oracle_roster_update.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.oracle_topk.argtypes = [P, ctypes.c_int, ctypes.c_int, P]
    lib.oracle_gate.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
    lib.oracle_gate_tokens.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, P, ctypes.c_int]
    lib.oracle_select.argtypes = [P, ctypes.c_int, _Sel, P]
    lib.oracle_expert.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.oracle_forward.argtypes = [ctypes.POINTER(_Layer), P, ctypes.c_int, _Sel, _Sel, P, P, P,
                                   P, P, P, P, P, P, ctypes.c_int]
    lib.oracle_calibrate.argtypes = [ctypes.POINTER(_Layer), P, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_double, P, P, ctypes.c_int]
    for f in ("oracle_route", "oracle_route_biased", "oracle_roster_bias", "oracle_roster_update",
              "oracle_route_weights", "oracle_topk", "oracle_gate",
              "oracle_gate_tokens", "oracle_select",
              "oracle_expert", "oracle_forward", "oracle_calibrate"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _sel(rule):
    if rule is None:
        return _Sel(0, 0.0, 0.0)
    kind, v = rule
    if kind == "topk":
        return _Sel(0, float(v), 0.0)
    if kind == "threshold":
        return _Sel(1, 0.0, float(v))
    raise ValueError(rule)


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with status {rc}")


def _elt(a):
    if a.dtype == np.uint16:
        return 2
    if a.dtype == np.float32:
        return 4
    raise TypeError("inputs must be uint16 (bf16 bits) or float32")


class Layer:
    """Weights of one layer for the oracle.

    ``router`` [E][H]; ``experts`` maps a routed expert index to (gate [I][H], up [I][H],
    down [H][I]); ``shared`` is a list of (gate, up, down) per shared expert.  Experts that no
    token routes to may be left out.
    """

    def __init__(self, shape, router, experts, shared=(), lib=None):
        self.shape = shape
        self.lib = lib or load()
        self._keep = [np.ascontiguousarray(router)]
        self.elt = _elt(router)
        E, S = shape.n_routed, shape.n_shared
        arr = ctypes.c_void_p * max(E, 1)
        sarr = ctypes.c_void_p * max(S, 1)
        self._g, self._u, self._d = arr(), arr(), arr()
        self._sg, self._su, self._sd = sarr(), sarr(), sarr()
        for e, (g, u, d) in experts.items():
            # up/down may be None when only the gate is needed (threshold calibration)
            g, u, d = (None if v is None else np.ascontiguousarray(v) for v in (g, u, d))
            assert g.shape == (shape.inter, shape.hidden)
            assert d is None or d.shape == (shape.hidden, shape.inter)
            self._keep += [v for v in (g, u, d) if v is not None]
            self._g[e] = g.ctypes.data
            self._u[e] = None if u is None else u.ctypes.data
            self._d[e] = None if d is None else d.ctypes.data
        for s, (g, u, d) in enumerate(shared):
            g, u, d = (np.ascontiguousarray(v) for v in (g, u, d))
            self._keep += [g, u, d]
            self._sg[s], self._su[s], self._sd[s] = g.ctypes.data, u.ctypes.data, d.ctypes.data
        self.c = _Layer(shape.hidden, E, shape.top_k, shape.inter, S, shape.inter_shared,
                        ROUTE[shape.route], self.elt, self._keep[0].ctypes.data,
                        ctypes.cast(self._g, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._u, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._d, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._sg, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._su, ctypes.POINTER(ctypes.c_void_p)),
                        ctypes.cast(self._sd, ctypes.POINTER(ctypes.c_void_p)))

    @property
    def imax(self):
        s = self.shape
        return max(s.inter, s.inter_shared if s.n_shared else 0)

    def route(self, x):
        x = np.ascontiguousarray(x)
        B, E, k = x.shape[0], self.shape.n_routed, self.shape.top_k
        logits = np.zeros((B, E)); idx = np.zeros((B, k), np.int32); w = np.zeros((B, k))
        _check(self.lib.oracle_route(ctypes.byref(self.c), _ptr(x), B, _ptr(logits), _ptr(idx),
                                     _ptr(w)), "oracle_route")
        return logits, idx, w

    def route_biased(self, x, bias):
        """Routing with an additive selection bias [B][E] (None: no bias): the top-k of
        logits + bias, the weights from the unbiased logits.  Returns (logits, idx, w)."""
        x = np.ascontiguousarray(x)
        B, E, k = x.shape[0], self.shape.n_routed, self.shape.top_k
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
        assert b is None or b.shape == (B, E)
        logits = np.zeros((B, E)); idx = np.zeros((B, k), np.int32); w = np.zeros((B, k))
        _check(self.lib.oracle_route_biased(ctypes.byref(self.c), _ptr(x), B, _ptr(b),
                                            _ptr(logits), _ptr(idx), _ptr(w)),
               "oracle_route_biased")
        return logits, idx, w

    def route_weights(self, logits_row, idx_row):
        lg = np.ascontiguousarray(logits_row, dtype=np.float64)
        ix = np.ascontiguousarray(idx_row, dtype=np.int32)
        w = np.zeros(self.shape.top_k)
        _check(self.lib.oracle_route_weights(ctypes.byref(self.c), _ptr(lg), _ptr(ix), _ptr(w)),
               "oracle_route_weights")
        return w

    def forward(self, x, routed, shared=None, idx_in=None, keep_in=None, keep_flag=None,
                nthreads=0):
        """Returns a dict: out [B][H], idx, w [B][k], keep [B][k+S][Imax] (uint8),
        a [B][k+S][Imax] (SiLU(g)), logits [B][E]."""
        x = np.ascontiguousarray(x)
        s = self.shape
        B, P, Im = x.shape[0], s.top_k + s.n_shared, self.imax
        out = np.zeros((B, s.hidden)); idx = np.zeros((B, s.top_k), np.int32)
        w = np.zeros((B, s.top_k)); keep = np.zeros((B, P, Im), np.uint8)
        a = np.zeros((B, P, Im)); logits = np.zeros((B, s.n_routed))
        if idx_in is not None:
            idx_in = np.ascontiguousarray(idx_in, dtype=np.int32)
        if keep_in is not None:
            keep_in = np.ascontiguousarray(keep_in, dtype=np.uint8)
            keep_flag = np.ascontiguousarray(keep_flag, dtype=np.uint8)
        _check(self.lib.oracle_forward(ctypes.byref(self.c), _ptr(x), B, _sel(routed), _sel(shared),
                                       _ptr(idx_in), _ptr(keep_in), _ptr(keep_flag), _ptr(out),
                                       _ptr(idx), _ptr(w), _ptr(keep), _ptr(a), _ptr(logits),
                                       int(nthreads)), "oracle_forward")
        return {"out": out, "idx": idx, "w": w, "keep": keep, "a": a, "logits": logits}

    def calibrate(self, x, s, shared=False, nthreads=0):
        """(t, N): the fp64 cut whose exceedances are the top N - floor(sN) calibration scores."""
        x = np.ascontiguousarray(x)
        t = ctypes.c_double(0.0); n = ctypes.c_longlong(0)
        _check(self.lib.oracle_calibrate(ctypes.byref(self.c), _ptr(x), x.shape[0], int(shared),
                                         float(s), ctypes.byref(t), ctypes.byref(n), int(nthreads)),
               "oracle_calibrate")
        return t.value, n.value


def keep_count(I, s, lib=None):
    return int((lib or load()).oracle_keep_count(int(I), float(s)))


def threads(lib=None):
    return int((lib or load()).oracle_threads())


def topk(logits_row, k, lib=None):
    """The k experts of one token's logits by (logit desc, index asc)."""
    lib = lib or load()
    lg = np.ascontiguousarray(logits_row, dtype=np.float64)
    idx = np.zeros(k, np.int32)
    _check(lib.oracle_topk(_ptr(lg), lg.shape[0], int(k), _ptr(idx)), "oracle_topk")
    return idx


def gate(x_t, wg, lib=None):
    """(g, a) of one pair: g = W_g x_t, a = SiLU(g)."""
    lib = lib or load()
    x_t = np.ascontiguousarray(x_t); wg = np.ascontiguousarray(wg)
    I, H = wg.shape
    g = np.zeros(I); a = np.zeros(I)
    _check(lib.oracle_gate(_ptr(x_t), _ptr(wg), _elt(wg), H, I, _ptr(g), _ptr(a)), "oracle_gate")
    return g, a


def roster_bias(counts, pinned, m, delta, lib=None):
    """Roster bias [B][E] (float64) from the selection counts [B][E] and pinned flags [B]."""
    lib = lib or load()
    c = np.ascontiguousarray(counts, dtype=np.int32)
    pn = np.ascontiguousarray(pinned, dtype=np.int32)
    B, E = c.shape
    b = np.zeros((B, E))
    _check(lib.oracle_roster_bias(_ptr(c), _ptr(pn), B, E, int(m), float(delta), _ptr(b)),
           "oracle_roster_bias")
    return b


def roster_update(counts, idx, lib=None):
    """counts[t][idx[t][j]] += 1, in place (counts: int32 [B][E], idx [B][k])."""
    lib = lib or load()
    assert counts.dtype == np.int32 and counts.flags.c_contiguous
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    B, E = counts.shape
    _check(lib.oracle_roster_update(_ptr(counts), _ptr(ix), B, E, ix.shape[1]),
           "oracle_roster_update")
    return counts


def gate_tokens(xs, wg, nthreads=0, lib=None):
    """a [T][I] = SiLU(W_g x_t) of one expert for the T tokens xs [T][H] (host threads)."""
    lib = lib or load()
    xs = np.ascontiguousarray(xs); wg = np.ascontiguousarray(wg)
    assert _elt(xs) == _elt(wg)
    I, H = wg.shape
    T = xs.shape[0]
    a = np.zeros((T, I))
    _check(lib.oracle_gate_tokens(_ptr(xs), T, _ptr(wg), _elt(wg), H, I, _ptr(a), int(nthreads)),
           "oracle_gate_tokens")
    return a


def select(score, rule, lib=None):
    """0/1 keep mask (uint8) of the scores under ``rule``."""
    lib = lib or load()
    sc = np.ascontiguousarray(score, dtype=np.float64)
    keep = np.zeros(sc.shape[0], np.uint8)
    _check(lib.oracle_select(_ptr(sc), sc.shape[0], _sel(rule), _ptr(keep)), "oracle_select")
    return keep


def expert(x_t, wu, wd, keep, a, lib=None):
    """y [H] of one pair for the mask ``keep`` and activations ``a``."""
    lib = lib or load()
    x_t = np.ascontiguousarray(x_t); wu = np.ascontiguousarray(wu); wd = np.ascontiguousarray(wd)
    keep = np.ascontiguousarray(keep, dtype=np.uint8); a = np.ascontiguousarray(a, dtype=np.float64)
    I, H = wu.shape
    y = np.zeros(H)
    _check(lib.oracle_expert(_ptr(x_t), _ptr(wu), _ptr(wd), _elt(wu), H, I, _ptr(keep), _ptr(a),
                             _ptr(y)), "oracle_expert")
    return y
