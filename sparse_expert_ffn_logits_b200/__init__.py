"""Python binding of libsparse_moe.so, the sparse-expert MoE FFN decode layer for B200.

Argument marshalling only: every step of the layer runs in the library's sm_100a kernels.
The entry points keep the C names of ``include/moe.h``; buffers may be passed as torch tensors
(their ``data_ptr()`` is used) or as raw addresses, streams as ``torch.cuda.Stream`` or raw
``cudaStream_t`` values (None = the current torch stream).  A non-OK status raises
``MoEError``.  There is no fallback: if the library is missing, importing the entry points
fails.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_moe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_OOM = 0, 1, 2, 3
MOE_ERR_CUDA, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT = 4, 5, 6
MOE_BF16, MOE_F32 = 0, 1
MOE_ROUTE_SOFTMAX_TOPK, MOE_ROUTE_SOFTMAX_ALL, MOE_ROUTE_SIGMOID = 0, 1, 2
MOE_SEL_TOPK, MOE_SEL_THRESHOLD = 0, 1

ROUTE = {"softmax_topk": MOE_ROUTE_SOFTMAX_TOPK, "softmax_all": MOE_ROUTE_SOFTMAX_ALL,
         "sigmoid": MOE_ROUTE_SIGMOID}
DTYPE = {"bf16": MOE_BF16, "f32": MOE_F32}


class MoEError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {_lib().moe_status_string(status).decode()} ({status})")


class MoEConfig(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_routed", ctypes.c_int), ("top_k", ctypes.c_int),
                ("inter", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("inter_shared", ctypes.c_int), ("max_tokens", ctypes.c_int),
                ("dtype", ctypes.c_int), ("route", ctypes.c_int)]


class MoESparsity(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("sparsity", ctypes.c_double),
                ("threshold", ctypes.c_float)]


class MoERoster(ctypes.Structure):
    _fields_ = [("counts", ctypes.c_void_p), ("pinned", ctypes.c_void_p), ("m", ctypes.c_int),
                ("delta", ctypes.c_float)]


class MoEExpertWeights(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("updown", ctypes.c_void_p)]


_LIB = None

# C entry points declared in include/moe.h
EXPORTS = ("moe_create", "moe_packed_bytes", "moe_pack_experts", "moe_forward",
           "moe_forward_roster",
           "moe_forward_host", "moe_debug_lists", "moe_profile_stages", "moe_read_trace",
           "moe_get_error", "moe_debug_force_timeout", "moe_set_dense_min_tokens", "moe_set_fused",
           "moe_last_launches", "moe_set_expert_range", "moe_forward_partial",
           "moe_cast_output", "moe_destroy",
           "moe_route_noalloc",
           "moe_status_string")
MOE_STAGE_EVENTS = 6
STAGES = ("router", "gate", "select", "updown", "finalize")


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built: run sparse_expert_ffn_logits_b200.build"
                              ".build() (nvcc, sm_100a); there is no fallback path")
        lib = ctypes.CDLL(LIB_PATH)
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.moe_create.argtypes = [ctypes.POINTER(MoEConfig), ctypes.POINTER(P)]
        lib.moe_packed_bytes.argtypes = [ctypes.POINTER(MoEConfig), I,
                                         ctypes.POINTER(ctypes.c_size_t),
                                         ctypes.POINTER(ctypes.c_size_t)]
        lib.moe_pack_experts.argtypes = [P, I, P, P, P, I, P, P, P]
        fwd = [P, P, I, P, ctypes.POINTER(MoEExpertWeights), ctypes.POINTER(MoEExpertWeights),
               ctypes.POINTER(MoESparsity), ctypes.POINTER(MoESparsity), P, P]
        lib.moe_forward.argtypes = fwd
        lib.moe_forward_host.argtypes = fwd
        lib.moe_forward_roster.argtypes = [P, P, I, P, ctypes.POINTER(MoERoster),
                                           ctypes.POINTER(MoEExpertWeights),
                                           ctypes.POINTER(MoEExpertWeights),
                                           ctypes.POINTER(MoESparsity), ctypes.POINTER(MoESparsity),
                                           P, P]
        lib.moe_debug_lists.argtypes = [P, I, P, P, P, P, P, P, P]
        lib.moe_profile_stages.argtypes = [P, ctypes.POINTER(P), I]
        lib.moe_read_trace.argtypes = [P, P, ctypes.c_size_t]
        lib.moe_get_error.argtypes = [P, ctypes.POINTER(I)]
        lib.moe_destroy.argtypes = [P]
        lib.moe_set_dense_min_tokens.argtypes = [P, I]
        lib.moe_set_fused.argtypes = [P, I]
        lib.moe_last_launches.argtypes = [P, ctypes.POINTER(I)]
        lib.moe_set_expert_range.argtypes = [P, I, I, ctypes.c_uint]
        lib.moe_forward_partial.argtypes = fwd
        lib.moe_cast_output.argtypes = [P, P, I, P, P]
        lib.moe_debug_force_timeout.argtypes = [P, P]
        lib.moe_route_noalloc.argtypes = [ctypes.POINTER(MoEConfig), P, I, P, P, P, P]
        lib.moe_status_string.argtypes = [I]
        lib.moe_status_string.restype = ctypes.c_char_p
        for f in EXPORTS[:-1]:
            getattr(lib, f).restype = I
        _LIB = lib
    return _LIB


def load():
    """Loads the library (raises if it is not built)."""
    return _lib()


def _ptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return ctypes.c_void_p(a)
    return ctypes.c_void_p(a.data_ptr())


def _stream(s):
    if s is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return ctypes.c_void_p(s)
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc, what):
    if rc != MOE_OK:
        raise MoEError(rc, what)


def make_config(hidden, n_routed, top_k, inter, n_shared=0, inter_shared=0, max_tokens=256,
                dtype="bf16", route="softmax_topk"):
    return MoEConfig(hidden, n_routed, top_k, inter, n_shared, inter_shared, max_tokens,
                     DTYPE[dtype] if isinstance(dtype, str) else dtype,
                     ROUTE[route] if isinstance(route, str) else route)


def sparsity(rule):
    """MoESparsity from ("topk", s) or ("threshold", t)."""
    kind, v = rule
    if kind == "topk":
        return MoESparsity(MOE_SEL_TOPK, float(v), 0.0)
    if kind == "threshold":
        return MoESparsity(MOE_SEL_THRESHOLD, 0.0, float(v))
    raise ValueError(rule)


def moe_create(cfg):
    h = ctypes.c_void_p()
    _check(_lib().moe_create(ctypes.byref(cfg), ctypes.byref(h)), "moe_create")
    return h.value


def moe_packed_bytes(cfg, shared=0):
    g, u = ctypes.c_size_t(), ctypes.c_size_t()
    _check(_lib().moe_packed_bytes(ctypes.byref(cfg), int(shared), ctypes.byref(g),
                                   ctypes.byref(u)), "moe_packed_bytes")
    return g.value, u.value


def moe_pack_experts(h, shared, w_gate, w_up, w_down, n, packed_gate, packed_updown, stream=None):
    _check(_lib().moe_pack_experts(ctypes.c_void_p(h), int(shared), _ptr(w_gate), _ptr(w_up),
                                   _ptr(w_down), int(n), _ptr(packed_gate), _ptr(packed_updown),
                                   _stream(stream)), "moe_pack_experts")


def expert_weights(gate, updown):
    return MoEExpertWeights(_ptr(gate), _ptr(updown))


def moe_forward(h, x, n_tokens, router, routed, shared, sp_routed, sp_shared, out, stream=None):
    _check(_lib().moe_forward(ctypes.c_void_p(h), _ptr(x), int(n_tokens), _ptr(router),
                              ctypes.byref(routed), ctypes.byref(shared) if shared else None,
                              ctypes.byref(sp_routed), ctypes.byref(sp_shared) if sp_shared else None,
                              _ptr(out), _stream(stream)), "moe_forward")


def roster(counts, pinned, m, delta):
    """MoERoster over device int32 tensors counts [B][E] and pinned [B]."""
    return MoERoster(_ptr(counts), _ptr(pinned), int(m), float(delta))


def moe_forward_roster(h, x, n_tokens, router, roster_state, routed, shared, sp_routed,
                       sp_shared, out, stream=None):
    _check(_lib().moe_forward_roster(ctypes.c_void_p(h), _ptr(x), int(n_tokens), _ptr(router),
                                     ctypes.byref(roster_state), ctypes.byref(routed),
                                     ctypes.byref(shared) if shared else None,
                                     ctypes.byref(sp_routed),
                                     ctypes.byref(sp_shared) if sp_shared else None, _ptr(out),
                                     _stream(stream)), "moe_forward_roster")


def moe_forward_host(h, x_host, n_tokens, router, routed, shared, sp_routed, sp_shared, out_host,
                     stream=None):
    _check(_lib().moe_forward_host(ctypes.c_void_p(h), _ptr(x_host), int(n_tokens), _ptr(router),
                                   ctypes.byref(routed), ctypes.byref(shared) if shared else None,
                                   ctypes.byref(sp_routed),
                                   ctypes.byref(sp_shared) if sp_shared else None,
                                   _ptr(out_host), _stream(stream)), "moe_forward_host")


def moe_debug_lists(h, n_tokens, idx=None, w=None, logits=None, cnt=None, lists=None, act=None,
                    stream=None):
    _check(_lib().moe_debug_lists(ctypes.c_void_p(h), int(n_tokens), _ptr(idx), _ptr(w),
                                  _ptr(logits), _ptr(cnt), _ptr(lists), _ptr(act),
                                  _stream(stream)), "moe_debug_lists")


def moe_profile_stages(h, events):
    """events: MOE_STAGE_EVENTS torch.cuda.Event objects (timing on) or None (timing off)."""
    if events is None:
        _check(_lib().moe_profile_stages(ctypes.c_void_p(h), None, 0), "moe_profile_stages")
        return
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    _check(_lib().moe_profile_stages(ctypes.c_void_p(h), arr, len(events)),
           "moe_profile_stages")


def moe_read_trace(h):
    """Phase timestamps as a numpy array [5 kernels][1024 CTAs][8 points] (ns, 0 = not reached)."""
    import numpy as np
    buf = np.zeros(5 * 1024 * 8, dtype=np.uint64)
    _check(_lib().moe_read_trace(ctypes.c_void_p(h), ctypes.c_void_p(buf.ctypes.data), buf.size),
           "moe_read_trace")
    return buf.reshape(5, 1024, 8)


def moe_get_error(h):
    """(status, device_code); status is MOE_OK, MOE_ERR_DEVICE or MOE_ERR_TIMEOUT (does not
    raise for those)."""
    code = ctypes.c_int(0)
    rc = _lib().moe_get_error(ctypes.c_void_p(h), ctypes.byref(code))
    if rc not in (MOE_OK, MOE_ERR_DEVICE, MOE_ERR_TIMEOUT):
        raise MoEError(rc, "moe_get_error")
    return rc, code.value


MOE_DENSE_AUTO = -1


def moe_debug_force_timeout(h, stream=None):
    """Test hook: a bounded wait that runs out (see include/moe.h)."""
    _check(_lib().moe_debug_force_timeout(ctypes.c_void_p(h) if h else None, _stream(stream)),
           "moe_debug_force_timeout")


def moe_set_dense_min_tokens(h, min_tokens):
    """Path choice: MOE_DENSE_AUTO (per call, the default), 0 (never dense) or a per-expert
    token threshold (see include/moe.h)."""
    _check(_lib().moe_set_dense_min_tokens(ctypes.c_void_p(h) if h else None, int(min_tokens)),
           "moe_set_dense_min_tokens")


def moe_set_fused(h, enable):
    """1: gate, selection and up/down as one fused kernel where it applies; 0 (the default): the
    chain of separate kernels (see include/moe.h)."""
    _check(_lib().moe_set_fused(ctypes.c_void_p(h) if h else None, int(enable)), "moe_set_fused")


def moe_last_launches(h):
    """Kernels launched by the handle's last moe_forward (see include/moe.h)."""
    n = ctypes.c_int(0)
    _check(_lib().moe_last_launches(ctypes.c_void_p(h) if h else None, ctypes.byref(n)),
           "moe_last_launches")
    return n.value


def moe_set_expert_range(h, e_begin, e_end, shared_mask):
    """Restricts the handle to routed experts [e_begin, e_end) and the masked shared experts."""
    _check(_lib().moe_set_expert_range(ctypes.c_void_p(h) if h else None, int(e_begin),
                                       int(e_end), int(shared_mask)), "moe_set_expert_range")


def moe_forward_partial(h, x, n_tokens, router, routed, shared, sp_routed, sp_shared, partial,
                        stream=None):
    _check(_lib().moe_forward_partial(ctypes.c_void_p(h), _ptr(x), int(n_tokens), _ptr(router),
                                      ctypes.byref(routed),
                                      ctypes.byref(shared) if shared else None,
                                      ctypes.byref(sp_routed),
                                      ctypes.byref(sp_shared) if sp_shared else None,
                                      _ptr(partial), _stream(stream)), "moe_forward_partial")


def moe_cast_output(h, partial_sum, n_tokens, out, stream=None):
    _check(_lib().moe_cast_output(ctypes.c_void_p(h), _ptr(partial_sum), int(n_tokens), _ptr(out),
                                  _stream(stream)), "moe_cast_output")


def moe_destroy(h):
    _check(_lib().moe_destroy(ctypes.c_void_p(h) if h else None), "moe_destroy")


def moe_route_noalloc(cfg, x, n_tokens, router, topk_idx, topk_w, stream=None):
    """Routing only, with no handle and no device allocation (see include/moe.h)."""
    _check(_lib().moe_route_noalloc(ctypes.byref(cfg), _ptr(x), int(n_tokens), _ptr(router),
                                    _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
           "moe_route_noalloc")
