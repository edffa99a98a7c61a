"""Seeded synthetic inputs for the sparse-expert MoE layer.

One counter-based generator (SplitMix64 + Box-Muller, defined in ``synth.h``) serves both
the CPU oracle and the CUDA library, with a host fill (``libsynth_host.so``) and a device
fill (``libsynth_cuda.so``) that produce identical bits.  Element ``i`` of a tensor depends
only on ``(seed, tensor_id, i)``, so any expert's weights can be generated on their own.

This module holds none of the layer's arithmetic: it only draws N(0, std) values, rounds
them to the workload's dtype and lays them out in the logical shapes

  x        [B][H]                       router  [E][H]
  gate     [E][I][H]   up [E][I][H]     down    [E][H][I]
  sh_gate  [S][Ish][H] sh_up [S][Ish][H] sh_down [S][H][Ish]
"""
import ctypes
import os

import numpy as np

from . import build as _build
from .configs import (DSV2L, GPTOSS, LLAMA4, OLMOE, SHAPES, TINY, LayerShape,  # noqa: F401
                      calib_seed, token_seed)

BF16, F32 = 0, 1

# tensor ids of the logical tensors (the seed is the workload seed, or a token seed for x)
TID = {"x": 1, "router": 2, "gate": 3, "up": 4, "down": 5,
       "sh_gate": 6, "sh_up": 7, "sh_down": 8}

_host = None
_cuda = None


def _host_lib():
    global _host
    if _host is None:
        path = _build.build_host()
        lib = ctypes.CDLL(path)
        lib.synth_fill_host.restype = ctypes.c_int
        lib.synth_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_int]
        lib.synth_host_threads.restype = ctypes.c_int
        _host = lib
    return _host


def _cuda_lib():
    global _cuda
    if _cuda is None:
        path = _build.CUDA_SO
        if not os.path.exists(path):
            path = _build.build_cuda()
        lib = ctypes.CDLL(path)
        lib.synth_fill_cuda.restype = ctypes.c_int
        lib.synth_fill_cuda.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                        ctypes.c_uint64, ctypes.c_uint64, ctypes.c_double,
                                        ctypes.c_int, ctypes.c_void_p]
        _cuda = lib
    return _cuda


def host_threads():
    return int(_host_lib().synth_host_threads())


def fill_host(n, seed, tensor_id, offset, std, dtype, nthreads=0):
    """Elements offset..offset+n-1 of (seed, tensor_id) as a numpy array:
    uint16 bf16 bit patterns for ``BF16``, float32 for ``F32``."""
    out = np.empty(int(n), dtype=np.uint16 if dtype == BF16 else np.float32)
    rc = _host_lib().synth_fill_host(out.ctypes.data, int(n), int(seed), int(tensor_id),
                                     int(offset), float(std), int(dtype), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"synth_fill_host failed ({rc})")
    return out


def fill_cuda(dst, seed, tensor_id, offset, std, stream=None):
    """Fills the contiguous CUDA tensor ``dst`` (torch.bfloat16 or torch.float32) with elements
    offset..offset+dst.numel()-1 of (seed, tensor_id)."""
    import torch
    if not dst.is_cuda or not dst.is_contiguous():
        raise ValueError("dst must be a contiguous CUDA tensor")
    if dst.dtype == torch.bfloat16:
        dt = BF16
    elif dst.dtype == torch.float32:
        dt = F32
    else:
        raise ValueError("dst must be bfloat16 or float32")
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = _cuda_lib().synth_fill_cuda(ctypes.c_void_p(dst.data_ptr()), dst.numel(), int(seed),
                                     int(tensor_id), int(offset), float(std), dt,
                                     ctypes.c_void_p(s.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"synth_fill_cuda failed ({rc})")
    return dst


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------------------------
# Tensor specifications of a workload
# ---------------------------------------------------------------------------------------------

def spec(shape: LayerShape, which: str, expert=None):
    """(seed, tensor_id, offset, count, std, logical_shape) of one tensor, or of one expert's
    slice of an expert tensor."""
    H, E, I = shape.hidden, shape.n_routed, shape.inter
    S, Ish = shape.n_shared, shape.inter_shared
    seed = shape.seed
    if which == "router":
        return seed, TID[which], 0, E * H, 0.02, (E, H)
    per = {"gate": (I * H, H ** -0.5, (I, H), E),
           "up": (I * H, H ** -0.5, (I, H), E),
           "down": (H * I, I ** -0.5 if I else 0.0, (H, I), E),
           "sh_gate": (Ish * H, H ** -0.5, (Ish, H), S),
           "sh_up": (Ish * H, H ** -0.5, (Ish, H), S),
           "sh_down": (H * Ish, Ish ** -0.5 if Ish else 0.0, (H, Ish), S)}
    if which not in per:
        raise KeyError(which)
    cnt, std, lshape, nexp = per[which]
    if expert is None:
        return seed, TID[which], 0, cnt * nexp, std, (nexp,) + lshape
    if not 0 <= expert < nexp:
        raise IndexError(f"expert {expert} out of range for {which}")
    return seed, TID[which], cnt * expert, cnt, std, lshape


def _dtype(shape):
    return BF16 if shape.dtype == "bf16" else F32


def host_tensor(shape: LayerShape, which: str, expert=None, nthreads=0):
    seed, tid, off, cnt, std, lshape = spec(shape, which, expert)
    return fill_host(cnt, seed, tid, off, std, _dtype(shape), nthreads).reshape(lshape)


def host_tokens(shape: LayerShape, n_tokens: int, seed: int, nthreads=0):
    """x [n_tokens][H] drawn from the token stream ``seed`` (std 1)."""
    return fill_host(n_tokens * shape.hidden, seed, TID["x"], 0, 1.0, _dtype(shape),
                     nthreads).reshape(n_tokens, shape.hidden)


def torch_dtype(shape):
    import torch
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def device_tensor(shape: LayerShape, which: str, expert=None, device="cuda", out=None):
    import torch
    seed, tid, off, cnt, std, lshape = spec(shape, which, expert)
    if out is None:
        out = torch.empty(lshape, dtype=torch_dtype(shape), device=device)
    return fill_cuda(out, seed, tid, off, std)


def device_tokens(shape: LayerShape, n_tokens: int, seed: int, device="cuda", out=None):
    import torch
    if out is None:
        out = torch.empty((n_tokens, shape.hidden), dtype=torch_dtype(shape), device=device)
    return fill_cuda(out, seed, TID["x"], 0, 1.0)
