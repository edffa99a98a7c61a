"""Shared test helpers: small synthetic layers drawn with the seeded generator."""
import numpy as np

import oracle
import synth
from synth.configs import LayerShape


def f32(a):
    """Exact float32 values of stored inputs (uint16 bf16 bits or float32)."""
    a = np.asarray(a)
    return synth.bf16_bits_to_f32(a) if a.dtype == np.uint16 else a.astype(np.float32)


def host_layer(shape, experts=None, lib=None):
    """oracle.Layer with the generator's weights for ``experts`` (default: all routed experts)."""
    if experts is None:
        experts = range(shape.n_routed)
    ex = {e: (synth.host_tensor(shape, "gate", e), synth.host_tensor(shape, "up", e),
              synth.host_tensor(shape, "down", e)) for e in experts}
    sh = [(synth.host_tensor(shape, "sh_gate", s), synth.host_tensor(shape, "sh_up", s),
           synth.host_tensor(shape, "sh_down", s)) for s in range(shape.n_shared)]
    return oracle.Layer(shape, synth.host_tensor(shape, "router"), ex, sh, lib=lib)


def small_shape(**kw):
    base = dict(name="small", hidden=48, n_routed=6, top_k=2, inter=40, n_shared=1,
                inter_shared=24, dtype="f32", route="softmax_topk", seed=11)
    base.update(kw)
    return LayerShape(**base)
