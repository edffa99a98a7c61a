"""moe_route_noalloc, the routing-only entry point that allocates nothing, against the routing
step of moe_forward (the existing entry point) through the C ABI.  This file is collected last
so that it also runs after every other test in the same process."""
import pytest
import torch

import synth
import sparse_expert_ffn_logits_b200 as moe
from sparse_expert_ffn_logits_b200 import MoEError, moe_route_noalloc
from sparse_expert_ffn_logits_b200 import build as moe_build
from sparse_expert_ffn_logits_b200.workload import DeviceLayer


def _cfg(shape, **kw):
    d = dict(hidden=shape.hidden, n_routed=shape.n_routed, top_k=shape.top_k, inter=shape.inter,
             n_shared=shape.n_shared, inter_shared=shape.inter_shared, max_tokens=64,
             dtype=shape.dtype, route=shape.route)
    d.update(kw)
    return moe.make_config(**d)


def test_rejects_before_touching_the_device():
    moe_build.build()
    cfg = _cfg(synth.OLMOE)
    moe_route_noalloc(cfg, None, 0, None, None, None, stream=0)  # n_tokens = 0: a no-op
    for n, status in ((257, moe.MOE_ERR_UNSUPPORTED), (-1, moe.MOE_ERR_INVALID_ARG),
                      (4, moe.MOE_ERR_INVALID_ARG)):  # 4 tokens with null pointers
        with pytest.raises(MoEError) as e:
            moe_route_noalloc(cfg, None, n, None, None, None, stream=0)
        assert e.value.status == status
    for bad, status in ((dict(top_k=65), moe.MOE_ERR_INVALID_ARG),
                        (dict(hidden=100), moe.MOE_ERR_UNSUPPORTED),
                        (dict(top_k=17, n_routed=64), moe.MOE_ERR_UNSUPPORTED)):
        with pytest.raises(MoEError) as e:
            moe_route_noalloc(_cfg(synth.OLMOE, **bad), None, 4, None, None, None, stream=0)
        assert e.value.status == status


# 512 experts x 100 tokens of logits exceed the single-cluster router's shared memory, so this
# shape takes the multi-CTA router, whose tickets start at zero on every call
WIDE = synth.configs.LayerShape("wide-router", 256, 512, 8, 64)


@pytest.mark.gpu
@pytest.mark.parametrize("shape,sizes", [(synth.OLMOE, (16, 64)), (synth.TINY, (16, 64)),
                                         (WIDE, (100, 96))], ids=lambda v: getattr(v, "name", ""))
def test_matches_forward_routing_on_two_calls_in_a_row(shape, sizes):
    dl = DeviceLayer(shape, max_tokens=max(sizes))
    try:
        cfg = _cfg(shape, max_tokens=max(sizes))
        batches = [(B, dl.tokens(B, synth.token_seed(shape, 3 + i))) for i, B in enumerate(sizes)]
        want = []
        for B, x in batches:
            out = torch.empty_like(x)
            dl.forward(x, ("topk", 0.5), ("topk", 0.5), out=out)
            d = dl.debug(B)
            want.append((d["idx"], d["w"]))
        # two calls in a row on the same stream, then one synchronisation
        got = []
        for B, x in batches:
            idx = torch.full((B, shape.top_k), -1, dtype=torch.int32, device=x.device)
            w = torch.full((B, shape.top_k), float("nan"), dtype=torch.float32, device=x.device)
            moe_route_noalloc(cfg, x, B, dl.router, idx, w)
            got.append((idx, w))
        torch.cuda.synchronize()
        for (wi, ww), (gi, gw) in zip(want, got):
            assert (gi.cpu().numpy() == wi).all()
            # the same kernel on the same inputs: the weights agree to fp32 rounding
            torch.testing.assert_close(gw.cpu(), torch.from_numpy(ww), rtol=1e-6, atol=0.0)
    finally:
        dl.close()
