"""The fused layer kernel (gate, selection and up/down in one persistent launch) against the
launch chain of separate kernels and against the fp64 oracle, through the C ABI.

Both paths run the same per-item arithmetic, so routing, activations and kept sets must be
bit-identical; the outputs differ only in how the fp32 up/down partial sums are grouped before
the bf16 cast.  Edge cases of the fused kernel's readiness protocol: one token, ragged token
tiles, every token on one expert (many tiles of one slot), empty unions (s = 1), everything
kept (s = 0), thresholds of +-inf, a restricted expert range, and graph replay."""
import numpy as np
import pytest
import torch

import synth
from sparse_expert_ffn_logits_b200 import moe_set_dense_min_tokens, moe_set_expert_range
from sparse_expert_ffn_logits_b200.workload import DeviceLayer
from tests import parity

pytestmark = pytest.mark.gpu

# small bf16 layer with a shared expert: H = 512 takes the register-fragment variant with one
# stage per row (NK = 1), I = 512 and Ish = 256 give 32 and 16 gate items per token tile
SMALL = synth.TINY.with_(name="small-bf16", hidden=512, dtype="bf16", n_shared=1,
                         inter_shared=256)


def _compare_paths(dl, x, rule_r, rule_s=None, out_tol=1e-2):
    """Runs x through the fused kernel and the chain; returns the fused output."""
    B = x.shape[0]
    dl.set_fused(True)
    out_f = dl.forward(x, rule_r, rule_s)
    n_f = dl.last_launches()
    dbg_f = dl.debug(B)
    dl.set_fused(False)
    out_c = dl.forward(x, rule_r, rule_s)
    n_c = dl.last_launches()
    dbg_c = dl.debug(B)
    dl.set_fused(True)
    assert n_f == 3 and n_c == 5, (n_f, n_c)
    for k in ("idx", "w", "logits", "cnt", "lists", "act"):
        a, b = dbg_f[k], dbg_c[k]
        if k == "lists":  # entries past each pair's count are not part of the result
            a = np.where(np.arange(a.shape[-1]) < dbg_f["cnt"][..., None], a, -1)
            b = np.where(np.arange(b.shape[-1]) < dbg_c["cnt"][..., None], b, -1)
        assert np.array_equal(a, b), f"{dl.shape.name} B={B}: {k} differs between the paths"
    f, c = out_f.float().cpu().numpy(), out_c.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(c.astype(np.float64) ** 2))) + 1e-30
    err = np.abs(f - c) / np.maximum(np.abs(c), rms)
    assert err.max() <= out_tol, f"{dl.shape.name} B={B}: outputs differ by {err.max():.3e}"
    return out_f


@pytest.fixture(scope="module")
def small():
    dl = DeviceLayer(SMALL, max_tokens=96)
    moe_set_dense_min_tokens(dl.h, 0)  # 8 experts: the automatic rule would go dense at B > 24
    yield dl
    dl.close()


def _tokens(dl, B, batch_index):
    seed = synth.token_seed(dl.shape, batch_index)
    return synth.host_tokens(dl.shape, B, seed), dl.tokens(B, seed)


@pytest.mark.parametrize("B", [1, 2, 9, 31, 64, 96])
def test_small_fused_matches_chain_and_oracle(small, B):
    xh, xd = _tokens(small, B, 1)
    _compare_paths(small, xd, ("topk", 0.7), ("topk", 0.5))
    rep = parity.compare(small, xh, xd, ("topk", 0.7), ("topk", 0.5),
                         name=f"fused small B={B}")
    assert small.last_launches() == 3
    print(rep)


@pytest.mark.parametrize("s,s_sh", [(0.0, 0.0), (1.0, 1.0), (1.0, 0.5), (0.5, 1.0),
                                    (0.9, 0.9)])
def test_small_fused_sparsity_extremes(small, s, s_sh):
    xh, xd = _tokens(small, 24, 2)
    _compare_paths(small, xd, ("topk", s), ("topk", s_sh))
    parity.compare(small, xh, xd, ("topk", s), ("topk", s_sh), name=f"fused small s={s}/{s_sh}")


def test_small_fused_thresholds(small):
    xh, xd = _tokens(small, 16, 3)
    for t in (-np.inf, np.inf, 0.05):
        _compare_paths(small, xd, ("threshold", t), ("threshold", t))
        parity.compare(small, xh, xd, ("threshold", t), ("threshold", t),
                       name=f"fused small threshold {t}")


def test_small_fused_one_expert_many_tiles(small):
    # every token is the same, so one routed expert holds all 80 tokens (10 token tiles)
    xh, _ = _tokens(small, 1, 4)
    xh = np.repeat(xh, 80, axis=0)
    xd = torch.from_numpy(xh).cuda().view(torch.bfloat16)  # the host copy holds bf16 bits
    _compare_paths(small, xd, ("topk", 0.5), ("topk", 0.75))
    parity.compare(small, xh, xd, ("topk", 0.5), ("topk", 0.75), name="fused one expert")


def test_small_fused_repeated_calls_and_graph(small):
    # the readiness state is cleared by every call: many calls of changing sizes, then replays
    # of a captured call, all against the chain
    for i, B in enumerate([5, 64, 1, 33, 8, 96, 2]):
        _, xd = _tokens(small, B, 10 + i)
        _compare_paths(small, xd, ("topk", 0.6), ("topk", 0.6))
    _, xd = _tokens(small, 40, 20)
    small.set_fused(False)
    ref = small.forward(xd, ("topk", 0.6), ("topk", 0.6)).clone()
    small.set_fused(True)
    out = torch.empty_like(xd)
    st = torch.cuda.Stream()
    small.forward(xd, ("topk", 0.6), ("topk", 0.6), out=out)  # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        small.forward(xd, ("topk", 0.6), ("topk", 0.6), out=out, stream=st.cuda_stream)
    for _ in range(5):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        f, c = out.float().cpu().numpy(), ref.float().cpu().numpy()
        rms = float(np.sqrt(np.mean(c.astype(np.float64) ** 2)))
        assert (np.abs(f - c) / np.maximum(np.abs(c), rms)).max() <= 1e-2
    del g


def test_small_fused_expert_range(small):
    # a handle restricted to half the routed experts and no shared expert still takes the
    # fused kernel; its partial output equals the chain's
    xh, xd = _tokens(small, 20, 5)
    try:
        moe_set_expert_range(small.h, 2, 6, 0)
        _compare_paths(small, xd, ("topk", 0.5), ("topk", 0.5))
    finally:
        moe_set_expert_range(small.h, 0, SMALL.n_routed, 1)


# --- the workload shapes ---------------------------------------------------------------------
@pytest.mark.parametrize("shape,Bs,rule_r,rule_s", [
    (synth.OLMOE, [1, 16, 40], ("topk", 0.9), None),
    (synth.DSV2L, [1, 16, 33], ("topk", 0.9), ("topk", 0.5)),
    (synth.GPTOSS, [1, 8, 64], ("topk", 0.5), None),
])
def test_shapes_fused_matches_chain(shape, Bs, rule_r, rule_s):
    dl = DeviceLayer(shape, max_tokens=max(Bs))
    try:
        for i, B in enumerate(Bs):
            _, xd = _tokens(dl, B, 30 + i)
            _compare_paths(dl, xd, rule_r, rule_s)
        # the chain against the oracle as well (the fused path is what the parity suite runs)
        xh, xd = _tokens(dl, Bs[1], 40)
        dl.set_fused(False)
        parity.compare(dl, xh, xd, rule_r, rule_s, name=f"chain {shape.name} B={Bs[1]}")
        assert dl.last_launches() == 5
        dl.set_fused(True)
    finally:
        dl.close()
