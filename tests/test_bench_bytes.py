"""bench.py's algorithmic bytes (the roofline numerator) on a hand-built call, counted by hand:
every touched expert's gate block is read once, every row in the union of an expert's kept
sets is read once (up row and down column), whatever the number of tokens that keep it."""
import importlib.util
import os

import numpy as np

from synth.configs import LayerShape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _dbg(idx, lists, imax):
    """A debug record as DeviceLayer.debug returns it: per (token, pair) an ascending kept list
    padded with -1, and its count."""
    B, P = len(lists), len(lists[0])
    cnt = np.zeros((B, P), np.int32)
    arr = np.full((B, P, imax), -1, np.int32)
    for t in range(B):
        for j in range(P):
            cnt[t][j] = len(lists[t][j])
            arr[t][j][: len(lists[t][j])] = sorted(lists[t][j])
    return {"idx": np.array(idx, np.int32), "cnt": cnt, "lists": arr}


def test_union_form_routed_only():
    shape = LayerShape("t", hidden=64, n_routed=4, top_k=2, inter=32, dtype="bf16")
    # token 0 -> experts 1, 3; token 1 -> experts 3, 0; expert 2 untouched
    idx = [[1, 3], [3, 0]]
    lists = [[[0, 5, 9], [1, 2]],        # expert 1 keeps {0,5,9}; expert 3 keeps {1,2}
             [[2, 7], [4]]]              # expert 3 keeps {2,7}; expert 0 keeps {4}
    got = _bench().algorithmic_bytes(shape, _dbg(idx, lists, 32), 2)
    H, elt = 64, 2
    assert got["gate"] == 3 * 32 * H * elt                 # experts 0, 1, 3 once each
    rows = 3 + len({1, 2} | {2, 7}) + 1                    # union per expert: 3 + 3 + 1
    assert got["rows"] == rows == 7
    assert got["updown"] == rows * 2 * H * elt
    assert got["router"] == 4 * H * elt + 2 * H * elt      # router weights plus the tokens
    assert got["select"] == 2 * 2 * 32 * 4                 # fp32 activations of every pair
    assert got["finalize"] == 2 * H * (8 + elt)


def test_union_form_with_shared_experts():
    shape = LayerShape("t", hidden=32, n_routed=4, top_k=1, inter=64, n_shared=2,
                       inter_shared=96, dtype="f32")
    idx = [[2], [2], [0]]
    lists = [[[1, 3], [0], [5, 6]],      # routed e2 {1,3}; shared 0 {0}; shared 1 {5,6}
             [[3, 4], [0, 1], []],       # routed e2 {3,4}; shared 0 {0,1}; shared 1 {}
             [[], [2], [6]]]             # routed e0 {} (touched, keeps nothing); shared ...
    got = _bench().algorithmic_bytes(shape, _dbg(idx, lists, 96), 3)
    H, elt = 32, 4
    # gate: routed experts 2 and 0 (a touched expert reads its gate block even if it keeps no
    # neuron), plus both shared experts
    assert got["gate"] == (2 * 64 + 2 * 96) * H * elt
    rows = len({1, 3, 4}) + 0 + len({0, 1, 2}) + len({5, 6})
    assert got["rows"] == rows == 8
    assert got["updown"] == rows * 2 * H * elt
    assert got["select"] == 3 * (1 + 2) * 96 * 4


def test_both_arms_describe_the_workload_with_the_same_keys():
    b = _bench()
    shape = LayerShape("olmoe", 2048, 64, 8, 1024)
    one = b.workload_config(shape, 16, 1, 0.9)
    four = b.workload_config(shape, 16, 4, 0.9)
    assert one["global_batch"] == 16 and four["global_batch"] == 64
    assert set(one) == {"workload", "hidden", "experts", "top_k", "inter", "shared",
                        "batch_per_gpu", "global_batch", "sparsity", "selection"}
