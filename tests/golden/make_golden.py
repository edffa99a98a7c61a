"""Writes tiny_fp32_oracle.json: the oracle's result on the tiny fp32 workload (H256 E8 top-2
I512, 4 tokens from token stream 1, s = 0.5), a regression record of the oracle itself.

It calls only the oracle and the input generator.  The pages print no worked example, so this
file pins nothing external; it guards the oracle against unintended change.  Regenerate it only
with a change of the oracle's arithmetic whose justification names the passage it follows.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def compute():
    s = synth.TINY
    layer = oracle.Layer(s, synth.host_tensor(s, "router"),
                         {e: (synth.host_tensor(s, "gate", e), synth.host_tensor(s, "up", e),
                              synth.host_tensor(s, "down", e)) for e in range(s.n_routed)})
    x = synth.host_tokens(s, 4, synth.token_seed(s, 0))
    r = layer.forward(x, ("topk", 0.5))
    kept = [[np.flatnonzero(r["keep"][t][j]).tolist() for j in range(s.top_k)] for t in range(4)]
    return {"workload": "tiny-fp32 H256 E8 top-2 I512, tokens seed 1, B=4, s=0.5",
            "idx": r["idx"].tolist(), "w": [[repr(float(v)) for v in row] for row in r["w"]],
            "kept": kept, "out": [[repr(float(v)) for v in row] for row in r["out"]]}


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_fp32_oracle.json"), "w") as f:
        json.dump(compute(), f, indent=0)
