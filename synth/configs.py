"""The five workload shapes of the sparse-expert MoE layer and their seeding rules.

The shapes follow the layers the paper's study covers (OLMoE, DeepSeek-V2, GPT-OSS, Llama-4
families; "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-Expert
Model Execution", technical summary, Methodology), instantiated with synthetic values:
x ~ N(0, 1), router ~ N(0, 0.02), gate/up ~ N(0, 1/sqrt(H)), down ~ N(0, 1/sqrt(I)),
all rounded to nearest-even into the layer dtype.

Seeds: the workload seed (0) for every weight tensor, ``seed + 1 + batch_index`` for the
token batch ``batch_index`` and ``seed + 1000`` for threshold-calibration tokens.
"""
from dataclasses import dataclass


@dataclass(frozen=True)
class LayerShape:
    name: str
    hidden: int          # H
    n_routed: int        # E
    top_k: int           # k
    inter: int           # I (routed expert intermediate size)
    n_shared: int = 0    # S (always-on shared experts)
    inter_shared: int = 0  # Ish
    dtype: str = "bf16"  # "bf16" | "f32"
    route: str = "softmax_topk"  # "softmax_topk" | "softmax_all" | "sigmoid"
    seed: int = 0

    @property
    def elt(self):
        return 2 if self.dtype == "bf16" else 4

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return LayerShape(**d)


# tiny fp32 layer: H256 E8 top-2 I512, no shared expert (parity at 4 tokens, s = 0.5)
TINY = LayerShape("tiny-fp32", 256, 8, 2, 512, dtype="f32")
# OLMoE-shaped: H2048 E64 top-8 I1024
OLMOE = LayerShape("olmoe", 2048, 64, 8, 1024)
# DeepSeek-V2-Lite-shaped: H2048, 64 routed top-6 + 2 shared, I = Ish = 1408
DSV2L = LayerShape("dsv2-lite", 2048, 64, 6, 1408, n_shared=2, inter_shared=1408)
# GPT-OSS-120B-shaped: H2880 E128 top-4 I2880, softmax over the top-k logits
GPTOSS = LayerShape("gpt-oss-120b", 2880, 128, 4, 2880)
# Llama-4-Maverick-shaped: H5120, 128 routed top-1 with a sigmoid gate + 1 shared, I = Ish = 8192
LLAMA4 = LayerShape("llama4-maverick", 5120, 128, 1, 8192, n_shared=1, inter_shared=8192,
                    route="sigmoid")

SHAPES = {s.name: s for s in (TINY, OLMOE, DSV2L, GPTOSS, LLAMA4)}


def token_seed(shape: LayerShape, batch_index: int) -> int:
    return shape.seed + 1 + batch_index


def calib_seed(shape: LayerShape) -> int:
    return shape.seed + 1000
