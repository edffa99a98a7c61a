"""Expert parallelism of the layer over G ranks (one process per GPU, torch.distributed).

The serving system of "Uncovering Intra-expert Activation Sparsity for Efficient Mixture-of-
Expert Model Execution" (technical summary, Methodology) keeps expert parallelism.  Here:
  * every rank holds the router and routes every token over all E experts (the tokens and the
    router are replicated), so the ranks agree on the routing;
  * rank r owns the routed experts ``expert_range(E, G, r)`` (contiguous, sizes differ by at
    most one) and the shared experts ``s`` with ``s % G == r``;
  * each rank runs the layer on its experts only and writes its part of the output in fp32
    (``moe_forward_partial``); one all-reduce (sum) over the ranks gives the layer output before
    rounding, which ``moe_cast_output`` rounds to the layer dtype.
Everything that computes runs in the library's kernels; the all-reduce is the process group's
(NCCL on GPUs).  The compute steps are a backend object so that the host logic (ranges,
ownership, the reduction and its order) can run against another implementation.
"""
import torch
import torch.distributed as dist

from . import (make_config, moe_cast_output, moe_create, moe_destroy, moe_forward_partial,
               moe_set_expert_range, sparsity)


def expert_range(E, world, rank):
    """Routed experts [begin, end) of ``rank``: contiguous, the first E % world ranks one more."""
    if not (0 <= rank < world) or E < 0:
        raise ValueError((E, world, rank))
    base, extra = divmod(E, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def shared_mask(S, world, rank):
    """Bit s set for each shared expert s that ``rank`` evaluates (s % world == rank)."""
    return sum(1 << s for s in range(S) if s % world == rank)


class LibraryBackend:
    """The library's kernels on this rank's device: a handle restricted to the rank's experts."""

    def __init__(self, cfg, rank, world, device):
        self.cfg = cfg
        self.h = moe_create(cfg)
        self.begin, self.end = expert_range(cfg.n_routed, world, rank)
        moe_set_expert_range(self.h, self.begin, self.end, shared_mask(cfg.n_shared, world, rank))
        self.partial_buf = torch.empty((cfg.max_tokens, cfg.hidden), dtype=torch.float32,
                                       device=device)

    def partial(self, x, router, routed_local, shared, rule_r, rule_s, stream=None):
        n = x.shape[0]
        buf = self.partial_buf[:n]
        moe_forward_partial(self.h, x, n, router, routed_local, shared, sparsity(rule_r),
                            sparsity(rule_s) if rule_s else None, buf, stream)
        return buf

    def cast(self, total, out, stream=None):
        moe_cast_output(self.h, total, total.shape[0], out, stream)
        return out

    def close(self):
        if self.h:
            moe_destroy(self.h)
            self.h = None


class ExpertParallelLayer:
    """One rank's share of an expert-parallel layer.  ``backend`` computes the rank's partial
    output and the final cast; ``group`` is the process group of the G ranks (None: default)."""

    def __init__(self, backend, group=None):
        self.backend = backend
        self.group = group

    def forward(self, x, router, routed_local, shared, rule_r, rule_s=None, out=None,
                stream=None):
        part = self.backend.partial(x, router, routed_local, shared, rule_r, rule_s, stream)
        if dist.is_initialized() and dist.get_world_size(self.group) > 1:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
        if out is None:
            return part
        return self.backend.cast(part, out, stream)


def library_layer(hidden, n_routed, top_k, inter, n_shared=0, inter_shared=0, max_tokens=256,
                  dtype="bf16", route="softmax_topk", rank=None, world=None, group=None,
                  device=None):
    """An ExpertParallelLayer on the library for this process's rank in ``group``."""
    rank = dist.get_rank(group) if rank is None else rank
    world = dist.get_world_size(group) if world is None else world
    cfg = make_config(hidden, n_routed, top_k, inter, n_shared, inter_shared, max_tokens, dtype,
                      route)
    return ExpertParallelLayer(LibraryBackend(cfg, rank, world, device), group)
