"""Synthetic device-resident workloads for the tests and the benchmark.

Draws a layer's logical weights on the GPU with the seeded generator (``synth``) and packs them
with ``moe_pack_experts``; the CPU oracle draws the same values with the generator's host fill.
This is harness code: the layer itself is the library (``moe_forward``).
"""
import torch

import synth

from . import (expert_weights, make_config, moe_create, moe_debug_lists, moe_destroy,
               moe_forward, moe_forward_roster, moe_last_launches, moe_pack_experts,
               moe_set_fused, roster, sparsity)


class DeviceLayer:
    """A packed, device-resident layer of the workload ``shape`` and its library handle."""

    def __init__(self, shape, max_tokens, device="cuda", expert_chunk=8):
        self.shape = shape
        self.max_tokens = max_tokens
        self.dtype = synth.torch_dtype(shape)
        self.cfg = make_config(shape.hidden, shape.n_routed, shape.top_k, shape.inter,
                               shape.n_shared, shape.inter_shared, max_tokens, shape.dtype,
                               shape.route)
        self.h = moe_create(self.cfg)
        H = shape.hidden
        self.router = synth.device_tensor(shape, "router", device=device)
        self.gate, self.updown = self._pack(False, shape.n_routed, shape.inter, expert_chunk, device)
        self.routed = expert_weights(self.gate, self.updown)
        if shape.n_shared:
            self.sh_gate, self.sh_updown = self._pack(True, shape.n_shared, shape.inter_shared,
                                                      expert_chunk, device)
            self.shared = expert_weights(self.sh_gate, self.sh_updown)
        else:
            self.shared = None
        self.roster = None  # (counts, pinned, m, delta): calls use roster routing when set
        torch.cuda.synchronize()

    def _pack(self, shared, n, I, chunk, device):
        s, H = self.shape, self.shape.hidden
        names = ("sh_gate", "sh_up", "sh_down") if shared else ("gate", "up", "down")
        gate = torch.empty((n, I, H), dtype=self.dtype, device=device)
        updown = torch.empty((n, I, 2, H), dtype=self.dtype, device=device)
        m = min(chunk, n)
        wu = torch.empty((m, I, H), dtype=self.dtype, device=device)
        wd = torch.empty((m, H, I), dtype=self.dtype, device=device)
        for e0 in range(0, n, m):
            c = min(m, n - e0)
            seed, tid, _, cnt, std, _ = synth.spec(s, names[0], e0)
            synth.fill_cuda(gate[e0:e0 + c], seed, tid, e0 * cnt, std)
            seed, tid, _, cnt, std, _ = synth.spec(s, names[1], e0)
            synth.fill_cuda(wu[:c], seed, tid, e0 * cnt, std)
            seed, tid, _, cnt, std, _ = synth.spec(s, names[2], e0)
            synth.fill_cuda(wd[:c], seed, tid, e0 * cnt, std)
            moe_pack_experts(self.h, int(shared), gate[e0:e0 + c], wu[:c], wd[:c], c,
                             gate[e0:e0 + c], updown[e0:e0 + c])
        torch.cuda.synchronize()
        return gate, updown

    def tokens(self, n_tokens, seed, out=None):
        return synth.device_tokens(self.shape, n_tokens, seed, out=out)

    def forward(self, x, rule_routed, rule_shared=None, out=None, stream=None):
        if out is None:
            out = torch.empty_like(x)
        sr = sparsity(rule_routed)
        ss = sparsity(rule_shared) if (self.shape.n_shared and rule_shared) else None
        if self.roster is not None:
            counts, pinned, m, delta = self.roster
            moe_forward_roster(self.h, x, x.shape[0], self.router,
                               roster(counts, pinned, m, delta), self.routed, self.shared, sr, ss,
                               out, stream)
        else:
            moe_forward(self.h, x, x.shape[0], self.router, self.routed, self.shared, sr, ss,
                        out, stream)
        return out

    def debug(self, n_tokens):
        """Intermediate results of the last call: idx, w, logits, cnt, lists, act (numpy)."""
        return {k: v.cpu().numpy() for k, v in self.debug_device(n_tokens).items()}

    def debug_device(self, n_tokens):
        """The same as debug(), as tensors on the layer's device."""
        s = self.shape
        P = s.top_k + s.n_shared
        imax = max(s.inter, s.inter_shared if s.n_shared else 0)
        dev = self.gate.device
        r = {"idx": torch.empty((n_tokens, s.top_k), dtype=torch.int32, device=dev),
             "w": torch.empty((n_tokens, s.top_k), dtype=torch.float32, device=dev),
             "logits": torch.empty((n_tokens, s.n_routed), dtype=torch.float32, device=dev),
             "cnt": torch.empty((n_tokens, P), dtype=torch.int32, device=dev),
             "lists": torch.empty((n_tokens, P, imax), dtype=torch.int32, device=dev),
             "act": torch.empty((n_tokens, P, imax), dtype=torch.float32, device=dev)}
        moe_debug_lists(self.h, n_tokens, r["idx"], r["w"], r["logits"], r["cnt"], r["lists"],
                        r["act"])
        torch.cuda.synchronize()
        return r

    def set_fused(self, enable):
        """Fused layer kernel where it applies (True) or the launch chain (False, the default)."""
        moe_set_fused(self.h, 1 if enable else 0)

    def last_launches(self):
        return moe_last_launches(self.h)

    def close(self):
        if self.h:
            moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
