"""Expert-parallel layers over G ranks, one process per GPU.

A layer's routed experts are split into contiguous blocks, rank r owning
experts [E*r/G, E*(r+1)/G); the shared expert of layer l belongs to rank
l mod G.  Every rank runs the whole router (it is a few hundred KB),
computes its pairs' weighted expert outputs into an fp32 partial m
(moe_layer_partial), the ranks' partials are summed by one all-reduce (NCCL
over NVLink / NVSwitch), and every rank finishes the layer with the same
post-norm, residual and layer scalar (moe_combine), so every rank holds the
layer's output.  Per layer a rank reads only its experts' weights: the split
pays off for batched prefill, where every expert is touched; at one decode
token the all-reduce latency outweighs 1/G of a layer's bytes.

The pages run one device, so the split is this library's multi-GPU form of
the same arithmetic, not one of the pages' designs.  Each rank keeps the
whole stack's weights here (the kernels index experts by global id); only
the owned experts' bytes are read.
"""
from __future__ import annotations

import torch

from . import moe, synth


def expert_range(E: int, world: int, rank: int) -> tuple[int, int]:
    """Routed experts [e_lo, e_hi) of `rank` in a split over `world` ranks."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside [0, {world})")
    return E * rank // world, E * (rank + 1) // world


def shared_owner(layer: int, world: int) -> int:
    """Rank that computes layer `layer`'s shared expert."""
    return layer % world


class EPStack:
    """A stack of MoE layers split over the ranks of a torch.distributed
    process group (NCCL), chained layer after layer."""

    def __init__(self, cfg: synth.MoEConfig, cfg_id: int, T: int, rank: int, world: int, layers: int | None = None,
                 device="cuda", group=None, device_layers: list | None = None, seed: int = 0):
        self.cfg, self.T, self.rank, self.world, self.group = cfg, T, rank, world, group
        self.L = cfg.layers if layers is None else layers
        self.device = torch.device(device)
        if device_layers is not None:
            self.layers = list(device_layers[:self.L])
        else:
            self.layers = []
            for l in range(self.L):
                w = synth.gen_layer(cfg, cfg_id, l, seed=seed, device=self.device)
                self.layers.append(moe.DeviceLayer.from_config(w, cfg, device=self.device))
                del w
        self.e_lo, self.e_hi = expert_range(cfg.E, world, rank)
        H = cfg.H
        self.buf = torch.zeros(self.L + 1, T, H, dtype=torch.bfloat16, device=self.device)
        self.m = torch.empty(T, H, dtype=torch.float32, device=self.device)
        self.ws = moe.workspace(self.layers[0], T, device=self.device)
        self.opts = moe.make_opts()

    def set_input(self, h: torch.Tensor):
        self.buf[0].copy_(h, non_blocking=True)

    def final_output(self) -> torch.Tensor:
        return self.buf[self.L]

    def run(self):
        import torch.distributed as dist
        for l in range(self.L):
            own_shared = shared_owner(l, self.world) == self.rank
            moe.moe_layer_partial(self.layers[l], self.buf[l], self.T, self.e_lo, self.e_hi, own_shared, self.m,
                                  self.ws, self.opts)
            if self.world > 1:
                dist.all_reduce(self.m, group=self.group)
            moe.moe_combine(self.buf[l], self.m, self.buf[l + 1], self.T, self.cfg.H, self.opts)

    def bytes_read_per_layer(self, distinct_in_range: float) -> float:
        """Algorithmic bytes one rank reads per layer (its distinct experts,
        the router, and the shared expert on the layers it owns, averaged)."""
        c = self.cfg
        per_expert = 3 * c.I * c.H * 4.5 / 8
        shared = 3 * c.Is * c.H * 4.5 / 8
        router = c.E * c.H * 8.5 / 8
        return distinct_in_range * per_expert + router + shared / self.world
