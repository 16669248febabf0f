"""Tiered expert residency: each layer's routed experts in a pool in pinned
host memory, with a cache of C experts per layer in device memory.

The pages stream experts from SSD into a 16-slot LFU cache per layer
(TurboFieldfare introduction page, section "TurboFieldfare's expert
streaming structure") and keep an LFU + recency pool (Swiftlet article,
section "why the same model runs in so little memory"); on a B200 the tiers
are host memory and HBM.  The decisions (hit, victim, copy) are made on the
GPU inside moe_layer_forward_cached, so no routing result crosses back to the
host; this module only owns the buffers.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import moe, synth


class CachedLayer:
    """One layer: router and shared expert resident (a DeviceLayer), the
    routed experts' tiled matrices moved to pinned host memory, and a device
    cache of `slots` experts with its bookkeeping."""

    def __init__(self, dl: moe.DeviceLayer, slots: int, device="cuda", free_resident: bool = False):
        """free_resident: drop dl's device copy of the routed experts (they are then
        served only through the cache; dl's routed pointers become null)."""
        dev = torch.device(device)
        self.dl, self.slots, self.E = dl, slots, dl.E
        self.pool, self.cache = {}, {}
        for name in ("gate", "up", "down"):
            for part in ("_qt", "_sbt"):
                full = dl.t[name + part]
                self.pool[name + part] = full.cpu().pin_memory()
                per = full.numel() // dl.E
                self.cache[name + part] = torch.empty(slots * per, dtype=full.dtype, device=dev)
            if free_resident:
                del dl.t[name + "_qt"], dl.t[name + "_sbt"]
                setattr(dl.struct, name, moe.QMat(None, None))
        self.slot_of = torch.empty(dl.E, dtype=torch.int32, device=dev)
        self.expert_of = torch.empty(slots, dtype=torch.int32, device=dev)
        self.uses = torch.empty(slots, dtype=torch.int32, device=dev)
        self.last = torch.empty(slots, dtype=torch.int32, device=dev)
        self.ctl = torch.zeros(4, dtype=torch.int32, device=dev)
        c = moe.ExpertCache(slots=slots)
        for name in ("gate", "up", "down"):
            setattr(c, name, moe.QMat(self.cache[name + "_qt"].data_ptr(), self.cache[name + "_sbt"].data_ptr()))
            setattr(c, "pool_" + name, moe.QMat(self.pool[name + "_qt"].data_ptr(), self.pool[name + "_sbt"].data_ptr()))
        c.slot_of, c.expert_of = self.slot_of.data_ptr(), self.expert_of.data_ptr()
        c.uses, c.last, c.ctl = self.uses.data_ptr(), self.last.data_ptr(), self.ctl.data_ptr()
        self.struct = c
        moe.moe_expert_cache_reset(c, dl.E)

    def stats(self) -> dict:
        calls, hits, misses, _ = (int(v) for v in self.ctl.cpu())
        return {"calls": calls, "hits": hits, "misses": misses}

    def reset(self):
        moe.moe_expert_cache_reset(self.struct, self.E)


class CachedStack:
    """A chained stack of layers served through per-layer expert caches."""

    def __init__(self, cfg: synth.MoEConfig, cfg_id: int, T: int, slots: int, layers: int | None = None,
                 device="cuda", device_layers: list | None = None, seed: int = 0):
        self.cfg, self.T = cfg, T
        self.L = cfg.layers if layers is None else layers
        self.device = torch.device(device)
        own = device_layers is None
        dls = device_layers[:self.L] if not own else [
            moe.DeviceLayer.from_config(synth.gen_layer(cfg, cfg_id, l, seed=seed, device=self.device), cfg,
                                        device=self.device) for l in range(self.L)]
        self.layers = [CachedLayer(dl, slots, self.device, free_resident=own) for dl in dls]
        self.buf = torch.zeros(self.L + 1, T, cfg.H, dtype=torch.bfloat16, device=self.device)
        self.ws = moe.workspace(dls[0], T, device=self.device)
        self.opts = moe.make_opts()

    def set_input(self, h):
        self.buf[0].copy_(h, non_blocking=True)

    def final_output(self):
        return self.buf[self.L]

    def run(self):
        for l, cl in enumerate(self.layers):
            moe.moe_layer_forward_cached(cl.dl, cl.struct, self.buf[l], self.buf[l + 1], self.T, self.ws, self.opts)

    def stats(self) -> dict:
        tot = {"calls": 0, "hits": 0, "misses": 0}
        for cl in self.layers:
            for k, v in cl.stats().items():
                tot[k] += v
        n = tot["hits"] + tot["misses"]
        tot["hit_rate"] = tot["hits"] / n if n else 0.0
        return tot
