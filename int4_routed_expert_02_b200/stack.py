"""A stack of MoE layers on one GPU: device-resident weights for L layers,
per-layer activation buffers and one workspace, driven through the C ABI.

Decode runs the layer loop one token batch at a time, prefill runs it per
chunk of up to 128 rows (TurboFieldfare introduction page, section
"TurboFieldfare's expert streaming structure", last paragraph).  Layers are
chained (layer l+1 consumes layer l's bf16 output) unless the configuration
feeds every layer its own input.  A whole step can be captured in one CUDA
graph, so the only host->device crossing per step is the graph launch.
"""
from __future__ import annotations

import torch

from . import moe, synth


class MoEStack:
    def __init__(self, cfg: synth.MoEConfig, cfg_id: int, T: int | None = None, layers: int | None = None,
                 seed: int = 0, device="cuda", keep_router_codes: bool = False):
        self.cfg, self.cfg_id, self.seed = cfg, cfg_id, seed
        self.T = cfg.T if T is None else T
        self.L = cfg.layers if layers is None else layers
        self.device = torch.device(device)
        self.layers = []
        self.router_codes = []
        for l in range(self.L):
            w = synth.gen_layer(cfg, cfg_id, l, seed=seed, device=self.device)
            if keep_router_codes and "router_codes" in w:
                self.router_codes.append(w["router_codes"].cpu())
            self.layers.append(moe.DeviceLayer.from_config(w, cfg, device=self.device))
            del w
        H = cfg.H
        # chained: buf[l] is layer l's input, buf[l+1] its output
        # unchained: inp[l] -> out[l]
        if cfg.chained:
            self.buf = torch.zeros(self.L + 1, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.inputs = [self.buf[l] for l in range(self.L)]
            self.outputs = [self.buf[l + 1] for l in range(self.L)]
        else:
            self.inp = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.out = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.inputs = [self.inp[l] for l in range(self.L)]
            self.outputs = [self.out[l] for l in range(self.L)]
        self.ws = moe.workspace(self.layers[0], self.T, device=self.device)
        self.opts = moe.make_opts()
        self.graph = None

    def weight_bytes(self) -> int:
        return sum(l.nbytes() for l in self.layers)

    def set_input(self, h: torch.Tensor):
        """h: [T, H] (chained) or [L, T, H] (one input per layer)."""
        if self.cfg.chained:
            self.buf[0].copy_(h, non_blocking=True)
        else:
            self.inp.copy_(h, non_blocking=True)

    def final_output(self) -> torch.Tensor:
        return self.outputs[-1]

    def enqueue(self, stream=None):
        """Enqueue one step (all L layers) on `stream` (default: torch's current stream)."""
        for l in range(self.L):
            moe.moe_layer_forward(self.layers[l], self.inputs[l], self.outputs[l], self.T, self.ws, self.opts,
                                  stream=stream)

    def capture(self):
        """Capture one step in a CUDA graph (replayed by run())."""
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.enqueue()  # warm-up outside capture (sets kernel attributes once)
        torch.cuda.current_stream(self.device).wait_stream(s)
        torch.cuda.synchronize(self.device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.enqueue()
        self.graph = g
        return g

    def run(self):
        if self.graph is not None:
            self.graph.replay()
        else:
            self.enqueue()
