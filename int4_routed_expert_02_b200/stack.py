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
                 seed: int = 0, device="cuda", keep_router_codes: bool = False, persistent: bool | None = None,
                 device_layers: list | None = None, opts=None):
        """device_layers: the weights of another stack of the same configuration
        to share (they are not regenerated)."""
        self.cfg, self.cfg_id, self.seed = cfg, cfg_id, seed
        self.T = cfg.T if T is None else T
        self.L = cfg.layers if layers is None else layers
        self.device = torch.device(device)
        self.layers = []
        self.router_codes = []
        for l in range(self.L if device_layers is None else 0):
            w = synth.gen_layer(cfg, cfg_id, l, seed=seed, device=self.device)
            if keep_router_codes and "router_codes" in w:
                self.router_codes.append(w["router_codes"].cpu())
            self.layers.append(moe.DeviceLayer.from_config(w, cfg, device=self.device))
            del w
        if device_layers is not None:
            assert len(device_layers) >= self.L
            self.layers = list(device_layers[:self.L])
        H = cfg.H
        if persistent is None:
            persistent = moe.moe_decode_stack_fits(self.layers[0], self.T, torch.cuda.current_stream(self.device))
        self.persistent = persistent
        if self.persistent:
            # one cooperative kernel per step: every layer's output in h_out[l]
            self.larr = moe.layer_array(self.layers)
            self.ws_dec = torch.empty(moe.moe_decode_stack_workspace_size(self.layers[0], self.T), dtype=torch.uint8,
                                      device=self.device)
            self.h_out = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
            if cfg.chained:
                self.buf = torch.zeros(1, self.T, H, dtype=torch.bfloat16, device=self.device)
                self.inputs = [self.buf[0]] + [self.h_out[l] for l in range(self.L - 1)]
            else:
                self.inp = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
                self.inputs = [self.inp[l] for l in range(self.L)]
            self.outputs = [self.h_out[l] for l in range(self.L)]
        elif cfg.chained:
            self.buf = torch.zeros(self.L + 1, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.inputs = [self.buf[l] for l in range(self.L)]
            self.outputs = [self.buf[l + 1] for l in range(self.L)]
        else:
            self.inp = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.out = torch.zeros(self.L, self.T, H, dtype=torch.bfloat16, device=self.device)
            self.inputs = [self.inp[l] for l in range(self.L)]
            self.outputs = [self.out[l] for l in range(self.L)]
        self.ws = moe.workspace(self.layers[0], self.T, device=self.device)  # per-layer calls
        self.opts = opts if opts is not None else moe.make_opts()
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

    def launches_per_step(self) -> int:
        """Kernels of the library launched per step."""
        return 1 if self.persistent else 6 * self.L

    def enqueue(self, stream=None):
        """Enqueue one step (all L layers) on `stream` (default: torch's current stream)."""
        if self.persistent:
            h_in = self.buf[0] if self.cfg.chained else self.inp
            moe.moe_decode_stack(self.larr, self.L, h_in, self.cfg.chained, self.h_out, self.T, self.ws_dec,
                                 self.opts, stream=stream)
            return
        for l in range(self.L):
            moe.moe_layer_forward(self.layers[l], self.inputs[l], self.outputs[l], self.T, self.ws, self.opts,
                                  stream=stream)

    def status(self):
        """Raise if the persistent kernel recorded a device-side error (synchronises)."""
        if self.persistent:
            moe.moe_decode_stack_status(self.ws_dec)

    def capture(self):
        """Capture one step in a CUDA graph (replayed by run()).  The persistent
        kernel is a single launch per step and is not captured."""
        if self.persistent:
            self.enqueue()
            torch.cuda.synchronize(self.device)
            return None
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
