"""Shared test helpers: seeded cases for the GPU path and the fp64 oracle.

The tolerances are the ones the layer is specified to meet:
  routing indices and bucketing: bit-exact;
  gate weights: relative error <= 1e-5;
  expert output m and layer output h_out: max |err| <= 2e-2 * rms(reference).
h_out is compared against the oracle's exact (fp64, unrounded) output, so
that the bf16 rounding of the GPU's result is part of the error budget.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from int4_routed_expert_02_b200 import synth

W_RTOL = 1e-5
OUT_TOL = 2e-2


def host(weights: dict) -> dict:
    return {k: v.detach().cpu() for k, v in weights.items()}


def oracle_layer(weights_host: dict, cfg, k=None) -> oracle.OracleLayer:
    return oracle.OracleLayer(weights_host, cfg.H, cfg.E, cfg.k if k is None else k, cfg.I, cfg.Is)


def min_topk_gap(logits_row: np.ndarray, k: int) -> float:
    """Smallest gap between consecutive sorted logits among the top k+1."""
    srt = np.sort(logits_row)[::-1][: k + 1]
    return float(np.min(srt[:-1] - srt[1:])) if len(srt) > 1 else np.inf


def hidden_with_gap(cfg, cfg_id, OL, stream, T, min_gap=1e-3, seed=0):
    """N(0,1) hidden rows; a row whose top-k logit gap is below min_gap is
    redrawn from the next independent draw (the tiny configuration's rule)."""
    h = synth.gen_hidden(cfg, cfg_id, stream, T, seed=seed)
    for t in range(T):
        d = 0
        while min_topk_gap(oracle.router(OL, h[t:t + 1])[0][0], cfg.k) < min_gap:
            d += 1
            h[t] = synth.gen_hidden(cfg, cfg_id, stream, 1, seed=seed, draw=d * 65536 + t + 1)[0]
    return h


def max_err_vs_rms(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / rms(ref)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-300)


def bf16_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().float().double().numpy()


def assert_same_up_to_one_rounding(a: torch.Tensor, b: torch.Tensor, max_frac=0.10):
    """Two bf16 results of the same fp32-accumulated computation along
    different kernel paths: every element within one bf16 ulp of the other at
    its magnitude, or within 1e-3 * rms (near zero, where ulps are tiny); and
    few elements differing at all (rounding flips only)."""
    a64 = a.detach().cpu().double()
    b64 = b.detach().cpu().double()
    rms = float(b64.pow(2).mean().sqrt())
    mag = torch.maximum(a64.abs(), b64.abs()).clamp_min(1e-30)
    ulp = torch.pow(2.0, torch.floor(torch.log2(mag)) - 7)      # bf16: 8 significant bits
    tol = torch.maximum(ulp, torch.full_like(ulp, 1e-3 * rms))
    diff = (a64 - b64).abs()
    worst = float((diff / tol).max())
    assert worst <= 1.0 + 1e-9, f"difference {worst:.2f} x (one ulp or 1e-3 rms)"
    frac = float((diff > 0).double().mean())
    assert frac <= max_frac, f"{frac:.2%} of elements differ"
