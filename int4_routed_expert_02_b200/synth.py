"""Seeded synthetic inputs for the int4 routed-expert MoE layer.

This module only DRAWS numbers: it holds none of the layer's arithmetic
(no dequantisation, no normalisation, no routing).  Both the fp64 CPU
oracle and the CUDA path are fed from here, and nothing else is shared
between them.

Weight format (TurboFieldfare page, section "memory saving"): MLX affine
quantisation, groups of 64 along the input dimension, one BF16 scale and one
BF16 bias per group, w = scale * q + bias.  Expert matrices hold 4-bit codes,
eight per uint32 word, low nibble first; the router projection holds 8-bit
codes, four per word, low byte first.  Scales are |N(0, 0.02)|, biases are
-mid * scale + N(0, 1e-3) with mid = 8 for int4 and 128 for int8, codes are
uniform over their range; router_scale and per_expert_scale are U(0.5, 1.5);
hidden states are N(0, 1).  Every value is rounded to BF16 (round to nearest
even) before it is handed to either side.

Tensors are generated with torch's counter-based Philox stream on the
requested device; each tensor has its own stream, seeded from
(seed, config, layer, tensor id), so any layer regenerates independently.

Shapes follow the pages' models (TurboFieldfare page, "streaming structure":
128 experts, top-8, shared expert without routing weight; Swiftlet page,
"why so little memory": 256 experts top-8 and 512 experts top-10).
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = [
    "MoEConfig", "CONFIGS", "tensor_seed", "gen_layer", "gen_router", "gen_experts", "gen_hidden",
    "gen_zipf_hidden", "load_redraws", "gen_hidden_redrawn", "pack_codes", "bf16_bits", "from_bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    H: int          # hidden size
    E: int          # routed experts
    k: int          # experts per token
    I: int          # routed expert intermediate size
    Is: int         # shared expert intermediate size
    layers: int
    T: int          # tokens per call
    zipf: float = 0.0   # > 0: router inputs planted so expert popularity ~ Zipf(zipf)
    chained: bool = True


CONFIGS = {
    0: MoEConfig("tiny", H=256, E=16, k=4, I=128, Is=128, layers=1, T=4),
    1: MoEConfig("gemma4-26b-a4b-shape-decode", H=2816, E=128, k=8, I=704, Is=2112, layers=30, T=1),
    2: MoEConfig("qwen3.6-35b-a3b-shape-decode", H=2048, E=256, k=8, I=512, Is=512, layers=40, T=1),
    3: MoEConfig("qwen3-next-80b-a3b-shape-decode", H=2048, E=512, k=10, I=512, Is=512, layers=48, T=1,
                 zipf=1.1, chained=False),
    4: MoEConfig("gemma4-26b-a4b-shape-prefill", H=2816, E=128, k=8, I=704, Is=2112, layers=30, T=128),
}

_TENSOR_IDS = {
    "router_q": 1, "router_s": 2, "router_b": 3, "router_scale": 4, "per_expert_scale": 5,
    "gate_q": 10, "gate_s": 11, "gate_b": 12,
    "up_q": 13, "up_s": 14, "up_b": 15,
    "down_q": 16, "down_s": 17, "down_b": 18,
    "sh_gate_q": 20, "sh_gate_s": 21, "sh_gate_b": 22,
    "sh_up_q": 23, "sh_up_s": 24, "sh_up_b": 25,
    "sh_down_q": 26, "sh_down_s": 27, "sh_down_b": 28,
    "hidden": 40, "zipf_perm": 41, "zipf_gumbel": 42,
    "head_q": 50, "head_s": 51, "head_b": 52,
}

_MASK64 = (1 << 64) - 1


def _splitmix64(x: int) -> int:
    """SplitMix64 finaliser (Steele, Lea, Flood 2014), used to mix seeds."""
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _MASK64
    return x ^ (x >> 31)


def tensor_seed(seed: int, cfg: int, layer: int, tensor: str, extra: int = 0) -> int:
    h = _splitmix64(seed)
    for v in (cfg, layer, _TENSOR_IDS[tensor], extra):
        h = _splitmix64(h ^ (v & _MASK64))
    return h & ((1 << 63) - 1)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def bf16_bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensor -> its raw bits as int16 (same storage layout)."""
    assert t.dtype == torch.bfloat16
    return t.view(torch.int16)


def from_bf16_bits(t: torch.Tensor) -> torch.Tensor:
    assert t.dtype == torch.int16
    return t.view(torch.bfloat16)


def pack_codes(q: torch.Tensor, bits: int) -> torch.Tensor:
    """Pack integer codes along the last dim into int32 words, low field first.

    q: integer tensor [..., n] with n % (32 // bits) == 0, values in [0, 2^bits).
    """
    per = 32 // bits
    q = q.to(torch.int64).reshape(*q.shape[:-1], q.shape[-1] // per, per)
    shifts = torch.arange(per, device=q.device, dtype=torch.int64) * bits
    words = (q << shifts).sum(-1)
    words = torch.where(words >= 2**31, words - 2**32, words)
    return words.to(torch.int32)


def _words(shape, device, seed):
    """Uniform 32-bit words == independent uniform codes in every field."""
    return torch.randint(-2**31, 2**31, shape, dtype=torch.int32, device=device,
                         generator=_gen(device, seed))


def _scales(shape, device, seed, std=0.02):
    n = torch.randn(shape, dtype=torch.float32, device=device, generator=_gen(device, seed))
    return (n * std).abs().to(torch.bfloat16)


def _biases(scale_bf16, mid, device, seed):
    n = torch.randn(scale_bf16.shape, dtype=torch.float32, device=device, generator=_gen(device, seed))
    return (-float(mid) * scale_bf16.float() + n * 1e-3).to(torch.bfloat16)


def _uniform(shape, lo, hi, device, seed):
    u = torch.rand(shape, dtype=torch.float32, device=device, generator=_gen(device, seed))
    return (lo + (hi - lo) * u).to(torch.bfloat16)


def _qmat(prefix, n_mat, rows, cols, bits, cfg_id, layer, seed, device, lead=True, scale_std=0.02):
    shape_w = (n_mat, rows, cols * bits // 32) if lead else (rows, cols * bits // 32)
    shape_g = (n_mat, rows, cols // 64) if lead else (rows, cols // 64)
    mid = 1 << (bits - 1)
    q = _words(shape_w, device, tensor_seed(seed, cfg_id, layer, prefix + "_q"))
    s = _scales(shape_g, device, tensor_seed(seed, cfg_id, layer, prefix + "_s"), scale_std)
    b = _biases(s, mid, device, tensor_seed(seed, cfg_id, layer, prefix + "_b"))
    return q, s, b


def gen_router(cfg: MoEConfig, cfg_id: int, layer: int, seed: int = 0, device="cpu") -> dict:
    """Router part of one layer (MLX layout):
      router_q [E, H/4] (8-bit codes), router_s, router_b [E, H/64],
      router_scale [H], per_expert_scale [E]  (+ router_codes [E, H] uint8 for Zipf configs)."""
    H, E = cfg.H, cfg.E
    out = {}
    out["router_q"], out["router_s"], out["router_b"] = _qmat("router", E, E, H, 8, cfg_id, layer, seed,
                                                               device, lead=False)
    if cfg.zipf > 0:
        # Draw the router codes explicitly (uniform bytes) and pack them, so the
        # Zipf input construction can use the codes without unpacking.
        g = _gen(device, tensor_seed(seed, cfg_id, layer, "router_q"))
        codes = torch.randint(0, 256, (E, H), dtype=torch.int32, device=device, generator=g)
        out["router_codes"] = codes.to(torch.uint8)
        out["router_q"] = pack_codes(codes, 8)
    out["router_scale"] = _uniform((H,), 0.5, 1.5, device, tensor_seed(seed, cfg_id, layer, "router_scale"))
    out["per_expert_scale"] = _uniform((E,), 0.5, 1.5, device,
                                       tensor_seed(seed, cfg_id, layer, "per_expert_scale"))
    return out


def gen_experts(cfg: MoEConfig, cfg_id: int, layer: int, seed: int = 0, device="cpu",
                scale_std: float = 0.02) -> dict:
    """Routed + shared expert matrices of one layer (MLX layout):
      gate_q, up_q [E, I, H/8]   gate_s/b, up_s/b [E, I, H/64]
      down_q [E, H, I/8]         down_s/b [E, H, I/64]
      sh_gate_q, sh_up_q [Is, H/8] (+ s/b [Is, H/64]);  sh_down_q [H, Is/8] (+ s/b [H, Is/64])
    scale_std: the group scales are |N(0, scale_std)| (0.02 in every workload;
    tests widen it to reach large scales)."""
    H, E, I, Is = cfg.H, cfg.E, cfg.I, cfg.Is
    out = {}
    for name, rows, cols in (("gate", I, H), ("up", I, H), ("down", H, I)):
        out[name + "_q"], out[name + "_s"], out[name + "_b"] = _qmat(name, E, rows, cols, 4, cfg_id, layer,
                                                                      seed, device, scale_std=scale_std)
    for name, rows, cols in (("sh_gate", Is, H), ("sh_up", Is, H), ("sh_down", H, Is)):
        out[name + "_q"], out[name + "_s"], out[name + "_b"] = _qmat(name, 1, rows, cols, 4, cfg_id, layer,
                                                                      seed, device, lead=False,
                                                                      scale_std=scale_std)
    return out


def gen_vocab_head(cfg: MoEConfig, cfg_id: int, V: int, seed: int = 0, device="cpu") -> dict:
    """A vocabulary-sized 4-bit matrix [V, H] (MLX layout), drawn like the
    expert matrices: the output head that shares the embedding's quantised
    weights.  head_q [V, H/8], head_s / head_b [V, H/64]."""
    q, s, b = _qmat("head", 1, V, cfg.H, 4, cfg_id, 0, seed, device, lead=False)
    return {"head_q": q, "head_s": s, "head_b": b}


def gen_layer(cfg: MoEConfig, cfg_id: int, layer: int, seed: int = 0, device="cpu",
              expert_scale_std: float = 0.02) -> dict:
    """All weights of one MoE layer in MLX layout (gen_router + gen_experts)."""
    out = gen_router(cfg, cfg_id, layer, seed, device)
    out.update(gen_experts(cfg, cfg_id, layer, seed, device, scale_std=expert_scale_std))
    return out


def gen_hidden(cfg: MoEConfig, cfg_id: int, stream: int, T: int, seed: int = 0, device="cpu",
               draw: int = 0) -> torch.Tensor:
    """N(0,1) hidden rows [T, H] in bf16.  `stream` picks a step / chunk,
    `draw` picks the next independent draw (used when a row is redrawn)."""
    g = _gen(device, tensor_seed(seed, cfg_id, stream, "hidden", draw))
    return torch.randn((T, cfg.H), dtype=torch.float32, device=device, generator=g).to(torch.bfloat16)


def load_redraws(path: str) -> dict:
    """A stored table of redrawn rows ({(stream, token): draw}), as written by
    tests/golden/make_tiny_redraws.py (lines 'stream token draw'; '#' comments)."""
    table = {}
    with open(path) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                stream, tok, draw = (int(v) for v in ln.split())
                table[(stream, tok)] = draw
    return table


def gen_hidden_redrawn(cfg: MoEConfig, cfg_id: int, stream: int, T: int, redraws: dict, seed: int = 0,
                       device="cpu") -> torch.Tensor:
    """gen_hidden with the rows that a stored redraw table names replaced by
    their redraws (draw d of token t: gen_hidden(..., draw=d * 65536 + t + 1))."""
    h = gen_hidden(cfg, cfg_id, stream, T, seed=seed)
    for t in range(T):
        d = redraws.get((stream, t), 0)
        if d:
            h[t] = gen_hidden(cfg, cfg_id, stream, 1, seed=seed, draw=d * 65536 + t + 1)[0]
    return h.to(device)


def gen_zipf_hidden(cfg: MoEConfig, cfg_id: int, layer: int, step: int, router_codes: torch.Tensor,
                    seed: int = 0, T: int | None = None, centred: torch.Tensor | None = None
                    ) -> tuple[torch.Tensor, torch.Tensor]:
    """Router inputs whose selected experts follow a Zipf(cfg.zipf) popularity.

    Per layer a random permutation assigns popularity ranks to experts; per
    token a target set of k experts is drawn without replacement with
    probability proportional to rank^-zipf (Gumbel top-k).  The hidden row is
    the sum of the target experts' centred router code rows (codes - 128),
    divided by the expected RMS of such a sum, sqrt(k * (256^2 - 1) / 12),
    and rounded to bf16.  Because the router codes are
    iid, the planted experts get logits far above the rest, so the router
    selects them; the test-side oracle confirms this per draw.

    router_codes: the layer's `router_codes` from gen_layer ([E, H] uint8).
    centred: optionally, router_codes - 128 as fp64 ([E, H], on the CPU),
    when the caller draws many steps of one layer.
    Returns (hidden [T, H] bf16, target expert ids [T, k] int64).
    """
    E, k = cfg.E, cfg.k
    T = cfg.T if T is None else T
    gp = _gen("cpu", tensor_seed(seed, cfg_id, layer, "zipf_perm"))
    perm = torch.randperm(E, generator=gp)            # perm[e] = popularity rank of expert e (0 = top)
    logp = -cfg.zipf * torch.log(perm.double() + 1.0)
    gg = _gen("cpu", tensor_seed(seed, cfg_id, layer, "zipf_gumbel", step))
    u = torch.rand((T, E), dtype=torch.float64, generator=gg).clamp_min(1e-300)
    keys = logp[None, :] - torch.log(-torch.log(u))
    target = torch.topk(keys, k, dim=1).indices      # [T, k]
    if centred is None:
        centred = router_codes.cpu().to(torch.float64) - 128.0  # [E, H]
    h = centred[target].sum(1) / math.sqrt(k * (256.0 ** 2 - 1.0) / 12.0)
    return h.to(torch.bfloat16), target
