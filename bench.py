"""Benchmark of the int4 routed-expert MoE layer stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C] [--tokens T]

Headline workload (config 1): Gemma-4-26B-A4B-shaped decode -- 30 stacked MoE
layers, H=2816, E=128 experts, top-8, expert intermediate 704, shared expert
intermediate 2112, one token per step, a fresh N(0,1) hidden row per step,
random weights drawn as the tiny configuration (synthetic, seeded).  One step
= one token through all layers (router, bucketing, routed + shared experts,
combine, post-norm, residual) in one persistent kernel launch.  Weights
(13.2 GB) are far larger than L2 and each step touches 1.1 GB of them, so no
step finds its weights in L2.

The default line also carries every other configuration of the workload set,
each with its own roofline, end-to-end number and oracle baseline:
  configs.tiny_T4            hidden 256, 16 experts, top-4, 4 tokens (latency; L2-resident)
  configs.qwen35b_T1/T4/T8   40 layers, H=2048, 256 experts, top-8, decode batches of 1, 4, 8
  configs.qwen80b_zipf_T1    48 layers, H=2048, 512 experts, top-10, Zipf(1.1) expert popularity
  prefill                    8 chunks of 128 tokens through the 30 Gemma-shaped layers
  prefill_fused              the same 1024 rows through each layer in one call
  prefill_batch64            64-token decode batches on the Gemma shape
  output_head                the 262,144 x 2816 4-bit head GEMV
`value` is tokens/s over all ranks (each rank runs an independent replica:
the layer fits one GPU, so multi-GPU is replicas only).  `--impl reference`
times the fp64 CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int4_routed_expert_02_b200 import synth  # noqa: E402

METRIC = "MoE-layer decode tok/s + HBM GB/s vs peak; prefill-chunk TFLOP/s vs peak"
TINY_REDRAWS = os.path.join(ROOT, "tests", "golden", "tiny_redraws.txt")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu
# capture, per unit of work; None where no capture of the current kernel
# exists.  Reset to None whenever the kernel changes.
# decode_stack_kernel, per layer, keyed by (configuration, tokens per step): one launch of 6 layers (Gemma
# shape) or 4 layers (Qwen shapes).  Only T = 1, where every layer reads exactly k experts, so bytes
# scale with layers; from T = 4 on a layer's bytes follow its routing (the distinct experts fall from
# ~57 in the first layers of the Qwen-35B-shaped stack to ~30 averaged over 40), so no capture stands
# for a whole stack and those lines carry null.
DECODE_TRAFFIC_PER_LAYER = {
    (1, 1): (223_362_304 + 4_370_944) / 6,
    (2, 1): (66_149_120 + 1_017_344) / 4,
    (3, 1): (82_535_424 + 1_690_368) / 4,
}
HEAD_TRAFFIC_PER_CALL = 415_259_392 + 3_848_192  # moe_qmat_gemv over the 262,144 x 2816 head, one token
PREFILL_FUSED_MMA_TRAFFIC_PER_LAYER = 369_931_520 + 15_747_328 + 162_025_216 + 65_058_816  # one 1024-token layer call
PREFILL_MMA_TRAFFIC_PER_LAYER_CHUNK = 296_960_000 + 5_408_000 + 147_004_672 + 8_862_720
PREFILL_WS_TRAFFIC_PER_LAYER_CHUNK = 298_698_496 + 5_197_056 + 148_107_776 + 5_612_800  # gateup + down_kernel


def expert_bytes(rows_cols: int) -> float:
    """Algorithmic bytes of an int4 matrix with rows*cols weights: 4 bits per
    code + a bf16 scale and a bf16 bias per 64 codes = 4.5 bits per weight."""
    return rows_cols * 0.5 + rows_cols / 64 * 4


def layer_bytes(cfg, distinct_experts: float) -> dict:
    H, E, I, Is = cfg.H, cfg.E, cfg.I, cfg.Is
    routed = distinct_experts * expert_bytes(3 * I * H)
    shared = expert_bytes(3 * Is * H)
    router = E * H * (1 + 4 / 64)  # 8-bit codes + bf16 scale/bias per 64
    return dict(routed=routed, shared=shared, router=router, total=routed + shared + router)


def pool_bytes(cfg) -> float:
    return cfg.layers * layer_bytes(cfg, cfg.E)["total"]


def workload_name(cfg, T, layers=None):
    L = cfg.layers if layers is None else layers
    extra = ", Zipf(%.1f) expert popularity" % cfg.zipf if cfg.zipf else ""
    return (f"{cfg.name}: {L} MoE layers, H={cfg.H}, E={cfg.E}, top-{cfg.k}, I={cfg.I}, "
            f"shared I={cfg.Is}, T={T} token(s) per step{extra}")


def l2_note(cfg, step_bytes):
    pool = pool_bytes(cfg)
    if pool < 100e6:
        return f"weights ({pool / 1e6:.2f} MB) fit in L2: a latency figure, no HBM roofline claim"
    return (f"inputs larger than L2 ({pool / 1e9:.1f} GB of weights, {step_bytes / 1e9:.2f} GB touched per step; "
            f"each layer's weights are revisited only a whole stack later)")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# --------------------------------------------------------------------------- inputs

class Inputs:
    """Device-resident inputs of every step of a decode run (generated up front)."""

    def __init__(self, cfg, cfg_id, st, T, n_steps, rank, dev):
        self.cfg = cfg
        if cfg.zipf > 0:
            centred = [c.to(torch.float64) - 128.0 for c in st.router_codes]
            self.h = [torch.stack([synth.gen_zipf_hidden(cfg, cfg_id, l, s, st.router_codes[l], T=T,
                                                         centred=centred[l])[0] for l in range(st.L)]).to(dev)
                      for s in range(n_steps)]
        elif cfg_id == 0:
            red = synth.load_redraws(TINY_REDRAWS)
            self.h = [synth.gen_hidden_redrawn(cfg, 0, 10_000 + s, T, red, device=dev) for s in range(n_steps)]
        else:
            self.h = [synth.gen_hidden(cfg, cfg_id, 10_000 + s + rank * 1_000_000, T, device=dev)
                      for s in range(n_steps)]

    def __getitem__(self, i):
        return self.h[i]


# --------------------------------------------------------------------------- ours

def _distinct_experts(st, moe, cfg, T):
    """Mean number of distinct experts per layer for the last step's routing."""
    if T == 1:
        return float(cfg.k)
    tot = 0
    for l in range(st.L):
        idx = torch.empty(T, cfg.k, dtype=torch.int32, device=st.device)
        wts = torch.empty(T, cfg.k, dtype=torch.float32, device=st.device)
        moe.moe_router(st.layers[l], st.inputs[l], T, idx, wts, None, st.ws)
        tot += int(torch.unique(idx).numel())
    return tot / st.L


def _expert_roofline(st, moe, cfg, T, hbm, dev, opts=None, split_shared=False):
    """Per-launch time of the expert part (moe_expert_ffn: gate/up + down +
    weighted sum) on each layer's real input, against the HBM roofline of
    the distinct experts it reads.  split_shared: also time the same calls
    without the shared expert, so that its share can be reported apart (the
    time with it minus the time without it)."""
    L = st.L
    bufs = []
    for l in range(L):
        idx = torch.empty(T, cfg.k, dtype=torch.int32, device=dev)
        wts = torch.empty(T, cfg.k, dtype=torch.float32, device=dev)
        xe = torch.empty(T, cfg.H, dtype=torch.bfloat16, device=dev)
        offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(T * cfg.k, dtype=torch.int32, device=dev)
        active = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
        moe.moe_router(st.layers[l], st.inputs[l], T, idx, wts, xe, st.ws)
        moe.moe_bucket(idx, T, cfg.k, cfg.E, offsets, perm, None, active)
        bufs.append((xe, idx, wts, offsets, perm, active))
    m = torch.empty(T, cfg.H, dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)
    ws2 = moe.workspace(st.layers[0], T, device=dev)
    stream = torch.cuda.current_stream(dev)
    reps = 3

    def timed(with_shared):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L * reps)]
        for r in range(reps):
            for l in range(L):
                xe, idx, wts, offsets, perm, active = bufs[l]
                a, b = evs[r * L + l]
                a.record(stream)
                moe.moe_expert_ffn(st.layers[l], xe, T, idx, wts, offsets, perm, active, with_shared, m, ws2, opts)
                b.record(stream)
        torch.cuda.synchronize(dev)
        moe.moe_workspace_status(ws2)
        times = [a.elapsed_time(b) for a, b in evs[L:]]  # drop the first (warm) repetition
        return statistics.mean(times) * 1e3

    us = timed(1)
    us_routed = timed(0) if split_shared else None
    d = statistics.mean(int(torch.unique(bufs[l][1]).numel()) for l in range(L))
    nbytes = d * expert_bytes(3 * cfg.I * cfg.H) + expert_bytes(3 * cfg.Is * cfg.H)
    achieved = nbytes / (us / 1e6) / 1e9
    out = {"kernel": "expert FFN per layer call (moe_expert_ffn)", "bound": "hbm", "achieved": round(achieved, 1),
           "peak": hbm["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / hbm["hbm_gbs"], 4),
           "peak_source": hbm["source"] + " (burst copy)", "traffic": None, "bytes_per_launch": int(nbytes),
           "us_per_launch": round(us, 3), "distinct_experts": round(d, 2)}
    if us_routed is not None:
        out["us_routed_only"] = round(us_routed, 3)
    return out


def _e2e(st, cfg, T, K, W, inputs, dev):
    """The same steps through the C ABI with host buffers: the step's input
    from pinned host memory to the device, all layers, the last layer's output
    back to pinned host memory, every step."""
    h_host = [inputs[i].cpu().pin_memory() for i in range(W + K)]
    out_host = torch.empty_like(st.final_output(), device="cpu").pin_memory()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    target = st.buf[0] if cfg.chained else st.inp

    def step(i):
        target.copy_(h_host[i], non_blocking=True)
        st.run()
        out_host.copy_(st.final_output(), non_blocking=True)

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for i in range(K):
        step(W + i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    return {"value": round(T * K / (ms / 1e3), 2), "unit": "tok/s",
            "h2d_bytes_per_step": int(h_host[0].numel() * h_host[0].element_size()),
            "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size())}


def decode_measure(cfg_id, T, K, W, dev, rank=0, world=1, clocks=False, cpu_budget=3.0, layers=None,
                   share=None, want_cpu=True, force_path=0):
    """One decode configuration: K timed steps of T tokens through the whole
    stack (device-resident inputs), its HBM roofline, the end-to-end number
    and the oracle on the host cores.  Returns (result, stack)."""
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.stack import MoEStack
    cfg = synth.CONFIGS[cfg_id]
    st = MoEStack(cfg, cfg_id, T=T, layers=layers, device=dev, keep_router_codes=cfg.zipf > 0,
                  device_layers=None if share is None else share.layers, opts=moe.make_opts(force_path=force_path))
    inputs = Inputs(cfg, cfg_id, st, T, W + K, rank, dev)
    stream = torch.cuda.current_stream(dev)
    st.capture()

    def step(i):
        st.set_input(inputs[i])
        st.run()

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    clk = ClockSampler(dev.index if dev.index is not None else 0)
    if clocks:
        clk.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        step(W + i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk_res = clk.stop() if clocks else None
    ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    st.status()
    ms_per_step = ms / K
    tok_s = world * T * K / (ms / 1e3)
    distinct = _distinct_experts(st, moe, cfg, T)
    step_bytes = st.L * layer_bytes(cfg, distinct)["total"]
    hbm = peaks()
    gbs = step_bytes / (ms_per_step / 1e3) / 1e9
    if st.persistent:
        traffic = (int(DECODE_TRAFFIC_PER_LAYER[(cfg_id, T)] * st.L)
                   if (cfg_id, T) in DECODE_TRAFFIC_PER_LAYER and layers is None else None)
        roof = {"kernel": "decode_stack_kernel (persistent: all layers of a step in one cooperative launch)",
                "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / hbm["hbm_gbs"], 4), "peak_source": hbm["source"] + " (burst copy)",
                "traffic": traffic, "bytes_per_launch": int(step_bytes), "us_per_launch": round(ms_per_step * 1e3, 2),
                "distinct_experts_per_layer": round(distinct, 2)}
    else:
        roof = _expert_roofline(st, moe, cfg, T, hbm, dev)
    res = {"workload": workload_name(cfg, T, st.L), "config_id": cfg_id, "tokens_per_step": T, "layers": st.L,
           "value": round(tok_s, 2), "unit": "tok/s", "ms_per_step": round(ms_per_step, 5), "steps": K, "warmup": W,
           "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm["hbm_gbs"], 4), "bytes_per_step": int(step_bytes),
           "roofline": roof, "l2": l2_note(cfg, step_bytes),
           "path": "persistent decode kernel" if st.persistent else "per-layer calls (CUDA graph)",
           "gpu_launches_per_step": st.launches_per_step()}
    res["e2e"] = _e2e(st, cfg, T, K, W, inputs, dev)
    if clocks:
        res["clocks"] = clk_res
    if want_cpu and rank == 0 and world == 1 and cpu_budget > 0:
        res["cpu_baseline"] = cpu_baseline(cfg, cfg_id, T, budget_s=cpu_budget)
    del inputs
    return res, st


def expert_flops(cfg, T: int) -> float:
    """Multiply-adds x 2 of the expert FFNs for T tokens: every token through
    k routed experts and the shared expert, three matrices each."""
    return 2.0 * T * (3.0 * cfg.I * cfg.H * cfg.k + 3.0 * cfg.Is * cfg.H)


PREFILL_KERNELS = {
    2: "expert_mma_kernel (tcgen05 grouped GEMM, FP16 operands) x2 + gather + combine",
    3: "gateup_kernel + down_kernel (weight-stationary warp MMA, exact FP16 codes) + gather + combine",
}


def expert_path_of(force_path, T):
    """The expert path a call of T tokens takes (the library's automatic rule when force_path is 0)."""
    if force_path:
        return force_path
    return 1 if T < 32 else (3 if T <= 448 else 2)


def prefill_measure(dev, chunks=8, layers=None, T=None, share=None, force_path=0):
    """Chunked prefill at the Gemma shape: `chunks` chunks of T tokens (128),
    each through every layer (chained), chunk after chunk; plus the per-launch
    expert FFN (tensor-core grouped GEMM) against the tensor and HBM peaks.
    With T = 1024, the 8 chunks' rows go through each layer in
    one call, so every expert's weights are read once for ~64 rows.  `share`:
    a stack whose weights to reuse; `force_path` the expert path (0 automatic).
    Returns (result, stack)."""
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.stack import MoEStack
    cfg = synth.CONFIGS[4]
    T = cfg.T if T is None else T
    opts = moe.make_opts(force_path=force_path)
    st = MoEStack(cfg, 4, T=T, layers=layers, device=dev, device_layers=None if share is None else share.layers,
                  opts=opts)
    inputs = [synth.gen_hidden(cfg, 4, 20_000 + c, T, device=dev) for c in range(chunks + 1)]
    stream = torch.cuda.current_stream(dev)
    st.set_input(inputs[0])
    st.run()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for c in range(chunks):
        st.set_input(inputs[1 + c])
        st.run()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    st.status()
    hbm = peaks()
    roof = _expert_roofline(st, moe, cfg, T, hbm, dev, opts, split_shared=True)
    fl = expert_flops(cfg, T)
    tflops = fl / (roof["us_per_launch"] / 1e6) / 1e12
    peak_t = hbm["bf16_tflops"]  # FP16 and BF16 share the dense tensor rate
    fused = T != cfg.T
    path = expert_path_of(force_path, T)
    traffic = ((PREFILL_FUSED_MMA_TRAFFIC_PER_LAYER if fused else PREFILL_MMA_TRAFFIC_PER_LAYER_CHUNK) if path == 2
               else PREFILL_WS_TRAFFIC_PER_LAYER_CHUNK if path == 3 and not fused else None)
    name = (workload_name(cfg, T) + ", the rows of 8 chunks of 128 through each layer in one call") if fused else \
        (workload_name(cfg, T) + f", {chunks} chunks chunk-major")
    bound_us = max(roof["bytes_per_launch"] / (hbm["hbm_gbs"] * 1e3), fl / (peak_t * 1e6))
    return {"workload": name, "tok_s": round(chunks * T / (ms / 1e3), 1),
            "ms_per_chunk": round(ms / chunks, 4),
            "force_path": force_path,
            "expert_ffn": {"kernel": PREFILL_KERNELS[path],
                           "us_per_launch": roof["us_per_launch"], "flops_per_launch": fl,
                           "tflops": round(tflops, 2), "tensor_peak_tflops": peak_t,
                           "tensor_frac": round(tflops / peak_t, 4), "hbm_gbs": roof["achieved"],
                           "hbm_frac": roof["frac"], "bytes_per_launch": roof["bytes_per_launch"],
                           "binding_roof_frac": round(bound_us / roof["us_per_launch"], 4),
                           "traffic": traffic,
                           "peak_source": hbm["source"] + " (bf16 dense burst; FP16 same rate; copy bandwidth)",
                           "split": split_roofline(cfg, T, roof, peak_t)}}, st


def split_roofline(cfg, T, roof, peak_t):
    """The routed experts and the shared expert apart: the routed part is the
    same call without the shared expert; the shared part is the difference
    (time with it minus time without it)."""
    us_r = roof["us_routed_only"]
    us_s = roof["us_per_launch"] - us_r
    fl_r = 2.0 * T * 3.0 * cfg.I * cfg.H * cfg.k
    fl_s = 2.0 * T * 3.0 * cfg.Is * cfg.H
    part = lambda fl, us: ({"us": round(us, 3), "tflops": round(fl / (us / 1e6) / 1e12, 2),
                           "tensor_frac": round(fl / (us / 1e6) / 1e12 / peak_t, 4)} if us > 0 else {"us": round(us, 3)})
    return {"routed": part(fl_r, us_r), "shared_expert": part(fl_s, us_s),
            "how": "routed: the call without the shared expert; shared: the call's time with it minus without it"}


HEAD_ROWS = 262_144  # vocabulary rows of the output head (synthetic: the pages give no vocabulary size)


def head_measure(dev, reps=50, warmup=5):
    """The output head that shares the embedding's quantised weights: one
    4-bit [262,144 x 2816] matrix times one token (moe_qmat_gemv), against the
    HBM roofline (4.5 bits per weight, every byte read once per call)."""
    from int4_routed_expert_02_b200 import moe
    cfg = synth.CONFIGS[1]
    V, H = HEAD_ROWS, cfg.H
    w = synth.gen_vocab_head(cfg, 1, V, device=dev)
    qt, sbt = moe.prepare_qmat(w["head_q"], w["head_s"], w["head_b"], 1, V, H)
    del w
    x = synth.gen_hidden(cfg, 1, 30_000, 1, device=dev)
    y = torch.empty(1, V, dtype=torch.float32, device=dev)
    ws = moe.qmat_gemv_workspace(device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        moe.moe_qmat_gemv(qt, sbt, V, H, x, 1, y, ws)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        moe.moe_qmat_gemv(qt, sbt, V, H, x, 1, y, ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / reps
    nbytes = int(expert_bytes(V * H) + V * 4 + H * 2)  # weights + fp32 output + bf16 input
    hbm = peaks()
    gbs = nbytes / (us / 1e6) / 1e9
    return {"workload": f"output head sharing the embedding's 4-bit weights: {V} x {H}, 1 token per call",
            "kernel": "qmat_gemv_kernel (dequant-GEMV, one 32-row block per warp at a time)",
            "us_per_call": round(us, 2), "bound": "hbm", "achieved": round(gbs, 1), "peak": hbm["hbm_gbs"],
            "unit": "GB/s", "frac": round(gbs / hbm["hbm_gbs"], 4), "bytes_per_call": nbytes,
            "traffic": HEAD_TRAFFIC_PER_CALL, "peak_source": hbm["source"] + " (burst copy)"}


def residency_measure(dev, slots=16, K=48, W=8, T=1):
    """Tiered expert residency on the Gemma-shaped decode: every layer's
    routed experts in pinned host memory, a device cache of `slots` experts
    per layer (the pages' 16-slot LFU), decisions and copies on the GPU
    (moe_layer_forward_cached, one layer call after another).  Reports tok/s,
    the hit rate and the bytes that crossed the host bus per token."""
    from int4_routed_expert_02_b200.residency import CachedStack
    cfg = synth.CONFIGS[1]
    cs = CachedStack(cfg, 1, T, slots=slots, device=dev)
    inputs = [synth.gen_hidden(cfg, 1, 10_000 + s, T, device=dev) for s in range(W + K)]
    stream = torch.cuda.current_stream(dev)
    for i in range(W):
        cs.set_input(inputs[i])
        cs.run()
    torch.cuda.synchronize(dev)
    s0 = cs.stats()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        cs.set_input(inputs[W + i])
        cs.run()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    s1 = cs.stats()
    hits, misses = s1["hits"] - s0["hits"], s1["misses"] - s0["misses"]
    per_expert = expert_bytes(3 * cfg.I * cfg.H)
    host_bytes = misses * per_expert / K
    res = {"workload": workload_name(cfg, T) + f", routed experts in pinned host memory, {slots}-slot device "
                                               "cache per layer (LFU, recency ties)",
           "value": round(T * K / (ms / 1e3), 2), "unit": "tok/s", "ms_per_step": round(ms / K, 4),
           "hit_rate": round(hits / max(hits + misses, 1), 4), "host_bytes_per_token": int(host_bytes),
           "host_gbs": round(host_bytes * K / (ms / 1e3) / 1e9, 2), "steps": K, "warmup": W,
           "resident_bytes": int(sum(sum(t.numel() * t.element_size() for t in l.cache.values()) +
                                     l.dl.nbytes() for l in cs.layers)),
           "launches_per_step": 7 * cs.L}
    del cs
    torch.cuda.empty_cache()
    return res


def ep_measure(dev, rank, world, T=1024, K=4, W=2):
    """Expert-parallel prefill over the world's GPUs: the Gemma-shaped stack's
    experts split in contiguous blocks, one all-reduce (NCCL) of each layer's
    fp32 partial combine, T rows per call through every layer.  The total
    work is fixed (strong scaling): tok/s = T * K / the slowest rank's time."""
    from int4_routed_expert_02_b200.ep import EPStack
    cfg = synth.CONFIGS[4]
    ep = EPStack(cfg, 4, T, rank, world, device=dev)
    inputs = [synth.gen_hidden(cfg, 4, 20_000 + c, T, device=dev) for c in range(W + K)]
    stream = torch.cuda.current_stream(dev)
    for i in range(W):
        ep.set_input(inputs[i])
        ep.run()
    torch.cuda.synchronize(dev)
    torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        ep.set_input(inputs[W + i])
        ep.run()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    t = torch.tensor([e0.elapsed_time(e1)], device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms = float(t.item())
    return {"workload": workload_name(cfg, T) + f", experts split over {world} GPUs, one NCCL all-reduce per layer",
            "value": round(T * K / (ms / 1e3), 1), "unit": "tok/s", "ms_per_call": round(ms / K, 3),
            "scaling": "strong", "n_gpus": world}


# --------------------------------------------------------------------------- oracle

def _oracle_layer_input(cfg, cfg_id, layer, w, T):
    if cfg.zipf > 0:
        return synth.gen_zipf_hidden(cfg, cfg_id, layer, 0, w["router_codes"], T=T)[0]
    if cfg_id == 0:
        return synth.gen_hidden_redrawn(cfg, 0, 10_000, T, synth.load_redraws(TINY_REDRAWS))
    return synth.gen_hidden(cfg, cfg_id, 10_000, T)


def cpu_baseline(cfg, cfg_id, T, budget_s=15.0, threads=None):
    """The fp64 oracle as it stands on a bounded sample of the workload: a few
    tokens (min(T, 4)) through consecutive layers of the stack (chained where
    the configuration chains) until the budget is spent, timed on one thread
    and on every host core (its row loops split over OpenMP threads; the same
    arithmetic, the same bits); tok/s scaled to T tokens and the full stack."""
    import oracle
    cores = threads or os.cpu_count() or 1
    Ts = min(T, 4)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    s1 = sall = 0.0
    n, h, used = 0, None, 1
    try:
        while n < cfg.layers and (n == 0 or s1 < budget_s):
            w = {k: v.cpu() for k, v in synth.gen_layer(cfg, cfg_id, n, device=dev).items()}
            OL = oracle.OracleLayer.from_config(w, cfg)
            if h is None or not cfg.chained:
                h = _oracle_layer_input(cfg, cfg_id, n, w, Ts)
            oracle.set_threads(1)
            t0 = time.perf_counter()
            r = oracle.layer_forward(OL, h)
            s1 += time.perf_counter() - t0
            used = oracle.set_threads(cores)
            t0 = time.perf_counter()
            oracle.layer_forward(OL, h)
            sall += time.perf_counter() - t0
            h = torch.from_numpy(r["out_bf16"].view("int16")).view(torch.bfloat16)
            n += 1
            del w, OL
    finally:
        oracle.set_threads(1)
    v1 = Ts * (n / cfg.layers) / s1
    vall = Ts * (n / cfg.layers) / sall
    cpu_model = ""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    cpu_model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"value": round(vall, 6), "unit": "tok/s", "cores": used, "kind": "oracle",
            "value_1_thread": round(v1, 6), "cpu_model": cpu_model,
            "sample": f"{Ts} token(s) through {n} of {cfg.layers} layers, fp64 C oracle: {sall:.2f} s on {used} "
                      f"threads, {s1:.2f} s on 1 thread; tok/s scaled to the full stack"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle on the host cores (OpenMP over
    its row loops).  Each step is a bounded sample: T fresh tokens through one
    layer (cycling over the first two layers); tok/s is scaled to the full
    layer stack."""
    import oracle
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.T
    if rank != 0:
        return None
    cores = os.cpu_count() or 1
    used = oracle.set_threads(cores)
    layers, hs = [], []
    for l in range(min(2, cfg.layers)):
        w = {k: v.cpu() for k, v in synth.gen_layer(cfg, args.config, l, device="cpu").items()}
        layers.append(oracle.OracleLayer.from_config(w, cfg))
        hs.append(w)
    times = []
    try:
        for s in range(args.warmup + args.steps):
            l = s % len(layers)
            if cfg.zipf > 0:
                h = synth.gen_zipf_hidden(cfg, args.config, l, s, hs[l]["router_codes"], T=T)[0]
            elif args.config == 0:
                h = synth.gen_hidden_redrawn(cfg, 0, 10_000 + s, T, synth.load_redraws(TINY_REDRAWS))
            else:
                h = synth.gen_hidden(cfg, args.config, 10_000 + s, T)
            t0 = time.perf_counter()
            oracle.layer_forward(layers[l], h)
            dt = time.perf_counter() - t0
            if s >= args.warmup:
                times.append(dt)
    finally:
        oracle.set_threads(1)
    per_layer = statistics.mean(times)
    v = T / (per_layer * cfg.layers)
    cpu = {"value": round(v, 6), "unit": "tok/s", "cores": used, "kind": "oracle",
           "sample": f"{args.steps} steps of {T} token(s) through 1 layer (fp64 C oracle, {used} threads, "
                     f"{per_layer * 1e3:.1f} ms/layer); tok/s scaled to {cfg.layers} layers"}
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_layer * cfg.layers * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(cfg, T), "config_id": args.config, "layers": cfg.layers,
                       "tokens_per_step": T, "parallelism": f"host CPU, {used} threads",
                       "l2": l2_note(cfg, cfg.layers * layer_bytes(cfg, cfg.k * T)["total"])},
            "cpu_baseline": cpu, "e2e": {"value": round(v, 6), "unit": "tok/s", "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- main

OTHER_DECODE = [("tiny_T4", 0, 4), ("qwen35b_T1", 2, 1), ("qwen35b_T4", 2, 4), ("qwen35b_T8", 2, 8),
                ("qwen80b_zipf_T1", 3, 1)]


def run_ours(args, rank, world, local_rank):
    from int4_routed_expert_02_b200 import build
    if rank == 0 or not os.path.exists(build.LIB):
        build.build()
    if world > 1:
        torch.distributed.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    T = args.tokens or synth.CONFIGS[args.config].T
    K, W = args.steps, args.warmup
    head_res, st = decode_measure(args.config, T, K, W, dev, rank, world, clocks=(rank == 0),
                                  cpu_budget=0 if args.no_cpu_baseline else args.cpu_budget,
                                  layers=args.layers or None, force_path=args.expert_path)
    cfg = synth.CONFIGS[args.config]
    res = {
        "metric": METRIC, "value": head_res["value"], "unit": "tok/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": head_res["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, bf16 activations, fp32 accumulate (router fp64)", "data": "synthetic",
        "config": {"workload": head_res["workload"], "config_id": args.config, "layers": head_res["layers"],
                   "tokens_per_step": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU", "l2": head_res["l2"]},
        "hbm_gbs": head_res["hbm_gbs"], "hbm_frac": head_res["hbm_frac"], "bytes_per_step": head_res["bytes_per_step"],
        "roofline": head_res["roofline"], "cpu_baseline": head_res.get("cpu_baseline"), "e2e": head_res["e2e"],
        "gpu_launches": head_res["gpu_launches_per_step"] * K, "clocks": head_res.get("clocks"),
    }
    if world > 1 and args.all_configs and not (args.layers or args.tokens) and args.config == 1:
        del st
        torch.cuda.empty_cache()
        try:
            res["ep_prefill"] = ep_measure(dev, rank, world)
        except Exception as exc:  # noqa: BLE001 -- report, keep the headline
            res["ep_prefill"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        return res
    if not args.all_configs or world > 1 or args.layers or args.tokens or args.config != 1:
        return res
    # the rest of the workload set, each on its own weights (freed in turn)
    del st
    torch.cuda.empty_cache()
    res["configs"] = {}
    for name, cid, t in OTHER_DECODE:
        k2 = K if t == 1 else max(64, K // 4)
        r, s2 = decode_measure(cid, t, k2, W, dev, cpu_budget=args.sub_cpu_budget)
        res["configs"][name] = r
        del s2
        torch.cuda.empty_cache()
    prefill, pst = prefill_measure(dev)
    res["prefill"] = prefill
    res["prefill_fused"], _ = prefill_measure(dev, chunks=2, T=1024, share=pst)
    # the other tensor-core path at each size, for comparison
    res["prefill_tcgen05"], _ = prefill_measure(dev, share=pst, force_path=2)
    res["prefill_fused_ws"], _ = prefill_measure(dev, chunks=2, T=1024, share=pst, force_path=3)
    r64, s64 = decode_measure(4, 64, 32, W, dev, cpu_budget=args.sub_cpu_budget, share=pst)
    r64["workload"] += " (64-token decode batches on the Gemma shape)"
    res["prefill_batch64"] = r64
    del pst, s64
    torch.cuda.empty_cache()
    res["output_head"] = head_measure(dev)
    res["residency"] = residency_measure(dev)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--tokens", type=int, default=0, help="tokens per step (default: the config's)")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: build this many layers instead of the config's (not a bench line)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="oracle seconds per leg for the headline")
    ap.add_argument("--sub-cpu-budget", type=float, default=3.0, help="oracle seconds per leg for the other configs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--head-only", action="store_true",
                    help="profiling only: time the output-head GEMV alone and print its object")
    ap.add_argument("--prefill-only", action="store_true",
                    help="profiling only: the 128-token prefill chunks alone (with --layers, --expert-path; "
                         "--tokens 1024 puts the rows of 8 chunks through each layer in one call)")
    ap.add_argument("--expert-path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="profiling only: force_path of the expert FFN (0 automatic) for --prefill-only or the headline")
    ap.add_argument("--headline-only", dest="all_configs", action="store_false",
                    help="only the headline configuration (skip the other configurations of the line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        elif args.prefill_only:
            from int4_routed_expert_02_b200 import build
            build.build()
            res = {"prefill": prefill_measure(torch.device("cuda", local_rank), chunks=2, layers=args.layers or None,
                                              T=args.tokens or None, force_path=args.expert_path)[0]} \
                if rank == 0 else None
        elif args.head_only:
            from int4_routed_expert_02_b200 import build
            build.build()
            res = {"output_head": head_measure(torch.device("cuda", local_rank))} if rank == 0 else None
        else:
            res = run_ours(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
