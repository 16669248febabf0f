"""Benchmark of the int4 routed-expert MoE layer stack on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

Workload (default, config 1): Gemma-4-26B-A4B-shaped decode -- 30 stacked MoE
layers, H=2816, E=128 experts, top-8, expert intermediate 704, shared expert
intermediate 2112, one token per step, a fresh N(0,1) hidden row per step,
random weights drawn as the tiny configuration (synthetic, seeded).  One step
= one token through all layers (router, bucketing, routed + shared experts,
combine) replayed as one CUDA graph.  Weights (13.2 GB) are far larger than
L2 and each step touches 1.1 GB of them, so no step finds its weights in L2.

Prints one JSON line.  `value` is tokens/s over all ranks (each rank runs an
independent replica: the layer fits one GPU, so multi-GPU is replicas only).
`--impl reference` times the fp64 CPU oracle on the host cores instead.
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


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu
# capture, per unit of work: decode_stack_kernel at the Gemma shape, T = 1,
# per layer (2-layer capture halved); the two grouped-GEMM kernels of one
# 128-token layer-chunk.  Reset to None whenever the kernel changes.
DECODE_TRAFFIC_PER_LAYER = (74_531_072 + 2_422_784) // 2
HEAD_TRAFFIC_PER_CALL = 415_259_392 + 3_848_192  # moe_qmat_gemv over the 262,144 x 2816 head, one token
PREFILL_FUSED_MMA_TRAFFIC_PER_LAYER = 369_931_520 + 15_747_328 + 162_025_216 + 65_058_816  # one 1024-token layer call
PREFILL_MMA_TRAFFIC_PER_LAYER_CHUNK = 296_960_000 + 5_408_000 + 147_004_672 + 8_862_720


def expert_bytes(rows_cols: int) -> float:
    """Algorithmic bytes of an int4 matrix with rows*cols weights: 4 bits per
    code + a bf16 scale and a bf16 bias per 64 codes = 4.5 bits per weight."""
    return rows_cols * 0.5 + rows_cols / 64 * 4


def layer_bytes(cfg, distinct_experts: int) -> dict:
    H, E, I, Is = cfg.H, cfg.E, cfg.I, cfg.Is
    routed = distinct_experts * expert_bytes(3 * I * H)
    shared = expert_bytes(3 * Is * H)
    router = E * H * (1 + 4 / 64)  # 8-bit codes + bf16 scale/bias per 64
    return dict(routed=routed, shared=shared, router=router, total=routed + shared + router)


def workload_name(cfg, T):
    return (f"{cfg.name}: {cfg.layers} MoE layers, H={cfg.H}, E={cfg.E}, top-{cfg.k}, I={cfg.I}, "
            f"shared I={cfg.Is}, T={T} token(s) per step")


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


# --------------------------------------------------------------------------- ours

def run_ours(args, rank, world, local_rank):
    from int4_routed_expert_02_b200 import build
    if rank == 0 or not os.path.exists(build.LIB):
        build.build()
    if world > 1:
        torch.distributed.barrier()
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.stack import MoEStack

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.T
    st = MoEStack(cfg, args.config, T=T, layers=args.layers or None, device=dev, keep_router_codes=cfg.zipf > 0)
    K, W = args.steps, args.warmup

    # one fresh input per step, generated up front (device-resident)
    def make_input(step):
        if cfg.zipf > 0:
            rows = [synth.gen_zipf_hidden(cfg, args.config, l, step, st.router_codes[l], T=T)[0]
                    for l in range(st.L)]
            return torch.stack(rows).to(dev)
        return synth.gen_hidden(cfg, args.config, 10_000 + step + rank * 1_000_000, T, device=dev)

    inputs = [make_input(s) for s in range(W + K)]
    stream = torch.cuda.current_stream(dev)
    st.capture()

    def step(i):
        st.set_input(inputs[i])
        st.run()

    for i in range(W):
        step(i)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    if rank == 0:
        clocks.start()
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
    clk = clocks.stop() if rank == 0 else None
    ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / K
    tok_s = world * T * K / (ms / 1e3)

    # algorithmic bytes: distinct experts actually selected, per layer, per step
    distinct = T * cfg.k if T == 1 else _distinct_experts(st, moe, cfg, T)
    step_bytes = st.L * layer_bytes(cfg, distinct)["total"]
    hbm = peaks()
    gbs = step_bytes / (ms_per_step / 1e3) / 1e9

    st.status()
    # dominant kernel: the persistent decode kernel is the whole step (one
    # launch); otherwise the expert GEMVs, timed per launch on the same inputs
    if st.persistent:
        achieved = step_bytes / (ms_per_step / 1e3) / 1e9
        roof = {"kernel": "decode_stack_kernel (persistent: all layers of a step in one cooperative launch)",
                "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / hbm["hbm_gbs"], 4), "peak_source": hbm["source"] + " (burst copy)",
                "traffic": (int(DECODE_TRAFFIC_PER_LAYER * st.L)
                            if DECODE_TRAFFIC_PER_LAYER and args.config == 1 and T == 1 else None),
                "bytes_per_launch": int(step_bytes), "us_per_launch": round(ms_per_step * 1e3, 2)}
    else:
        roof = _expert_roofline(st, moe, cfg, T, hbm, dev)

    # end to end through the C ABI with host buffers: pinned input -> device,
    # all layers, result -> pinned host buffer, every step
    e2e = _e2e(st, cfg, T, K, W, inputs, dev)

    # cpu baseline (oracle) on rank 0 at N = 1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, args.config, T, budget_s=args.cpu_budget)

    launches_per_step = st.launches_per_step()
    n_layers = st.L
    prefill = prefill_fused = head = None
    if args.prefill and world == 1 and args.config == 1 and not args.layers:
        del st
        torch.cuda.empty_cache()
        prefill, pst = prefill_measure(dev)
        prefill_fused, _ = prefill_measure(dev, chunks=2, T=1024, share=pst)
        del pst
        torch.cuda.empty_cache()
        head = head_measure(dev)
    res = {
        "metric": METRIC, "value": round(tok_s, 2), "unit": "tok/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 weights, bf16 activations, fp32 accumulate (router fp64)", "data": "synthetic",
        "config": {"workload": workload_name(cfg, T), "config_id": args.config, "layers": n_layers, "tokens_per_step": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (13.2 GB of weights, 1.1 GB touched per step)"},
        "hbm_gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm["hbm_gbs"], 4),
        "bytes_per_step": int(step_bytes),
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    if prefill is not None:
        res["prefill"] = prefill
        res["prefill_fused"] = prefill_fused
        res["output_head"] = head
    return res


def _distinct_experts(st, moe, cfg, T):
    """Mean number of distinct experts per layer for the last step's routing."""
    ws = st.ws
    tot = 0
    for l in range(st.L):
        idx = torch.empty(T, cfg.k, dtype=torch.int32, device=st.device)
        wts = torch.empty(T, cfg.k, dtype=torch.float32, device=st.device)
        moe.moe_router(st.layers[l], st.inputs[l], T, idx, wts, None, ws)
        tot += int(torch.unique(idx).numel())
    return tot / st.L


def _expert_roofline(st, moe, cfg, T, hbm, dev):
    """Per-launch time of the expert part (gate/up GEMV + down GEMV + weighted
    sum: three launches of moe_expert_ffn) on each layer's real input."""
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
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L * reps)]
    for r in range(reps):
        for l in range(L):
            xe, idx, wts, offsets, perm, active = bufs[l]
            a, b = evs[r * L + l]
            a.record(stream)
            moe.moe_expert_ffn(st.layers[l], xe, T, idx, wts, offsets, perm, active, 1, m, ws2)
            b.record(stream)
    torch.cuda.synchronize(dev)
    times = [a.elapsed_time(b) for a, b in evs[L:]]  # drop the first (warm) repetition
    us = statistics.mean(times) * 1e3
    if T == 1:
        nbytes = cfg.k * expert_bytes(3 * cfg.I * cfg.H) + expert_bytes(3 * cfg.Is * cfg.H)
    else:
        d = statistics.mean(int(torch.unique(bufs[l][1]).numel()) for l in range(L))
        nbytes = d * expert_bytes(3 * cfg.I * cfg.H) + expert_bytes(3 * cfg.Is * cfg.H)
    achieved = nbytes / (us / 1e6) / 1e9
    return {"kernel": "expert FFN: gate/up dequant-GEMV + down dequant-GEMV + weighted sum (moe_expert_ffn)",
            "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / hbm["hbm_gbs"], 4), "peak_source": hbm["source"] + " (burst copy)",
            "traffic": None, "bytes_per_launch": int(nbytes), "us_per_launch": round(us, 3)}


def expert_flops(cfg, T: int) -> float:
    """Multiply-adds x 2 of the expert FFNs for T tokens: every token through
    k routed experts and the shared expert, three matrices each."""
    return 2.0 * T * (3.0 * cfg.I * cfg.H * cfg.k + 3.0 * cfg.Is * cfg.H)


def prefill_measure(dev, chunks=8, layers=None, T=None, share=None):
    """Chunked prefill at the Gemma shape: `chunks` chunks of T tokens (128),
    each through every layer (chained), chunk after chunk; plus the per-launch
    expert FFN (tensor-core grouped GEMM) against the tensor and HBM peaks.
    With T = 1024, the 8 chunks' rows go through each layer in
    one call, so every expert's weights are read once for ~64 rows.  `share`:
    a stack whose weights to reuse.  Returns (result, stack)."""
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.stack import MoEStack
    cfg = synth.CONFIGS[4]
    T = cfg.T if T is None else T
    st = MoEStack(cfg, 4, T=T, layers=layers, device=dev, device_layers=None if share is None else share.layers)
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
    roof = _expert_roofline(st, moe, cfg, T, hbm, dev)
    fl = expert_flops(cfg, T)
    tflops = fl / (roof["us_per_launch"] / 1e6) / 1e12
    peak_t = hbm["bf16_tflops"]  # FP16 and BF16 share the dense tensor rate
    fused = T != cfg.T
    traffic = PREFILL_FUSED_MMA_TRAFFIC_PER_LAYER if fused else PREFILL_MMA_TRAFFIC_PER_LAYER_CHUNK
    name = (workload_name(cfg, T) + ", the rows of 8 chunks of 128 through each layer in one call") if fused else \
        (workload_name(cfg, T) + f", {chunks} chunks chunk-major")
    return {"workload": name, "tok_s": round(chunks * T / (ms / 1e3), 1),
            "ms_per_chunk": round(ms / chunks, 4),
            "expert_ffn": {"kernel": "expert_mma_kernel (tcgen05 grouped GEMM, FP16 operands) x2 + gather + combine",
                           "us_per_launch": roof["us_per_launch"], "flops_per_launch": fl,
                           "tflops": round(tflops, 2), "tensor_peak_tflops": peak_t,
                           "tensor_frac": round(tflops / peak_t, 4), "hbm_gbs": roof["achieved"],
                           "hbm_frac": roof["frac"], "bytes_per_launch": roof["bytes_per_launch"],
                           "traffic": traffic,
                           "peak_source": hbm["source"] + " (bf16 dense burst; FP16 same rate; copy bandwidth)"}}, st


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


def _e2e(st, cfg, T, K, W, inputs, dev):
    from int4_routed_expert_02_b200 import moe  # noqa: F401
    h_host = [inp.cpu().pin_memory() for inp in inputs]
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


# --------------------------------------------------------------------------- oracle

class OracleSample:
    """The fp64 CPU oracle as it stands (plain C, one thread) on host copies
    of the first few layers of a configuration."""

    def __init__(self, cfg, cfg_id, n_layers):
        import oracle
        self.oracle = oracle
        self.cfg, self.cfg_id = cfg, cfg_id
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.layers = []
        self.router_codes = []
        for l in range(n_layers):
            w = {k: v.cpu() for k, v in synth.gen_layer(cfg, cfg_id, l, device=dev).items()}
            self.router_codes.append(w.get("router_codes"))
            self.layers.append(oracle.OracleLayer.from_config(w, cfg))

    def hidden(self, layer, step):
        if self.cfg.zipf > 0:
            return synth.gen_zipf_hidden(self.cfg, self.cfg_id, layer, step, self.router_codes[layer], T=1)[0]
        return synth.gen_hidden(self.cfg, self.cfg_id, 10_000 + step, 1)

    def time_layer(self, layer, h):
        t0 = time.perf_counter()
        r = self.oracle.layer_forward(self.layers[layer], h)
        dt = time.perf_counter() - t0
        return dt, torch.from_numpy(r["out_bf16"].view("int16")).view(torch.bfloat16)


def cpu_baseline(cfg, cfg_id, T, budget_s=15.0):
    """Oracle tok/s on a bounded sample: one token through consecutive layers
    until the time budget is spent, scaled to the full layer stack."""
    import oracle
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    spent, n, h = 0.0, 0, None
    while n < cfg.layers and spent < budget_s:
        w = {k: v.cpu() for k, v in synth.gen_layer(cfg, cfg_id, n, device=dev).items()}
        OL = oracle.OracleLayer.from_config(w, cfg)
        if h is None or not cfg.chained:
            h = (synth.gen_zipf_hidden(cfg, cfg_id, n, 0, w["router_codes"], T=1)[0] if cfg.zipf > 0
                 else synth.gen_hidden(cfg, cfg_id, 0, 1))
        t0 = time.perf_counter()
        r = oracle.layer_forward(OL, h)
        spent += time.perf_counter() - t0
        h = torch.from_numpy(r["out_bf16"].view("int16")).view(torch.bfloat16)
        n += 1
        del w, OL
    tok_s = (n / cfg.layers) / spent
    return {"value": round(tok_s, 6), "unit": "tok/s", "cores": 1, "kind": "oracle",
            "sample": f"1 token through {n} of {cfg.layers} layers (fp64 C oracle, 1 thread, {spent:.1f} s); "
                      f"tok/s scaled to the full {cfg.layers}-layer stack"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle on the host cores.  Each step is
    a bounded sample: one fresh token through one layer (cycling over the
    first two layers); tok/s is scaled to the full layer stack."""
    cfg = synth.CONFIGS[args.config]
    T = args.tokens or cfg.T
    if rank != 0:
        return None
    smp = OracleSample(cfg, args.config, min(2, cfg.layers))
    times = []
    for s in range(args.warmup + args.steps):
        l = s % len(smp.layers)
        dt, _ = smp.time_layer(l, smp.hidden(l, s))
        if s >= args.warmup:
            times.append(dt)
    per_layer = statistics.mean(times)
    v = 1.0 / (per_layer * cfg.layers)
    cpu = {"value": round(v, 6), "unit": "tok/s", "cores": 1, "kind": "oracle",
           "sample": f"{args.steps} steps of 1 token through 1 layer (fp64 C oracle, 1 thread, "
                     f"{per_layer * 1e3:.1f} ms/layer); tok/s scaled to {cfg.layers} layers"}
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "tok/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_layer * cfg.layers * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_name(cfg, T), "config_id": args.config, "layers": cfg.layers,
                       "tokens_per_step": 1, "parallelism": "host CPU, 1 thread"},
            "cpu_baseline": cpu, "e2e": {"value": round(v, 6), "unit": "tok/s", "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}


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
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--head-only", action="store_true",
                    help="profiling only: time the output-head GEMV alone and print its object")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false",
                    help="skip the chunked-prefill measurement that the default line carries")
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
