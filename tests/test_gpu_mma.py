"""Tensor-core (tcgen05) grouped-GEMM expert path vs the fp64 oracle and vs the
CUDA-core dequant-GEMV path, through the C ABI.

The grouped GEMM multiplies FP16 weights (s*q + b rounded once) by FP16
activations with FP32 accumulation in tensor memory, and hands the SwiGLU
output to the down GEMM in FP16; both roundings are far inside the bar
max|err| <= 2e-2 * rms(reference) (checked here at 5e-3).  Cases cover several 128-row tiles, half
tiles (I = 704 = 5.5 tiles), one-k-block inputs (H = 64), ragged token
counts, experts with more than 128 tokens (two token tiles), the shared
expert on and off, and the 128-token prefill chunk at the Gemma shape.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth
from tests.moe_cases import OUT_TOL, assert_same_up_to_one_rounding, bf16_host, hidden_with_gap, host, max_err_vs_rms, oracle_layer

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe

MMA = 2
GEMV = 1


def _layer(cfg, cfg_id, layer=0):
    w = synth.gen_layer(cfg, cfg_id, layer, device="cuda")
    return w, moe.DeviceLayer.from_config(w, cfg), oracle_layer(host(w), cfg)


def _expert_ffn(cfg, D, xe_d, idx_np, w_np, path, with_shared=True):
    T = xe_d.shape[0]
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w_np, np.float32)).cuda()
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
    active = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    moe.moe_bucket(idx, T, cfg.k, cfg.E, offsets, perm, None, active)
    m = torch.empty(T, cfg.H, dtype=torch.float32, device="cuda")
    ws = moe.workspace(D, T)
    moe.moe_expert_ffn(D, xe_d, T, idx, wts, offsets, perm, active, with_shared, m, ws,
                       moe.make_opts(force_path=path))
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    return m.cpu().double().numpy()


def _routed_inputs(cfg, OL, h):
    _, idx, wr, xn = oracle.router(OL, h)
    xe_bits = oracle.f64_to_bf16(xn)
    xe_d = torch.from_numpy(xe_bits.view(np.int16)).cuda().view(torch.bfloat16)
    return idx, wr, oracle.bf16_to_f64(xe_bits), xe_d


@pytest.mark.parametrize("cfg_id,T,sample", [
    (0, 4, None),                 # tiny: one tile per matrix, four k-blocks
    (1, 33, [0, 17, 32]),         # Gemma shape, ragged token count, half tiles of I = 704
    (2, 8, None),                 # Qwen-35B shape, 8-token decode batch
    (4, 128, [0, 1, 77, 127]),    # the 128-token prefill chunk
])
def test_mma_expert_ffn_matches_oracle_and_gemv(cfg_id, T, sample):
    cfg = synth.CONFIGS[cfg_id]
    base_id = 1 if cfg_id == 4 else cfg_id
    w, D, OL = _layer(synth.CONFIGS[base_id], base_id)
    h = hidden_with_gap(cfg, cfg_id, OL, 5, T) if cfg_id == 0 else synth.gen_hidden(cfg, cfg_id, 5, T)
    idx, wr, xe, xe_d = _routed_inputs(cfg, OL, h)
    m_mma = _expert_ffn(cfg, D, xe_d, idx, wr, MMA)
    m_gemv = _expert_ffn(cfg, D, xe_d, idx, wr, GEMV)
    rows = list(range(T)) if sample is None else sample
    ref = oracle.expert_ffn(OL, xe[rows], idx[rows], wr[rows].astype(np.float32).astype(np.float64))
    err = max_err_vs_rms(m_mma[rows], ref)
    assert err <= OUT_TOL, err
    assert err <= 5e-3, err                     # FP16 weights and activations: well inside the bar
    assert max_err_vs_rms(m_mma, m_gemv) <= 5e-3
    assert np.all(np.isfinite(m_mma))


def test_mma_without_shared_expert_and_dense_equivalence():
    """k = E with unit gates equals the dense mixture; shared expert on and off."""
    base = synth.CONFIGS[0]
    cfg = synth.MoEConfig("dense", H=256, E=16, k=16, I=128, Is=128, layers=1, T=40)
    w = synth.gen_layer(base, 0, 0, device="cuda")
    D = moe.DeviceLayer.from_config(w, cfg)
    OL = oracle_layer(host(w), cfg)
    rng = np.random.default_rng(3)
    T = 40
    x = torch.from_numpy(rng.standard_normal((T, cfg.H)).astype(np.float32)).to(torch.bfloat16)
    idx = np.stack([rng.permutation(cfg.E) for _ in range(T)]).astype(np.int32)
    ones = np.ones((T, cfg.E))
    rows = [0, 13, 39]
    for with_shared in (True, False):
        m = _expert_ffn(cfg, D, x.cuda(), idx, ones, MMA, with_shared)
        ref = oracle.expert_ffn(OL, x.double().numpy()[rows], idx[rows], ones[rows], with_shared)
        assert max_err_vs_rms(m[rows], ref) <= 5e-3


@pytest.mark.parametrize("dims", [
    dict(H=64, E=8, k=8, I=64, Is=64, T=40),         # one k-block, half tiles, k = E
    dict(H=320, E=24, k=5, I=192, Is=320, T=33),     # ragged k-blocks / row tiles
    dict(H=256, E=8, k=8, I=128, Is=192, T=130),     # every expert holds 130 tokens: two token tiles
    dict(H=512, E=16, k=2, I=256, Is=128, T=300),    # shared expert over three token tiles
])
def test_mma_edge_shapes(dims):
    T = dims.pop("T")
    cfg = synth.MoEConfig("edge", layers=1, T=T, **dims)
    w, D, OL = _layer(cfg, 98)
    h = synth.gen_hidden(cfg, 98, 0, T)
    hd = h.cuda()
    out = torch.empty_like(hd)
    ws = moe.workspace(D, T)
    moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=MMA))
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    rows = sorted({0, 1, T // 2, T - 1})
    ref = oracle.layer_forward(OL, h[rows])
    assert max_err_vs_rms(bf16_host(out)[rows], ref["out_f64"]) <= OUT_TOL


def test_prefill_chunk_layer_paths_are_deterministic():
    """A 128-token chunk at the Gemma shape, on the automatic path (the
    weight-stationary warp-MMA path at this size) and on the tcgen05 path:
    reruns are bit-identical, sampled rows match the oracle, and the two paths
    agree to one bf16 ulp element by element."""
    cfg = synth.CONFIGS[4]
    w, D, OL = _layer(synth.CONFIGS[1], 1, layer=3)
    T = 128
    h = synth.gen_hidden(cfg, 4, 2, T)
    hd = h.cuda()
    ws = moe.workspace(D, T)
    rows = [3, 64, 100]
    ref = oracle.layer_forward(OL, h[rows])
    first = {}
    for path in (0, MMA):
        outs = []
        for _ in range(2):
            out = torch.empty_like(hd)
            moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=path))
            torch.cuda.synchronize()
            moe.moe_workspace_status(ws)
            outs.append(out)
        assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
        assert max_err_vs_rms(bf16_host(outs[0])[rows], ref["out_f64"]) <= OUT_TOL
        first[path] = outs[0]
    # the two paths accumulate in another order: rounding flips only
    assert_same_up_to_one_rounding(first[0], first[MMA], max_frac=0.25)


def test_prefill_rows_of_eight_chunks_in_one_call():
    """The rows of 8 chunks of 128 through a Gemma-shaped layer in ONE call
    (T = 1024, ~64 rows per expert tile): sampled rows match the oracle, and
    every row matches the same rows run as 8 separate 128-token chunks."""
    cfg = synth.CONFIGS[4]
    w, D, OL = _layer(synth.CONFIGS[1], 1, layer=5)
    T = 1024
    h = synth.gen_hidden(cfg, 4, 7, T)
    hd = h.cuda()
    out = torch.empty_like(hd)
    ws = moe.workspace(D, T)
    moe.moe_layer_forward(D, hd, out, T, ws)
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    rows = [0, 127, 128, 555, 1023]
    ref = oracle.layer_forward(OL, h[rows])
    assert max_err_vs_rms(bf16_host(out)[rows], ref["out_f64"]) <= OUT_TOL
    ws128 = moe.workspace(D, 128)
    chunked = torch.empty_like(hd)
    for c in range(8):
        moe.moe_layer_forward(D, hd[c * 128:(c + 1) * 128], chunked[c * 128:(c + 1) * 128], 128, ws128)
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws128)
    # one call of 1024 rows and the 128-row chunks may take different expert paths
    assert_same_up_to_one_rounding(out, chunked, max_frac=0.25)


def test_grouped_gemm_wait_timeout_is_reported_and_the_next_call_is_fine(monkeypatch):
    """A test hook makes the epilogue's first wait run out (about 1 s): every
    role of both grouped-GEMM kernels stops as on a real timeout, the status
    call reports MOE_EDEVICE, and the next call on the same context is right."""
    cfg = synth.CONFIGS[0]
    T = 32
    w, D, OL = _layer(cfg, 0)
    h = hidden_with_gap(cfg, 0, OL, 6, T)
    hd = h.cuda()
    out = torch.empty_like(hd)
    ws = moe.workspace(D, T)
    monkeypatch.setenv("MOE_TEST_MMA_STALL", "1")
    moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=MMA))
    torch.cuda.synchronize()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_workspace_status(ws)
    assert ei.value.code == moe.MOE_EDEVICE and "timed out" in str(ei.value)
    monkeypatch.delenv("MOE_TEST_MMA_STALL")
    moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=MMA))
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    ref = oracle.layer_forward(OL, h)
    assert max_err_vs_rms(bf16_host(out), ref["out_f64"]) <= OUT_TOL
