"""Weight-stationary warp-MMA expert path (force_path 3) vs the fp64 oracle,
the CUDA-core dequant-GEMV path and the tcgen05 path, through the C ABI.

The codes enter the tensor cores as exact FP16 values (q * 2^-24), the group
scales and biases stay FP32, and the token rows and SwiGLU outputs are
rounded once to FP16; the bar is max|err| <= 2e-2 * rms(reference), checked
here at 5e-3.  Cases cover the tiny shape, every decode shape, the 128-token
prefill chunk, a 512-expert layer, K of a single 64-column group, ragged row
blocks, experts holding more than one token group (8 tokens for gate/up, 16
for down), the shared expert over many token groups and switched off, and
bit-identical reruns (the warps' partial sums are added in a fixed order).
Because the weights are never formed in FP16, group scales far outside the
workloads' range are computed to the bar with no report, while a SwiGLU value
beyond the FP16 range is reported as on the tcgen05 path.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth
from tests.moe_cases import OUT_TOL, bf16_host, hidden_with_gap, host, max_err_vs_rms, oracle_layer

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe

WS, TC, GEMV = 3, 2, 1


def _layer(cfg, cfg_id, layer=0, **kw):
    w = synth.gen_layer(cfg, cfg_id, layer, device="cuda", **kw)
    return w, moe.DeviceLayer.from_config(w, cfg), oracle_layer(host(w), cfg)


def _routed(cfg, OL, h):
    _, idx, wr, xn = oracle.router(OL, h)
    xe_bits = oracle.f64_to_bf16(xn)
    xe_d = torch.from_numpy(xe_bits.view(np.int16)).cuda().view(torch.bfloat16)
    return idx, wr, oracle.bf16_to_f64(xe_bits), xe_d


def _ffn(cfg, D, xe_d, idx_np, w_np, path, with_shared=True, check=True):
    T = xe_d.shape[0]
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    wts = torch.from_numpy(np.ascontiguousarray(w_np, np.float32)).cuda()
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * cfg.k, dtype=torch.int32, device="cuda")
    active = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    moe.moe_bucket(idx, T, cfg.k, cfg.E, offsets, perm, None, active)
    m = torch.full((T, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = moe.workspace(D, T)
    moe.moe_expert_ffn(D, xe_d, T, idx, wts, offsets, perm, active, int(with_shared), m, ws,
                       moe.make_opts(force_path=path))
    torch.cuda.synchronize()
    if check:
        moe.moe_workspace_status(ws)
    return m, ws


@pytest.mark.parametrize("cfg_id,T,sample", [
    (0, 4, None),                  # tiny: 4 row blocks, 4 groups of K
    (0, 40, None),                 # tiny, 10 tokens per expert: two gate/up token groups
    (1, 1, None),                  # Gemma shape, one token
    (1, 33, [0, 17, 32]),          # ragged token count, I = 704 = 22 row blocks, Is = 2112
    (2, 8, None),                  # Qwen-35B shape, 8-token batch
    (3, 16, [0, 7, 15]),           # 512 experts, k = 10
    (4, 128, [0, 1, 77, 127]),     # the 128-token prefill chunk
])
def test_ws_expert_ffn_matches_oracle_and_other_paths(cfg_id, T, sample):
    cfg = synth.CONFIGS[cfg_id]
    base_id = 1 if cfg_id == 4 else cfg_id
    w, D, OL = _layer(synth.CONFIGS[base_id], base_id)
    h = hidden_with_gap(cfg, cfg_id, OL, 5, T) if cfg_id == 0 else synth.gen_hidden(cfg, cfg_id, 5, T)
    idx, wr, xe, xe_d = _routed(cfg, OL, h)
    m_ws, _ = _ffn(cfg, D, xe_d, idx, wr, WS)
    m_ws2, _ = _ffn(cfg, D, xe_d, idx, wr, WS)
    assert torch.equal(m_ws, m_ws2)                                 # fixed summation order
    m_ws = m_ws.cpu().double().numpy()
    assert np.all(np.isfinite(m_ws))
    rows = list(range(T)) if sample is None else sample
    ref = oracle.expert_ffn(OL, xe[rows], idx[rows], wr[rows].astype(np.float32).astype(np.float64))
    err = max_err_vs_rms(m_ws[rows], ref)
    assert err <= OUT_TOL, err
    assert err <= 5e-3, err
    m_gemv = _ffn(cfg, D, xe_d, idx, wr, GEMV)[0].cpu().double().numpy()
    assert max_err_vs_rms(m_ws, m_gemv) <= 5e-3
    if T >= 4:
        m_tc = _ffn(cfg, D, xe_d, idx, wr, TC)[0].cpu().double().numpy()
        assert max_err_vs_rms(m_ws, m_tc) <= 5e-3


def test_ws_dense_mixture_with_and_without_shared_expert():
    """k = E with unit gates equals the dense mixture of all 16 experts."""
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
        m = _ffn(cfg, D, x.cuda(), idx, ones, WS, with_shared)[0].cpu().double().numpy()
        ref = oracle.expert_ffn(OL, x.double().numpy()[rows], idx[rows], ones[rows], with_shared)
        assert max_err_vs_rms(m[rows], ref) <= 5e-3


@pytest.mark.parametrize("dims", [
    dict(H=64, E=8, k=8, I=64, Is=64, T=40),          # K of one group: one warp of eight does the sums
    dict(H=320, E=24, k=5, I=192, Is=320, T=33),      # 5 and 3 groups of K, 6 and 10 row blocks
    dict(H=256, E=8, k=8, I=128, Is=192, T=130),      # every expert holds 130 tokens: 17 / 9 token groups
    dict(H=512, E=16, k=2, I=256, Is=128, T=300),     # the shared expert over 38 / 19 token groups
    dict(H=1024, E=8, k=1, I=1088, Is=64, T=9),       # 17 groups of K in down: warps take 3 or 2
])
def test_ws_edge_shapes(dims):
    T = dims.pop("T")
    cfg = synth.MoEConfig("edge", layers=1, T=T, **dims)
    w, D, OL = _layer(cfg, 98)
    h = synth.gen_hidden(cfg, 98, 0, T)
    hd = h.cuda()
    out = torch.empty_like(hd)
    ws = moe.workspace(D, T)
    moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=WS))
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    rows = sorted({0, 1, T // 2, T - 1})
    ref = oracle.layer_forward(OL, h[rows])
    assert max_err_vs_rms(bf16_host(out)[rows], ref["out_f64"]) <= OUT_TOL


def test_ws_large_scales_and_weights_beyond_fp16():
    """Scales |N(0, 0.3)| and one group of the shared expert's down matrix
    with s = 8192, b = -65536 (weights from -65536 to 57344: beyond FP16,
    which the tcgen05 path reports): the warp-MMA path keeps scale and bias in
    FP32 and the down output is FP32, so it computes the layer to the bar and
    reports nothing."""
    cfg = synth.CONFIGS[0]
    w = synth.gen_layer(cfg, 0, 0, device="cuda", expert_scale_std=0.3)
    w["sh_down_s"][5, 1] = 8192.0                                  # both exact in bf16
    w["sh_down_b"][5, 1] = -65536.0
    D = moe.DeviceLayer.from_config(w, cfg)
    OL = oracle_layer(host(w), cfg)
    T = 32
    h = hidden_with_gap(cfg, 0, OL, 13, T)
    idx, wr, xe, xe_d = _routed(cfg, OL, h)
    m, _ = _ffn(cfg, D, xe_d, idx, wr, WS)                         # status read: no report
    ref = oracle.expert_ffn(OL, xe, idx, wr.astype(np.float32).astype(np.float64))
    # row 5 sums terms up to 65536 * |a| that cancel to a much smaller value, so
    # the FP16 rounding of the SwiGLU inputs a (2^-12 relative) weighs more there
    assert max_err_vs_rms(m.cpu().double().numpy(), ref) <= OUT_TOL
    rest = [r for r in range(cfg.H) if r != 5]                     # the other rows on their own scale
    assert max_err_vs_rms(m.cpu().double().numpy()[:, rest], ref[:, rest]) <= 5e-3
    _, ws = _ffn(cfg, D, xe_d, idx, wr, TC, check=False)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_workspace_status(ws)
    assert "weight" in str(ei.value)


def test_ws_swiglu_outside_fp16_range_is_reported():
    cfg = synth.CONFIGS[0]
    w = synth.gen_layer(cfg, 0, 0, device="cuda", expert_scale_std=10.0)
    D = moe.DeviceLayer.from_config(w, cfg)
    OL = oracle_layer(host(w), cfg)
    h = hidden_with_gap(cfg, 0, OL, 13, 32)
    idx, wr, _, xe_d = _routed(cfg, OL, h)
    _, ws = _ffn(cfg, D, xe_d, idx, wr, WS, check=False)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_workspace_status(ws)
    assert ei.value.code == moe.MOE_EDEVICE and "SwiGLU" in str(ei.value)
    w2 = synth.gen_layer(cfg, 0, 0, device="cuda")
    D2 = moe.DeviceLayer.from_config(w2, cfg)
    OL2 = oracle_layer(host(w2), cfg)
    idx2, wr2, _, xe2_d = _routed(cfg, OL2, h)
    _ffn(cfg, D2, xe2_d, idx2, wr2, WS)                            # the next in-range call: no report


def test_ws_prefill_layer_rows_match_chunked_rows():
    """T = 1024 through the Gemma-shaped layer on this path in one call equals
    the same rows as 8 calls of 128 (the items of a call do not interact),
    and sampled rows match the oracle."""
    cfg = synth.CONFIGS[4]
    w, D, OL = _layer(synth.CONFIGS[1], 1, layer=5)
    T = 1024
    h = synth.gen_hidden(cfg, 4, 7, T)
    hd = h.cuda()
    opts = moe.make_opts(force_path=WS)
    out = torch.empty_like(hd)
    ws = moe.workspace(D, T)
    moe.moe_layer_forward(D, hd, out, T, ws, opts)
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    rows = [0, 127, 128, 555, 1023]
    ref = oracle.layer_forward(OL, h[rows])
    assert max_err_vs_rms(bf16_host(out)[rows], ref["out_f64"]) <= OUT_TOL
    ws128 = moe.workspace(D, 128)
    chunked = torch.empty_like(hd)
    for c in range(8):
        moe.moe_layer_forward(D, hd[c * 128:(c + 1) * 128], chunked[c * 128:(c + 1) * 128], 128, ws128, opts)
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws128)
    assert max_err_vs_rms(bf16_host(out), bf16_host(chunked)) <= 5e-3


@pytest.mark.parametrize("T,path", [(32, WS), (448, WS), (449, TC)])
def test_automatic_path_at_its_boundaries(T, path):
    """force_path 0 takes this path for 32..448 tokens and the tcgen05 GEMM
    above (both measured on B200; the GEMV below 32): the automatic output
    equals the forced path's bit for bit, and sampled rows match the oracle."""
    cfg = synth.CONFIGS[0]
    w, D, OL = _layer(cfg, 0, layer=1)
    h = hidden_with_gap(cfg, 0, OL, 11, T)
    hd = h.cuda()
    ws = moe.workspace(D, T)
    outs = []
    for fp in (0, path):
        out = torch.empty_like(hd)
        moe.moe_layer_forward(D, hd, out, T, ws, moe.make_opts(force_path=fp))
        torch.cuda.synchronize()
        moe.moe_workspace_status(ws)
        outs.append(out)
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    rows = sorted({0, T // 2, T - 1})
    ref = oracle.layer_forward(OL, h[rows])
    assert max_err_vs_rms(bf16_host(outs[0])[rows], ref["out_f64"]) <= OUT_TOL
