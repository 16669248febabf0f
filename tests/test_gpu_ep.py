"""The expert-parallel split through the C ABI on one GPU: every rank's part
(moe_layer_partial with that rank's expert block, and the shared expert on
its owner) computed in turn; their sum must be the whole layer's expert
output (the same fp32 products in another summation order), and moe_combine
of that sum must give moe_layer_forward's output up to one bf16 rounding and
the oracle's within the layer's bar.  The collective itself runs only on
several GPUs; its host logic is tested on CPU ranks (test_ep_gloo.py)."""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth
from int4_routed_expert_02_b200.ep import EPStack, expert_range, shared_owner
from tests.moe_cases import (OUT_TOL, assert_same_up_to_one_rounding, bf16_host, hidden_with_gap, host,
                             max_err_vs_rms, oracle_layer)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe


@pytest.mark.parametrize("cfg_id,T,path", [(0, 4, 0), (0, 64, 2), (1, 33, 0), (2, 8, 1), (1, 40, 3)])
def test_rank_parts_sum_to_the_layer(cfg_id, T, path):
    cfg = synth.CONFIGS[cfg_id]
    w = synth.gen_layer(cfg, cfg_id, 0, device="cuda")
    D = moe.DeviceLayer.from_config(w, cfg)
    OL = oracle_layer(host(w), cfg)
    h = hidden_with_gap(cfg, cfg_id, OL, 3, T) if cfg_id == 0 else synth.gen_hidden(cfg, cfg_id, 3, T)
    hd = h.cuda()
    ws = moe.workspace(D, T)
    opts = moe.make_opts(force_path=path)
    whole = torch.empty(T, cfg.H, dtype=torch.float32, device="cuda")
    moe.moe_layer_partial(D, hd, T, 0, cfg.E, 1, whole, ws, opts)
    ref_out = torch.empty_like(hd)
    moe.moe_layer_forward(D, hd, ref_out, T, ws, opts)
    torch.cuda.synchronize()
    moe.moe_workspace_status(ws)
    ref = oracle.layer_forward(OL, h)
    rows = list(range(T)) if T <= 8 else [0, T // 2, T - 1]
    assert max_err_vs_rms(whole.cpu().double().numpy()[rows], ref["m"][rows]) <= OUT_TOL
    for G in (2, 4):
        total = torch.zeros(T, cfg.H, dtype=torch.float32, device="cuda")
        part = torch.empty_like(total)
        for r in range(G):
            e_lo, e_hi = expert_range(cfg.E, G, r)
            moe.moe_layer_partial(D, hd, T, e_lo, e_hi, shared_owner(0, G) == r, part, ws, opts)
            total += part
        out = torch.empty_like(hd)
        moe.moe_combine(hd, total, out, T, cfg.H)
        torch.cuda.synchronize()
        moe.moe_workspace_status(ws)
        rms = float(whole.double().pow(2).mean().sqrt())
        assert float((total - whole).abs().max()) <= 1e-5 * rms
        assert_same_up_to_one_rounding(out, ref_out)
        assert max_err_vs_rms(bf16_host(out)[rows], ref["out_f64"][rows]) <= OUT_TOL


def test_partial_rejects_bad_ranges():
    cfg = synth.CONFIGS[0]
    D = moe.DeviceLayer.from_config(synth.gen_layer(cfg, 0, 0, device="cuda"), cfg)
    h = torch.zeros(4, cfg.H, dtype=torch.bfloat16, device="cuda")
    m = torch.zeros(4, cfg.H, dtype=torch.float32, device="cuda")
    ws = moe.workspace(D, 4)
    for lo, hi in ((-1, 4), (3, 2), (0, cfg.E + 1)):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_layer_partial(D, h, 4, lo, hi, 1, m, ws)
        assert ei.value.code == moe.MOE_EINVAL
    assert float(m.abs().max()) == 0.0


def test_single_rank_ep_stack_matches_the_per_layer_path():
    """EPStack on one rank (no collective) runs the same chained layers."""
    from int4_routed_expert_02_b200.stack import MoEStack
    cfg = synth.CONFIGS[1]
    T, L = 16, 3
    st = MoEStack(cfg, 1, T=T, layers=L, persistent=False)
    ep = EPStack(cfg, 1, T, rank=0, world=1, layers=L, device_layers=st.layers)
    h = synth.gen_hidden(cfg, 1, 9, T).cuda()
    st.set_input(h)
    st.run()
    ep.set_input(h)
    ep.run()
    torch.cuda.synchronize()
    for l in range(L):
        assert_same_up_to_one_rounding(ep.buf[l + 1], st.outputs[l])
