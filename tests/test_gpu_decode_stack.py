"""The persistent decode kernel (moe_decode_stack) against the per-layer path
(moe_layer_forward) and the fp64 oracle.  Each layer is checked teacher-forced:
on exactly the bf16 input the kernel gave it."""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth
from tests.moe_cases import (OUT_TOL, assert_same_up_to_one_rounding, bf16_host, host, max_err_vs_rms,
                             oracle_layer)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.stack import MoEStack


def _check_stack(st, cfg, cfg_id, oracle_layers=(0,), tol=OUT_TOL):
    st.status()
    ws = moe.workspace(st.layers[0], st.T)
    for l in range(st.L):
        h_in = st.inputs[l]
        ref = torch.empty_like(h_in)
        moe.moe_layer_forward(st.layers[l], h_in, ref, st.T, ws)
        torch.cuda.synchronize()
        assert_same_up_to_one_rounding(st.outputs[l], ref)
    for l in oracle_layers:
        w = host(synth.gen_layer(cfg, cfg_id, l, device="cuda"))
        OL = oracle_layer(w, cfg)
        ref = oracle.layer_forward(OL, st.inputs[l].cpu())
        err = max_err_vs_rms(bf16_host(st.outputs[l]), ref["out_f64"])
        assert err <= tol, f"layer {l}: {err:.3e} vs the oracle"


@pytest.mark.parametrize("cfg_id,T,L,path", [(0, 4, 3, 0), (0, 1, 2, 0), (1, 1, 4, 0), (1, 8, 2, 0), (2, 4, 3, 0),
                                              (2, 8, 2, 0), (0, 4, 2, 1), (1, 1, 3, 2), (2, 2, 2, 1), (2, 3, 2, 2),
                                              (2, 8, 2, 1)])
def test_decode_stack_matches_per_layer_path_and_oracle(cfg_id, T, L, path):
    """path 0: automatic (CUDA-core FMAs for T = 1, tensor cores for T >= 2);
    1 and 2 force the CUDA-core and the tensor-core variants."""
    cfg = synth.CONFIGS[cfg_id]
    st = MoEStack(cfg, cfg_id, T=T, layers=L, opts=moe.make_opts(force_path=path))
    assert st.persistent
    for step in range(2):   # second call reuses the workspace and the ring state
        st.set_input(synth.gen_hidden(cfg, cfg_id, 500 + step, T).cuda())
        st.run()
        torch.cuda.synchronize()
        _check_stack(st, cfg, cfg_id, oracle_layers=(0, L - 1) if step == 1 else ())


@pytest.mark.parametrize("T", [1, 2])
def test_decode_stack_unchained_zipf_inputs(T):
    """512 experts (16 groups of 32 in the kernel's top-k) with the Zipf-routed
    inputs, on the CUDA-core (T = 1) and the tensor-core (T = 2) variants."""
    cfg = synth.CONFIGS[3]
    L = 3
    st = MoEStack(cfg, 3, T=T, layers=L, keep_router_codes=True)
    h = torch.stack([synth.gen_zipf_hidden(cfg, 3, l, 0, st.router_codes[l], T=T)[0] for l in range(L)])
    st.set_input(h.cuda())
    st.run()
    torch.cuda.synchronize()
    _check_stack(st, cfg, 3, oracle_layers=(1,))


@pytest.mark.parametrize("cfg_id,T,tie", [(1, 1, "all"), (1, 2, "pairs"), (2, 1, "pairs"), (3, 1, "all"),
                                           (3, 2, "pairs")])
def test_decode_stack_top_k_ties_go_to_the_lower_index(cfg_id, T, tie):
    """Router rows made identical, so that logits tie exactly: "all" (every
    expert the same: the top k must be experts 0..k-1) or "pairs" (expert e
    and e + E/2 the same: the two sit in different groups of 32 for E >= 64,
    and the lower one must win where the pair straddles the k-th place).  The
    experts' own weights differ, so a wrong pick changes the output far beyond
    the bar; the kernel is checked against the oracle and the per-layer path."""
    cfg = synth.CONFIGS[cfg_id]
    L = 2
    ws_, OLs, Ds = [], [], []
    for l in range(L):
        w = synth.gen_layer(cfg, cfg_id, l, device="cuda")
        if tie == "all":
            for key in ("router_q", "router_s", "router_b"):
                w[key][:] = w[key][0]
        else:
            half = cfg.E // 2
            for key in ("router_q", "router_s", "router_b"):
                w[key][half:] = w[key][:half]
        Ds.append(moe.DeviceLayer.from_config(w, cfg))
        OLs.append(oracle_layer(host(w), cfg))
    st = MoEStack(cfg, cfg_id, T=T, layers=L, device_layers=Ds)
    assert st.persistent
    h = synth.gen_hidden(cfg, cfg_id, 900, T).cuda()
    if not cfg.chained:
        h = h.unsqueeze(0).expand(L, T, cfg.H).contiguous()
    st.set_input(h)
    st.run()
    torch.cuda.synchronize()
    st.status()
    ws = moe.workspace(st.layers[0], T)
    for l in range(L):
        h_in = st.inputs[l]
        ref = torch.empty_like(h_in)
        moe.moe_layer_forward(st.layers[l], h_in, ref, T, ws)
        torch.cuda.synchronize()
        assert_same_up_to_one_rounding(st.outputs[l], ref)
        out = oracle.layer_forward(OLs[l], h_in.cpu())
        if tie == "all":
            assert all(list(r) == list(range(cfg.k)) for r in out["idx"])
        assert max_err_vs_rms(bf16_host(st.outputs[l]), out["out_f64"]) <= OUT_TOL


@pytest.mark.parametrize("dims", [
    dict(H=64, E=8, k=8, I=64, Is=64, T=3),           # k = E: every token uses every expert
    dict(H=320, E=24, k=5, I=192, Is=1088, T=5),      # ragged groups, 2 shared down parts
    dict(H=4096, E=32, k=2, I=1088, Is=128, T=2),     # widest hidden, 2 routed down parts
])
def test_decode_stack_edge_shapes(dims):
    T = dims.pop("T")
    cfg = synth.MoEConfig("edge", layers=2, T=T, **dims)
    st = MoEStack(cfg, 98, T=T)
    st.set_input(synth.gen_hidden(cfg, 98, 1, T).cuda())
    st.run()
    torch.cuda.synchronize()
    _check_stack(st, cfg, 98, oracle_layers=(0,))


def test_decode_stack_is_deterministic_and_rejects_bad_sizes():
    cfg = synth.CONFIGS[1]
    st = MoEStack(cfg, 1, T=1, layers=2)
    st.set_input(synth.gen_hidden(cfg, 1, 3, 1).cuda())
    st.run()
    a = st.h_out.clone()
    st.run()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), st.h_out.view(torch.int16))
    assert moe.moe_decode_stack_workspace_size(st.layers[0], 9) == 0
    with pytest.raises(moe.MoEError):
        moe.moe_decode_stack(st.larr, 2, st.buf[0], 1, st.h_out, 9, st.ws_dec)


def test_barrier_timeout_is_reported_and_the_context_survives(monkeypatch):
    """The grid barrier's bounded wait runs out (a test hook makes it wait for
    one arrival more than the grid has): the kernel records the code, every CTA
    returns, the status call reports MOE_EDEVICE, and the next call is fine."""
    cfg = synth.CONFIGS[0]
    st = MoEStack(cfg, 0, T=1, layers=1)
    st.set_input(synth.gen_hidden(cfg, 0, 3, 1).cuda())
    monkeypatch.setenv("MOE_TEST_BARRIER_EXTRA", "1")
    st.run()
    torch.cuda.synchronize()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_decode_stack_status(st.ws_dec)
    assert ei.value.code == moe.MOE_EDEVICE and "grid barrier timed out" in str(ei.value)
    monkeypatch.delenv("MOE_TEST_BARRIER_EXTRA")
    st.run()
    torch.cuda.synchronize()
    moe.moe_decode_stack_status(st.ws_dec)
    assert torch.isfinite(st.final_output().float()).all()
