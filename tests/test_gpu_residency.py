"""Tiered expert residency through the C ABI (moe_layer_forward_cached): the
routed experts in pinned host memory, a device cache of C slots per layer.

The cached layer must give moe_layer_forward's output bit for bit (the same
kernels on the same bytes, reached through slot ids), and its decisions must
be the replacement rule's: the test replays every call's selected experts
through the CPU model of the rule (tests/test_residency_policy.py) and
compares the hit and miss counts and the slot of every expert."""
import pytest
import torch

from int4_routed_expert_02_b200 import synth
from tests.test_residency_policy import CacheModel

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe
    from int4_routed_expert_02_b200.residency import CachedLayer, CachedStack


def _selected(D, h, T, cfg, ws):
    idx = torch.empty(T, cfg.k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, cfg.k, dtype=torch.float32, device="cuda")
    moe.moe_router(D, h, T, idx, wts, None, ws)
    torch.cuda.synchronize()
    return idx.flatten().tolist()


@pytest.mark.parametrize("cfg_id,T,slots,path", [(0, 1, 6, 0), (0, 4, 16, 0), (1, 1, 16, 0), (2, 4, 40, 1),
                                                 (0, 40, 16, 2), (0, 24, 16, 3)])
def test_cached_layer_matches_the_resident_layer_and_the_rule(cfg_id, T, slots, path):
    cfg = synth.CONFIGS[cfg_id]
    D = moe.DeviceLayer.from_config(synth.gen_layer(cfg, cfg_id, 0, device="cuda"), cfg)
    cl = CachedLayer(D, slots)
    model = CacheModel(cfg.E, slots)
    ws = moe.workspace(D, T)
    opts = moe.make_opts(force_path=path)
    for step in range(12):
        h = synth.gen_hidden(cfg, cfg_id, 300 + step % 7, T).cuda()   # streams repeat: some hits
        ref = torch.empty_like(h)
        got = torch.full_like(h, float("nan"))
        moe.moe_layer_forward(D, h, ref, T, ws, opts)
        moe.moe_layer_forward_cached(D, cl.struct, h, got, T, ws, opts)
        torch.cuda.synchronize()
        moe.moe_workspace_status(ws)
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"step {step}"
        model.call(_selected(D, h, T, cfg, ws))
        st = cl.stats()
        assert (st["calls"], st["hits"], st["misses"]) == (step + 1, model.hits, model.misses)
        assert cl.slot_of.cpu().tolist() == model.slot_of
        assert cl.expert_of.cpu().tolist() == model.expert_of


def test_cached_stack_serves_a_chained_stack_from_host_memory():
    """Three Gemma-shaped layers with the pages' 16 slots each, their routed
    experts only in host memory, against the resident stack."""
    from int4_routed_expert_02_b200.stack import MoEStack
    cfg = synth.CONFIGS[1]
    L, T = 3, 1
    ref = MoEStack(cfg, 1, T=T, layers=L, persistent=False)
    cs = CachedStack(cfg, 1, T, slots=16, layers=L)
    for step in range(6):
        h = synth.gen_hidden(cfg, 1, 40 + step, T).cuda()
        ref.set_input(h)
        ref.run()
        cs.set_input(h)
        cs.run()
        torch.cuda.synchronize()
        assert torch.equal(cs.final_output().view(torch.int16), ref.final_output().view(torch.int16))
    s = cs.stats()
    assert s["calls"] == 6 * L and s["hits"] + s["misses"] == 6 * L * cfg.k
    assert all(l.dl.struct.gate.q is None for l in cs.layers)   # the routed experts left HBM


def test_cached_layer_rejects_too_few_slots():
    cfg = synth.CONFIGS[0]
    D = moe.DeviceLayer.from_config(synth.gen_layer(cfg, 0, 0, device="cuda"), cfg)
    cl = CachedLayer(D, 3)                    # T = 1 selects 4 experts
    h = torch.zeros(1, cfg.H, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(h)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_forward_cached(D, cl.struct, h, out, 1, moe.workspace(D, 1))
    assert ei.value.code == moe.MOE_EINVAL and "slots" in str(ei.value)
