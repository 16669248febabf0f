"""moe_layer_forward_noalloc: the layer for callers that cannot allocate.

Callers inside a CUDA-graph capture (where cudaMalloc is not allowed),
serving loops that cannot afford an allocation's device synchronisation, and
plugins whose host framework owns all device memory cannot hand the library
a workspace.  For them the library keeps a fixed scratch array in device
memory.  This test calls that entry point through the C ABI and checks its
output against moe_layer_forward with a caller-provided workspace, on two
calls in a row (the scratch keeps the first call's contents when the second
one starts).  Both run the same kernels on the same inputs, so the outputs
must be bit-identical.  The cases cover the CUDA-core path (T < 32) and the
tensor-core paths (T >= 32 in auto mode, and force_path 2 and 3), whose status words
live in the static scratch and are read back with moe_noalloc_status.  It
lives in its own file, collected last.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from int4_routed_expert_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg_id,T,force_path", [(0, 4, 0), (1, 1, 0), (2, 8, 0), (2, 32, 0), (0, 4, 2),
                                                        (0, 40, 3)])
def test_noalloc_matches_the_workspace_entry_point(cfg_id, T, force_path):
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe

    cfg = synth.CONFIGS[cfg_id]
    w = synth.gen_layer(cfg, cfg_id, 0, device="cuda")
    D = moe.DeviceLayer.from_config(w, cfg)
    assert moe.moe_workspace_size(D, T) <= moe.moe_noalloc_scratch_bytes()
    ws = moe.workspace(D, T)
    opts = moe.make_opts(force_path=force_path)
    lib = moe.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        h = synth.gen_hidden(cfg, cfg_id, 700 + call, T).cuda()
        ref = torch.empty_like(h)
        got = torch.full_like(h, float("nan"))
        moe.moe_layer_forward(D, h, ref, T, ws, opts)
        moe.moe_workspace_status(ws)
        rc = lib.moe_layer_forward_noalloc(D.ptr(), h.data_ptr(), got.data_ptr(), T, C.byref(opts), stream)
        assert rc == moe.MOE_OK, moe.last_error()
        assert lib.moe_noalloc_status(stream) == moe.MOE_OK, moe.last_error()
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"call {call}: outputs differ"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from int4_routed_expert_02_b200 import moe
    cfg = synth.CONFIGS[1]
    w = synth.gen_layer(cfg, 1, 0, device="cuda")
    D = moe.DeviceLayer.from_config(w, cfg)
    T = 256
    assert moe.moe_workspace_size(D, T) > moe.moe_noalloc_scratch_bytes()
    h = torch.zeros(T, cfg.H, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(h)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_forward_noalloc(D, h, out, T)
    assert ei.value.code == moe.MOE_EWORKSPACE and "static scratch" in str(ei.value)
    assert np.all(out.cpu().float().numpy() == 0.0)     # nothing was launched
