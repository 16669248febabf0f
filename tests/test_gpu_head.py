"""One 4-bit matrix times a few rows through the C ABI (moe_qmat_gemv), e.g. the
vocabulary-sized output head that shares the embedding's quantised weights,
against the fp64 oracle.

Each group's products are exact on the GPU (code times pre-scaled input) and
accumulate in fp32, so the bar is fp32 summation error: max|err| <= 1e-4 *
rms(reference).  Cases: small shapes with every row checked (1, 3 and 8 input
rows; one-group and widest inputs), the full vocabulary shape (262,144 x 2816)
on sampled rows, and argument errors.
"""
import numpy as np
import pytest
import torch

import oracle
from int4_routed_expert_02_b200 import synth
from tests.moe_cases import max_err_vs_rms

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from int4_routed_expert_02_b200 import build
    build.build()
    from int4_routed_expert_02_b200 import moe

TOL = 1e-4


def _head(rows, cols, seed):
    cfg = synth.MoEConfig("head", H=cols, E=8, k=1, I=64, Is=64, layers=1, T=1)
    w = synth.gen_vocab_head(cfg, 97, rows, seed=seed, device="cuda")
    qt, sbt = moe.prepare_qmat(w["head_q"], w["head_s"], w["head_b"], 1, rows, cols)
    return w, qt, sbt


def _run(qt, sbt, rows, cols, x):
    T = x.shape[0]
    y = torch.empty(T, rows, dtype=torch.float32, device="cuda")
    moe.moe_qmat_gemv(qt, sbt, rows, cols, x, T, y, moe.qmat_gemv_workspace())
    torch.cuda.synchronize()
    return y.cpu().double().numpy()


def _x(T, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(T, cols, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols,T", [(256, 256, 1), (96, 320, 3), (128, 64, 8), (64, 8192, 2), (1024, 2816, 4)])
def test_qmat_gemv_matches_oracle_every_row(rows, cols, T):
    w, qt, sbt = _head(rows, cols, seed=rows + cols)
    x = _x(T, cols, seed=T)
    y = _run(qt, sbt, rows, cols, x.cuda())
    ref = oracle.qmat_gemv(w["head_q"], w["head_s"], w["head_b"], rows, cols, x.float().double().numpy())
    assert max_err_vs_rms(y, ref) <= TOL


def test_qmat_gemv_full_vocabulary_sampled_rows():
    V, H = 262144, 2816
    w, qt, sbt = _head(V, H, seed=1)
    x = _x(1, H, seed=11)
    y = _run(qt, sbt, V, H, x.cuda())
    rows = [0, 31, 32, 4095, 131071, 200000, V - 33, V - 1]
    sub = {k: w[k][rows] for k in ("head_q", "head_s", "head_b")}
    ref = oracle.qmat_gemv(sub["head_q"], sub["head_s"], sub["head_b"], len(rows), H, x.float().double().numpy())
    assert max_err_vs_rms(y[:, rows], ref) <= TOL
    assert np.all(np.isfinite(y))
    # a second call reuses the workspace (its work counter is reset by the call)
    y2 = _run(qt, sbt, V, H, x.cuda())
    assert np.array_equal(y, y2)


def test_qmat_gemv_rejects_bad_arguments():
    rows, cols = 64, 128
    w, qt, sbt = _head(rows, cols, seed=3)
    x = _x(9, cols, seed=0).cuda()
    y = torch.empty(9, rows, dtype=torch.float32, device="cuda")
    ws = moe.qmat_gemv_workspace()
    for T in (0, 9):
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_qmat_gemv(qt, sbt, rows, cols, x, T, y, ws)
        assert ei.value.code == moe.MOE_EINVAL
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_qmat_gemv(qt, sbt, 48, cols, x, 1, y, ws)
    assert ei.value.code == moe.MOE_EINVAL
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_qmat_gemv(qt, sbt, rows, cols, x, 1, y, ws[:8])
    assert ei.value.code == moe.MOE_EWORKSPACE


def test_qmat_gemv_replays_from_a_cuda_graph_on_a_side_stream():
    """Captured on a non-default stream after one eager call, the head GEMV
    replays to the eager result bit for bit (the launch sizes its grid for
    the stream's device without a query that the capture refuses)."""
    rows, cols, T = 1024, 2816, 2
    _, qt, sbt = _head(rows, cols, 5)
    x = _x(T, cols, 6).cuda()
    ws = moe.qmat_gemv_workspace()
    eager = torch.empty(T, rows, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        moe.moe_qmat_gemv(qt, sbt, rows, cols, x, T, eager, ws, stream=s)
    s.synchronize()
    out = torch.full_like(eager, float("nan"))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_qmat_gemv(qt, sbt, rows, cols, x, T, out, ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
