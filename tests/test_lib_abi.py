"""The C-ABI library loads, exports every symbol include/*.h declares, and
rejects bad arguments on the host before touching the GPU.  CPU only: no
call here reaches a kernel launch (invalid arguments are refused first, and
T == 0 enqueues nothing)."""
import ctypes as C
import glob
import os
import re

import pytest

from int4_routed_expert_02_b200 import build

build.build()
from int4_routed_expert_02_b200 import moe  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        for m in re.finditer(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", open(h).read(), re.M):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    names = declared_symbols()
    assert len(names) >= 10
    lib = C.CDLL(moe.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(moe.EXPORTED) <= set(names)


def test_version_and_empty_error():
    assert "sm_100a" in moe.version()


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first


def fake_layer(H=256, E=16, k=4, I=128, Is=128, ptr=FAKE):
    st = moe.LayerW(H=H, E=E, k=k, I=I, Is=Is)
    for n in ("router_q", "router_s", "router_b", "router_scale", "per_expert_scale"):
        setattr(st, n, ptr)
    for n in ("gate", "up", "down", "sh_gate", "sh_up", "sh_down"):
        setattr(st, n, moe.QMat(ptr, ptr))
    return st


def fwd(st, T=4, h_in=FAKE, h_out=FAKE * 4, ws=FAKE * 8, ws_bytes=1 << 40, opts=None):
    o = opts if opts is not None else moe.make_opts()
    return moe.lib().moe_layer_forward(C.addressof(st), h_in, h_out, T, ws, ws_bytes, C.byref(o), None)


@pytest.mark.parametrize("kw,frag", [
    (dict(H=100), "H=100"), (dict(H=0), "H=0"), (dict(I=96), "I=96"), (dict(Is=32), "Is=32"),
    (dict(E=12), "E=12"), (dict(E=2048), "E=2048"), (dict(k=0), "k=0"), (dict(k=17), "k=17"),
    (dict(E=64, k=33), "k=33"), (dict(H=16384), "H=16384"),
])
def test_bad_dims_are_rejected(kw, frag):
    rc = fwd(fake_layer(**kw))
    assert rc == moe.MOE_EINVAL
    assert frag in moe.last_error()


def test_null_and_misaligned_pointers():
    st = fake_layer()
    st.router_q = None
    assert fwd(st) == moe.MOE_EINVAL and "router_q" in moe.last_error()
    st = fake_layer()
    st.down = moe.QMat(FAKE + 4, FAKE)
    assert fwd(st) == moe.MOE_EALIGN and "down.q" in moe.last_error()
    assert fwd(fake_layer(), h_in=FAKE + 2) == moe.MOE_EALIGN
    assert fwd(fake_layer(), h_out=None) == moe.MOE_EINVAL


def test_negative_T_and_overlap_and_workspace():
    assert fwd(fake_layer(), T=-1) == moe.MOE_EINVAL
    assert fwd(fake_layer(), T=70000) == moe.MOE_EINVAL
    assert fwd(fake_layer(), h_in=FAKE, h_out=FAKE + 256) == moe.MOE_EINVAL and "overlaps" in moe.last_error()
    st = fake_layer()
    need = moe.lib().moe_workspace_size(C.addressof(st), 4)
    assert need > 0
    assert fwd(st, ws_bytes=need - 1) == moe.MOE_EWORKSPACE
    assert fwd(st, ws=None) == moe.MOE_EWORKSPACE
    assert fwd(st, ws=FAKE + 8) == moe.MOE_EALIGN


def test_empty_call_is_a_valid_no_op():
    assert fwd(fake_layer(), T=0, ws_bytes=0, ws=FAKE) == moe.MOE_OK
    assert moe.lib().moe_bucket(FAKE, 0, 4, 16, FAKE, FAKE, None, None, None) == moe.MOE_OK


def test_opts_validation():
    assert fwd(fake_layer(), opts=moe.make_opts(force_path=7)) == moe.MOE_EINVAL
    assert fwd(fake_layer(), opts=moe.make_opts(eps=-1.0)) == moe.MOE_EINVAL


def test_workspace_size_grows_with_T_and_rejects_bad_dims():
    st = fake_layer()
    ws = [moe.lib().moe_workspace_size(C.addressof(st), T) for T in (0, 1, 4, 128)]
    assert ws[0] > 0 and ws == sorted(ws) and ws[3] > ws[2]
    assert moe.lib().moe_workspace_size(C.addressof(fake_layer(H=100)), 4) == 0
    assert moe.lib().moe_workspace_size(C.addressof(st), -1) == 0


def test_other_entry_points_validate():
    L = moe.lib()
    st = fake_layer()
    assert L.moe_router_topk(FAKE, 4, 16, 17, FAKE, FAKE, FAKE, None) == moe.MOE_EINVAL
    assert L.moe_router_topk(FAKE, 4, 2000, 4, FAKE, FAKE, FAKE, None) == moe.MOE_EINVAL
    assert L.moe_bucket(FAKE, 10000, 8, 16, FAKE, FAKE, None, None, None) == moe.MOE_EINVAL   # T*k > 65536
    assert L.moe_bucket(FAKE + 1, 4, 4, 16, FAKE, FAKE, None, None, None) == moe.MOE_EALIGN
    assert L.moe_prepare_qmat(FAKE, FAKE, FAKE, 1, 48, 64, FAKE, FAKE, None) == moe.MOE_EINVAL
    assert L.moe_prepare_qmat(FAKE, FAKE, FAKE, 1, 32, 96, FAKE, FAKE, None) == moe.MOE_EINVAL
    assert L.moe_router_logits(C.addressof(st), None, 4, FAKE, None, None) == moe.MOE_EINVAL
    assert L.moe_router(C.addressof(st), FAKE, 4, FAKE, FAKE, None, FAKE, 16, None) == moe.MOE_EWORKSPACE
    assert L.moe_expert_ffn(C.addressof(st), FAKE, 4, FAKE, FAKE, FAKE, FAKE, None, 1, FAKE, FAKE, 1 << 40,
                            None, None) == moe.MOE_EINVAL


def _stack(layers, L, T, ws_bytes=1 << 40, h_in=FAKE, h_out=FAKE * 4):
    arr = (moe.LayerW * len(layers))(*layers)
    return moe.lib().moe_decode_stack(C.addressof(arr), L, h_in, 1, h_out, T, FAKE * 8, ws_bytes,
                                      C.byref(moe.make_opts()), None)


def test_decode_stack_validation():
    a = fake_layer()
    assert _stack([a], 0, 1) == moe.MOE_EINVAL
    assert _stack([a] * 65, 65, 1) == moe.MOE_EINVAL
    assert _stack([a], 1, 9) == moe.MOE_EINVAL and "T=9" in moe.last_error()
    assert _stack([a, fake_layer(I=192)], 2, 1) == moe.MOE_EINVAL and "different shape" in moe.last_error()
    assert _stack([fake_layer(H=8192)], 1, 1) == moe.MOE_EINVAL
    assert _stack([fake_layer(H=4096)], 1, 8) == moe.MOE_EINVAL and "T*H" in moe.last_error()
    assert _stack([a], 1, 0) == moe.MOE_OK
    assert _stack([a], 1, 2, ws_bytes=16) == moe.MOE_EWORKSPACE
    assert moe.lib().moe_decode_stack_workspace_size(C.addressof(a), 9) == 0
    assert moe.lib().moe_decode_stack_workspace_size(C.addressof(a), 8) > 0


def test_qmat_gemv_validation():
    L = moe.lib()
    ws = L.moe_qmat_gemv_workspace_size()
    assert ws >= 4
    m = moe.QMat(FAKE, FAKE)

    def call(rows, cols, T, x=FAKE, y=FAKE, wsp=FAKE, wsb=ws, mat=m):
        return L.moe_qmat_gemv(C.byref(mat) if mat is not None else None, rows, cols, x, T, y, wsp, wsb, None)

    assert call(48, 64, 1) == moe.MOE_EINVAL                     # rows not a multiple of 32
    assert call(64, 96, 1) == moe.MOE_EINVAL                     # cols not a multiple of 64
    assert call(64, 16384, 1) == moe.MOE_EINVAL                  # cols above the limit
    assert call(64, 64, 0) == moe.MOE_EINVAL and call(64, 64, 9) == moe.MOE_EINVAL
    assert call(64, 8192, 8) == moe.MOE_EINVAL and "shared-memory" in moe.last_error()
    assert call(64, 64, 1, mat=None) == moe.MOE_EINVAL
    assert call(64, 64, 1, mat=moe.QMat(FAKE + 4, FAKE)) == moe.MOE_EALIGN
    assert call(64, 64, 1, x=FAKE + 2) == moe.MOE_EALIGN
    assert call(64, 64, 1, y=None) == moe.MOE_EINVAL
    assert call(64, 64, 1, wsb=ws - 1) == moe.MOE_EWORKSPACE


def test_new_entry_points_reject_bad_arguments_before_any_launch():
    st = fake_layer()
    lib = moe.lib()
    o = moe.make_opts()
    # expert-parallel part: an empty or reversed expert range, an out-of-range end
    for lo, hi in ((3, 2), (-1, 4), (0, 17)):
        rc = lib.moe_layer_partial(C.addressof(st), FAKE, 4, lo, hi, 1, FAKE * 2, FAKE * 8, 1 << 40, C.byref(o), None)
        assert rc == moe.MOE_EINVAL and "expert range" in moe.last_error()
    # combine: hidden size not a multiple of 64, a null pointer, T = 0 enqueues nothing
    assert lib.moe_combine(FAKE, FAKE * 2, FAKE * 4, 4, 100, C.byref(o), None) == moe.MOE_EINVAL
    assert lib.moe_combine(None, FAKE * 2, FAKE * 4, 4, 256, C.byref(o), None) == moe.MOE_EINVAL
    assert lib.moe_combine(FAKE, FAKE * 2, FAKE * 4, 0, 256, C.byref(o), None) == moe.MOE_OK
    # expert cache: no slots; fewer slots than one call can select (T=4, k=4 -> 16 of E=16)
    c = moe.ExpertCache(slots=0)
    assert lib.moe_expert_cache_reset(C.addressof(c), 16, None) == moe.MOE_EINVAL
    c = moe.ExpertCache(slots=8)
    for n in ("gate", "up", "down", "pool_gate", "pool_up", "pool_down"):
        setattr(c, n, moe.QMat(FAKE, FAKE))
    c.slot_of = c.expert_of = c.uses = c.last = c.ctl = FAKE
    rc = lib.moe_layer_forward_cached(C.addressof(st), C.addressof(c), FAKE, FAKE * 4, 4, FAKE * 8, 1 << 40,
                                      C.byref(o), None)
    assert rc == moe.MOE_EINVAL and "slots" in moe.last_error()
    # T = 1 selects 4 experts: 8 slots pass the size check, and a null pool pointer is then caught
    c.pool_down = moe.QMat(None, FAKE)
    rc = lib.moe_layer_forward_cached(C.addressof(st), C.addressof(c), FAKE, FAKE * 4, 1, FAKE * 8, 1 << 40,
                                      C.byref(o), None)
    assert rc == moe.MOE_EINVAL
    # the decode kernel's fit query answers 0 on bad sizes (and without a device)
    assert lib.moe_decode_stack_fits(C.addressof(st), 9, None) == 0
    assert lib.moe_decode_stack_fits(C.addressof(fake_layer(H=100)), 1, None) == 0
