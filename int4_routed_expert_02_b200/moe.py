"""Thin ctypes binding of libmoe.so (see include/moe_api.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  torch tensors are used as device buffers; the CUDA stream
defaults to torch's current stream.  Importing this module loads the library
and raises ImportError when it is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libmoe.so not built ({LIB_PATH}); run `python -m int4_routed_expert_02_b200.build`")
_lib = C.CDLL(LIB_PATH)

MOE_OK, MOE_EINVAL, MOE_EALIGN, MOE_EWORKSPACE, MOE_ECUDA, MOE_EDEVICE = 0, -1, -2, -3, -4, -5
EXPORTED = ("moe_last_error", "moe_version", "moe_prepare_qmat", "moe_workspace_size", "moe_router_logits",
            "moe_router_topk", "moe_router", "moe_bucket", "moe_expert_ffn", "moe_layer_forward",
            "moe_noalloc_scratch_bytes", "moe_layer_forward_noalloc", "moe_decode_stack_workspace_size",
            "moe_decode_stack", "moe_decode_stack_status", "moe_workspace_status", "moe_qmat_gemv_workspace_size",
            "moe_qmat_gemv", "moe_noalloc_status", "moe_decode_stack_fits", "moe_layer_partial", "moe_combine",
            "moe_expert_cache_reset", "moe_layer_forward_cached")


class MoEError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


class QMat(C.Structure):
    _fields_ = [("q", C.c_void_p), ("sb", C.c_void_p)]


class LayerW(C.Structure):
    _fields_ = [("H", C.c_int), ("E", C.c_int), ("k", C.c_int), ("I", C.c_int), ("Is", C.c_int),
                ("router_q", C.c_void_p), ("router_s", C.c_void_p), ("router_b", C.c_void_p),
                ("router_scale", C.c_void_p), ("per_expert_scale", C.c_void_p),
                ("gate", QMat), ("up", QMat), ("down", QMat),
                ("sh_gate", QMat), ("sh_up", QMat), ("sh_down", QMat)]


class ExpertCache(C.Structure):
    _fields_ = [("slots", C.c_int), ("gate", QMat), ("up", QMat), ("down", QMat),
                ("pool_gate", QMat), ("pool_up", QMat), ("pool_down", QMat),
                ("slot_of", C.c_void_p), ("expert_of", C.c_void_p), ("uses", C.c_void_p), ("last", C.c_void_p),
                ("ctl", C.c_void_p)]


class Opts(C.Structure):
    _fields_ = [("post_norm", C.c_int), ("layer_scalar", C.c_float), ("eps", C.c_float), ("force_path", C.c_int)]


_P, _I = C.c_void_p, C.c_int
_lib.moe_last_error.restype = C.c_char_p
_lib.moe_version.restype = C.c_char_p
_lib.moe_prepare_qmat.argtypes = [_P, _P, _P, _I, _I, _I, _P, _P, _P]
_lib.moe_workspace_size.argtypes = [_P, _I]
_lib.moe_workspace_size.restype = C.c_size_t
_lib.moe_router_logits.argtypes = [_P, _P, _I, _P, _P, _P]
_lib.moe_router_topk.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
_lib.moe_router.argtypes = [_P, _P, _I, _P, _P, _P, _P, C.c_size_t, _P]
_lib.moe_bucket.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P, _P]
_lib.moe_expert_ffn.argtypes = [_P, _P, _I, _P, _P, _P, _P, _P, _I, _P, _P, C.c_size_t, _P, _P]
_lib.moe_layer_forward.argtypes = [_P, _P, _P, _I, _P, C.c_size_t, _P, _P]
_lib.moe_noalloc_scratch_bytes.restype = C.c_size_t
_lib.moe_decode_stack_workspace_size.argtypes = [_P, _I]
_lib.moe_decode_stack_workspace_size.restype = C.c_size_t
_lib.moe_decode_stack.argtypes = [_P, _I, _P, _I, _P, _I, _P, C.c_size_t, _P, _P]
_lib.moe_decode_stack_status.argtypes = [_P]
_lib.moe_decode_stack_fits.argtypes = [_P, _I, _P]
_lib.moe_layer_partial.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, C.c_size_t, _P, _P]
_lib.moe_combine.argtypes = [_P, _P, _P, _I, _I, _P, _P]
_lib.moe_expert_cache_reset.argtypes = [_P, _I, _P]
_lib.moe_layer_forward_cached.argtypes = [_P, _P, _P, _P, _I, _P, C.c_size_t, _P, _P]
_lib.moe_workspace_status.argtypes = [_P]
_lib.moe_layer_forward_noalloc.argtypes = [_P, _P, _P, _I, _P, _P]
_lib.moe_noalloc_status.argtypes = [_P]
_lib.moe_qmat_gemv_workspace_size.restype = C.c_size_t
_lib.moe_qmat_gemv.argtypes = [_P, _I, _I, _P, _I, _P, _P, C.c_size_t, _P]


def lib():
    return _lib


def last_error() -> str:
    return _lib.moe_last_error().decode()


def version() -> str:
    return _lib.moe_version().decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != MOE_OK:
        raise MoEError(rc, last_error())


def _opts(post_norm=True, layer_scalar=1.0, eps=1e-6, force_path=0):
    return Opts(int(post_norm), float(layer_scalar), float(eps), int(force_path))


# ---------------------------------------------------------------- weights

def moe_prepare_qmat(q, scale, bias, n_mat, rows, cols, q_out, sb_out, stream=None):
    _check(_lib.moe_prepare_qmat(_ptr(q), _ptr(scale), _ptr(bias), n_mat, rows, cols, _ptr(q_out), _ptr(sb_out),
                                 _stream(stream)))


def prepare_qmat(q, scale, bias, n_mat, rows, cols, stream=None):
    """MLX-layout matrices (device tensors) -> (q_tiled, sb_tiled) device tensors."""
    q_out = torch.empty(n_mat * rows * cols // 8, dtype=torch.int32, device=q.device)
    sb_out = torch.empty(n_mat * rows * cols // 64, dtype=torch.int32, device=q.device)
    moe_prepare_qmat(q, scale, bias, n_mat, rows, cols, q_out, sb_out, stream)
    return q_out, sb_out


class DeviceLayer:
    """One layer's weights on the device in the library's layout, and the
    moe_layer_w struct that points at them.  `weights` is a dict of MLX-layout
    tensors as produced by synth.gen_layer (moved to `device` if needed)."""

    _MATS = (("gate", "I", "H", True), ("up", "I", "H", True), ("down", "H", "I", True),
             ("sh_gate", "Is", "H", False), ("sh_up", "Is", "H", False), ("sh_down", "H", "Is", False))

    def __init__(self, weights: dict, H: int, E: int, k: int, I: int, Is: int, device="cuda", keep_mlx=False):
        self.H, self.E, self.k, self.I, self.Is = H, E, k, I, Is
        dims = dict(H=H, E=E, I=I, Is=Is)
        dev = torch.device(device)
        self.t = {}
        for n in ("router_q", "router_s", "router_b", "router_scale", "per_expert_scale"):
            self.t[n] = weights[n].to(dev).contiguous()
        st = LayerW(H=H, E=E, k=k, I=I, Is=Is)
        for n in ("router_q", "router_s", "router_b", "router_scale", "per_expert_scale"):
            setattr(st, n, self.t[n].data_ptr())
        for name, r, c, routed in self._MATS:
            rows, cols = dims[r], dims[c]
            n_mat = E if routed else 1
            q = weights[name + "_q"].to(dev).contiguous()
            s = weights[name + "_s"].to(dev).contiguous()
            b = weights[name + "_b"].to(dev).contiguous()
            qt, sbt = prepare_qmat(q, s, b, n_mat, rows, cols)
            self.t[name + "_qt"], self.t[name + "_sbt"] = qt, sbt
            if keep_mlx:
                self.t[name + "_q"], self.t[name + "_s"], self.t[name + "_b"] = q, s, b
            setattr(st, name, QMat(qt.data_ptr(), sbt.data_ptr()))
        self.struct = st

    @classmethod
    def from_config(cls, weights, cfg, device="cuda", keep_mlx=False):
        return cls(weights, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is, device=device, keep_mlx=keep_mlx)

    def ptr(self):
        return C.addressof(self.struct)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.t.values())


# ---------------------------------------------------------------- calls

def moe_workspace_size(layer, T_max: int) -> int:
    return int(_lib.moe_workspace_size(layer.ptr(), T_max))


def workspace(layer, T_max: int, device="cuda") -> torch.Tensor:
    n = moe_workspace_size(layer, T_max)
    if n == 0:
        raise MoEError(MOE_EINVAL, "moe_workspace_size returned 0")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_router_logits(layer, h, logits, xe=None, stream=None):
    _check(_lib.moe_router_logits(layer.ptr(), _ptr(h), h.shape[0] if hasattr(h, "shape") else 0, _ptr(logits),
                                  _ptr(xe), _stream(stream)))


def moe_router_topk(logits, T, E, k, per_expert_scale, idx, wts, stream=None):
    _check(_lib.moe_router_topk(_ptr(logits), T, E, k, _ptr(per_expert_scale), _ptr(idx), _ptr(wts),
                                _stream(stream)))


def moe_router(layer, h, T, idx, wts, xe, ws, stream=None):
    _check(_lib.moe_router(layer.ptr(), _ptr(h), T, _ptr(idx), _ptr(wts), _ptr(xe), _ptr(ws),
                           ws.numel() if ws is not None else 0, _stream(stream)))


def moe_qmat_gemv(q_tiled, sb_tiled, rows, cols, x, T, y, ws, stream=None):
    """y[T, rows] (fp32) = W x for one tiled 4-bit matrix (prepare_qmat with n_mat = 1)."""
    m = QMat(q_tiled.data_ptr(), sb_tiled.data_ptr())
    _check(_lib.moe_qmat_gemv(C.byref(m), rows, cols, _ptr(x), T, _ptr(y), _ptr(ws),
                              ws.numel() * ws.element_size(), _stream(stream)))


def qmat_gemv_workspace(device="cuda") -> torch.Tensor:
    return torch.empty(int(_lib.moe_qmat_gemv_workspace_size()), dtype=torch.uint8, device=device)


def moe_bucket(idx, T, k, E, offsets, perm, inv=None, active=None, stream=None):
    _check(_lib.moe_bucket(_ptr(idx), T, k, E, _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(active),
                           _stream(stream)))


def moe_expert_ffn(layer, xe, T, idx, wts, offsets, perm, active, with_shared, m_out, ws, opts=None, stream=None):
    o = opts if opts is not None else _opts()
    _check(_lib.moe_expert_ffn(layer.ptr(), _ptr(xe), T, _ptr(idx), _ptr(wts), _ptr(offsets), _ptr(perm),
                               _ptr(active), int(with_shared), _ptr(m_out), _ptr(ws),
                               ws.numel() if ws is not None else 0, C.byref(o), _stream(stream)))


def moe_layer_forward(layer, h_in, h_out, T, ws, opts=None, stream=None):
    o = opts if opts is not None else _opts()
    _check(_lib.moe_layer_forward(layer.ptr(), _ptr(h_in), _ptr(h_out), T, _ptr(ws),
                                  ws.numel() if ws is not None else 0, C.byref(o), _stream(stream)))


def moe_layer_forward_noalloc(layer, h_in, h_out, T, opts=None, stream=None):
    """moe_layer_forward without a workspace: the library's static scratch
    (moe_noalloc_scratch_bytes()) is used instead; see include/moe_api.h."""
    o = opts if opts is not None else _opts()
    _check(_lib.moe_layer_forward_noalloc(layer.ptr(), _ptr(h_in), _ptr(h_out), T, C.byref(o), _stream(stream)))


def layer_array(layers):
    """A contiguous host array of moe_layer_w for moe_decode_stack."""
    arr = (LayerW * len(layers))()
    for i, l in enumerate(layers):
        arr[i] = l.struct
    return arr


def moe_decode_stack_workspace_size(layer, T: int) -> int:
    return int(_lib.moe_decode_stack_workspace_size(layer.ptr(), T))


def moe_decode_stack(layer_arr, L, h_in, chained, h_out, T, ws, opts=None, stream=None):
    o = opts if opts is not None else _opts()
    _check(_lib.moe_decode_stack(C.addressof(layer_arr), L, _ptr(h_in), int(chained), _ptr(h_out), T, _ptr(ws),
                                 ws.numel() if ws is not None else 0, C.byref(o), _stream(stream)))


def moe_decode_stack_status(ws):
    _check(_lib.moe_decode_stack_status(_ptr(ws)))


def moe_layer_partial(layer, h_in, T, e_lo, e_hi, with_shared, m_out, ws, opts=None, stream=None):
    """This rank's part of an expert-parallel layer: m_out = the weighted sum
    over its routed experts [e_lo, e_hi) (+ the shared expert)."""
    o = opts if opts is not None else _opts()
    _check(_lib.moe_layer_partial(layer.ptr(), _ptr(h_in), T, e_lo, e_hi, int(with_shared), _ptr(m_out), _ptr(ws),
                                  ws.numel() if ws is not None else 0, C.byref(o), _stream(stream)))


def moe_combine(h_in, m, h_out, T, H, opts=None, stream=None):
    """h_out = bf16((h_in + rmsnorm_no_scale(m)) * layer_scalar)."""
    o = opts if opts is not None else _opts()
    _check(_lib.moe_combine(_ptr(h_in), _ptr(m), _ptr(h_out), T, H, C.byref(o), _stream(stream)))


def moe_expert_cache_reset(cache, E, stream=None):
    _check(_lib.moe_expert_cache_reset(C.addressof(cache), E, _stream(stream)))


def moe_layer_forward_cached(layer, cache, h_in, h_out, T, ws, opts=None, stream=None):
    """moe_layer_forward with the routed experts served from a device cache
    filled from a host pool (see moe_layer_forward_cached in the header)."""
    o = opts if opts is not None else _opts()
    _check(_lib.moe_layer_forward_cached(layer.ptr(), C.addressof(cache), _ptr(h_in), _ptr(h_out), T, _ptr(ws),
                                         ws.numel() if ws is not None else 0, C.byref(o), _stream(stream)))


def moe_decode_stack_fits(layer, T, stream=None) -> bool:
    """True if the persistent decode kernel can run layers shaped like
    `layer` with T tokens on the stream's device."""
    return bool(_lib.moe_decode_stack_fits(layer.ptr(), T, _stream(stream)))


def moe_workspace_status(ws):
    _check(_lib.moe_workspace_status(_ptr(ws)))


def moe_noalloc_scratch_bytes() -> int:
    return int(_lib.moe_noalloc_scratch_bytes())


def moe_noalloc_status(stream=None):
    """Raise if the last moe_layer_forward_noalloc call on the stream's device
    left a device-side error in the static scratch (synchronises the stream)."""
    _check(_lib.moe_noalloc_status(_stream(stream)))


def make_opts(post_norm=True, layer_scalar=1.0, eps=1e-6, force_path=0) -> Opts:
    return _opts(post_norm, layer_scalar, eps, force_path)
