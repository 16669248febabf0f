"""fp64 CPU oracle for the int4 routed-expert MoE layer -- TEST INFRASTRUCTURE.

Only the test suite, `__graft_entry__.smoke()` and the CPU-baseline leg of
`bench.py` may import this package.  The product path (the CUDA library and
its binding) never imports or calls it, and the oracle shares no code with
that path.  The arithmetic is in plain C (`moe_oracle.c`); this module
compiles it with gcc on first use and marshals numpy arrays to it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

EPS = 1e-6  # reading: eps inside rmsnorm_no_scale (the pages give none)


def build_oracle(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so with gcc (plain C, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-fopenmp", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("H", "E", "k", "I", "Is")] + [
        ("router_q", C.c_void_p), ("router_s", C.c_void_p), ("router_b", C.c_void_p),
        ("router_scale", C.c_void_p), ("per_expert_scale", C.c_void_p),
        ("gate_q", C.c_void_p), ("up_q", C.c_void_p), ("down_q", C.c_void_p),
        ("gate_s", C.c_void_p), ("gate_b", C.c_void_p), ("up_s", C.c_void_p), ("up_b", C.c_void_p),
        ("down_s", C.c_void_p), ("down_b", C.c_void_p),
        ("sh_gate_q", C.c_void_p), ("sh_up_q", C.c_void_p), ("sh_down_q", C.c_void_p),
        ("sh_gate_s", C.c_void_p), ("sh_gate_b", C.c_void_p), ("sh_up_s", C.c_void_p), ("sh_up_b", C.c_void_p),
        ("sh_down_s", C.c_void_p), ("sh_down_b", C.c_void_p),
    ]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build_oracle())
            P, I = C.c_void_p, C.c_int
            L.oracle_bf16_to_double.restype = C.c_double
            L.oracle_bf16_to_double.argtypes = [C.c_uint16]
            L.oracle_double_to_bf16.restype = C.c_uint16
            L.oracle_double_to_bf16.argtypes = [C.c_double]
            L.oracle_dequant.argtypes = [P, P, P, I, I, I, P]
            L.oracle_qmat_gemv.argtypes = [P, P, P, I, I, I, P, I, P]
            L.oracle_rmsnorm_no_scale.argtypes = [P, I, C.c_double, P]
            L.oracle_rmsnorm_no_scale.restype = None
            L.oracle_topk.argtypes = [P, I, I, P]
            L.oracle_gate_weights.argtypes = [P, P, I, P, P, P]
            L.oracle_gate_weights.restype = None
            L.oracle_router.argtypes = [P, P, I, C.c_double, P, P, P, P]
            L.oracle_bucket.argtypes = [P, I, I, I, P, P, P]
            L.oracle_expert.argtypes = [P, I, P, P]
            L.oracle_expert_ffn.argtypes = [P, P, I, P, P, I, P]
            L.oracle_combine.argtypes = [P, P, I, I, I, C.c_double, C.c_double, P, P]
            L.oracle_combine.restype = None
            L.oracle_layer_forward.argtypes = [P, P, I, C.c_double, I, C.c_double, P, P, P, P, P]
            L.oracle_set_threads.argtypes = [I]
            L.oracle_set_threads.restype = I
            L.oracle_set_threads(1)  # the plain sequential oracle unless a caller asks for more
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def set_threads(n: int) -> int:
    """Threads of the oracle's row loops (1: sequential); returns the count in
    effect.  Results do not depend on it."""
    return int(lib().oracle_set_threads(int(n)))


def _np(t, dtype):
    """torch tensor or numpy array -> C-contiguous numpy array viewed as dtype."""
    if hasattr(t, "detach"):
        t = t.detach().cpu().contiguous()
        if str(t.dtype) == "torch.bfloat16":
            import torch
            t = t.view(torch.int16)
        a = t.numpy()
    else:
        a = np.ascontiguousarray(t)
    return np.ascontiguousarray(a).view(dtype)


_WORDS = ("router_q", "gate_q", "up_q", "down_q", "sh_gate_q", "sh_up_q", "sh_down_q")


class OracleLayer:
    """Holds one layer's weights (MLX layout, host) and the C struct pointing at them."""

    def __init__(self, weights: dict, H: int, E: int, k: int, I: int, Is: int):
        self.H, self.E, self.k, self.I, self.Is = H, E, k, I, Is
        self._keep = {}
        st = _Layer(H=H, E=E, k=k, I=I, Is=Is)
        for name, _ in _Layer._fields_[5:]:
            a = _np(weights[name], np.uint32 if name in _WORDS else np.uint16)
            self._keep[name] = a
            setattr(st, name, a.ctypes.data)
        self.struct = st

    @classmethod
    def from_config(cls, weights, cfg):
        return cls(weights, cfg.H, cfg.E, cfg.k, cfg.I, cfg.Is)

    def ptr(self):
        return C.byref(self.struct)


def bf16_to_f64(bits) -> np.ndarray:
    b = _np(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    f = lib().oracle_double_to_bf16
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def dequant(q, s, b, rows, cols, bits) -> np.ndarray:
    out = np.empty((rows, cols), np.float64)
    qa, sa, ba = _np(q, np.uint32), _np(s, np.uint16), _np(b, np.uint16)
    rc = lib().oracle_dequant(_p(qa), _p(sa), _p(ba), rows, cols, bits, _p(out))
    assert rc == 0
    return out


def qmat_gemv(q, s, b, rows, cols, x, bits=4) -> np.ndarray:
    """Y [T, rows] = dequant(W) x for x [T, cols] (fp64), one matrix in MLX layout."""
    xa = np.ascontiguousarray(np.atleast_2d(x), np.float64)
    qa, sa, ba = _np(q, np.uint32), _np(s, np.uint16), _np(b, np.uint16)
    y = np.empty((xa.shape[0], rows), np.float64)
    rc = lib().oracle_qmat_gemv(_p(qa), _p(sa), _p(ba), rows, cols, bits, _p(xa), xa.shape[0], _p(y))
    assert rc == 0
    return y


def rmsnorm_no_scale(h, eps=EPS) -> np.ndarray:
    h = np.ascontiguousarray(h, np.float64)
    out = np.empty_like(h)
    lib().oracle_rmsnorm_no_scale(_p(h), h.shape[-1], eps, _p(out))
    return out


def topk(logits, k) -> np.ndarray:
    lg = np.ascontiguousarray(logits, np.float64)
    idx = np.empty(k, np.int32)
    rc = lib().oracle_topk(_p(lg), lg.shape[0], k, _p(idx))
    assert rc == 0
    return idx


def gate_weights(logits, idx, per_expert_scale):
    lg = np.ascontiguousarray(logits, np.float64)
    ix = np.ascontiguousarray(idx, np.int32)
    pes = _np(per_expert_scale, np.uint16)
    w = np.empty(ix.shape[0], np.float64)
    p = np.empty(ix.shape[0], np.float64)
    lib().oracle_gate_weights(_p(lg), _p(ix), ix.shape[0], _p(pes), _p(w), _p(p))
    return w, p


def router(layer: OracleLayer, h, eps=EPS):
    """-> logits [T,E], idx [T,k], w [T,k], xn [T,H] (fp64)."""
    ha = _np(h, np.uint16)
    T = ha.shape[0]
    logits = np.empty((T, layer.E), np.float64)
    idx = np.empty((T, layer.k), np.int32)
    w = np.empty((T, layer.k), np.float64)
    xn = np.empty((T, layer.H), np.float64)
    rc = lib().oracle_router(layer.ptr(), _p(ha), T, eps, _p(logits), _p(idx), _p(w), _p(xn))
    assert rc == 0
    return logits, idx, w, xn


def bucket(idx, E):
    ix = np.ascontiguousarray(idx, np.int32)
    T, k = ix.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = lib().oracle_bucket(_p(ix), T, k, E, _p(offsets), _p(perm), _p(inv))
    assert rc == 0
    return offsets, perm, inv


def expert(layer: OracleLayer, e: int, x) -> np.ndarray:
    xa = np.ascontiguousarray(x, np.float64)
    y = np.empty(layer.H, np.float64)
    rc = lib().oracle_expert(layer.ptr(), e, _p(xa), _p(y))
    assert rc == 0
    return y


def expert_ffn(layer: OracleLayer, x, idx, w, with_shared=True) -> np.ndarray:
    xa = np.ascontiguousarray(x, np.float64)
    ix = np.ascontiguousarray(idx, np.int32)
    wa = np.ascontiguousarray(w, np.float64)
    T = xa.shape[0]
    m = np.empty((T, layer.H), np.float64)
    rc = lib().oracle_expert_ffn(layer.ptr(), _p(xa), T, _p(ix), _p(wa), int(with_shared), _p(m))
    assert rc == 0
    return m


def combine(h, m, post_norm=True, layer_scalar=1.0, eps=EPS):
    ha = _np(h, np.uint16)
    ma = np.ascontiguousarray(m, np.float64)
    T, H = ma.shape
    of = np.empty((T, H), np.float64)
    ob = np.empty((T, H), np.uint16)
    lib().oracle_combine(_p(ha), _p(ma), T, H, int(post_norm), layer_scalar, eps, _p(of), _p(ob))
    return of, ob


def layer_forward(layer: OracleLayer, h, post_norm=True, layer_scalar=1.0, eps=EPS) -> dict:
    """Whole layer.  -> dict(idx, w, m, out_f64, out_bf16)."""
    ha = _np(h, np.uint16)
    T = ha.shape[0]
    H, k = layer.H, layer.k
    r = dict(idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float64), m=np.empty((T, H), np.float64),
             out_f64=np.empty((T, H), np.float64), out_bf16=np.empty((T, H), np.uint16))
    rc = lib().oracle_layer_forward(layer.ptr(), _p(ha), T, eps, int(post_norm), layer_scalar, _p(r["idx"]),
                                    _p(r["w"]), _p(r["m"]), _p(r["out_f64"]), _p(r["out_bf16"]))
    assert rc == 0
    return r
