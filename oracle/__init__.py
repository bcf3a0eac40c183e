"""CPU oracle of the LeapQuant decode path (FP64, plain loops, in C).

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline / reference leg import this package.  The CUDA library and its Python
binding never import it, and it imports nothing from them: the two share no
code.  The inputs both sides consume come from the seeded generator module.

This module only marshals numpy arrays into ``liblq_oracle.so`` (built from
``lq_oracle.c`` by ``oracle/build.py``); every step of the arithmetic is in
the C file, which cites the passages it follows.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblq_oracle.so")

KIND_COL = 0x80000000
NONE = 0xFFFFFFFF


class _Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("dk", "dv", "window", "num_comp", "bits", "kda", "smoothing", "scale_f16",
                 "per_step")]


@dataclass(frozen=True)
class Params:
    dk: int = 128
    dv: int = 128
    window: int = 16
    num_comp: int = 4
    bits: int = 8
    kda: bool = False
    smoothing: bool = True
    scale_f16: bool = False
    per_step: bool = False  # naive baselines: bits 16 = BF16, bits 8 = FP8 E4M3 state

    @property
    def qmax(self) -> int:
        return (1 << (self.bits - 1)) - 1

    @property
    def maxd(self) -> int:
        return max(self.dk, self.dv)

    def c(self) -> _Params:
        return _Params(self.dk, self.dv, self.window, self.num_comp, self.bits,
                       int(self.kda), int(self.smoothing), int(self.scale_f16), int(self.per_step))

    @staticmethod
    def of(wl) -> "Params":
        """Parameters of a generator Workload."""
        return Params(dk=wl.dk, dv=wl.dv, window=wl.window, num_comp=wl.num_comp,
                      bits=wl.bits, kda=(wl.decay_kind == "kda"), smoothing=wl.smoothing,
                      scale_f16=(wl.scale_dtype == "f16"))


_lib = None


def bind(path: str):
    """Load an oracle shared library and declare its C signatures."""
    L = ctypes.CDLL(path)
    P = ctypes.POINTER
    vp = ctypes.c_void_p
    L.lqo_compress.restype = ctypes.c_int
    L.lqo_compress.argtypes = [P(_Params), vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.lqo_dequant.argtypes = [P(_Params), vp, vp, vp, vp, vp, vp]
    L.lqo_reconstruct_f32.argtypes = [P(_Params), vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp]
    L.lqo_step.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, ctypes.c_double, vp, vp, vp]
    L.lqo_run.restype = ctypes.c_int
    L.lqo_run.argtypes = [P(_Params), ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, vp,
                          vp, vp, ctypes.c_int]
    L.lqo_prefill.restype = ctypes.c_int
    L.lqo_prefill.argtypes = [ctypes.c_int] * 5 + [vp] * 9 + [ctypes.c_int]
    L.lqo_window_buffered.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                      vp, vp, vp, vp, vp]
    L.lqo_round_f16.restype = ctypes.c_double
    L.lqo_round_f16.argtypes = [ctypes.c_double]
    L.lqo_round_bf16.restype = ctypes.c_double
    L.lqo_round_bf16.argtypes = [ctypes.c_double]
    L.lqo_round_e4m3.restype = ctypes.c_double
    L.lqo_round_e4m3.argtypes = [ctypes.c_double]
    L.lqo_fp8_columns.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp]
    L.lqo_row_bytes.restype = ctypes.c_int
    L.lqo_row_bytes.argtypes = [ctypes.c_int, ctypes.c_int]
    L.lqo_pack_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    L.lqo_unpack_rows.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    return L


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            from . import build as _b
            _b.build()
        _lib = bind(_LIB_PATH)
    return _lib


def use(L):
    """Swap the loaded library (the mutation tests plant mistakes this way);
    returns the previous one."""
    global _lib
    prev, _lib = _lib, L
    return prev


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def compress(p: Params, S, forced=None) -> dict:
    """Compensators + smoothed quantized residual of one head's FP32 state."""
    S, Sp = _c(S, np.float32)
    assert S.shape == (p.dk, p.dv)
    codes = np.zeros((p.dv, p.dk), np.int8)
    qs = np.zeros(p.dv, np.float32)
    sm = np.zeros(p.dk, np.float32)
    meta = np.zeros(p.num_comp, np.uint32)
    vec = np.zeros((p.num_comp, p.maxd), np.float32)
    top2 = np.zeros((p.num_comp, 2), np.float64)
    R = np.zeros((p.dk, p.dv), np.float64)
    fp = None
    if forced is not None:
        forced, fp = _c(forced, np.uint32)
    n = lib().lqo_compress(ctypes.byref(p.c()), Sp, fp, codes.ctypes.data, qs.ctypes.data,
                           sm.ctypes.data, meta.ctypes.data, vec.ctypes.data, top2.ctypes.data,
                           R.ctypes.data)
    return {"codes": codes, "qs": qs, "sm": sm, "meta": meta, "vec": vec, "ncomp": n,
            "top2": top2, "R": R}


def dequant(p: Params, codes, qs, sm, meta, vec) -> np.ndarray:
    """FP64 dense state of a compact state (exact)."""
    args = [_c(codes, np.int8), _c(qs, np.float32), _c(sm, np.float32), _c(meta, np.uint32),
            _c(vec, np.float32)]
    S = np.zeros((p.dk, p.dv), np.float64)
    lib().lqo_dequant(ctypes.byref(p.c()), *[a[1] for a in args], S.ctypes.data)
    return S


def reconstruct_f32(p: Params, codes, qs, sm, meta, vec, pairs, g) -> np.ndarray:
    """FP32 window-end state: diag(g) (base + compensators + buffered pairs)."""
    pairs = np.ascontiguousarray(pairs, np.float32).reshape(-1, p.dk + p.dv)
    args = [_c(codes, np.int8), _c(qs, np.float32), _c(sm, np.float32), _c(meta, np.uint32),
            _c(vec, np.float32)]
    pr, pp = _c(pairs, np.float32)
    gg, gp = _c(np.broadcast_to(np.asarray(g, np.float32), (p.dk,)), np.float32)
    S = np.zeros((p.dk, p.dv), np.float32)
    lib().lqo_reconstruct_f32(ctypes.byref(p.c()), *[a[1] for a in args], pairs.shape[0], pp, gp,
                              S.ctypes.data)
    return S


def step(S, q, k, v, beta, a):
    """One FP64 delta-rule step; returns (S_new, o, u)."""
    S = np.array(S, dtype=np.float64, copy=True, order="C")
    dk, dv = S.shape
    q, qp = _c(q, np.float64)
    k, kp = _c(k, np.float64)
    v, vp = _c(v, np.float64)
    a, ap = _c(np.broadcast_to(np.asarray(a, np.float64), (dk,)), np.float64)
    o = np.zeros(dv, np.float64)
    u = np.zeros(dv, np.float64)
    lib().lqo_step(dk, dv, S.ctypes.data, qp, kp, vp, float(beta), ap, o.ctypes.data, u.ctypes.data)
    return S, o, u


def run(p: Params, S0, q, k, v, beta, decay, threads: int = 0):
    """Whole decode sequences for nh heads.

    S0 [nh, dk, dv]; q, k [T, nh, dk]; v [T, nh, dv]; beta [T, nh];
    decay [T, nh] (GDN) or [T, nh, dk] (KDA).  Returns (o [T, nh, dv], S_end
    [nh, dk, dv], threads used).
    """
    S0, s0p = _c(S0, np.float32)
    nh = S0.shape[0]
    q, qp = _c(q, np.float32)
    T = q.shape[0]
    k, kp = _c(k, np.float32)
    v, vp = _c(v, np.float32)
    beta, bp = _c(beta, np.float32)
    decay, dp = _c(decay, np.float32)
    assert q.shape == (T, nh, p.dk) and v.shape == (T, nh, p.dv) and beta.shape == (T, nh)
    assert decay.shape == ((T, nh, p.dk) if p.kda else (T, nh))
    o = np.zeros((T, nh, p.dv), np.float64)
    S_end = np.zeros((nh, p.dk, p.dv), np.float64)
    used = lib().lqo_run(ctypes.byref(p.c()), nh, T, s0p, qp, kp, vp, bp, dp, o.ctypes.data,
                         S_end.ctypes.data, int(threads))
    return o, S_end, used


def prefill(p: Params, S0, q, k, v, beta, decay, lengths=None, threads: int = 0):
    """Prompt handoff: the FP64 delta rule over each head's prompt from S0,
    then the FP32 rounding of the final state compressed as at a window
    boundary.  Layouts as run(); lengths [nh] (None: all T).  Returns
    (o [T, nh, dv] with zeros past a head's length, S_end [nh, dk, dv] FP64,
    [compress(p, fl32(S_end[h])) for each head])."""
    S0, s0p = _c(S0, np.float32)
    nh = S0.shape[0]
    q, qp = _c(q, np.float32)
    T = q.shape[0]
    k, kp = _c(k, np.float32)
    v, vp = _c(v, np.float32)
    beta, bp = _c(beta, np.float32)
    decay, dp = _c(decay, np.float32)
    assert q.shape == (T, nh, p.dk) and v.shape == (T, nh, p.dv) and beta.shape == (T, nh)
    assert decay.shape == ((T, nh, p.dk) if p.kda else (T, nh))
    lp = None
    if lengths is not None:
        lengths, lp = _c(np.asarray(lengths).reshape(nh), np.int32)
    o = np.zeros((T, nh, p.dv), np.float64)
    S_end = np.zeros((nh, p.dk, p.dv), np.float64)
    lib().lqo_prefill(p.dk, p.dv, int(p.kda), nh, T, lp, s0p, qp, kp, vp, bp, dp, o.ctypes.data,
                      S_end.ctypes.data, int(threads))
    return o, S_end, [compress(p, S_end[h].astype(np.float32)) for h in range(nh)]


def window_buffered(S_base, q, k, v, beta, a):
    """Buffered window form with explicit decay products (one head).

    q, k [T, dk]; v [T, dv]; beta [T]; a [T, dk].  Returns (o [T, dv], S_end).
    """
    S_base, sp = _c(S_base, np.float64)
    dk, dv = S_base.shape
    q, qp = _c(q, np.float64)
    T = q.shape[0]
    k, kp = _c(k, np.float64)
    v, vp = _c(v, np.float64)
    beta, bp = _c(beta, np.float64)
    a, ap = _c(np.broadcast_to(np.asarray(a, np.float64), (T, dk)), np.float64)
    o = np.zeros((T, dv), np.float64)
    S_end = np.zeros((dk, dv), np.float64)
    lib().lqo_window_buffered(dk, dv, T, sp, qp, kp, vp, bp, ap, o.ctypes.data, S_end.ctypes.data)
    return o, S_end


def round_f16(x: float) -> float:
    return lib().lqo_round_f16(float(x))


def round_bf16(x: float) -> float:
    return lib().lqo_round_bf16(float(x))


def round_e4m3(x: float) -> float:
    return lib().lqo_round_e4m3(float(x))


def fp8_columns(S32):
    """Per-value-column FP8 E4M3 quantization of an FP32 state [dk, dv]:
    (scale [dv] float32, code values [dk, dv] float32)."""
    S32, sp = _c(S32, np.float32)
    dk, dv = S32.shape
    scale = np.zeros(dv, np.float32)
    val = np.zeros((dk, dv), np.float32)
    lib().lqo_fp8_columns(dk, dv, sp, scale.ctypes.data, val.ctypes.data)
    return scale, val


def row_bytes(bits: int, dk: int) -> int:
    return lib().lqo_row_bytes(bits, dk)


def pack_rows(bits: int, codes) -> np.ndarray:
    codes, cp = _c(codes, np.int8)
    rows, dk = codes.shape
    out = np.zeros((rows, row_bytes(bits, dk)), np.uint8)
    lib().lqo_pack_rows(bits, dk, rows, cp, out.ctypes.data)
    return out


def unpack_rows(bits: int, packed, dk: int) -> np.ndarray:
    packed, pp = _c(packed, np.uint8)
    rows = packed.shape[0]
    out = np.zeros((rows, dk), np.int8)
    lib().lqo_unpack_rows(bits, dk, rows, pp, out.ctypes.data)
    return out
