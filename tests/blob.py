"""Test-side reading and writing of state blobs, from the layout documented
in include/leapquant.h (restated here; nothing is imported from the library).
Code rows are packed/unpacked with the oracle's routines."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import oracle

MAGIC = 0x4C515354
KIND_COL = 0x80000000
NONE = 0xFFFFFFFF


def _al(x, a):
    return (x + a - 1) // a * a


@dataclass
class Layout:
    blob: int
    g_off: int
    qs_off: int
    sm_off: int
    cvec_off: int
    codes_off: int
    pairs_off: int
    row_bytes: int
    sbytes: int


def layout(dk, dv, window, num_comp, bits, kda, f16) -> Layout:
    if bits == 32:
        return Layout(_al(128 + dk * dv * 4, 256), 0, 128, 128, 128, 128, 128 + dk * dv * 4, 0, 4)
    sb = 2 if f16 else 4
    off = 128
    g_off = 0
    if kda:
        g_off = off
        off += _al(dk * 4, 128)
    qs = off; off += _al(dv * sb, 128)
    sm = off; off += _al(dk * sb, 128)
    cv = off; off += _al(num_comp * max(dk, dv) * 4, 128)
    cd = off; off += _al(dv * dk * bits // 8, 128)
    pr = off; off += window * (dk + dv) * 4
    return Layout(_al(off, 256), g_off, qs, sm, cv, cd, pr, dk * bits // 8, sb)


def layout_of(p: oracle.Params) -> Layout:
    return layout(p.dk, p.dv, p.window, p.num_comp, p.bits, p.kda, p.scale_f16)


def _scales(raw: np.ndarray, n: int, f16: bool) -> np.ndarray:
    if f16:
        return raw[: 2 * n].view(np.float16).astype(np.float32)
    return raw[: 4 * n].view(np.float32).copy()


def parse(p: oracle.Params, b: np.ndarray) -> dict:
    """One blob (uint8 array) -> its fields."""
    L = layout_of(p)
    b = np.ascontiguousarray(b, dtype=np.uint8)
    h = b[:16].view(np.uint32)
    out = {"count": int(h[0]), "status": int(h[1]), "ncomp": int(h[2]), "magic": int(h[3]),
           "g_scalar": float(b[16:20].view(np.float32)[0]),
           "meta": b[64:128].view(np.uint32)[: p.num_comp].copy()}
    if p.bits == 32:
        out["S"] = b[128:128 + p.dk * p.dv * 4].view(np.float32).reshape(p.dk, p.dv).copy()
        return out
    out["g"] = (b[L.g_off:L.g_off + 4 * p.dk].view(np.float32).copy() if p.kda
                else np.full(p.dk, out["g_scalar"], np.float32))
    out["qs"] = _scales(b[L.qs_off:], p.dv, p.scale_f16)
    out["sm"] = _scales(b[L.sm_off:], p.dk, p.scale_f16)
    out["vec"] = b[L.cvec_off:L.cvec_off + 4 * p.num_comp * p.maxd].view(np.float32).reshape(
        p.num_comp, p.maxd).copy()
    packed = b[L.codes_off:L.codes_off + p.dv * L.row_bytes].reshape(p.dv, L.row_bytes)
    out["codes"] = oracle.unpack_rows(p.bits, packed, p.dk)
    n = out["count"] if out["count"] <= p.window else 0
    out["pairs"] = b[L.pairs_off:L.pairs_off + n * (p.dk + p.dv) * 4].view(np.float32).reshape(
        n, p.dk + p.dv).copy()
    return out


def pack(p: oracle.Params, comp: dict, pairs=None, g=None, status=0) -> np.ndarray:
    """Build one blob from oracle-style fields (codes value-major int8, qs, sm,
    meta, vec), optional buffered pairs [count, dk+dv] and decay product g."""
    L = layout_of(p)
    b = np.zeros(L.blob, np.uint8)
    pairs = np.zeros((0, p.dk + p.dv), np.float32) if pairs is None else np.asarray(pairs, np.float32)
    g = np.ones(p.dk, np.float32) if g is None else np.broadcast_to(np.asarray(g, np.float32), (p.dk,))
    ncomp = int(np.sum(comp["meta"] != NONE))
    b[:16] = np.array([pairs.shape[0], status, ncomp, MAGIC], np.uint32).view(np.uint8)
    b[16:20] = np.array([g[0]], np.float32).view(np.uint8)
    meta = np.full(16, NONE, np.uint32)
    meta[: p.num_comp] = comp["meta"]
    b[64:128] = meta.view(np.uint8)
    if p.kda:
        b[L.g_off:L.g_off + 4 * p.dk] = g.astype(np.float32).view(np.uint8)
    sdt = np.float16 if p.scale_f16 else np.float32
    qs = np.asarray(comp["qs"], np.float32).astype(sdt)
    sm = np.asarray(comp["sm"], np.float32).astype(sdt)
    b[L.qs_off:L.qs_off + qs.nbytes] = qs.view(np.uint8)
    b[L.sm_off:L.sm_off + sm.nbytes] = sm.view(np.uint8)
    vec = np.asarray(comp["vec"], np.float32)
    b[L.cvec_off:L.cvec_off + vec.nbytes] = vec.view(np.uint8).ravel()
    packed = oracle.pack_rows(p.bits, comp["codes"])
    b[L.codes_off:L.codes_off + packed.nbytes] = packed.ravel()
    b[L.pairs_off:L.pairs_off + pairs.nbytes] = pairs.view(np.uint8).ravel()
    return b
