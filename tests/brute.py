"""Brute-force NumPy restatement of the method for tiny heads (dk, dv <= 16).

Independent of the C oracle (no shared code): every line energy is enumerated
explicitly each round, the state is kept dense, and the FP32 decisions use
numpy float32 scalars.  Used only to cross-check the oracle on tiny inputs.
"""
from __future__ import annotations

import numpy as np

KIND_COL = 0x80000000
NONE = 0xFFFFFFFF


def compress(S, bits, r, smoothing, scale_f16=False):
    S = np.asarray(S, np.float32)
    dk, dv = S.shape
    qmax = 2 ** (bits - 1) - 1
    R = S.astype(np.float64).copy()
    picks, vecs = [], []
    for _ in range(r):
        cands = []
        for i in range(dk):
            cands.append((float(sum(R[i, j] ** 2 for j in range(dv))), 0, i))
        for j in range(dv):
            cands.append((float(sum(R[i, j] ** 2 for i in range(dk))), 1, j))
        # larger energy first, then row (0) before column (1), then lower index
        best = sorted(cands, key=lambda c: (-c[0], c[1], c[2]))[0]
        if best[0] <= 0.0:
            break
        e, kind, idx = best
        if kind == 0:
            vecs.append(R[idx, :].astype(np.float32).copy())
            R[idx, :] = 0.0
            picks.append(idx)
        else:
            vecs.append(R[:, idx].astype(np.float32).copy())
            R[:, idx] = 0.0
            picks.append(KIND_COL | idx)
    sm = np.ones(dk, np.float32)
    lo, hi = (2.0 ** -14, 2.0 ** 15) if scale_f16 else (2.0 ** -126, 2.0 ** 127)
    for i in range(dk):
        m = np.max(np.abs(R[i]))
        if smoothing and m > 0:
            s = 1.0
            while s < m:
                s *= 2.0
            while s / 2.0 >= m:
                s /= 2.0
            sm[i] = min(max(s, lo), hi)
    Rp = np.zeros((dk, dv), np.float32)
    for i in range(dk):
        for j in range(dv):
            Rp[i, j] = np.float32(R[i, j]) / sm[i]
    qs = np.zeros(dv, np.float32)
    codes = np.zeros((dv, dk), np.int8)
    for j in range(dv):
        m = np.float32(np.max(np.abs(Rp[:, j])))
        s = m / np.float32(qmax)
        if scale_f16:
            s = np.float32(np.float16(s))
        if m > 0 and s == 0:
            s = np.float32(2.0 ** -24 if scale_f16 else 2.0 ** -149)
        qs[j] = s
        for i in range(dk):
            if s != 0:
                t = np.float32(Rp[i, j] / s)
                codes[j, i] = int(np.clip(np.rint(t), -qmax, qmax))
    return {"meta": picks, "vec": vecs, "sm": sm, "qs": qs, "codes": codes, "R": R}


def dequant(c, dk, dv):
    S = (c["sm"].astype(np.float64)[:, None] * c["qs"].astype(np.float64)[None, :]
         * c["codes"].T.astype(np.float64))
    for pick, w in zip(c["meta"], c["vec"]):
        if pick & KIND_COL:
            S[:, pick & 0x7FFFFFFF] += w
        else:
            S[pick, :] += w
    return S


def run(S0, q, k, v, beta, a, W, bits, r, smoothing, scale_f16=False):
    """One head: S0 [dk, dv], q/k [T, dk], v [T, dv], beta [T], a [T, dk]."""
    dk, dv = S0.shape
    quant = bits != 32

    def requant(S):
        return dequant(compress(S.astype(np.float32), bits, r, smoothing, scale_f16), dk, dv)

    S = requant(S0) if quant else S0.astype(np.float64)
    outs = []
    for t in range(q.shape[0]):
        Sd = np.diag(a[t].astype(np.float64)) @ S
        u = beta[t] * (v[t] - Sd.T @ k[t])
        S = Sd + np.outer(k[t], u)
        outs.append(S.T @ q[t])
        if quant and (t + 1) % W == 0:
            S = requant(S)
    return np.array(outs), S


def f32_round(x):
    """Round an exact rational (fractions.Fraction or int) to the nearest
    binary32, ties to even, with gradual underflow; written from the format's
    definition (24 significant bits, smallest normal 2^-126) with integer
    arithmetic only, so no intermediate rounding can creep in."""
    from fractions import Fraction
    x = Fraction(x)
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    # e = floor(log2(a))
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    quantum = Fraction(2) ** (e - 23)
    n, rem = divmod(a, quantum)        # a = n * quantum + rem, 0 <= rem < quantum
    n = int(n)
    if rem * 2 > quantum or (rem * 2 == quantum and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n * quantum))


def reconstruct_f32(codes, qs, sm, meta, vec, pairs, g):
    """The FP32 window-end state, written independently of the C oracle:
    S_ij = g_i * ( ((qs_j * C_ji) * sm_i) + compensators in round order
                   + fused multiply-add over the pairs in buffer order ),
    each operation one FP32 rounding.  The fused multiply-add is taken
    exactly in rationals, then rounded once (f32_round).
    codes [dv, dk] (value-major); meta / vec as the compressor returns them;
    pairs [count, dk + dv] (khat then u); g [dk]."""
    from fractions import Fraction
    dv, dk = codes.shape
    S = np.zeros((dk, dv), np.float32)
    for i in range(dk):
        for j in range(dv):
            acc = (np.float32(qs[j]) * np.float32(codes[j, i])) * np.float32(sm[i])
            for c, m in enumerate(meta):
                m = int(m)
                if m == NONE:
                    continue
                if m & KIND_COL:
                    if (m & 0x7FFFFFFF) == j:
                        acc = np.float32(acc + np.float32(vec[c][i]))
                elif m == i:
                    acc = np.float32(acc + np.float32(vec[c][j]))
            for pr in pairs:
                acc = f32_round(Fraction(float(pr[i])) * Fraction(float(pr[dk + j])) + Fraction(float(acc)))
            S[i, j] = np.float32(g[i]) * acc
    return S
