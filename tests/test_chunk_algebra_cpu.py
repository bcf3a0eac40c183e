"""The chunkwise form of the delta rule that the tensor-core prefill evaluates,
restated step by step in float64 and held to the oracle's token-by-token
recurrence (oracle.prefill, FP64).

Per chunk of at most C tokens starting at t0: the first token's gate scales
the incoming state, G_t is the product of the gates of tokens t0+1 .. t (per
key channel), and
    A = strictly lower part of diag(beta) (K.G)(K/G)^T,
    U = (I + A)^-1 diag(beta) (V - (K.G) S'),
    O = (Q.G) S' + lower((Q.G)(K/G)^T, diagonal included) U,
    S = diag(G_last . a_next) S' + (K . G_last . a_next / G)^T U,
with a_next the next chunk's first gate folded in; a chunk ends before a token
whose gate product would fall below 2^-40.  The check covers ragged prompt
lengths, zero gates and gates so small that chunks split early.  Source: the
state a prefill leaves enters the quantized cache (news post "Linear attention
has to move state every token it generates; LeapQuant compresses it to 8-bit
without losing accuracy", per-window paragraph); the recurrence is the delta
rule of the decode step.
"""
import numpy as np
import pytest

import oracle

THR = 2.0 ** -40


def chunked(S0, q, k, v, beta, a, C):
    """One head: S0 [dk, dv]; q, k [T, dk]; v [T, dv]; beta [T]; a [T, dk]."""
    T, dk = k.shape
    dv = v.shape[1]
    S = S0.astype(np.float64)
    if T:
        S = a[0][:, None] * S
    out = np.zeros((T, dv))
    t0 = 0
    while t0 < T:
        nt = min(C, T - t0)
        n = nt
        for i in range(dk):          # the chunk ends before an out-of-range product
            g = 1.0
            for x in range(1, nt):
                g *= a[t0 + x, i]
                if not g >= THR:
                    n = min(n, x)
                    break
        G = np.ones((n, dk))
        for x in range(1, n):
            G[x] = G[x - 1] * a[t0 + x]
        K, Q, V, B = k[t0:t0 + n], q[t0:t0 + n], v[t0:t0 + n], beta[t0:t0 + n]
        Kt, Qt, Kh = K * G, Q * G, K / G
        A = np.tril(B[:, None] * (Kt @ Kh.T), -1)
        U = np.linalg.solve(np.eye(n) + A, B[:, None] * (V - Kt @ S))
        out[t0:t0 + n] = Qt @ S + np.tril(Qt @ Kh.T) @ U
        gl = G[-1] * (a[t0 + n] if t0 + n < T else 1.0)
        S = gl[:, None] * S + (K * (gl / G)).T @ U
        t0 += n
    return out, S


@pytest.mark.parametrize("kda", [False, True])
def test_chunkwise_form_equals_token_recurrence(oracle_lib, kda):
    rng = np.random.default_rng(400 + int(kda))
    dk = dv = 16
    nh, T = 4, 45
    lengths = [45, 0, 17, 33]
    S0 = rng.normal(0, 0.5, (nh, dk, dv)).astype(np.float32)
    q = rng.normal(size=(T, nh, dk)).astype(np.float32)
    k = rng.normal(size=(T, nh, dk))
    k = (k / np.linalg.norm(k, axis=-1, keepdims=True)).astype(np.float32)
    v = rng.normal(size=(T, nh, dv)).astype(np.float32)
    beta = rng.uniform(0.05, 1.0, (T, nh)).astype(np.float32)
    if kda:
        a = rng.uniform(0.5, 1.0, (T, nh, dk)).astype(np.float32)
        a[10, 0, 3] = 0.0            # a zero gate
        a[20, :, :] = 1e-9           # every channel tiny: the chunk splits
        a[30, 3, 5] = 1e-30
        decay = a
    else:
        g = rng.uniform(0.5, 1.0, (T, nh)).astype(np.float32)
        g[12, 0] = 0.0
        g[25, :] = 1e-13
        decay = g
        a = np.repeat(g[..., None], dk, -1)
    p = oracle.Params(dk=dk, dv=dv, kda=kda, bits=8, num_comp=2)
    o_ref, S_ref, _ = oracle.prefill(p, S0, q, k, v, beta, decay, lengths=np.array(lengths))
    for h in range(nh):
        L = lengths[h]
        f64 = lambda x: x[:L, h].astype(np.float64)
        o, S = chunked(S0[h], f64(q), f64(k), f64(v), beta[:L, h].astype(np.float64),
                       a[:L, h].astype(np.float64), C=8)
        np.testing.assert_allclose(o, o_ref[:L, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(S, S_ref[h], rtol=1e-10, atol=1e-12)
