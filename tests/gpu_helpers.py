"""Shared helpers of the GPU parity tests: upload seeded inputs, drive the
C ABI through the binding, and compare against the oracle."""
from __future__ import annotations

import numpy as np

import oracle
from tests import blob

# FP32-accumulation tolerance on outputs and states (relative L2).
REL_L2 = 2e-3
# One decode step from a given state.  The step quantizes the decay-folded
# vectors x_k, x_q to int16 per 16-key chunk (error <= 2^-16 of the chunk's
# largest entry) and accumulates code products exactly in int32, so the code
# term carries a relative error of order 1e-5 (random signs over 128 keys,
# codes up to 127); everything else is FP32.  2e-4 leaves a 10x margin.
STEP_REL = 2e-4
# Bound on the fraction of codes that may differ by one step when the two
# sides start from the same FP32 state.
CODE_FLIP_FRACTION = 1e-5
# Line energies closer than this (relative) count as a tie between lines.
NEAR_TIE = 1e-5


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def device_inputs(wl, d):
    """Upload all drawn tokens: dict of cuda tensors with a leading token axis."""
    from linear_attention_recurrent_lq_b200 import inputs
    return inputs.to_device(wl, d)


def run_gpu(wl, d, n_tokens, cfg=None, flush=True, hook=None):
    """Init from S0, then n_tokens decode steps with a flush after every
    window.  Returns (outputs [T, B, H, dv] float32, LQState)."""
    import torch
    from linear_attention_recurrent_lq_b200 import binding as B
    cfg = cfg or B.config_for(wl)
    st = B.LQState(cfg)
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = device_inputs(wl, d)
    out = torch.empty((n_tokens, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    for t in range(n_tokens):
        st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out[t])
        if hook:
            hook(t, st)
        if flush and cfg.bits != 32 and (t + 1) % cfg.window == 0:
            st.flush()
    torch.cuda.synchronize()
    return out.cpu().numpy(), st


def oracle_inputs(wl, d, heads, n_tokens):
    """Inputs of the selected flat head indices in the oracle's layout."""
    nh = wl.batch * wl.heads
    S0 = d["S0"].reshape(nh, wl.dk, wl.dv)[heads]
    q = d["q"][:n_tokens].reshape(n_tokens, nh, wl.dk)[:, heads]
    k = d["k"][:n_tokens].reshape(n_tokens, nh, wl.dk)[:, heads]
    v = d["v"][:n_tokens].reshape(n_tokens, nh, wl.dv)[:, heads]
    beta = d["beta"][:n_tokens].reshape(n_tokens, nh)[:, heads]
    if wl.decay_kind == "kda":
        decay = d["decay"][:n_tokens].reshape(n_tokens, nh, wl.dk)[:, heads]
    else:
        decay = d["decay"][:n_tokens].reshape(n_tokens, nh)[:, heads]
    return S0, q, k, v, beta, decay


def residual_energy_ok(S, picks, tol=NEAR_TIE) -> bool:
    """Every pick is (within tol) a line of largest residual energy at its round."""
    R = np.asarray(S, np.float64).copy()
    for p in picks:
        if p == blob.NONE:
            break
        er = (R ** 2).sum(1)
        ec = (R ** 2).sum(0)
        emax = max(er.max(), ec.max())
        if p & blob.KIND_COL:
            j = p & 0x7FFFFFFF
            e = ec[j]
            R[:, j] = 0
        else:
            e = er[p]
            R[p, :] = 0
        if e < emax * (1 - tol):
            return False
    return True


def compare_compressed(p: oracle.Params, S_f32, got: dict) -> dict:
    """Compare a GPU-compressed blob with the oracle's compression of the same
    FP32 state.  The compensator choice must agree, or differ only at a near
    tie (then the oracle is re-run with the GPU's valid choice); codes, scales
    and compensator lines must then agree bit for bit.  Returns diagnostics."""
    ref = oracle.compress(p, S_f32)
    gm = [int(x) for x in got["meta"]]
    rm = [int(x) for x in ref["meta"]]
    tie = False
    if gm != rm:
        assert residual_energy_ok(S_f32, gm), f"compensator choice {gm} is not a max-energy line ({rm})"
        ref = oracle.compress(p, S_f32, forced=np.array(gm, np.uint32))
        tie = True
    np.testing.assert_array_equal(got["sm"], ref["sm"])
    np.testing.assert_array_equal(got["qs"], ref["qs"])
    np.testing.assert_array_equal(got["vec"], ref["vec"])
    diff = got["codes"].astype(np.int32) - ref["codes"].astype(np.int32)
    assert np.abs(diff).max() <= 1
    flips = int(np.count_nonzero(diff))
    return {"near_tie": tie, "flips": flips, "codes": diff.size}
