"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed
form, a textbook special case of the delta rule, an invariant of the method,
a hand-derived fixture under tests/golden/, a library routine, or a
brute-force enumeration on tiny heads.  Together they are meant to fail on a
dropped term, a wrong sign or index, or a transposed operand anywhere in the
oracle.  Sources: news post "Linear attention has to move state every token it
generates; LeapQuant compresses it to 8-bit without losing accuracy" (the
per-window, Compensator Tokens and residual smoothing paragraphs) and
"LeapQuant: Efficient Linear Attention with Accurate Recurrent State
Quantization" (original abstract).
"""
import json
import os

import numpy as np
import pytest

import oracle
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_state(rng, dk, dv, rows=(), cols=(), gain=50.0):
    S = rng.normal(0, 0.1, (dk, dv))
    for i in rows:
        S[i] *= gain
    for j in cols:
        S[:, j] *= gain
    return S


def _unit(rng, n):
    x = rng.normal(size=n)
    return x / np.linalg.norm(x)


# --------------------------------------------------------------------------
# the delta-rule step (GDN / KDA)

def test_step_delta_rule_overwrites_key_row(oracle_lib):
    """k = e_i, beta = 1: the step writes v into key row i after the decay,
    every other row is only decayed, and o = S_t^T q with q = e_i returns v."""
    rng = np.random.default_rng(1)
    dk, dv = 8, 6
    S = rng.normal(size=(dk, dv))          # not symmetric, not square
    a = rng.uniform(0.5, 1.0, dk)
    i = 3
    e = np.zeros(dk)
    e[i] = 1.0
    v = rng.normal(size=dv)
    S1, o, u = oracle.step(S, e, e, v, 1.0, a)
    expect = a[:, None] * S
    expect[i] = v
    np.testing.assert_allclose(S1, expect, rtol=0, atol=1e-14)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
    np.testing.assert_allclose(u, v - a[i] * S[i], rtol=0, atol=1e-14)


def test_step_beta_zero_is_pure_decay(oracle_lib):
    rng = np.random.default_rng(2)
    dk, dv = 8, 8
    S = rng.normal(size=(dk, dv))
    a = rng.uniform(0.3, 1.0, dk)
    q, k, v = _unit(rng, dk), _unit(rng, dk), rng.normal(size=dv)
    S1, o, u = oracle.step(S, q, k, v, 0.0, a)
    np.testing.assert_array_equal(S1, a[:, None] * S)
    np.testing.assert_allclose(o, (a[:, None] * S).T @ q, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(u, np.zeros(dv))


@pytest.mark.parametrize("alpha", [1.0, 0.93])
def test_step_matches_textbook_gated_delta_rule(oracle_lib, alpha):
    """Textbook form S_t = alpha (I - beta k k^T) S_{t-1} + beta k v^T
    (alpha = 1: plain DeltaNet), o_t = S_t^T q_t."""
    rng = np.random.default_rng(3)
    dk, dv = 16, 12
    S = rng.normal(size=(dk, dv))
    for _ in range(5):
        q, k, v = _unit(rng, dk), _unit(rng, dk), rng.normal(size=dv)
        beta = rng.uniform(0.1, 0.9)
        ref = alpha * (np.eye(dk) - beta * np.outer(k, k)) @ S + beta * np.outer(k, v)
        S, o, _ = oracle.step(S, q, k, v, beta, np.full(dk, alpha))
        np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(o, ref.T @ q, rtol=1e-12, atol=1e-13)


def test_step_matches_textbook_kda(oracle_lib):
    """KDA: S_t = (I - beta k k^T) diag(a) S_{t-1} + beta k v^T."""
    rng = np.random.default_rng(4)
    dk, dv = 16, 8
    S = rng.normal(size=(dk, dv))
    for _ in range(5):
        q, k, v = _unit(rng, dk), _unit(rng, dk), rng.normal(size=dv)
        a = rng.uniform(0.4, 1.0, dk)
        beta = rng.uniform(0.1, 0.9)
        ref = (np.eye(dk) - beta * np.outer(k, k)) @ np.diag(a) @ S + beta * np.outer(k, v)
        S, o, _ = oracle.step(S, q, k, v, beta, a)
        np.testing.assert_allclose(S, ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(o, ref.T @ q, rtol=1e-12, atol=1e-13)


def test_kda_with_uniform_decay_is_gdn(oracle_lib):
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=40)
    d = inputs.draw(wl)
    nh = 1
    S0 = d["S0"].reshape(nh, 128, 128)
    q, k, v = (d[x].reshape(40, nh, 128) for x in "qkv")
    beta = d["beta"].reshape(40, nh)
    alpha = d["decay"].reshape(40, nh)
    pg = oracle.Params.of(wl)
    pk = oracle.Params(**{**pg.__dict__, "kda": True})
    og, Sg, _ = oracle.run(pg, S0, q, k, v, beta, alpha)
    ok, Sk, _ = oracle.run(pk, S0, q, k, v, beta, np.repeat(alpha[..., None], 128, -1))
    np.testing.assert_array_equal(og, ok)
    np.testing.assert_array_equal(Sg, Sk)


def test_rank_grows_by_at_most_one_per_token(oracle_lib):
    rng = np.random.default_rng(5)
    dk = dv = 16
    p = oracle.Params(dk=dk, dv=dv, bits=32, num_comp=0)
    T = 6
    q = np.stack([_unit(rng, dk) for _ in range(T)])[:, None].astype(np.float32)
    k = np.stack([_unit(rng, dk) for _ in range(T)])[:, None].astype(np.float32)
    v = rng.normal(size=(T, 1, dv)).astype(np.float32)
    beta = rng.uniform(0.2, 0.9, (T, 1)).astype(np.float32)
    a = rng.uniform(0.8, 1.0, (T, 1)).astype(np.float32)
    for t in range(1, T + 1):
        _, S, _ = oracle.run(p, np.zeros((1, dk, dv), np.float32), q[:t], k[:t], v[:t],
                             beta[:t], a[:t])
        assert np.linalg.matrix_rank(S[0], tol=1e-9) == t


# --------------------------------------------------------------------------
# per-window buffering is exact algebra

@pytest.mark.parametrize("kda", [False, True])
def test_buffered_window_equals_dense_recurrence(oracle_lib, kda):
    """With no quantization inside the window, outputs computed from the
    window-start state plus the buffered rank-one updates equal the
    step-by-step recurrence (per-window paragraph; abstract)."""
    rng = np.random.default_rng(6 + kda)
    dk, dv, T = 32, 24, 16
    S = _rand_state(rng, dk, dv, rows=(3,), cols=(5,))
    q = np.stack([_unit(rng, dk) for _ in range(T)])
    k = np.stack([_unit(rng, dk) for _ in range(T)])
    v = rng.normal(size=(T, dv))
    beta = rng.uniform(0.1, 0.9, T)
    a = rng.uniform(0.5, 1.0, (T, dk)) if kda else np.repeat(rng.uniform(0.5, 1.0, (T, 1)), dk, 1)
    ob, Sb = oracle.window_buffered(S, q, k, v, beta, a)
    Sd = S.copy()
    od = []
    for t in range(T):
        Sd, o, _ = oracle.step(Sd, q[t], k[t], v[t], beta[t], a[t])
        od.append(o)
    od = np.array(od)
    assert np.linalg.norm(ob - od) <= 1e-12 * np.linalg.norm(od)
    assert np.linalg.norm(Sb - Sd) <= 1e-12 * np.linalg.norm(Sd)


def test_window_one_is_per_step_quantization(oracle_lib):
    """W = 1 reduces to quantizing after every token."""
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=8, window=1)
    d = inputs.draw(wl)
    p = oracle.Params.of(wl)
    o_run, S_run, _ = oracle.run(p, d["S0"].reshape(1, 128, 128), d["q"].reshape(8, 1, 128),
                                 d["k"].reshape(8, 1, 128), d["v"].reshape(8, 1, 128),
                                 d["beta"].reshape(8, 1), d["decay"].reshape(8, 1))

    def requant(S):
        c = oracle.compress(p, S.astype(np.float32))
        return oracle.dequant(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"])

    S = requant(d["S0"][0, 0])
    for t in range(8):
        S, o, _ = oracle.step(S, d["q"][t, 0, 0], d["k"][t, 0, 0], d["v"][t, 0, 0],
                              d["beta"][t, 0, 0], np.full(128, d["decay"][t, 0, 0], np.float64))
        np.testing.assert_array_equal(o, o_run[t, 0])
        S = requant(S)
    np.testing.assert_array_equal(S, S_run[0])


def test_partial_window_stays_unquantized(oracle_lib):
    """Tokens after the last boundary are not requantized: running 20 tokens
    with W = 16 equals 16 quantized tokens followed by 4 dense steps."""
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=20)
    d = inputs.draw(wl)
    p = oracle.Params.of(wl)
    args = lambda n: (d["q"][:n].reshape(n, 1, 128), d["k"][:n].reshape(n, 1, 128),
                      d["v"][:n].reshape(n, 1, 128), d["beta"][:n].reshape(n, 1),
                      d["decay"][:n].reshape(n, 1))
    _, S16, _ = oracle.run(p, d["S0"].reshape(1, 128, 128), *args(16))
    o20, S20, _ = oracle.run(p, d["S0"].reshape(1, 128, 128), *args(20))
    S = S16[0]
    for t in range(16, 20):
        S, o, _ = oracle.step(S, d["q"][t, 0, 0], d["k"][t, 0, 0], d["v"][t, 0, 0],
                              d["beta"][t, 0, 0], np.full(128, d["decay"][t, 0, 0], np.float64))
        np.testing.assert_array_equal(o, o20[t, 0])
    np.testing.assert_array_equal(S, S20[0])


# --------------------------------------------------------------------------
# compress: compensators, smoothing, quantization

def _params(dk, dv, bits=8, r=4, smoothing=True, f16=False):
    return oracle.Params(dk=dk, dv=dv, bits=bits, num_comp=r, smoothing=smoothing, scale_f16=f16)


@pytest.mark.parametrize("bits", [8, 6, 4])
def test_compensators_plus_residual_reconstruct_state_exactly(oracle_lib, bits):
    rng = np.random.default_rng(10 + bits)
    dk, dv = 32, 48
    S = _rand_state(rng, dk, dv, rows=(1, 7), cols=(4, 40)).astype(np.float32)
    p = _params(dk, dv, bits=bits, r=5)
    c = oracle.compress(p, S)
    rebuilt = c["R"].copy()
    lines = set()
    for m, w in zip(c["meta"][:c["ncomp"]], c["vec"]):
        assert m not in lines
        lines.add(int(m))
        if m & oracle.KIND_COL:
            j = m & 0x7FFFFFFF
            assert np.all(c["R"][:, j] == 0)
            rebuilt[:, j] += w[:dk]
        else:
            assert np.all(c["R"][m] == 0)
            rebuilt[m] += w[:dv]
    np.testing.assert_array_equal(rebuilt, S.astype(np.float64))
    # the planted outlier lines are the ones taken
    assert {1, 7, oracle.KIND_COL | 4, oracle.KIND_COL | 40} <= lines


def test_greedy_choice_matches_brute_force(oracle_lib):
    rng = np.random.default_rng(20)
    for trial in range(40):
        dk, dv = rng.choice([2, 4, 8]), rng.choice([2, 4, 8])
        S = rng.normal(size=(dk, dv)).astype(np.float32)
        if trial % 3 == 0:      # exact ties between a row and a column
            S = np.round(S * 2) / 2
            S[:, 0] = 0
            S[0, :] = 0
            S[0, 0] = 2.0
        r = int(rng.integers(1, min(dk, dv) + 1))
        p = _params(dk, dv, bits=8, r=r, smoothing=bool(trial % 2))
        c = oracle.compress(p, S)
        b = brute.compress(S, 8, r, bool(trial % 2))
        assert list(c["meta"][:c["ncomp"]]) == b["meta"]
        np.testing.assert_array_equal(c["sm"], b["sm"])
        np.testing.assert_array_equal(c["qs"], b["qs"])
        np.testing.assert_array_equal(c["codes"], b["codes"])


@pytest.mark.parametrize("name", ["compress_ties.json"])
def test_golden_tie_order(oracle_lib, name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    for case in g["cases"]:
        S = np.array(case["S"], np.float32)
        p = _params(S.shape[0], S.shape[1], bits=8, r=case["num_comp"])
        c = oracle.compress(p, S)
        assert [int(x) for x in c["meta"]] == case["meta"]


@pytest.mark.parametrize("name", ["compress_4x4_int4.json", "compress_fp32_quotient.json"])
def test_golden_compress(oracle_lib, name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    pr = g["params"]
    p = oracle.Params(dk=pr["dk"], dv=pr["dv"], bits=pr["bits"], num_comp=pr["num_comp"],
                      smoothing=pr["smoothing"], scale_f16=pr["scale_f16"])
    c = oracle.compress(p, np.array(g["S"], np.float32))
    if "meta" in g:
        assert [int(x) for x in c["meta"]] == g["meta"]
        np.testing.assert_array_equal(c["vec"], np.array(g["vec"], np.float32))
    if "sm" in g:
        np.testing.assert_array_equal(c["sm"], np.array(g["sm"], np.float32))
    np.testing.assert_array_equal(c["qs"], np.array(g["qs"], np.float32))
    np.testing.assert_array_equal(c["codes"], np.array(g["codes_value_major"], np.int8))


@pytest.mark.parametrize("f16", [False, True])
def test_smoothing_is_power_of_two_and_exactly_invertible(oracle_lib, f16):
    rng = np.random.default_rng(30)
    dk, dv = 64, 64
    S = _rand_state(rng, dk, dv, rows=(2, 9), cols=(11,), gain=100.0).astype(np.float32)
    S[5] = 0.0          # an all-zero key row
    S[6] *= 1e-3        # a tiny one
    p = _params(dk, dv, bits=8, r=2, f16=f16)
    c = oracle.compress(p, S)
    R = c["R"].astype(np.float32)
    sm = c["sm"]
    mant, _ = np.frexp(sm)
    assert np.all(mant == 0.5), "smoothing scales must be powers of two"
    Rs = R / sm[:, None]
    np.testing.assert_array_equal(Rs * sm[:, None], R)
    rowmax = np.abs(Rs).max(axis=1)
    nz = np.abs(R).max(axis=1) > 0
    assert np.all((rowmax[nz] > 0.5) & (rowmax[nz] <= 1.0))
    assert np.all(sm[~nz] == 1.0)
    p0 = _params(dk, dv, bits=8, r=2, smoothing=False, f16=f16)
    assert np.all(oracle.compress(p0, S)["sm"] == 1.0)


@pytest.mark.parametrize("bits,f16,smoothing", [(8, False, True), (8, False, False),
                                                 (6, True, True), (4, True, True)])
def test_quantization_error_bound(oracle_lib, bits, f16, smoothing):
    """Symmetric rounding per value column of the smoothed residual: every
    entry off a compensated line is within half a step sm_i*qs_j/2, entries on
    compensated lines are exact, and each nonzero column reaches Qmax."""
    rng = np.random.default_rng(40 + bits)
    dk, dv = 64, 32
    S = _rand_state(rng, dk, dv, rows=(0, 13), cols=(7,), gain=80.0).astype(np.float32)
    p = _params(dk, dv, bits=bits, r=3, smoothing=smoothing, f16=f16)
    c = oracle.compress(p, S)
    D = oracle.dequant(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"])
    err = np.abs(D - S.astype(np.float64))
    bound = 0.5 * c["sm"].astype(np.float64)[:, None] * c["qs"].astype(np.float64)[None, :]
    comp_rows = [int(m) for m in c["meta"] if m != oracle.NONE and not m & oracle.KIND_COL]
    comp_cols = [int(m & 0x7FFFFFFF) for m in c["meta"] if m != oracle.NONE and m & oracle.KIND_COL]
    mask = np.ones_like(err, bool)
    mask[comp_rows, :] = False
    mask[:, comp_cols] = False
    # the stored scale is rounded, so allow its relative rounding on top
    slack = 2.0 ** -10 if f16 else 2.0 ** -22
    assert np.all(err[mask] <= bound[mask] * (1 + slack) + 1e-30)
    assert np.all(err[~mask] == 0)
    assert np.abs(c["codes"]).max() <= p.qmax
    colmax = np.abs(c["codes"].astype(int)).max(axis=1)
    live = c["qs"] > 0
    assert np.all(colmax[live] >= p.qmax - (1 if f16 else 0))


def test_f16_scale_rounding_matches_numpy(oracle_lib):
    rng = np.random.default_rng(50)
    xs = np.concatenate([rng.uniform(-1, 1, 2000) * 10.0 ** rng.integers(-9, 5, 2000),
                         [2 ** -24, 2 ** -25, 3 * 2 ** -26, 65504.0, 65519.0, 1.0 + 2 ** -11,
                          1.0 + 3 * 2 ** -11, 2 ** -14 * (1 + 2 ** -10)]]).astype(np.float32)
    for x in xs:
        assert oracle.round_f16(float(x)) == float(np.float16(x)), x


def test_pack_unpack_round_trip(oracle_lib):
    rng = np.random.default_rng(60)
    for bits in (8, 6, 4):
        q = 2 ** (bits - 1)
        codes = rng.integers(-q, q, size=(9, 128)).astype(np.int8)
        packed = oracle.pack_rows(bits, codes)
        assert packed.shape == (9, 128 * bits // 8)
        np.testing.assert_array_equal(oracle.unpack_rows(bits, packed, 128), codes)


def test_golden_packed_rows(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "packed_rows.json")))
    for key, bits in (("int4", 4), ("int6", 6)):
        codes = np.array([g[key]["codes"]], np.int8)
        packed = oracle.pack_rows(bits, codes)
        assert packed.tobytes().hex() == g[key]["bytes_hex"]
        np.testing.assert_array_equal(oracle.unpack_rows(bits, packed, 16), codes)


# --------------------------------------------------------------------------
# whole sequences

def test_run_matches_brute_force_on_tiny_heads(oracle_lib):
    rng = np.random.default_rng(70)
    for kda, bits, smoothing in ((False, 8, True), (True, 4, True), (False, 6, False)):
        dk = dv = 16
        T, W, r = 13, 4, 2
        S0 = _rand_state(rng, dk, dv, rows=(2,), cols=(9,), gain=20.0).astype(np.float32)
        q = np.stack([_unit(rng, dk) for _ in range(T)]).astype(np.float32)
        k = np.stack([_unit(rng, dk) for _ in range(T)]).astype(np.float32)
        v = rng.normal(size=(T, dv)).astype(np.float32)
        beta = rng.uniform(0.1, 0.9, T).astype(np.float32)
        a = (rng.uniform(0.6, 1.0, (T, dk)) if kda else
             np.repeat(rng.uniform(0.6, 1.0, (T, 1)), dk, 1)).astype(np.float32)
        p = oracle.Params(dk=dk, dv=dv, window=W, num_comp=r, bits=bits, kda=kda,
                          smoothing=smoothing)
        dec = a[:, None, :] if kda else a[:, :1]
        o, S, _ = oracle.run(p, S0[None], q[:, None], k[:, None], v[:, None], beta[:, None], dec)
        ob, Sb = brute.run(S0, q, k, v, beta, a, W, bits, r, smoothing)
        np.testing.assert_allclose(o[:, 0], ob, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(S[0], Sb, rtol=1e-9, atol=1e-12)


def _err_vs_fp32(wl, **kw):
    from linear_attention_recurrent_lq_b200 import inputs
    d = inputs.draw(wl)
    T = wl.tokens
    args = (d["S0"].reshape(1, 128, 128), d["q"].reshape(T, 1, 128), d["k"].reshape(T, 1, 128),
            d["v"].reshape(T, 1, 128), d["beta"].reshape(T, 1), d["decay"].reshape(T, 1))
    p = oracle.Params.of(wl)
    o_ref, _, _ = oracle.run(oracle.Params(**{**p.__dict__, "bits": 32}), *args)
    o, _, _ = oracle.run(oracle.Params(**{**p.__dict__, **kw}), *args)
    return np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref)


def test_window_quantization_accumulates_less_error_than_per_step(oracle_lib):
    """Per-window paragraph: quantizing once per window instead of every
    token keeps rounding error from compounding."""
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=64, bits=6, smoothing=True)
    e_step = _err_vs_fp32(wl, window=1)
    e_win = _err_vs_fp32(wl, window=16)
    assert e_win < 0.5 * e_step, (e_win, e_step)


def test_compensators_and_smoothing_reduce_error(oracle_lib):
    """Compensator Tokens paragraph: taking the outlier lines out as FP32
    pairs lowers the quantization error.  Residual smoothing paragraph: when
    the residual's key rows are still uneven, balancing them before
    quantizing lowers it further.  More bits lower it too."""
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=32, bits=6)
    plain = _err_vs_fp32(wl, num_comp=0, smoothing=False)
    comp = _err_vs_fp32(wl, num_comp=3, smoothing=False)
    assert comp < 0.1 * plain, (plain, comp)
    # one compensator for three outlier lines leaves uneven key rows behind
    assert _err_vs_fp32(wl, num_comp=1, smoothing=True) < 0.5 * _err_vs_fp32(
        wl, num_comp=1, smoothing=False)
    graded = wl.replace(outlier_rows=6, row_gain=8.0, outlier_cols=0)
    assert _err_vs_fp32(graded, num_comp=1, smoothing=True) < 0.7 * _err_vs_fp32(
        graded, num_comp=1, smoothing=False)
    e = [_err_vs_fp32(wl, bits=b, num_comp=3, smoothing=True) for b in (8, 6, 4)]
    assert e[0] < e[1] < e[2], e


# --------------------------------------------------------------------------
# the naive per-step baselines of the accuracy table (BF16 and FP8 states)

def test_bf16_rounding_matches_torch(oracle_lib):
    """bfloat16 rounding (ties to even, subnormals included) against
    PyTorch's float32 -> bfloat16 conversion."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    mags = 10.0 ** rng.uniform(-44, 37, 20000)
    x = np.concatenate([rng.standard_normal(20000) * mags,
                        [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -9, -(1 + 2.0 ** -8), 1.5 * 2.0 ** -126,
                         2.0 ** -133, 3 * 2.0 ** -134, 0.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    got = np.array([oracle_lib.round_bf16(float(v)) for v in x], np.float32)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_rounding_matches_torch_and_saturates(oracle_lib):
    """FP8 E4M3 rounding against PyTorch's float32 -> float8_e4m3fn
    conversion inside the finite range, and saturation to 448 beyond it (the
    format's largest finite value)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(8)
    x = rng.standard_normal(20000) * 2.0 ** rng.integers(-12, 8, 20000)
    x = np.concatenate([x[np.abs(x) <= 448], [2.0 ** -10, 3 * 2.0 ** -10, 1 + 2.0 ** -4, 1 + 3 * 2.0 ** -4,
                                              248.0, -248.0, 448.0, 0.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle_lib.round_e4m3(float(v)) for v in x], np.float32)
    np.testing.assert_array_equal(got, ref)
    for v, want in ((449.0, 448.0), (464.0, 448.0), (470.0, 448.0), (1e6, 448.0), (-1e6, -448.0)):
        assert oracle_lib.round_e4m3(v) == want, v


def test_fp8_column_quantization_by_hand(oracle_lib):
    """Per-value-column FP8: scale = fl32(column max / 448), codes = E4M3 of
    the FP32 quotient; an all-zero column has scale 0."""
    S = np.zeros((4, 3), np.float32)
    S[:, 0] = [1.0, -0.5, 0.25, 0.0]
    S[:, 2] = [1344.0, 3.0, -1344.0, 1.0]
    scale, val = oracle_lib.fp8_columns(S)
    assert scale[0] == np.float32(1.0) / np.float32(448.0)
    assert scale[1] == 0.0 and scale[2] == 3.0
    np.testing.assert_array_equal(val[:, 0], [448.0, -224.0, 112.0, 0.0])
    np.testing.assert_array_equal(val[:, 1], [0.0, 0.0, 0.0, 0.0])
    # 1/3 lies between the E4M3 values 0.3125 and 0.34375 (spacing 1/32 in [1/4, 1/2))
    np.testing.assert_array_equal(val[:, 2], [448.0, 1.0, -448.0, 0.34375])


@pytest.mark.parametrize("bits", [16, 8])
def test_per_step_store_keeps_representable_states(oracle_lib, bits):
    """With beta = 0 and decay 1/2 every state of the run is 2^-t S0.  If S0
    is exactly representable in the per-step format (BF16 values; for FP8,
    E4M3 values times a power-of-two column scale whose column maximum is
    448 times that scale), storing it after every token changes nothing, and
    the outputs equal those of the unquantized state exactly."""
    rng = np.random.default_rng(9)
    dk = dv = 16
    grid = np.array([oracle_lib.round_e4m3(v) for v in rng.uniform(-448, 448, dk * dv)]).reshape(dk, dv)
    if bits == 16:
        S0 = np.array([oracle_lib.round_bf16(v) for v in rng.normal(0, 1, dk * dv)]).reshape(dk, dv)
    else:
        grid[0, :] = 448.0
        S0 = grid * 2.0 ** -rng.integers(3, 9, dv)[None, :]
    T = 8
    q = np.stack([_unit(rng, dk) for _ in range(T)])[:, None]
    k = np.stack([_unit(rng, dk) for _ in range(T)])[:, None]
    v = rng.normal(size=(T, 1, dv))
    beta = np.zeros((T, 1))
    decay = np.full((T, 1), 0.5)
    base = dict(dk=dk, dv=dv, window=1, num_comp=0, smoothing=False)
    o_ref, S_ref, _ = oracle_lib.run(oracle_lib.Params(**base, bits=32), S0[None], q, k, v, beta, decay)
    o, S, _ = oracle_lib.run(oracle_lib.Params(**base, bits=bits, per_step=True), S0[None], q, k, v, beta,
                             decay)
    np.testing.assert_array_equal(o, o_ref)
    np.testing.assert_array_equal(S, S_ref)


def test_naive_per_step_baselines_lose_more_than_leapquant(oracle_lib):
    """Accuracy table of the news post: at the same 8 bits, states stored
    naively after every token (FP8 E4M3, or INT8 without compensators and
    smoothing) drift much further from the FP32 state than LeapQuant's
    windowed INT8; BF16, with more mantissa bits than E4M3, drifts less than
    FP8, and still more than LeapQuant INT8."""
    from linear_attention_recurrent_lq_b200 import inputs
    wl = inputs.WORKLOADS["gdn_int8_b1h1"].replace(tokens=96)
    e_lq = _err_vs_fp32(wl, window=16, num_comp=2, smoothing=True)
    e_int8 = _err_vs_fp32(wl, window=1, num_comp=0, smoothing=False)
    e_fp8 = _err_vs_fp32(wl, bits=8, per_step=True)
    e_bf16 = _err_vs_fp32(wl, bits=16, per_step=True)
    assert e_lq < 0.5 * e_int8, (e_lq, e_int8)
    assert e_lq < 0.5 * e_fp8, (e_lq, e_fp8)
    assert e_bf16 < e_fp8, (e_bf16, e_fp8)
    # the table's headline: 8-bit LeapQuant also beats the per-step BF16 state
    assert e_lq < e_bf16, (e_lq, e_bf16)


# --------------------------------------------------------------------------
# prompt handoff (prefill, then the state enters the quantized cache)

def test_prefill_matches_brute_force_on_tiny_heads(oracle_lib):
    """The dense recurrence over the prompt and the compression of its FP32
    rounding, against the independent NumPy restatement, per head with its
    own prompt length."""
    rng = np.random.default_rng(91)
    for kda, bits, smoothing in ((False, 8, True), (True, 4, True), (False, 6, False)):
        dk = dv = 16
        T, nh, r = 11, 3, 2
        lengths = [11, 0, 6]
        S0 = np.stack([_rand_state(rng, dk, dv, rows=(1,), cols=(7,), gain=20.0) for _ in range(nh)])
        S0 = S0.astype(np.float32)
        q = rng.normal(size=(T, nh, dk)).astype(np.float32) / 4
        k = rng.normal(size=(T, nh, dk)).astype(np.float32) / 4
        v = rng.normal(size=(T, nh, dv)).astype(np.float32)
        beta = rng.uniform(0.1, 0.9, (T, nh)).astype(np.float32)
        a = rng.uniform(0.6, 1.0, (T, nh, dk) if kda else (T, nh)).astype(np.float32)
        p = oracle.Params(dk=dk, dv=dv, window=4, num_comp=r, bits=bits, kda=kda, smoothing=smoothing)
        o, S, comp = oracle.prefill(p, S0, q, k, v, beta, a, lengths=lengths)
        for h in range(nh):
            n = lengths[h]
            ah = a[:, h] if kda else np.repeat(a[:, h:h + 1], dk, 1)
            ob, Sb = brute.run(S0[h], q[:n, h], k[:n, h], v[:n, h], beta[:n, h], ah[:n], 4, 32, r,
                               smoothing)
            if n:
                np.testing.assert_allclose(o[:n, h], ob, rtol=1e-9, atol=1e-12)
            assert not o[n:, h].any()
            np.testing.assert_allclose(S[h], Sb, rtol=1e-9, atol=1e-12)
            cb = brute.compress(Sb.astype(np.float32), bits, r, smoothing)
            np.testing.assert_array_equal(comp[h]["codes"], cb["codes"])
            np.testing.assert_array_equal(comp[h]["qs"], cb["qs"])
            np.testing.assert_array_equal(comp[h]["sm"], cb["sm"])


def test_prefill_without_writes_is_pure_decay(oracle_lib):
    """beta = 0: nothing is written, so after t tokens the state is the decay
    product times S0 (powers of two keep it exact) and o_t = S_t^T q_t."""
    rng = np.random.default_rng(92)
    dk, dv, T = 8, 6, 5
    S0 = rng.normal(size=(1, dk, dv)).astype(np.float32)
    q = rng.normal(size=(T, 1, dk)).astype(np.float32)
    k = rng.normal(size=(T, 1, dk)).astype(np.float32)
    v = rng.normal(size=(T, 1, dv)).astype(np.float32)
    beta = np.zeros((T, 1), np.float32)
    for kda in (False, True):
        a = (2.0 ** -rng.integers(0, 3, (T, 1, dk)) if kda else 2.0 ** -rng.integers(0, 3, (T, 1)))
        a = a.astype(np.float32)
        p = oracle.Params(dk=dk, dv=dv, num_comp=1, kda=kda)
        o, S, _ = oracle.prefill(p, S0, q, k, v, beta, a)
        G = np.ones(dk)
        for t in range(T):
            G = G * a[t, 0]
            St = G[:, None] * S0[0].astype(np.float64)
            np.testing.assert_allclose(o[t, 0], St.T @ q[t, 0].astype(np.float64), rtol=1e-13, atol=1e-13)
        np.testing.assert_array_equal(S[0], G[:, None] * S0[0].astype(np.float64))


def test_prefill_one_token_from_zero_writes_beta_k_v(oracle_lib):
    """From a zero state one token leaves S = beta k v^T (u = beta v, nothing
    to subtract) and o = beta (k . q) v: the orientation of the update."""
    dk, dv = 4, 3
    k = np.array([[[1.0, 2.0, 0.0, -1.0]]], np.float32)
    q = np.array([[[0.5, 0.0, 1.0, 2.0]]], np.float32)
    v = np.array([[[3.0, -1.0, 2.0]]], np.float32)
    p = oracle.Params(dk=dk, dv=dv, num_comp=0)
    o, S, _ = oracle.prefill(p, np.zeros((1, dk, dv), np.float32), q, k, v,
                             np.array([[0.5]], np.float32), np.array([[0.75]], np.float32))
    np.testing.assert_array_equal(S[0], 0.5 * np.outer(k[0, 0], v[0, 0]))
    np.testing.assert_array_equal(o[0, 0], 0.5 * float(k[0, 0] @ q[0, 0]) * v[0, 0])


# --------------------------------------------------------------------------
# the FP32 window-end rebuild (what the flush requantizes and dequant returns)

def _hexf(x):
    return np.array([[float.fromhex(v) for v in row] for row in x] if isinstance(x[0], list)
                    else [float.fromhex(v) for v in x], np.float32)


def test_golden_rebuild_order(oracle_lib):
    """Hand-derived 3 x 2 rebuild whose FP32 result depends on the order the
    rule fixes: fused pair terms, compensators in round order, pairs in buffer
    order, the decay of the key row applied last (tests/golden)."""
    g = json.load(open(os.path.join(GOLDEN, "rebuild_3x2_f32.json")))
    pr = g["params"]
    p = oracle.Params(dk=pr["dk"], dv=pr["dv"], bits=pr["bits"], num_comp=pr["num_comp"])
    codes = np.array(g["codes_value_major"], np.int8)
    args = (codes, _hexf(g["qs"]), _hexf(g["sm"]), np.array(g["meta"], np.uint32), _hexf(g["vec"]),
            _hexf(g["pairs_khat_then_u"]), _hexf(g["g"]))
    expect = _hexf(g["S"])
    np.testing.assert_array_equal(oracle.reconstruct_f32(p, *args), expect)
    np.testing.assert_array_equal(brute.reconstruct_f32(*args), expect)


def _rand_compact(rng, dk, dv, r, count, bits=8):
    """A compressed random head plus `count` random pairs and a decay vector."""
    S = _rand_state(rng, dk, dv, rows=(1,), cols=(dv - 2,), gain=30.0).astype(np.float32)
    p = oracle.Params(dk=dk, dv=dv, bits=bits, num_comp=r, window=max(count, 1))
    c = oracle.compress(p, S)
    pairs = np.concatenate([rng.normal(size=(count, dk)), rng.normal(0, 0.3, (count, dv))],
                           axis=1).astype(np.float32)
    g = rng.uniform(0.2, 1.0, dk).astype(np.float32)
    return p, c, pairs, g


def test_rebuild_within_fp32_rounding_bound_of_exact_sum(oracle_lib):
    """Against the exact (FP64) matrix the blob stands for,
    diag(g) (Dequant(compact) + sum_m khat_m u_m^T): each entry is within the
    forward error bound of the FP32 evaluation.  The rebuild rounds once for
    qs*C (the power-of-two smoothing scale multiplies exactly), once per
    compensator addition and fused pair term, and once for the decay:
        |S32 - S| <= (n + 2) 2^-24 |g_i| (|B_ij| + sum of |added terms|),
    with n the number of additions.  A dropped, doubled or misplaced term
    moves an entry by far more."""
    rng = np.random.default_rng(90)
    u = 2.0 ** -24
    for dk, dv, r, count in ((16, 16, 3, 5), (24, 16, 4, 9), (8, 8, 0, 0), (32, 32, 2, 15)):
        p, c, pairs, g = _rand_compact(rng, dk, dv, r, count)
        S32 = oracle.reconstruct_f32(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"], pairs, g)
        base = (c["sm"].astype(np.float64)[:, None] * c["qs"].astype(np.float64)[None, :]
                * c["codes"].T.astype(np.float64))
        mag = np.abs(base)
        inner = oracle.dequant(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"])
        mag = mag + np.abs(inner - base)        # the compensator entries (exact in FP64)
        for m in range(count):
            t = np.outer(pairs[m, :dk].astype(np.float64), pairs[m, dk:].astype(np.float64))
            inner = inner + t
            mag = mag + np.abs(t)
        exact = g.astype(np.float64)[:, None] * inner
        n = 1 + r + count
        bound = 1.0001 * (n + 2) * u * g.astype(np.float64)[:, None] * mag + 1e-45
        err = np.abs(S32.astype(np.float64) - exact)
        assert np.all(err <= bound), (dk, dv, r, count, float(np.max(err / bound)))
        if count:   # the bound is far tighter than one pair's contribution
            one = np.abs(g.astype(np.float64)[:, None] * np.outer(pairs[-1, :dk], pairs[-1, dk:]))
            assert np.median(one / bound) > 100


def test_rebuild_matches_brute_force_bit_for_bit(oracle_lib):
    """Random tiny heads, non-square, f32 scales: the C rebuild equals an
    independent NumPy restatement (exact rational fused multiply-add, one
    rounding per operation) in every bit."""
    rng = np.random.default_rng(91)
    for trial in range(12):
        dk, dv = (int(x) for x in rng.choice([4, 6, 8], 2))
        if dv > dk:
            dk, dv = dv, dk
        r = int(rng.integers(0, 4))
        count = int(rng.integers(0, 6))
        p, c, pairs, g = _rand_compact(rng, dk, dv, r, count, bits=int(rng.choice([8, 6, 4])))
        args = (c["codes"], c["qs"], c["sm"], c["meta"], c["vec"], pairs, g)
        a = oracle.reconstruct_f32(p, *args)
        b = brute.reconstruct_f32(*args)
        np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))
