"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Bars: quantization codes, scales and compensator lines bit-exact when both
sides compress the same FP32 state (a near tie between compensator lines may
resolve either way; the rest must then agree); decode outputs and dense
states within 2e-3 relative L2 over whole sequences (FP32 accumulation), and
within 2e-4 for a single step from a given state (the step's int16
quantization of the decay-folded vectors, see gpu_helpers.STEP_REL).
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests import blob
from tests.gpu_helpers import (REL_L2, STEP_REL, compare_compressed, device_inputs, oracle_inputs,
                               rel_l2, run_gpu)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
SMALL = {
    "gdn_int8": W["gdn_int8_b64h32"].replace(batch=3, heads=5, tokens=40),
    "gdn_int8_d64": W["gdn_int8_b64h32"].replace(batch=3, heads=5, tokens=40, dk=64, dv=64),
    "kda_int8": W["kda_int8_b128h32"].replace(batch=3, heads=5, tokens=40),
    "gdn_6bit": W["gdn_6bit_b256h32"].replace(batch=3, heads=5, tokens=40),
    "gdn_4bit": W["gdn_4bit_b256h32"].replace(batch=3, heads=5, tokens=40),
    "kda_4bit_d64": W["kda_int8_b128h32"].replace(batch=2, heads=3, tokens=40, bits=4, dk=64,
                                                   dv=64, scale_dtype="f16"),
    "tiny_f32in": W["gdn_int8_b1h1"],
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _params(wl):
    return oracle.Params.of(wl)


def _blobs(st):
    torch.cuda.synchronize()
    return st.blobs().cpu().numpy()


@pytest.mark.parametrize("name", sorted(SMALL))
def test_init_compression_bit_exact(name):
    wl = SMALL[name]
    d = I.draw(wl, 0)
    from linear_attention_recurrent_lq_b200 import binding as B
    st = B.LQState(B.config_for(wl))
    st.init(torch.from_numpy(d["S0"]).cuda())
    blobs = _blobs(st)
    p = _params(wl)
    S0 = d["S0"].reshape(-1, wl.dk, wl.dv)
    for h in range(S0.shape[0]):
        got = blob.parse(p, blobs[h])
        assert (got["count"], got["status"], got["magic"]) == (0, 0, blob.MAGIC)
        np.testing.assert_array_equal(got["g"], np.ones(wl.dk, np.float32))
        r = compare_compressed(p, S0[h], got)
        assert r["flips"] == 0, r
    assert st.check() == 0


@pytest.mark.parametrize("name", sorted(SMALL))
def test_dequant_equals_fp32_rebuild(name):
    """lq_dequant_state after init evaluates the rebuild rule bit for bit, and
    stays within FP32 rounding of the exact dequantized state."""
    wl = SMALL[name]
    d = I.draw(wl, 0)
    from linear_attention_recurrent_lq_b200 import binding as B
    st = B.LQState(B.config_for(wl))
    st.init(torch.from_numpy(d["S0"]).cuda())
    S = st.dequant().cpu().numpy().reshape(-1, wl.dk, wl.dv)
    blobs = _blobs(st)
    p = _params(wl)
    for h in range(S.shape[0]):
        f = blob.parse(p, blobs[h])
        ref32 = oracle.reconstruct_f32(p, f["codes"], f["qs"], f["sm"], f["meta"], f["vec"],
                                       f["pairs"], f["g"])
        np.testing.assert_array_equal(S[h], ref32)
        ref64 = oracle.dequant(p, f["codes"], f["qs"], f["sm"], f["meta"], f["vec"])
        assert rel_l2(S[h], ref64) < 1e-6


def _oracle_window(wl, d, h, n_pairs):
    """A window state built by the oracle: the compressed S0 of head h plus
    n_pairs buffered pairs from the dense FP64 recurrence.  Returns (comp,
    pairs [n, dk+dv] f32, g [dk] f32, dense FP64 state after n_pairs tokens)."""
    p = _params(wl)
    nh = wl.batch * wl.heads
    S0 = d["S0"].reshape(nh, wl.dk, wl.dv)[h]
    comp = oracle.compress(p, S0)
    S = oracle.dequant(p, comp["codes"], comp["qs"], comp["sm"], comp["meta"], comp["vec"])
    g = np.ones(wl.dk, np.float32)
    pairs = []
    for t in range(n_pairs):
        q = d["q"][t].reshape(nh, -1)[h]
        k = d["k"][t].reshape(nh, -1)[h]
        v = d["v"][t].reshape(nh, -1)[h]
        beta = d["beta"][t].reshape(nh)[h]
        a = (d["decay"][t].reshape(nh, -1)[h] if wl.decay_kind == "kda"
             else np.full(wl.dk, d["decay"][t].reshape(nh)[h], np.float32))
        S, _, u = oracle.step(S, q, k, v, beta, a)
        g = (g * a).astype(np.float32)
        pairs.append(np.concatenate([(k / g).astype(np.float32), u.astype(np.float32)]))
    pairs = np.array(pairs, np.float32).reshape(n_pairs, wl.dk + wl.dv)
    return comp, pairs, g, S


def _upload_blobs(wl, blobs_np):
    from linear_attention_recurrent_lq_b200 import binding as B
    st = B.LQState(B.config_for(wl))
    st.buf.copy_(torch.from_numpy(np.concatenate(blobs_np)).cuda())
    return st


@pytest.mark.parametrize("name", sorted(SMALL))
def test_flush_bit_exact_on_oracle_window(name):
    """A full window built by the oracle: the GPU rebuild equals the FP32
    rebuild rule bit for bit, and the GPU flush compresses it to exactly the
    oracle's codes, scales and compensators."""
    wl = SMALL[name]
    p = _params(wl)
    d = I.draw(wl, wl.window)
    nh = wl.batch * wl.heads
    heads = list(range(min(nh, 6)))
    made = [_oracle_window(wl, d, h, wl.window) for h in heads]
    blobs_np = [blob.pack(p, c, pairs, g) for c, pairs, g, _ in made]
    sub = wl.replace(batch=len(heads), heads=1)
    st = _upload_blobs(sub, blobs_np)
    S_pre = st.dequant().cpu().numpy().reshape(-1, wl.dk, wl.dv)
    st.flush()
    after = _blobs(st)
    for x, (c, pairs, g, S64) in enumerate(made):
        ref32 = oracle.reconstruct_f32(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"], pairs, g)
        np.testing.assert_array_equal(S_pre[x], ref32)
        assert rel_l2(ref32, S64) < 1e-5  # the FP32 rebuild stands for the FP64 window state
        got = blob.parse(p, after[x])
        assert (got["count"], got["status"]) == (0, 0)
        np.testing.assert_array_equal(got["g"], np.ones(wl.dk, np.float32))
        r = compare_compressed(p, ref32, got)
        assert r["flips"] == 0, r


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("n_pairs", [0, 5, 15])
def test_decode_step_matches_oracle(name, n_pairs):
    wl = SMALL[name]
    n_pairs = min(n_pairs, wl.window - 1)
    p = _params(wl)
    d = I.draw(wl, n_pairs + 1)
    nh = wl.batch * wl.heads
    heads = list(range(min(nh, 6)))
    made = [_oracle_window(wl, d, h, n_pairs) for h in heads]
    blobs_np = [blob.pack(p, c, pairs, g) for c, pairs, g, _ in made]
    sub = wl.replace(batch=len(heads), heads=1)
    st = _upload_blobs(sub, blobs_np)
    t = n_pairs
    names = ("q", "k", "v", "beta", "decay") + (
        ("q_bits", "k_bits", "v_bits") if wl.in_dtype == "bf16" else ())
    dev = device_inputs(wl, {x: d[x][t:t + 1] for x in names})
    q, k, v = (dev[x][0].reshape(nh, -1)[heads].contiguous() for x in ("q", "k", "v"))
    beta = dev["beta"][0].reshape(nh)[heads].contiguous()
    decay = (dev["decay"][0].reshape(nh, -1)[heads].contiguous() if wl.decay_kind == "kda"
             else dev["decay"][0].reshape(nh)[heads].contiguous())
    out = torch.empty((len(heads), wl.dv), dtype=torch.float32, device="cuda")
    st.step(q, k, v, beta, decay, out)
    o_gpu = out.cpu().numpy()
    after = _blobs(st)
    for x, h in enumerate(heads):
        c, pairs, g, S = made[x]
        qh = d["q"][t].reshape(nh, -1)[h]
        kh = d["k"][t].reshape(nh, -1)[h]
        vh = d["v"][t].reshape(nh, -1)[h]
        bh = d["beta"][t].reshape(nh)[h]
        a = (d["decay"][t].reshape(nh, -1)[h] if wl.decay_kind == "kda"
             else np.full(wl.dk, d["decay"][t].reshape(nh)[h], np.float32))
        # the oracle starts from exactly the state the blob stands for
        S_blob = oracle.dequant(p, c["codes"], c["qs"], c["sm"], c["meta"], c["vec"])
        for m in range(n_pairs):
            S_blob += np.outer(pairs[m, :wl.dk].astype(np.float64), pairs[m, wl.dk:])
        S_blob *= g.astype(np.float64)[:, None]
        _, o_ref, u_ref = oracle.step(S_blob, qh, kh, vh, bh, a)
        assert rel_l2(o_gpu[x], o_ref) < STEP_REL
        got = blob.parse(p, after[x])
        assert got["count"] == n_pairs + 1 and got["status"] == 0
        g_new = (g * a.astype(np.float32)).astype(np.float32)
        np.testing.assert_array_equal(got["g"], g_new)
        np.testing.assert_array_equal(got["pairs"][:n_pairs], pairs)
        np.testing.assert_array_equal(got["pairs"][n_pairs, :wl.dk], (kh / g_new).astype(np.float32))
        assert rel_l2(got["pairs"][n_pairs, wl.dk:], u_ref) < STEP_REL


@pytest.mark.parametrize("name", sorted(SMALL))
def test_sequence_matches_oracle(name):
    """Init, then whole windows of decode steps with flushes and a partial
    last window: every window's outputs and the final state within 2e-3
    relative L2 of the FP64 oracle."""
    wl = SMALL[name]
    T = wl.tokens
    d = I.draw(wl, T)
    o_gpu, st = run_gpu(wl, d, T)
    S_gpu = st.dequant().cpu().numpy().reshape(-1, wl.dk, wl.dv)
    heads = np.arange(wl.batch * wl.heads)
    o_ref, S_ref, _ = oracle.run(_params(wl), *oracle_inputs(wl, d, heads, T))
    o_gpu = o_gpu.reshape(T, -1, wl.dv)
    for w0 in range(0, T, wl.window):
        sl = slice(w0, min(T, w0 + wl.window))
        assert rel_l2(o_gpu[sl], o_ref[sl]) < REL_L2, (w0, rel_l2(o_gpu[sl], o_ref[sl]))
    assert rel_l2(S_gpu, S_ref) < REL_L2
    assert st.check() == 0


def test_fp32_state_kernel_matches_oracle():
    from linear_attention_recurrent_lq_b200 import binding as B
    for wl in (SMALL["gdn_int8"], SMALL["kda_int8"], SMALL["gdn_int8_d64"]):
        T = 24
        d = I.draw(wl, T)
        cfg = B.config_for(wl, bits=32)
        o_gpu, st = run_gpu(wl, d, T, cfg=cfg)
        S_gpu = st.dequant().cpu().numpy().reshape(-1, wl.dk, wl.dv)
        p = oracle.Params(**{**_params(wl).__dict__, "bits": 32})
        heads = np.arange(wl.batch * wl.heads)
        o_ref, S_ref, _ = oracle.run(p, *oracle_inputs(wl, d, heads, T))
        assert rel_l2(o_gpu.reshape(T, -1, wl.dv), o_ref) < 1e-5
        assert rel_l2(S_gpu, S_ref) < 1e-5


@pytest.mark.parametrize("kind", ["gdn_int8_b64h32", "kda_int8_b128h32"])
def test_fp32_state_kernel_at_scale_sampled_heads(kind):
    """1200 heads: eight per CTA of the FP32 kernel (one CTA per SM), so its
    ring of stages is reused across heads; 32 seeded heads against the
    oracle over 12 tokens."""
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = W[kind].replace(batch=40, heads=30)
    T = 12
    d = I.draw(wl, T)
    o_gpu, st = run_gpu(wl, d, T, cfg=B.config_for(wl, bits=32))
    nh = wl.batch * wl.heads
    heads = np.sort(np.random.default_rng(5).choice(nh, 32, replace=False))
    p = oracle.Params(**{**_params(wl).__dict__, "bits": 32})
    o_ref, S_ref, _ = oracle.run(p, *oracle_inputs(wl, d, heads, T))
    assert rel_l2(o_gpu.reshape(T, nh, wl.dv)[:, heads], o_ref) < 1e-5
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)[heads]
    assert rel_l2(S_gpu, S_ref) < 1e-5


@pytest.mark.parametrize("key", ["gdn_int8_b64h32", "kda_int8_b128h32", "gdn_6bit_b256h32",
                                 "gdn_4bit_b256h32"])
def test_full_size_sampled_heads(key):
    """The full batch of each workload (the benchmark's launch configuration),
    two windows and a ragged third: 64 seeded heads are checked against the
    oracle (init codes bit-exact, outputs and final state within 2e-3)."""
    wl = W[key]
    T = 2 * wl.window + 3
    d = I.draw(wl, T)
    o_gpu, st = run_gpu(wl, d, T)
    nh = wl.batch * wl.heads
    heads = np.sort(np.random.default_rng(123).choice(nh, 64, replace=False))
    o_ref, S_ref, _ = oracle.run(_params(wl), *oracle_inputs(wl, d, heads, T))
    o_gpu = o_gpu.reshape(T, nh, wl.dv)[:, heads]
    assert rel_l2(o_gpu, o_ref) < REL_L2
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)[heads]
    assert rel_l2(S_gpu, S_ref) < REL_L2
    assert st.check() == 0
    # init of the same heads, bit for bit
    from linear_attention_recurrent_lq_b200 import binding as B
    st2 = B.LQState(B.config_for(wl))
    st2.init(torch.from_numpy(d["S0"]).cuda())
    blobs = _blobs(st2)
    p = _params(wl)
    S0 = d["S0"].reshape(nh, wl.dk, wl.dv)
    for h in heads:
        r = compare_compressed(p, S0[h], blob.parse(p, blobs[h]))
        assert r["flips"] == 0


# ------------------------------------------------------------------ edges

def test_window_of_one_and_no_compensators():
    wl = SMALL["gdn_int8"].replace(window=1, num_comp=0, tokens=6)
    d = I.draw(wl, 6)
    o_gpu, st = run_gpu(wl, d, 6)
    heads = np.arange(wl.batch * wl.heads)
    o_ref, S_ref, _ = oracle.run(_params(wl), *oracle_inputs(wl, d, heads, 6))
    assert rel_l2(o_gpu.reshape(6, -1, wl.dv), o_ref) < REL_L2


def test_largest_window_and_compensator_count():
    wl = SMALL["gdn_int8"].replace(batch=2, heads=2, window=64, num_comp=16, tokens=70)
    d = I.draw(wl, 70)
    o_gpu, st = run_gpu(wl, d, 70)
    heads = np.arange(4)
    o_ref, S_ref, _ = oracle.run(_params(wl), *oracle_inputs(wl, d, heads, 70))
    assert rel_l2(o_gpu.reshape(70, -1, wl.dv), o_ref) < REL_L2
    assert rel_l2(st.dequant().cpu().numpy().reshape(4, 128, 128), S_ref) < REL_L2


def test_empty_flush_leaves_state_unchanged():
    wl = SMALL["gdn_int8"]
    d = I.draw(wl, 0)
    from linear_attention_recurrent_lq_b200 import binding as B
    st = B.LQState(B.config_for(wl))
    st.init(torch.from_numpy(d["S0"]).cuda())
    before = st.buf.clone()
    st.flush()
    torch.cuda.synchronize()
    assert torch.equal(before, st.buf)


def test_step_into_full_window_is_flagged_and_skipped():
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = SMALL["gdn_int8"].replace(window=2)
    d = I.draw(wl, 3)
    cfg = B.config_for(wl)
    st = B.LQState(cfg)
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = device_inputs(wl, d)
    out = torch.empty((wl.batch, wl.heads, wl.dv), device="cuda")
    for t in range(2):
        st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out)
    assert st.check() == 0
    before = st.buf.clone()
    st.step(dev["q"][2], dev["k"][2], dev["v"][2], dev["beta"][2], dev["decay"][2], out)
    assert st.check() == 4  # LQ_ERR_WINDOW_FULL
    assert torch.count_nonzero(out) == 0
    changed = (before != st.buf).view(-1, st.blob_bytes)
    # only the status words changed
    assert changed[:, :4].sum() == 0 and changed[:, 8:].sum() == 0


def test_decay_underflow_moves_the_window_frame():
    """Gates of 2^-40: the third token takes the decay product below 2^-96,
    so the frame moves to it (no status bit, the stored product restarts at
    1).  A zero gate then forgets everything: the state is beta k v^T."""
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = SMALL["gdn_int8"].replace(window=8)
    d = I.draw(wl, 4)
    cfg = B.config_for(wl)
    st = B.LQState(cfg)
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = device_inputs(wl, d)
    out = torch.empty((wl.batch, wl.heads, wl.dv), device="cuda")
    tiny = torch.full_like(dev["decay"][0], 2.0 ** -40)
    for t in range(3):  # 2^-40, 2^-80, then 2^-120 < 2^-96
        st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], tiny, out)
    assert st.check() == 0
    g = st.blobs().cpu().numpy()[:, 16:20].copy().view(np.float32)[:, 0]
    np.testing.assert_array_equal(g, np.ones_like(g))
    st.step(dev["q"][3], dev["k"][3], dev["v"][3], dev["beta"][3], torch.zeros_like(tiny), out)
    assert st.check() == 0
    S = st.dequant().cpu().numpy().reshape(-1, wl.dk, wl.dv)
    nh = wl.batch * wl.heads
    k = d["k"][3].reshape(nh, wl.dk).astype(np.float64)
    v = d["v"][3].reshape(nh, wl.dv).astype(np.float64)
    beta = d["beta"][3].reshape(nh).astype(np.float64)
    for h in range(nh):
        np.testing.assert_allclose(S[h], beta[h] * np.outer(k[h], v[h]), rtol=1e-6, atol=1e-30)


def test_snapshot_restore_continues_bitwise():
    """The blob is pointer-free: copy it after a flush, run on, restore the
    copy, run the same tokens again: identical outputs and states."""
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = SMALL["kda_int8"]
    d = I.draw(wl, 24)
    cfg = B.config_for(wl)
    st = B.LQState(cfg)
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = device_inputs(wl, d)
    out = torch.empty((24, wl.batch, wl.heads, wl.dv), device="cuda")

    def steps(t0, t1):
        for t in range(t0, t1):
            st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out[t])
            if (t + 1) % wl.window == 0:
                st.flush()

    steps(0, 16)
    snap = st.buf.clone()
    steps(16, 24)
    first = out[16:24].clone()
    end = st.buf.clone()
    st.buf.copy_(snap)
    steps(16, 24)
    torch.cuda.synchronize()
    assert torch.equal(first, out[16:24])
    assert torch.equal(end, st.buf)
