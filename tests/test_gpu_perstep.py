"""The naive per-step baselines on the GPU against the oracle: a dense state
stored after every token in BF16, or in FP8 E4M3 with one FP32 scale per
value column (the BF16 and FP8 rows of the news post's accuracy table).

Bars: entering a sequence stores exactly the oracle's rounding of S0 (BF16
values; FP8 scales and values), bit for bit.  Each decode token, taken from
the state the GPU holds (read back exactly), gives outputs within 2e-4
relative L2 of the oracle's FP64 step from that same state.  The stored state
after the token is teacher-forced: the same FP32 values the per-step kernel
rounds are produced by the library's FP32-state step from the same stored
state (the two share their arithmetic), and the oracle's rounding of those
values (BF16 entry by entry; FP8 column scales and codes) must equal what the
GPU stored, with at most 1e-5 of the entries differing.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import REL_L2, STEP_REL, device_inputs, oracle_inputs, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "gdn": W["gdn_int8_b64h32"].replace(batch=3, heads=5),
    "kda": W["kda_int8_b128h32"].replace(batch=3, heads=5),
    "gdn_d64": W["gdn_int8_b64h32"].replace(batch=3, heads=5, dk=64, dv=64),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _params(wl, bits):
    return oracle.Params(dk=wl.dk, dv=wl.dv, window=1, num_comp=0, bits=bits,
                         kda=(wl.decay_kind == "kda"), smoothing=False, per_step=True)


def _stored(bits, S32):
    """The oracle's per-step storage of FP32 states [n, dk, dv] (values)."""
    out = np.empty_like(S32)
    for h in range(S32.shape[0]):
        if bits == 16:
            out[h] = np.vectorize(oracle.round_bf16)(S32[h].astype(np.float64))
        else:
            scale, val = oracle.fp8_columns(S32[h])
            out[h] = (val.astype(np.float64) * scale.astype(np.float64)[None, :]).astype(np.float32)
    return out


def _state(wl, bits):
    from linear_attention_recurrent_lq_b200 import binding as B
    return B.LQState(B.config_for(wl, bits=bits, per_step=True))


@pytest.mark.parametrize("bits", [16, 8])
@pytest.mark.parametrize("name", sorted(CASES))
def test_init_stores_the_oracle_rounding(name, bits):
    wl = CASES[name]
    d = I.draw(wl, 0)
    st = _state(wl, bits)
    st.init(torch.from_numpy(d["S0"]).cuda())
    nh = wl.batch * wl.heads
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)
    S0 = d["S0"].reshape(nh, wl.dk, wl.dv)
    np.testing.assert_array_equal(S_gpu, _stored(bits, S0))
    if bits == 8:
        torch.cuda.synchronize()
        blobs = st.blobs().cpu().numpy()
        for h in range(nh):
            scale_gpu = blobs[h, 128:128 + 4 * wl.dv].view(np.float32)
            np.testing.assert_array_equal(scale_gpu, oracle.fp8_columns(S0[h])[0])
    assert st.check() == 0


@pytest.mark.parametrize("bits", [16, 8])
@pytest.mark.parametrize("name", sorted(CASES))
def test_decode_steps_from_the_stored_state(name, bits):
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = CASES[name]
    T = 6
    d = I.draw(wl, T)
    dev = device_inputs(wl, d)
    st = _state(wl, bits)
    st.init(torch.from_numpy(d["S0"]).cuda())
    st32 = B.LQState(B.config_for(wl, bits=32))
    nh = wl.batch * wl.heads
    heads = np.arange(nh)
    _, q, k, v, beta, decay = oracle_inputs(wl, d, heads, T)
    out = torch.empty((wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    out32 = torch.empty_like(out)
    p = _params(wl, bits)
    for t in range(T):
        S_prev_t = st.dequant()
        S_prev = S_prev_t.cpu().numpy().reshape(nh, wl.dk, wl.dv)
        # the FP32 values the per-step kernel rounds: the FP32-state step from
        # the same stored state (init copies it exactly)
        st32.init(S_prev_t)
        st32.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out32)
        st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out)
        torch.cuda.synchronize()
        o_gpu = out.cpu().numpy().reshape(nh, wl.dv)
        S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)
        S32 = st32.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)
        # the output comes before the store's rounding: the same bits as FP32
        np.testing.assert_array_equal(o_gpu, out32.cpu().numpy().reshape(nh, wl.dv))
        o_ref, S_ref, _ = oracle.run(p, S_prev, q[t:t + 1], k[t:t + 1], v[t:t + 1], beta[t:t + 1],
                                     decay[t:t + 1])
        assert rel_l2(o_gpu, o_ref[0]) < STEP_REL, (t, rel_l2(o_gpu, o_ref[0]))
        assert rel_l2(S_gpu, S_ref) < (STEP_REL if bits == 16 else REL_L2), (t, rel_l2(S_gpu, S_ref))
        # teacher-forced storage: the oracle's rounding of the same FP32 values
        expect = _stored(bits, S32)
        off = S_gpu.view(np.uint32) != expect.view(np.uint32)
        assert off.mean() <= 1e-5, (t, off.mean())
        if bits == 8:
            blobs = st.blobs().cpu().numpy()
            for h in range(nh):
                scale_gpu = blobs[h, 128:128 + 4 * wl.dv].view(np.float32)
                np.testing.assert_array_equal(scale_gpu, oracle.fp8_columns(S32[h])[0])
    assert st.check() == 0


def test_flush_is_a_no_op_for_per_step_states():
    wl = CASES["gdn"]
    d = I.draw(wl, 0)
    st = _state(wl, 8)
    st.init(torch.from_numpy(d["S0"]).cuda())
    before = st.buf.clone()
    st.flush()
    torch.cuda.synchronize()
    assert torch.equal(before, st.buf)
