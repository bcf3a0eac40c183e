"""Extreme gates on the GPU: when a window's decay product falls below 2^-96
the decode moves the window frame (the stored base scales, compensator
entries and buffered keys take the factor; the product restarts at 1)
instead of refusing the token.

The oracle is the dense recurrence, which has no frame: the bar is the same
as for ordinary gates (outputs per window and the final state within 2e-3
relative L2, no status bits).  Multi-token calls that rebase mid-call stay
bitwise equal to single-token calls.  Negative or NaN gates are input
errors: the head is skipped with the RANGE bit.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import REL_L2, oracle_inputs, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
NAMES = ("q", "k", "v", "beta", "decay")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _extreme(wl, d, rng, kda_channels=8):
    """Overwrite the drawn gates: GDN heads get alpha between 2^-45 and 2^-20
    on every token (the product leaves the frame's range within 2 to 5
    tokens); KDA heads get such gates on their first channels only."""
    dec = d["decay"].copy()
    if wl.decay_kind == "kda":
        dec[..., :kda_channels] = 2.0 ** -rng.uniform(20, 45, dec[..., :kda_channels].shape)
    else:
        dec[...] = 2.0 ** -rng.uniform(20, 45, dec.shape)
    d["decay"] = dec.astype(np.float32)
    return d


def _run(wl, d, cfg, T, flush=True):
    from linear_attention_recurrent_lq_b200 import binding as B
    st = B.LQState(cfg)
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = I.to_device(wl, d)
    out = torch.empty((T, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    for t in range(T):
        st.step(*[dev[x][t] for x in NAMES], out[t])
        if flush and (t + 1) % cfg.window == 0:
            st.flush()
    torch.cuda.synchronize()
    return out.cpu().numpy(), st


CASES = {
    "gdn_int8": W["gdn_int8_b64h32"].replace(batch=3, heads=4),
    "gdn_int4_f16": W["gdn_int8_b64h32"].replace(batch=3, heads=4, scale_dtype="f16"),
    "kda_int8": W["kda_int8_b128h32"].replace(batch=3, heads=4),
    "kda_int6_d64_f16": W["kda_int8_b128h32"].replace(batch=3, heads=4, dk=64, dv=64, scale_dtype="f16"),
}
BITS = {"gdn_int8": 8, "gdn_int4_f16": 4, "kda_int8": 8, "kda_int6_d64_f16": 6}


@pytest.mark.parametrize("name", sorted(CASES))
def test_extreme_gates_match_the_dense_recurrence(name):
    from linear_attention_recurrent_lq_b200 import binding as B
    wl, bits = CASES[name], BITS[name]
    T = 40  # two windows of 16 and a partial one
    d = _extreme(wl, I.draw(wl, T), np.random.default_rng(3))
    cfg = B.config_for(wl, bits=bits)
    o_gpu, st = _run(wl, d, cfg, T)
    assert st.check() == 0
    nh = wl.batch * wl.heads
    heads = np.arange(nh)
    p = oracle.Params(**{**oracle.Params.of(wl).__dict__, "bits": bits})
    o_ref, S_ref, _ = oracle.run(p, *oracle_inputs(wl, d, heads, T))
    o_gpu = o_gpu.reshape(T, nh, wl.dv)
    for w0 in range(0, T, wl.window):
        sl = slice(w0, min(T, w0 + wl.window))
        assert rel_l2(o_gpu[sl], o_ref[sl]) < REL_L2, (w0, rel_l2(o_gpu[sl], o_ref[sl]))
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)
    assert rel_l2(S_gpu, S_ref) < REL_L2


def test_multi_token_rebase_equals_single_tokens_bitwise():
    from linear_attention_recurrent_lq_b200 import binding as B
    for name in ("gdn_int8", "kda_int8"):
        wl = CASES[name]
        Tm = 5
        d = _extreme(wl, I.draw(wl, 2 * Tm), np.random.default_rng(4))
        cfg = B.config_for(wl)
        a, b = B.LQState(cfg), B.LQState(cfg)
        a.buf.zero_()
        b.buf.zero_()
        S0 = torch.from_numpy(d["S0"]).cuda()
        a.init(S0)
        b.init(S0)
        dev = I.to_device(wl, d)
        for t0 in (0, Tm):
            ref = torch.empty((Tm, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
            for i in range(Tm):
                a.step(*[dev[x][t0 + i] for x in NAMES], ref[i])
            args = [torch.stack([dev[x][t0 + i] for i in range(Tm)], dim=1).contiguous() for x in NAMES]
            out = torch.empty((wl.batch, Tm, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
            b.steps(Tm, *args, out)
            torch.cuda.synchronize()
            assert torch.equal(out, ref.transpose(0, 1)), name
            assert torch.equal(a.buf, b.buf), name
        assert b.check() == 0


@pytest.mark.parametrize("bad", [-0.5, float("nan")])
def test_invalid_gate_is_an_input_error(bad):
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = CASES["gdn_int8"]
    d = I.draw(wl, 2)
    d["decay"][1, 0, 1] = bad  # token 1, row 0, head 1
    cfg = B.config_for(wl)
    o, st = _run(wl, d, cfg, 2, flush=False)
    assert st.check() == B.LQ_ERR_RANGE
    assert not o[1, 0, 1].any()
    assert np.abs(o[1, 0, 0]).sum() > 0 and np.abs(o[0, 0, 1]).sum() > 0
