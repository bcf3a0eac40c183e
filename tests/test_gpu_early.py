"""The early-state flag of lq_decode_step_ex: with states taking turns on
the stream (the previous launch never writes the next one's state), a
window of flagged steps and its flush give, bit for bit, the outputs and
blobs of unflagged steps; for the LeapQuant formats, the FP32-state
reference and the per-step BF16 / FP8 baselines."""
import pytest

from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import device_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "beta", "decay")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


@pytest.mark.parametrize("kind,bits,per_step", [("gdn_int8_b64h32", 8, False), ("kda_int8_b128h32", 4, False),
                                                ("gdn_int8_b64h32", 6, False), ("gdn_int8_b64h32", 32, False),
                                                ("kda_int8_b128h32", 32, False), ("gdn_int8_b64h32", 16, True),
                                                ("kda_int8_b128h32", 8, True)])
def test_early_state_steps_equal_plain_steps(kind, bits, per_step):
    from linear_attention_recurrent_lq_b200 import binding as B
    # 900 heads: two or three per CTA of the LeapQuant decode (three CTAs per
    # SM), so the heads after the early-staged first one take the ordinary
    # path; with 1200 heads the dense kernels (one CTA per SM) walk several
    # heads per CTA as well
    wl = I.WORKLOADS[kind].replace(batch=100 if bits in (8, 6, 4) and not per_step else 40,
                                   heads=9 if bits in (8, 6, 4) and not per_step else 30, window=8)
    L, T = 3, 12  # three layer-states taking turns; a flush after token 8
    draws = [I.InputStream(wl, stream=l) for l in range(L)]
    st0 = [s.state() for s in draws]
    toks = [s.tokens(T) for s in draws]
    cfg = B.config_for(wl, bits=bits, per_step=per_step)
    plain, early = [], []
    for l in range(L):
        for group in (plain, early):
            st = B.LQState(cfg)
            st.buf.zero_()
            st.init(torch.from_numpy(st0[l]["S0"]).cuda())
            group.append(st)
    dev = [device_inputs(wl, toks[l]) for l in range(L)]
    outs = {}
    for name, group, flags in (("plain", plain, 0), ("early", early, B.LQ_STEP_EARLY_STATE)):
        out = torch.empty((T, L, wl.batch, wl.heads, wl.dv), device="cuda")
        for t in range(T):
            for l in range(L):
                group[l].step(*[dev[l][x][t] for x in NAMES], out[t, l], flags=flags)
            if t + 1 == wl.window:
                for l in range(L):
                    group[l].flush()
        torch.cuda.synchronize()
        outs[name] = out
    assert torch.equal(outs["plain"], outs["early"])
    for a, b in zip(plain, early):
        assert torch.equal(a.buf, b.buf)
        assert b.check() == 0
