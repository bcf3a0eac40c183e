"""Speculative verify / accept on the GPU: after accepting a tokens of a
T-token verify step, every row's state is bit for bit the state of an
a-token decode of the same inputs, and the rows' next tokens agree too."""
import pytest

from linear_attention_recurrent_lq_b200 import inputs as I

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "beta", "decay")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def test_accepted_prefix_equals_direct_decode():
    from linear_attention_recurrent_lq_b200 import binding as B
    from linear_attention_recurrent_lq_b200.speculative import SpeculativeDecoder
    wl = I.WORKLOADS["kda_int8_b128h32"].replace(batch=5, heads=3)
    T = 4
    d = I.draw(wl, T + 1)
    dev = I.to_device(wl, d)
    cfg = B.config_for(wl)
    spec, ref = B.LQState(cfg), B.LQState(cfg)
    for st in (spec, ref):
        st.buf.zero_()
        st.init(torch.from_numpy(d["S0"]).cuda())
    slots = torch.tensor([3, 0, 4, 1, 2], dtype=torch.int32, device="cuda")
    rows = slots.long()  # row n is the sequence in slot slots[n]
    draft = [dev[x][:T].transpose(0, 1)[rows].contiguous() for x in NAMES]
    out = torch.empty((5, T, wl.heads, wl.dv), device="cuda")
    sd = SpeculativeDecoder(spec, max_rows=8)
    sd.verify(slots, T, *draft, out)
    accepted = [4, 0, 2, 1, 3]
    sd.accept(accepted, *draft)
    # the reference: each sequence decoded for exactly its accepted tokens
    for n, a in enumerate(accepted):
        if a == 0:
            continue
        s1 = slots[n:n + 1]
        o = torch.empty((1, a, wl.heads, wl.dv), device="cuda")
        ref.steps_slots(s1, a, *[x[n:n + 1, :a].contiguous() for x in draft], o)
        torch.cuda.synchronize()
        assert torch.equal(o[0], out[n, :a]), n  # the verify step's outputs of the kept tokens
    torch.cuda.synchronize()
    assert torch.equal(spec.buf, ref.buf)
    assert spec.check() == 0
