"""Failure detection on the GPU, without faulting it.

A bounded wait that nothing satisfies gives up after its limit and the
kernel records LQ_DEV_TIMEOUT instead of hanging; the context stays usable.
Blobs whose headers fail their checks (bad magic, too many compensators, a
compensator index out of range, a window count past W) are flagged CORRUPT
and skipped by decode and flush, every other (slot, head) running exactly as
without them; the checks come before any index from the header is used.
"""
import numpy as np
import pytest

from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import device_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def test_bounded_wait_gives_up_and_the_context_survives():
    from linear_attention_recurrent_lq_b200 import binding as B
    status = torch.full((1,), 0x5A5A, dtype=torch.int32, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    B.lq_selftest_wait(status)
    b.record()
    torch.cuda.synchronize()
    assert int(status.item()) == 0x4  # LQ_DEV_TIMEOUT
    assert 900.0 <= a.elapsed_time(b) < 10000.0  # the one-second limit, then it returns
    # the context still runs work
    wl = I.WORKLOADS["gdn_int8_b64h32"].replace(batch=2, heads=2)
    d = I.draw(wl, 1)
    st = B.LQState(B.config_for(wl))
    st.init(torch.from_numpy(d["S0"]).cuda())
    dev = device_inputs(wl, d)
    out = torch.empty((wl.batch, wl.heads, wl.dv), device="cuda")
    st.step(dev["q"][0], dev["k"][0], dev["v"][0], dev["beta"][0], dev["decay"][0], out)
    assert st.check() == 0 and out.abs().sum() > 0


def test_corrupt_headers_are_flagged_and_skipped():
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = I.WORKLOADS["kda_int8_b128h32"].replace(batch=2, heads=3)
    d = I.draw(wl, 2)
    cfg = B.config_for(wl)
    good, bad = B.LQState(cfg), B.LQState(cfg)
    good.buf.zero_()  # the unused pair slots compare equal too
    bad.buf.zero_()
    S0 = torch.from_numpy(d["S0"]).cuda()
    good.init(S0)
    bad.init(S0)
    torch.cuda.synchronize()
    u32 = bad.blobs().view(torch.int32)  # [N*H, blob/4]
    u32[1, 3] = 0x12345678           # magic
    u32[2, 2] = cfg.num_comp + 1     # compensators in use
    u32[3, 16] = 0x7FFFFFFF & 500    # a compensator index past dk (meta[0], key row)
    u32[4, 0] = cfg.window + 3       # window count
    corrupt = [1, 2, 3, 4]
    dev = device_inputs(wl, d)
    nh = wl.batch * wl.heads
    og = torch.empty((wl.batch, wl.heads, wl.dv), device="cuda")
    ob = torch.full_like(og, float("nan"))
    before = bad.blobs().clone()
    good.step(dev["q"][0], dev["k"][0], dev["v"][0], dev["beta"][0], dev["decay"][0], og)
    bad.step(dev["q"][0], dev["k"][0], dev["v"][0], dev["beta"][0], dev["decay"][0], ob)
    good.flush()
    bad.flush()
    torch.cuda.synchronize()
    assert bad.check() == B.LQ_ERR_CORRUPT and good.check() == 0
    og, ob = og.reshape(nh, -1), ob.reshape(nh, -1)
    gb, bb = good.blobs(), bad.blobs()
    for h in range(nh):
        if h in corrupt:
            assert not ob[h].any() and not ob[h].isnan().any()
            # only the status word changed
            assert torch.equal(bb[h, :4], before[h, :4]) and torch.equal(bb[h, 8:], before[h, 8:])
            assert int(bb[h].view(torch.int32)[1].item()) & 0x8  # LQ_DEV_CORRUPT
        else:
            assert torch.equal(ob[h], og[h])
            assert torch.equal(bb[h], gb[h])
    # the read-back of a corrupt blob is zeros, the others are unaffected
    Sb, Sg = bad.dequant().reshape(nh, -1), good.dequant().reshape(nh, -1)
    for h in range(nh):
        if h in corrupt:
            assert not Sb[h].any()
        else:
            assert torch.equal(Sb[h], Sg[h])
