"""Multi-token decode on the GPU: T consecutive tokens per (slot, head) in
one launch (lq_decode_steps), the compact state read once.

The bar is bitwise: token t of a multi-token call runs the same arithmetic
as the t-th of T single-token calls (the same decay products, the same
window-frame keys, the same pairs, read back from the stage instead of the
blob), so outputs and blob bytes must equal those of the single-token path,
which the parity tests hold against the oracle.  One case is also checked
against the oracle directly.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import REL_L2, device_inputs, oracle_inputs, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "gdn_int8": (W["gdn_int8_b64h32"].replace(batch=5, heads=3), 8),
    "kda_int4": (W["kda_int8_b128h32"].replace(batch=5, heads=3), 4),
    "gdn_int6_d64": (W["gdn_int8_b64h32"].replace(batch=5, heads=3, dk=64, dv=64), 6),
    "kda_int8_f16": (W["kda_int8_b128h32"].replace(batch=5, heads=3, scale_dtype="f16"), 8),
    "gdn_int8_d64_f32in": (W["gdn_int8_b64h32"].replace(batch=5, heads=3, dk=64, dv=64, in_dtype="f32"), 8),
}
NAMES = ("q", "k", "v", "beta", "decay")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _state(wl, bits, window, num_slots=None):
    from linear_attention_recurrent_lq_b200 import binding as B
    cfg = B.config_for(wl, bits=bits)
    cfg.window = window
    if num_slots is not None:
        cfg.num_slots = num_slots
    st = B.LQState(cfg)
    st.buf.zero_()
    return st


def _stack(dev, t0, T, rows=None):
    """Tokens t0 .. t0+T-1 of every input as [rows, T, ...]."""
    out = []
    for x in NAMES:
        a = torch.stack([dev[x][t0 + i] for i in range(T)], dim=1)
        out.append((a if rows is None else a[rows]).contiguous())
    return out


def _single(st, dev, t0, T, out_tok):
    for i in range(T):
        st.step(*[dev[x][t0 + i] for x in NAMES], out_tok[i])


@pytest.mark.parametrize("name", sorted(CASES))
def test_multi_token_equals_single_tokens_bitwise(name):
    wl, bits = CASES[name]
    Wn = 8
    plan = [3, 3, 2, "flush", 4, 4, "flush", 8, "flush", 1, 5]  # tokens per call
    n_tok = sum(p for p in plan if p != "flush")
    d = I.draw(wl, n_tok)
    dev = device_inputs(wl, d)
    S0 = torch.from_numpy(d["S0"]).cuda()
    a, b = _state(wl, bits, Wn), _state(wl, bits, Wn)
    a.init(S0)
    b.init(S0)
    t0 = 0
    for p in plan:
        if p == "flush":
            a.flush()
            b.flush()
            continue
        ref = torch.empty((p, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        _single(a, dev, t0, p, ref)
        out = torch.full((wl.batch, p, wl.heads, wl.dv), float("nan"), device="cuda")
        b.steps(p, *_stack(dev, t0, p), out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref.transpose(0, 1)), (name, t0, p)
        assert torch.equal(a.buf, b.buf), (name, t0, p)
        t0 += p
    assert b.check() == 0


def test_multi_token_sequence_matches_oracle():
    wl, bits = CASES["gdn_int8"]
    Wn, T = 8, 4
    n_tok = 16
    d = I.draw(wl, n_tok)
    dev = device_inputs(wl, d)
    st = _state(wl, bits, Wn)
    st.init(torch.from_numpy(d["S0"]).cuda())
    outs = []
    for t0 in range(0, n_tok, T):
        out = torch.empty((wl.batch, T, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        st.steps(T, *_stack(dev, t0, T), out)
        if (t0 + T) % Wn == 0:
            st.flush()
        outs.append(out.transpose(0, 1))
    torch.cuda.synchronize()
    o_gpu = torch.cat(outs).cpu().numpy().reshape(n_tok, -1, wl.dv)
    nh = wl.batch * wl.heads
    heads = np.arange(nh)
    p = oracle.Params(**{**oracle.Params.of(wl).__dict__, "window": Wn})
    o_ref, S_ref, _ = oracle.run(p, *oracle_inputs(wl, d, heads, n_tok))
    assert rel_l2(o_gpu, o_ref) < REL_L2
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)
    assert rel_l2(S_gpu, S_ref) < REL_L2


def test_window_without_room_skips_the_whole_head():
    wl, bits = CASES["gdn_int8"]
    Wn = 8
    d = I.draw(wl, 10)
    dev = device_inputs(wl, d)
    st = _state(wl, bits, Wn)
    st.init(torch.from_numpy(d["S0"]).cuda())
    out = torch.empty((wl.batch, 6, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    st.steps(6, *_stack(dev, 0, 6), out)
    torch.cuda.synchronize()
    before = st.buf.clone()
    out3 = torch.full((wl.batch, 3, wl.heads, wl.dv), float("nan"), device="cuda")
    st.steps(3, *_stack(dev, 6, 3), out3)  # 6 + 3 > 8
    torch.cuda.synchronize()
    assert not out3.any() and not out3.isnan().any()
    from linear_attention_recurrent_lq_b200 import binding as B
    assert st.check() == B.LQ_ERR_WINDOW_FULL
    # only the status words changed
    v, bv = st.blobs(), before.view(-1, st.blob_bytes)
    assert torch.equal(v[:, :4], bv[:, :4]) and torch.equal(v[:, 8:], bv[:, 8:])


def test_invalid_gate_mid_call_keeps_the_earlier_tokens():
    """A NaN gate at the third token of a head: tokens 0 and 1 commit; the
    rest of that head is skipped with the RANGE bit, exactly as single-token
    calls behave."""
    wl, bits = CASES["gdn_int8"]
    Wn, T = 8, 5
    d = I.draw(wl, T)
    dev = device_inputs(wl, d)
    dev["decay"][2, 1, 2] = float("nan")  # token 2, row 1, head 2
    a, b = _state(wl, bits, Wn), _state(wl, bits, Wn)
    S0 = torch.from_numpy(d["S0"]).cuda()
    a.init(S0)
    b.init(S0)
    ref = torch.empty((T, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    _single(a, dev, 0, T, ref)
    out = torch.full((wl.batch, T, wl.heads, wl.dv), float("nan"), device="cuda")
    b.steps(T, *_stack(dev, 0, T), out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.transpose(0, 1))
    assert torch.equal(a.buf, b.buf)
    assert out[1, :2, 2].abs().sum() > 0 and not out[1, 2:, 2].any()
    assert out[0].abs().sum() > 0
    from linear_attention_recurrent_lq_b200 import binding as B
    assert b.check() == B.LQ_ERR_RANGE


def test_multi_token_through_a_slot_list():
    wl, bits = CASES["kda_int4"]
    Wn, T = 8, 4
    d = I.draw(wl, 2 * T)
    dev = device_inputs(wl, d)
    sel, slots = [3, 0, 4], [1, 6, 2]
    full, alone = _state(wl, bits, Wn, num_slots=7), _state(wl, bits, Wn, num_slots=3)
    S0 = torch.from_numpy(d["S0"]).cuda()[sel].contiguous()
    alone.init(S0)
    sl = torch.tensor(slots, dtype=torch.int32, device="cuda")
    full.init_slots(sl, S0)
    torch.cuda.synchronize()
    H = wl.heads
    for n, s in enumerate(slots):  # same bytes to start from
        full.blobs()[s * H:(s + 1) * H] = alone.blobs()[n * H:(n + 1) * H]
    for t0 in (0, T):
        args = _stack(dev, t0, T, rows=sel)
        oa = torch.empty((3, T, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        of = torch.empty_like(oa)
        alone.steps(T, *args, oa)
        full.steps_slots(sl, T, *args, of)
        torch.cuda.synchronize()
        assert torch.equal(oa, of)
        for n, s in enumerate(slots):
            assert torch.equal(full.blobs()[s * H:(s + 1) * H], alone.blobs()[n * H:(n + 1) * H])


def test_multi_token_at_the_largest_window_and_compensator_count():
    """W = 64, r = 16, T = 8 (KDA, the largest stage): a whole window in
    eight calls, then the flush, bitwise equal to single-token calls."""
    wl = W["kda_int8_b128h32"].replace(batch=2, heads=2, num_comp=16)
    bits, Wn, T = 8, 64, 8
    d = I.draw(wl, Wn)
    dev = device_inputs(wl, d)
    a, b = _state(wl, bits, Wn), _state(wl, bits, Wn)
    S0 = torch.from_numpy(d["S0"]).cuda()
    a.init(S0)
    b.init(S0)
    for t0 in range(0, Wn, T):
        ref = torch.empty((T, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        _single(a, dev, t0, T, ref)
        out = torch.empty((wl.batch, T, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        b.steps(T, *_stack(dev, t0, T), out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref.transpose(0, 1)), t0
    a.flush()
    b.flush()
    torch.cuda.synchronize()
    assert torch.equal(a.buf, b.buf)
    assert b.check() == 0


@pytest.mark.parametrize("kind,bits", [("gdn_int8_b64h32", 8), ("kda_int8_b128h32", 4)])
def test_multi_token_with_several_heads_per_cta_bitwise(kind, bits):
    """900 heads: two or three per CTA of the multi-token kernel, so the
    prep warp runs a head ahead, stages and prep buffers are reused and the
    next head's codes load during the current one; T = 4 and 3 (four-token
    instance) and T = 5 (eight-token instance), across a flush, bitwise equal
    to single-token calls."""
    wl = W[kind].replace(batch=100, heads=9)
    Wn = 8
    plan = [4, 3, 1, "flush", 5, 3]
    n_tok = sum(p for p in plan if p != "flush")
    d = I.draw(wl, n_tok)
    dev = device_inputs(wl, d)
    S0 = torch.from_numpy(d["S0"]).cuda()
    a, b = _state(wl, bits, Wn), _state(wl, bits, Wn)
    a.init(S0)
    b.init(S0)
    t0 = 0
    for p in plan:
        if p == "flush":
            a.flush()
            b.flush()
            continue
        ref = torch.empty((p, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        _single(a, dev, t0, p, ref)
        out = torch.full((wl.batch, p, wl.heads, wl.dv), float("nan"), device="cuda")
        if p == 1:
            b.step(*[dev[x][t0] for x in NAMES], out[:, 0])
        else:
            b.steps(p, *_stack(dev, t0, p), out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref.transpose(0, 1)), (kind, t0, p)
        assert torch.equal(a.buf, b.buf), (kind, t0, p)
        t0 += p
    assert b.check() == 0
