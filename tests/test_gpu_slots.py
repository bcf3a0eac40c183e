"""Serving through a slot list on the GPU: decode, flush and init over a
subset of the sequences of a larger state buffer, and whole-sequence copies
between buffers (prefix-cache snapshots).

The bar is bitwise: a row run through a slot list goes through the same
kernels and arithmetic as the same sequence run alone, so its outputs and
its blob bytes must equal those of a plain run on a buffer holding only the
active sequences; slots outside the list keep every byte.  Rows whose slot
is out of range touch no blob and get zero outputs.
"""
import numpy as np
import pytest

from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import device_inputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "gdn_int8": (W["gdn_int8_b64h32"].replace(batch=6, heads=3), 8),
    "kda_int4": (W["kda_int8_b128h32"].replace(batch=6, heads=3), 4),
    "gdn_int6_d64": (W["gdn_int8_b64h32"].replace(batch=6, heads=3, dk=64, dv=64), 6),
    "kda_int8_f16": (W["kda_int8_b128h32"].replace(batch=6, heads=3, scale_dtype="f16"), 8),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _state(wl, bits, num_slots, window=4):
    from linear_attention_recurrent_lq_b200 import binding as B
    cfg = B.config_for(wl, bits=bits)
    cfg.window = window
    cfg.num_slots = num_slots
    st = B.LQState(cfg)
    st.buf.zero_()  # padding and unused pair rows compare equal too
    return st


def _rows(x, sel):
    """Rows of the batch axis (the first) of one token's input."""
    return x[sel].contiguous()


def _blob_rows(st, slots):
    H = st.cfg.num_heads
    return torch.cat([st.blobs()[s * H:(s + 1) * H] for s in slots])


def _i32(v):
    return torch.tensor(v, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("name", sorted(CASES))
def test_subset_equals_a_plain_run_bitwise(name):
    wl, bits = CASES[name]
    T = 10  # two flushes, then a partial window
    d = I.draw(wl, T)
    dev = device_inputs(wl, d)
    sel = [4, 1, 3]              # sequences running now
    slots = [5, 0, 2]            # where the server keeps them (N = 7 slots)
    full = _state(wl, bits, num_slots=7)
    alone = _state(wl, bits, num_slots=len(sel))
    # slots the list never names start with a known pattern
    full.buf.copy_(torch.randint(0, 256, full.buf.shape, dtype=torch.uint8, device="cuda"))
    S0 = torch.from_numpy(d["S0"]).cuda()[sel].contiguous()
    alone.init(S0)
    sl = _i32(slots)
    full.init_slots(sl, S0)
    torch.cuda.synchronize()
    untouched = [s for s in range(7) if s not in slots]
    before = _blob_rows(full, untouched).clone()
    # init writes what the plain init writes (padding bytes aside, which the
    # random fill left in the full buffer): compare the dequantized states
    assert torch.equal(full.dequant()[slots], alone.dequant())
    # from here, compare bytes: copy the plain run's blobs in
    H = wl.heads
    for n, s in enumerate(slots):
        full.blobs()[s * H:(s + 1) * H] = alone.blobs()[n * H:(n + 1) * H]
    out_a = torch.empty((len(sel), wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    out_f = torch.full_like(out_a, float("nan"))
    for t in range(T):
        args = [_rows(dev[x][t], sel) for x in ("q", "k", "v", "beta", "decay")]
        alone.step(*args, out_a)
        full.step_slots(sl, *args, out_f)
        if (t + 1) % alone.cfg.window == 0:
            alone.flush()
            full.flush_slots(sl)
        torch.cuda.synchronize()
        assert torch.equal(out_f, out_a), t
        assert torch.equal(_blob_rows(full, slots), alone.blobs()), t
    assert torch.equal(_blob_rows(full, untouched), before)
    assert alone.check() == 0


def test_rows_with_slots_out_of_range_are_skipped():
    wl, bits = CASES["gdn_int8"]
    d = I.draw(wl, 3)
    dev = device_inputs(wl, d)
    N = 4
    st = _state(wl, bits, num_slots=N)
    st.init(torch.from_numpy(d["S0"]).cuda()[:N].contiguous())
    ref = _state(wl, bits, num_slots=N)
    ref.buf.copy_(st.buf)
    sel = [0, 1, 2, 3, 5]
    slots = [2, -1, N, 0, 2 ** 31 - 1]
    sl = _i32(slots)
    out = torch.full((len(sel), wl.heads, wl.dv), float("nan"), device="cuda")
    ref_out = torch.empty((N, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    for t in range(3):
        args = [_rows(dev[x][t], sel) for x in ("q", "k", "v", "beta", "decay")]
        st.step_slots(sl, *args, out)
        st.flush_slots(sl)
        # the reference: the same rows as a plain run on slots 2 and 0 only
        full_args = []
        for x in ("q", "k", "v", "beta", "decay"):
            a = dev[x][t][:N].clone()
            a[2], a[0] = dev[x][t][0], dev[x][t][3]
            full_args.append(a)
        keep = ref.buf.clone()
        ref.step(*full_args, ref_out)
        ref.flush()
        torch.cuda.synchronize()
        # slots 1 and 3 are not in the list: put their bytes back
        H = wl.heads
        for s in (1, 3):
            ref.buf.view(-1, ref.blob_bytes)[s * H:(s + 1) * H] = keep.view(-1, ref.blob_bytes)[s * H:(s + 1) * H]
        assert torch.equal(st.buf, ref.buf), t
        assert torch.equal(out[0], ref_out[2]) and torch.equal(out[3], ref_out[0])
        for n in (1, 2, 4):
            assert not out[n].any() and not out[n].isnan().any()
    # init through a list with bad entries writes only the good ones
    before = st.buf.clone()
    S0 = torch.from_numpy(d["S0"]).cuda()[:2].contiguous()
    st.init_slots(_i32([-3, N + 1]), S0)
    torch.cuda.synchronize()
    assert torch.equal(st.buf, before)
    assert st.check() == 0


def test_copy_restore_continues_bit_for_bit():
    from linear_attention_recurrent_lq_b200 import binding as B
    wl, bits = CASES["kda_int4"]
    T = 9
    d = I.draw(wl, T)
    dev = device_inputs(wl, d)
    N = 6
    st = _state(wl, bits, num_slots=N)
    st.init(torch.from_numpy(d["S0"]).cuda())
    out = torch.empty((N, wl.heads, wl.dv), dtype=torch.float32, device="cuda")

    def steps(t0, t1):
        res = []
        for t in range(t0, t1):
            st.step(*[dev[x][t] for x in ("q", "k", "v", "beta", "decay")], out)
            if (t + 1) % st.cfg.window == 0:
                st.flush()
            res.append(out.clone())
        return res

    steps(0, 3)  # mid-window: pending pairs are part of the snapshot
    P = 5
    pool = torch.zeros(P * wl.heads * st.blob_bytes, dtype=torch.uint8, device="cuda")
    src, dst = [1, 4, 0], [3, 0, 4]
    B.lq_copy_slots(st.cfg, pool, P, _i32(dst), st.buf, N, _i32(src))
    snap = st.buf.clone()
    first = steps(3, T)
    after = st.buf.clone()
    # wreck the snapshotted slots, restore them from the pool, run again
    H = wl.heads
    for s in src:
        st.blobs()[s * H:(s + 1) * H] = 0
    st.buf.view(-1, st.blob_bytes)[2 * H:3 * H] = snap.view(-1, st.blob_bytes)[2 * H:3 * H]
    for s in (3, 5):
        st.buf.view(-1, st.blob_bytes)[s * H:(s + 1) * H] = snap.view(-1, st.blob_bytes)[s * H:(s + 1) * H]
    B.lq_copy_slots(st.cfg, st.buf, N, _i32(src + [7]), pool, P, _i32(dst + [1]))  # last pair out of range
    torch.cuda.synchronize()
    assert torch.equal(st.buf, snap)
    second = steps(3, T)
    torch.cuda.synchronize()
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    assert torch.equal(st.buf, after)


def test_prefix_cache_round_trip_with_eviction():
    from linear_attention_recurrent_lq_b200.prefix_cache import PrefixCache
    wl, bits = CASES["gdn_int8"]
    d = I.draw(wl, 0)
    N = 6
    st = _state(wl, bits, num_slots=N)
    st.init(torch.from_numpy(d["S0"]).cuda())
    st.flush()
    torch.cuda.synchronize()
    snap = st.buf.clone()
    cache = PrefixCache.for_state(st, capacity=2)
    cache.store([("p0", 0), ("p1", 1)])
    cache.store([("p2", 2)])                     # evicts p0
    st.buf.zero_()
    hits = cache.restore([("p2", 5), ("p0", 3), ("p1", 4)])
    torch.cuda.synchronize()
    assert hits == [True, False, True]
    H = wl.heads
    v, sv = st.buf.view(-1, st.blob_bytes), snap.view(-1, st.blob_bytes)
    assert torch.equal(v[5 * H:6 * H], sv[2 * H:3 * H])
    assert torch.equal(v[4 * H:5 * H], sv[1 * H:2 * H])
    assert not v[:4 * H].any()


def test_subset_at_scale_equals_a_plain_run_bitwise():
    """100 of 150 slots with 9 heads: 900 work items, two or three per CTA of
    the decode and multi-token kernels and three or four per CTA of the flush,
    so the slot instances walk several blobs per CTA; single-token steps, a
    four-token step and two flushes, bitwise against a plain run."""
    wl = W["gdn_int8_b64h32"].replace(batch=130, heads=9)
    bits, N, T = 8, 150, 10
    d = I.draw(wl, T)
    dev = device_inputs(wl, d)
    rng = np.random.default_rng(7)
    sel = sorted(rng.choice(wl.batch, 100, replace=False).tolist())
    slots = rng.choice(N, 100, replace=False).tolist()
    full = _state(wl, bits, num_slots=N)
    alone = _state(wl, bits, num_slots=len(sel))
    full.buf.copy_(torch.randint(0, 256, full.buf.shape, dtype=torch.uint8, device="cuda"))
    S0 = torch.from_numpy(d["S0"]).cuda()[sel].contiguous()
    alone.init(S0)
    sl = _i32(slots)
    H = wl.heads
    for n, s in enumerate(slots):
        full.blobs()[s * H:(s + 1) * H] = alone.blobs()[n * H:(n + 1) * H]
    untouched = [s for s in range(N) if s not in slots]
    before = _blob_rows(full, untouched).clone()
    names = ("q", "k", "v", "beta", "decay")
    t = 0
    for p in (1, 1, 1, 1, "flush", 4, "flush", 1, 1):
        if p == "flush":
            alone.flush()
            full.flush_slots(sl)
            continue
        if p == 1:
            args = [_rows(dev[x][t], sel) for x in names]
            out_a = torch.empty((len(sel), H, wl.dv), dtype=torch.float32, device="cuda")
            out_f = torch.full_like(out_a, float("nan"))
            alone.step(*args, out_a)
            full.step_slots(sl, *args, out_f)
        else:
            args = [torch.stack([dev[x][t + i][sel] for i in range(p)], dim=1).contiguous() for x in names]
            out_a = torch.empty((len(sel), p, H, wl.dv), dtype=torch.float32, device="cuda")
            out_f = torch.full_like(out_a, float("nan"))
            alone.steps(p, *args, out_a)
            full.steps_slots(sl, p, *args, out_f)
        torch.cuda.synchronize()
        assert torch.equal(out_f, out_a), t
        assert torch.equal(_blob_rows(full, slots), alone.blobs()), t
        t += p
    assert torch.equal(_blob_rows(full, untouched), before)
    assert alone.check() == 0
