"""Prompt handoff on the GPU (lq_prefill): the FP32 delta rule over each
row's prompt with the state on chip, then its compression into a fresh blob.

Bars: outputs and the final FP32 state within 2e-3 relative L2 of the FP64
oracle (FP32 accumulation over the prompt); the blob compresses the GPU's own
final FP32 state bit for bit as the oracle does (no code flips), as the init
does; outputs past a row's length are zero; T = 0 is the init; a slot-list
prefill writes exactly the blobs a plain prefill of those rows writes.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests import blob
from tests.gpu_helpers import REL_L2, compare_compressed, oracle_inputs, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

W = I.WORKLOADS
CASES = {
    "gdn_int8": (W["gdn_int8_b64h32"].replace(batch=5, heads=3), 8),
    "kda_int4": (W["kda_int8_b128h32"].replace(batch=5, heads=3), 4),
    "gdn_int6_d64": (W["gdn_int8_b64h32"].replace(batch=5, heads=3, dk=64, dv=64), 6),
    "kda_int8_f16_f32in": (W["kda_int8_b128h32"].replace(batch=5, heads=3, scale_dtype="f16",
                                                         in_dtype="f32"), 8),
}
NAMES = ("q", "k", "v", "beta", "decay")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


def _state(wl, bits, num_slots=None):
    from linear_attention_recurrent_lq_b200 import binding as B
    cfg = B.config_for(wl, bits=bits)
    if num_slots is not None:
        cfg.num_slots = num_slots
    st = B.LQState(cfg)
    st.buf.zero_()
    return st


def _row_major(wl, d, T, rows=None):
    """Prompt inputs [rows, T, H, .] on the device, in the library's dtypes."""
    dev = I.to_device(wl, d)
    out = []
    for x in NAMES:
        a = dev[x][:T].transpose(0, 1)
        out.append((a if rows is None else a[rows]).contiguous())
    return out


def _params(wl, bits):
    return oracle.Params(**{**oracle.Params.of(wl).__dict__, "bits": bits})


@pytest.mark.parametrize("name", sorted(CASES))
def test_prefill_matches_oracle(name):
    wl, bits = CASES[name]
    T = 40  # two chunks of 16 and a ragged one
    lens = [40, 0, 17, 33, 16]
    d = I.draw(wl, T)
    st = _state(wl, bits)
    nh, H = wl.batch * wl.heads, wl.heads
    out = torch.full((wl.batch, T, H, wl.dv), float("nan"), device="cuda")
    S_fin = torch.empty((wl.batch, H, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
    lengths = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st.prefill(T, *_row_major(wl, d, T), S0=torch.from_numpy(d["S0"]).cuda(), lengths=lengths,
               out=out, S_final=S_fin)
    torch.cuda.synchronize()
    p = _params(wl, bits)
    heads = np.arange(nh)
    o_ref, S_ref, _ = oracle.prefill(p, *oracle_inputs(wl, d, heads, T), lengths=np.repeat(lens, H))
    o_gpu = out.transpose(0, 1).cpu().numpy().reshape(T, nh, wl.dv)
    S_gpu = S_fin.cpu().numpy().reshape(nh, wl.dk, wl.dv)
    for h in range(nh):
        n = lens[h // H]
        assert not o_gpu[n:, h].any() and not np.isnan(o_gpu[:, h]).any()
        if n:
            assert rel_l2(o_gpu[:n, h], o_ref[:n, h]) < REL_L2, (h, rel_l2(o_gpu[:n, h], o_ref[:n, h]))
        assert rel_l2(S_gpu[h], S_ref[h]) < REL_L2, h
    blobs = st.blobs().cpu().numpy()
    for h in range(nh):
        got = blob.parse(p, blobs[h])
        assert (got["count"], got["status"], got["magic"]) == (0, 0, blob.MAGIC)
        np.testing.assert_array_equal(got["g"], np.ones(wl.dk, np.float32))
        r = compare_compressed(p, S_gpu[h], got)
        assert r["flips"] == 0, (h, r)
    assert st.check() == 0


def test_zero_tokens_is_the_init_and_null_S0_is_zero():
    wl, bits = CASES["gdn_int8"]
    d = I.draw(wl, 4)
    S0 = torch.from_numpy(d["S0"]).cuda()
    a, b = _state(wl, bits), _state(wl, bits)
    a.init(S0)
    b.prefill(0, None, None, None, None, None, S0=S0)
    torch.cuda.synchronize()
    assert torch.equal(a.buf, b.buf)
    # a prompt from S0 = 0 and from no S0 at all
    T = 4
    c, e = _state(wl, bits), _state(wl, bits)
    args = _row_major(wl, d, T)
    c.prefill(T, *args, S0=torch.zeros_like(S0))
    e.prefill(T, *args)
    torch.cuda.synchronize()
    assert torch.equal(c.buf, e.buf)


def test_prefill_through_a_slot_list():
    wl, bits = CASES["kda_int4"]
    T = 21
    d = I.draw(wl, T)
    sel, slots = [4, 1, 2], [0, 5, 3]
    lens = torch.tensor([21, 9, 0], dtype=torch.int32, device="cuda")
    full, alone = _state(wl, bits, num_slots=6), _state(wl, bits, num_slots=3)
    full.buf.copy_(torch.randint(0, 256, full.buf.shape, dtype=torch.uint8, device="cuda"))
    before = full.buf.clone()
    S0 = torch.from_numpy(d["S0"]).cuda()[sel].contiguous()
    args = _row_major(wl, d, T, rows=sel)
    oa = torch.empty((3, T, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    of = torch.empty_like(oa)
    alone.prefill(T, *args, S0=S0, lengths=lens, out=oa)
    from linear_attention_recurrent_lq_b200 import binding as B
    B.lq_prefill_slots(full.cfg, full.buf, torch.tensor(slots, dtype=torch.int32, device="cuda"), T, *args,
                       S0=S0, lengths=lens, out=of)
    torch.cuda.synchronize()
    assert torch.equal(oa, of)
    H = wl.heads
    # the written blobs equal the plain prefill's in every byte the init writes;
    # compare their dense read-back, and the untouched slots byte for byte
    Sf, Sa = full.dequant(), alone.dequant()
    for n, s in enumerate(slots):
        assert torch.equal(Sf[s], Sa[n])
    fb, bb = full.blobs(), before.view(-1, full.blob_bytes)
    for s in (1, 2, 4):
        assert torch.equal(fb[s * H:(s + 1) * H], bb[s * H:(s + 1) * H])


def test_full_size_prefill_sampled_heads():
    """The bench's prefill shape (64 rows x 32 heads, dk = dv = 128, INT8), a
    prompt of 64 tokens; eight sampled heads against the oracle."""
    wl, bits = W["gdn_int8_b64h32"], 8
    T = 64
    d = I.draw(wl, T)
    st = _state(wl, bits)
    H, nh = wl.heads, wl.batch * wl.heads
    out = torch.empty((wl.batch, T, H, wl.dv), dtype=torch.float32, device="cuda")
    S_fin = torch.empty((wl.batch, H, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
    st.prefill(T, *_row_major(wl, d, T), S0=torch.from_numpy(d["S0"]).cuda(), out=out, S_final=S_fin)
    torch.cuda.synchronize()
    heads = np.random.default_rng(5).choice(nh, 8, replace=False)
    p = _params(wl, bits)
    o_ref, S_ref, _ = oracle.prefill(p, *oracle_inputs(wl, d, heads, T))
    o_gpu = out.transpose(0, 1).reshape(T, nh, wl.dv)[:, torch.from_numpy(heads).cuda()].cpu().numpy()
    S_gpu = S_fin.reshape(nh, wl.dk, wl.dv)[torch.from_numpy(heads).cuda()].cpu().numpy()
    assert rel_l2(o_gpu, o_ref) < REL_L2
    assert rel_l2(S_gpu, S_ref) < REL_L2
    blobs = st.blobs().cpu().numpy()
    for x, h in enumerate(heads):
        r = compare_compressed(p, S_gpu[x], blob.parse(p, blobs[h]))
        assert r["flips"] == 0, (h, r)
    assert st.check() == 0


def test_one_token_prompts_and_empty_prompts():
    """T = 1, and a length list of zeros (every row keeps S0: the blob equals
    the init's, the outputs are zero)."""
    wl, bits = CASES["gdn_int8"]
    d = I.draw(wl, 1)
    S0 = torch.from_numpy(d["S0"]).cuda()
    st = _state(wl, bits)
    out = torch.empty((wl.batch, 1, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    st.prefill(1, *_row_major(wl, d, 1), S0=S0, out=out)
    torch.cuda.synchronize()
    nh, H = wl.batch * wl.heads, wl.heads
    o_ref, _, _ = oracle.prefill(_params(wl, bits), *oracle_inputs(wl, d, np.arange(nh), 1))
    assert rel_l2(out.transpose(0, 1).cpu().numpy().reshape(1, nh, wl.dv), o_ref) < REL_L2
    z, ini = _state(wl, bits), _state(wl, bits)
    outz = torch.full((wl.batch, 1, wl.heads, wl.dv), float("nan"), device="cuda")
    z.prefill(1, *_row_major(wl, d, 1), S0=S0, out=outz,
              lengths=torch.zeros(wl.batch, dtype=torch.int32, device="cuda"))
    ini.init(S0)
    torch.cuda.synchronize()
    assert not outz.any() and not outz.isnan().any()
    assert torch.equal(z.buf, ini.buf)
    assert z.check() == 0 and st.check() == 0


@pytest.mark.parametrize("name", ["gdn_int8", "kda_int8_f16_f32in"])
def test_prefill_extreme_gates_split_chunks(name):
    """Gates of 0 and gate products far below the chunk range (1e-13 on every
    channel, 1e-30 on one key channel), over a prompt of several chunks with
    ragged lengths: the chunkwise prefill ends a chunk before each such token
    and stays within 2e-3 of the FP64 oracle."""
    wl, bits = CASES[name]
    T = 150
    lens = [150, 63, 130, 1, 97]
    d = I.draw(wl, T)
    dec = d["decay"]
    if wl.decay_kind == "kda":
        dec[20, :, :, 7] = 0.0          # one channel's gate is 0
        dec[70] = 1e-13                 # every channel, every head
        dec[90, :, :, 3] = 1e-30
        dec[0, 1, :, 5] = 0.0           # a zero gate on a row's first token
    else:
        dec[20] = 0.0
        dec[70] = 1e-13
        dec[0, 1] = 0.0
    st = _state(wl, bits)
    nh, H = wl.batch * wl.heads, wl.heads
    out = torch.empty((wl.batch, T, H, wl.dv), dtype=torch.float32, device="cuda")
    S_fin = torch.empty((wl.batch, H, wl.dk, wl.dv), dtype=torch.float32, device="cuda")
    lengths = torch.tensor(lens, dtype=torch.int32, device="cuda")
    st.prefill(T, *_row_major(wl, d, T), S0=torch.from_numpy(d["S0"]).cuda(), lengths=lengths,
               out=out, S_final=S_fin)
    torch.cuda.synchronize()
    p = _params(wl, bits)
    o_ref, S_ref, _ = oracle.prefill(p, *oracle_inputs(wl, d, np.arange(nh), T), lengths=np.repeat(lens, H))
    o_gpu = out.transpose(0, 1).cpu().numpy().reshape(T, nh, wl.dv)
    S_gpu = S_fin.cpu().numpy().reshape(nh, wl.dk, wl.dv)
    for h in range(nh):
        n = lens[h // H]
        assert np.isfinite(o_gpu[:, h]).all() and not o_gpu[n:, h].any()
        assert rel_l2(o_gpu[:n, h], o_ref[:n, h]) < REL_L2, (h, rel_l2(o_gpu[:n, h], o_ref[:n, h]))
        assert rel_l2(S_gpu[h], S_ref[h]) < REL_L2, (h, rel_l2(S_gpu[h], S_ref[h]))
    assert st.check() == 0
