"""The prefix-cache-scale sweep on the GPU: a 48-head layer mixed 3:1 GDN:KDA
(held as two states, 36 GDN and 12 KDA heads per sequence) over windows
W in {8, 16, 32} and compensator counts r in {2, 4, 8}, at a reduced batch;
and the restore of cached compact blobs into another sequence's slot, which
must continue exactly like the sequence the blobs came from.
"""
import numpy as np
import pytest

import oracle
from linear_attention_recurrent_lq_b200 import inputs as I
from tests.gpu_helpers import REL_L2, device_inputs, oracle_inputs, rel_l2, run_gpu

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

PARTS = ("mix_gdn_b512h36", "mix_kda_b512h12")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from linear_attention_recurrent_lq_b200 import build
    build.build()


@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("window", [8, 16, 32])
@pytest.mark.parametrize("num_comp", [2, 4, 8])
def test_window_and_compensator_sweep(part, window, num_comp):
    """Two windows and a ragged third on two sequences of the layer part:
    every window's outputs and the final state of 24 seeded heads within
    2e-3 relative L2 of the FP64 oracle."""
    wl = I.WORKLOADS[part].replace(batch=2, window=window, num_comp=num_comp)
    T = 2 * window + 3
    d = I.draw(wl, T)
    o_gpu, st = run_gpu(wl, d, T)
    nh = wl.batch * wl.heads
    heads = np.sort(np.random.default_rng(window * 10 + num_comp).choice(nh, min(24, nh), replace=False))
    o_ref, S_ref, _ = oracle.run(oracle.Params.of(wl), *oracle_inputs(wl, d, heads, T))
    o_gpu = o_gpu.reshape(T, nh, wl.dv)[:, heads]
    for w0 in range(0, T, window):
        sl = slice(w0, min(T, w0 + window))
        assert rel_l2(o_gpu[sl], o_ref[sl]) < REL_L2, (w0, rel_l2(o_gpu[sl], o_ref[sl]))
    S_gpu = st.dequant().cpu().numpy().reshape(nh, wl.dk, wl.dv)[heads]
    assert rel_l2(S_gpu, S_ref) < REL_L2
    assert st.check() == 0


@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("at", ["window_start", "mid_window"])
def test_restored_cached_blobs_continue_bitwise(part, at):
    """A blob holds no pointers and no slot index: copying the blobs of
    sequence 0 into the slot of sequence 3 (a prefix-cache hit) and feeding
    both the same tokens gives bit-identical outputs and states, whether the
    copy is taken at a window boundary (after the flush) or mid-window (with
    buffered pairs)."""
    from linear_attention_recurrent_lq_b200 import binding as B
    wl = I.WORKLOADS[part].replace(batch=4, heads=5)
    W = wl.window
    t_copy = W if at == "window_start" else W + 5
    T = t_copy + W + 3
    d = I.draw(wl, T)
    # after the copy, sequence 3 receives sequence 0's tokens
    for key in ("q", "k", "v", "q_bits", "k_bits", "v_bits", "beta", "decay"):
        if key in d:
            d[key][t_copy:, 3] = d[key][t_copy:, 0]
    dev = device_inputs(wl, d)
    st = B.LQState(B.config_for(wl))
    st.init(torch.from_numpy(d["S0"]).cuda())
    out = torch.empty((T, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    H = wl.heads
    for t in range(T):
        if t == t_copy:
            blobs = st.blobs()
            cache = blobs[0:H].clone()       # a cached copy of sequence 0's state
            blobs[3 * H:4 * H].copy_(cache)  # restored into sequence 3's slot
        st.step(dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t], dev["decay"][t], out[t])
        if (t + 1) % W == 0:
            st.flush()
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert np.array_equal(o[t_copy:, 3], o[t_copy:, 0])
    blobs = st.blobs().cpu().numpy()
    assert np.array_equal(blobs[3 * H:4 * H], blobs[0:H])
    assert st.check() == 0
