"""The host-I/O pipeline (uploads, windows and downloads on three streams,
ordered by events) gives, step after step, exactly the outputs and states of
the plain sequential calls on the same inputs."""
import numpy as np
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


@pytest.mark.parametrize("kind", ["gdn_int8_b64h32", "kda_int8_b128h32"])
def test_pipeline_equals_sequential_calls(kind):
    from linear_attention_recurrent_lq_b200 import binding as B
    from linear_attention_recurrent_lq_b200.pipeline import HostIOPipeline, Layer
    wl = I.WORKLOADS[kind].replace(batch=3, heads=4, window=4)
    Wn, L, steps = wl.window, 3, 3
    # per layer: its own initial state and one window of tokens per step
    draws = []
    for l in range(L):
        s = I.InputStream(wl, stream=l)
        st0 = s.state()
        toks = [s.tokens(Wn) for _ in range(steps)]
        draws.append((st0, toks))
    cfg = B.config_for(wl)
    ref_states, pipe_layers = [], []
    for l, (st0, toks) in enumerate(draws):
        a, b = B.LQState(cfg), B.LQState(cfg)
        a.buf.zero_()
        b.buf.zero_()
        S0 = torch.from_numpy(st0["S0"]).cuda()
        a.init(S0)
        b.init(S0)
        ref_states.append(a)
        dev0 = I.to_device(wl, toks[0])
        host_in = {n: dev0[n].cpu().pin_memory() for n in NAMES}
        dev_in = {n: torch.empty_like(dev0[n]) for n in NAMES}
        dev_out = torch.empty((Wn, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
        pipe_layers.append(Layer(b, dev_in, dev_out, host_in, torch.empty_like(dev_out, device="cpu").pin_memory()))
    torch.cuda.synchronize()
    pipe = HostIOPipeline(pipe_layers, Wn)
    # the capture runs each window once eagerly: give it real inputs, then
    # bring the pipeline's states back to the initial state
    for lay in pipe_layers:
        for n in NAMES:
            lay.dev_in[n].copy_(lay.host_in[n])
    snap = [lay.state.buf.clone() for lay in pipe_layers]
    pipe.capture()
    for lay, s0 in zip(pipe_layers, snap):
        lay.state.buf.copy_(s0)
    torch.cuda.synchronize()
    out_ref = torch.empty((Wn, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda")
    for step in range(steps):
        for l, lay in enumerate(pipe_layers):  # this step's tokens into the pinned buffers
            dev = I.to_device(wl, draws[l][1][step])
            for n in NAMES:
                lay.host_in[n].copy_(dev[n].cpu())
        pipe.fork()
        pipe.step()
        pipe.join()
        torch.cuda.synchronize()
        for l, lay in enumerate(pipe_layers):
            dev = I.to_device(wl, draws[l][1][step])
            a = ref_states[l]
            for t in range(Wn):
                a.step(*[dev[n][t] for n in NAMES], out_ref[t])
            a.flush()
            torch.cuda.synchronize()
            np.testing.assert_array_equal(lay.host_out.numpy(), out_ref.cpu().numpy())
            assert torch.equal(lay.state.buf, a.buf), (step, l)
    for lay in pipe_layers:
        assert lay.state.check() == 0
