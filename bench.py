#!/usr/bin/env python
"""Decode throughput of the LeapQuant low-bit recurrent state on B200.

Metric: decode head-tokens/s (one head-token = one (sequence, head) state
advanced by one generated token) and the achieved HBM bandwidth of the decode
kernel against the measured copy bandwidth, next to the library's own
FP32-state kernel on the same inputs.

Workload (default gdn_int8_b64h32): Gated DeltaNet heads, batch 64 x 32 heads,
dk = dv = 128, INT8 state with smoothing, W = 16, r = 4 compensators, bf16
q/k/v.  One step = one window: W decode tokens over L layer-states (each its
own 64 x 32 heads, as consecutive linear-attention layers of a model), then
the L window flushes.  Rotating L = 8 layers keeps the working set (~0.6 GB of
state) well above the 126 MB L2, so every token re-reads its state from HBM;
no L2 flush is needed.  Inputs are seeded synthetic draws, resident in HBM
before timing; every step reuses the same window of inputs on an evolving
state.  The decodes go through lq_decode_step_ex with LQ_STEP_EARLY_STATE
when two or more layer-states rotate (the launch before each decode is then
always another state's).

Besides the headline line, the JSON carries, each timed on its own:
fp32_state (the FP32-state kernel on the same inputs), per_step_baselines
(BF16, FP8 E4M3 and INT8 states stored every token), multi_token (T tokens
per launch), prefill (a 256-token prompt then compression), serving_slots
(decode and flush through a shuffled slot list), e2e (host buffers, the
transfers overlapped with the kernels) and cpu_baseline (the oracle on the
host cores).

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run, one process per GPU, each rank advancing its own
replica of the workload (independent sequences: no collective on the data
path), timed as the max over ranks.  --impl reference times the CPU oracle
(the FP64 restatement of the method) on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gdn_int8_b64h32")
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--fp32-steps", type=int, default=0, help="0: steps/4")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0: steps/10")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp32", action="store_true")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip the naive per-step BF16 / FP8 / INT8 states")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mt-tokens", type=int, default=4,
                    help="tokens per launch of the multi-token decode line (0: skip it)")
    ap.add_argument("--prefill-tokens", type=int, default=256,
                    help="prompt length of the prefill line (0: skip it)")
    ap.add_argument("--no-slots", action="store_true",
                    help="skip the serving path (decode and flush through a slot list)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per_config lines (KDA INT8, GDN 6-bit and 4-bit, the mixed sweep)")
    ap.add_argument("--config-steps", type=int, default=40,
                    help="timed window-steps of each per_config workload")
    ap.add_argument("--sweep-tokens", type=int, default=4096,
                    help="decode tokens of each point of the prefix-cache-scale sweep")
    ap.add_argument("--sweep", default="8x2,8x4,8x8,16x2,16x4,16x8,32x2,32x4,32x8",
                    help="WxR points of the prefix-cache-scale sweep (empty: skip it)")
    return ap.parse_args()


# ------------------------------------------------------------ byte model

def field_bytes(wl):
    """Bytes of every blob field and input, per head (no padding)."""
    dk, dv, r = wl.dk, wl.dv, wl.num_comp
    sb = 2 if wl.scale_dtype == "f16" else 4
    ib = 2 if wl.in_dtype == "bf16" else 4
    kda = wl.decay_kind == "kda"
    return dict(
        hdr=20, meta=4 * r, qs=sb * dv, sm=sb * dk, cvec=4 * r * max(dk, dv),
        codes=dv * dk * wl.bits // 8, pair=4 * (dk + dv), g=4 * dk if kda else 0,
        inputs=ib * (2 * dk + dv) + 4 + (4 * dk if kda else 4), out=4 * dv)


def decode_bytes(wl, count):
    """Algorithmic bytes one decode step moves for one head with `count`
    pairs already buffered: it reads the header, scales, compensators, codes,
    the buffered pairs, the decay product and the token's inputs, and writes
    the output, the new pair, the decay product and the count."""
    f = field_bytes(wl)
    read = (f["hdr"] + f["meta"] + f["qs"] + f["sm"] + f["cvec"] + f["codes"] + count * f["pair"]
            + f["g"] + f["inputs"])
    write = f["out"] + f["pair"] + f["g"] + 8
    return read + write


def multi_decode_bytes(wl, count, T):
    """Algorithmic bytes of one T-token decode launch for one head with
    `count` pairs buffered before it: the compact state, the pairs and the
    decay product are read once; every token reads its inputs and writes its
    output and its pair."""
    f = field_bytes(wl)
    read = (f["hdr"] + f["meta"] + f["qs"] + f["sm"] + f["cvec"] + f["codes"] + count * f["pair"]
            + f["g"] + T * f["inputs"])
    write = T * (f["out"] + f["pair"]) + f["g"] + 8
    return read + write


def flush_bytes(wl):
    """Algorithmic bytes of one window flush per head: read the compact state,
    W pairs and the decay product; write the new compact state and header."""
    f = field_bytes(wl)
    compact = f["qs"] + f["sm"] + f["cvec"] + f["codes"]
    return (f["hdr"] + f["meta"] + compact + wl.window * f["pair"] + f["g"]) + \
           (compact + f["meta"] + 16 + f["g"])


def per_step_bytes(wl, fmt):
    """Per-step baseline per head-token: read and write the stored state
    (BF16 entries, or FP8 codes plus f32 column scales), read the inputs,
    write the output."""
    f = field_bytes(wl)
    state = 2 * wl.dk * wl.dv if fmt == "bf16" else wl.dk * wl.dv + 4 * wl.dv
    return 2 * state + f["inputs"] + f["out"]


def state_memory(wl, B):
    """Bytes of state per (sequence, head): the LeapQuant blob (window buffer
    included), its compact part alone (what a flushed prefix-cache entry
    holds), and the FP32-state blob; plus the whole layer at this workload."""
    lq = B.lq_state_bytes(B.config_for(wl))
    f32 = B.lq_state_bytes(B.config_for(wl, bits=32))
    f = field_bytes(wl)
    compact = f["hdr"] + f["meta"] + f["qs"] + f["sm"] + f["cvec"] + f["codes"] + f["g"]
    nh = wl.batch * wl.heads
    return {"leapquant_blob_bytes": lq, "leapquant_compact_bytes": compact, "fp32_blob_bytes": f32,
            "layer_leapquant_mb": nh * lq / 1e6, "layer_fp32_mb": nh * f32 / 1e6,
            "compact_vs_fp32": f32 / compact}


def fp32_bytes(wl):
    """FP32-state step per head: read and write the dense state, read inputs,
    write the output."""
    f = field_bytes(wl)
    return 2 * 4 * wl.dk * wl.dv + f["inputs"] + f["out"]


def restore_bytes(wl):
    """A prefix-cache hit: the compact part of a flushed blob is read from the
    pool and written into a live slot (algorithmic bytes per head; the copy
    itself moves whole blobs)."""
    f = field_bytes(wl)
    compact = f["hdr"] + f["meta"] + f["qs"] + f["sm"] + f["cvec"] + f["codes"] + f["g"]
    return 2 * compact


def head_token_bytes(wl):
    """Window-mean algorithmic bytes per head-token, the flush amortised."""
    W = wl.window
    return (sum(decode_bytes(wl, c) for c in range(W)) + flush_bytes(wl)) / W


# ------------------------------------------------------------ helpers

def strip_comments(src: str) -> str:
    """C/C++ source without comments and blank space: what the compiler sees
    of it (string literals with comment markers do not occur in these files)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


# NVIDIA's HBM3e figure for a B200 (8 TB/s), the second denominator beside
# the measured copy bandwidth
SPEC_HBM_GBS = 8000.0


def kernel_source_sha():
    """Hash of the CUDA sources and the C header, comments left out, so a
    profile taken on the same code stays valid across comment edits."""
    h = hashlib.sha256()
    paths = sorted(os.path.join(ROOT, "linear_attention_recurrent_lq_b200", "csrc", n)
                   for n in os.listdir(os.path.join(ROOT, "linear_attention_recurrent_lq_b200", "csrc")))
    for p in paths + [os.path.join(ROOT, "include", "leapquant.h")]:
        with open(p, encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "kernel_source_sha")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha") != kernel_source_sha():
        return None
    try:
        return int(float(vals["traffic_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            return json.load(fh), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class Clocks:
    """nvidia-smi samples of one GPU while the timed region runs."""

    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and self.uuid not in parts[1]:
                continue
            rows.append(parts)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][3]) if rows[0][3].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[4]) for r in rows
                                   if r[4].replace(".", "").isdigit()) if rows else None}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(vals, torch, dist, world, device):
    """Element-wise maximum of a list of times over all ranks (the job takes
    as long as its slowest rank); the identity on one rank."""
    if world <= 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def rank_workload(wl, rank):
    """Each rank runs its own independent sequences (weak scaling: replicas,
    no exchange between ranks): same shapes, another seed."""
    return wl if rank == 0 else wl.replace(seed=wl.seed + 1000 * rank)


def whole_job_rate(units_per_rank, world, ms):
    """Units per second of the whole job: every rank's units over the
    slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


# ------------------------------------------------------------ our arm

class Arm:
    """L layer-states of one workload on this GPU, with captured graphs."""

    def __init__(self, wl, layers_data, bits, torch, B, per_step=False):
        self.wl, self.torch, self.B = wl, torch, B
        self.cfg = B.config_for(wl, bits=bits, per_step=per_step)
        self.bits = bits
        self.has_flush = bits != 32 and not per_step
        self.L = len(layers_data)
        # token-major order over two or more layer-states: the launch before a
        # decode is always another state's decode or flush
        self.flags = B.LQ_STEP_EARLY_STATE if (self.has_flush and self.L >= 2) else 0
        self.states, self.inp, self.out = [], [], []
        for ld in layers_data:
            st = B.LQState(self.cfg)
            st.init(ld["S0"])
            self.states.append(st)
            self.inp.append(ld["dev"])
            self.out.append(torch.empty((wl.window, wl.batch, wl.heads, wl.dv), dtype=torch.float32,
                                        device="cuda"))
        torch.cuda.synchronize()

    def decode_all(self):
        W = self.wl.window
        for t in range(W):
            for l in range(self.L):
                x = self.inp[l]
                self.states[l].step(x["q"][t], x["k"][t], x["v"][t], x["beta"][t], x["decay"][t],
                                    self.out[l][t], flags=self.flags)

    def flush_all(self):
        if not self.has_flush:
            return
        for l in range(self.L):
            self.states[l].flush()

    def capture(self):
        torch = self.torch
        # one eager window first: sets kernel attributes outside capture
        self.decode_all()
        self.flush_all()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        self.g_dec, self.g_fl = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_dec, stream=s):
            self.decode_all()
        if self.has_flush:
            with torch.cuda.graph(self.g_fl, stream=s):
                self.flush_all()
        torch.cuda.synchronize()

    def step(self):
        self.g_dec.replay()
        if self.has_flush:
            self.g_fl.replay()

    def launches_per_step(self):
        return self.wl.window * self.L + (self.L if self.has_flush else 0)


class SlotArm(Arm):
    """The same layers served through a slot list: each layer's state buffer
    holds 2x the running sequences, and the batch rows map to a seeded random
    subset of those slots in shuffled order (continuous batching)."""

    def __init__(self, wl, layers_data, torch, B, seed=12345):
        import numpy as np
        self.wl, self.torch, self.B = wl, torch, B
        self.cfg = B.config_for(wl)
        self.cfg.num_slots = 2 * wl.batch
        self.bits, self.has_flush, self.L = wl.bits, True, len(layers_data)
        rng = np.random.default_rng(seed)
        pick = rng.permutation(2 * wl.batch)[:wl.batch]
        self.slots = torch.from_numpy(pick.astype(np.int32)).cuda()
        self.states, self.inp, self.out = [], [], []
        for ld in layers_data:
            st = B.LQState(self.cfg)
            st.init_slots(self.slots, ld["S0"])
            self.states.append(st)
            self.inp.append(ld["dev"])
            self.out.append(torch.empty((wl.window, wl.batch, wl.heads, wl.dv), dtype=torch.float32,
                                        device="cuda"))
        torch.cuda.synchronize()

    def decode_all(self):
        for t in range(self.wl.window):
            for l in range(self.L):
                x = self.inp[l]
                self.states[l].step_slots(self.slots, x["q"][t], x["k"][t], x["v"][t], x["beta"][t],
                                          x["decay"][t], self.out[l][t])

    def flush_all(self):
        for l in range(self.L):
            self.states[l].flush_slots(self.slots)


class MultiArm(Arm):
    """The same layers decoded T tokens per launch (lq_decode_steps): a
    window is W / T launches per layer, inputs regrouped [batch, T, H, .]."""

    NAMES = ("q", "k", "v", "beta", "decay")

    def __init__(self, wl, layers_data, torch, B, tokens):
        super().__init__(wl, layers_data, wl.bits, torch, B)
        self.T = tokens
        W = wl.window
        self.chunks = [[{n: torch.stack([x[n][t0 + i] for i in range(tokens)], dim=1).contiguous()
                         for n in self.NAMES} for t0 in range(0, W, tokens)] for x in self.inp]
        self.mout = [torch.empty((W // tokens, wl.batch, tokens, wl.heads, wl.dv), dtype=torch.float32,
                                 device="cuda") for _ in layers_data]
        torch.cuda.synchronize()

    def decode_all(self):
        for c in range(self.wl.window // self.T):
            for l in range(self.L):
                x = self.chunks[l][c]
                self.states[l].steps(self.T, x["q"], x["k"], x["v"], x["beta"], x["decay"], self.mout[l][c])

    def launches_per_step(self):
        return (self.wl.window // self.T) * self.L + self.L


def time_arm(arm, steps, warmup, torch, dist, world):
    """Time `steps` window-steps; returns total ms (max over ranks) and the
    per-step decode / flush split from events recorded between the graphs."""
    for _ in range(warmup):
        arm.step()
    torch.cuda.synchronize()
    E = torch.cuda.Event
    marks = [(E(enable_timing=True), E(enable_timing=True), E(enable_timing=True)) for _ in range(steps)]
    start, end = E(enable_timing=True), E(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for s in range(steps):
        a, b, c = marks[s]
        a.record()
        arm.g_dec.replay()
        b.record()
        if arm.has_flush:
            arm.g_fl.replay()
        c.record()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total = start.elapsed_time(end)
    dec = sum(a.elapsed_time(b) for a, b, _ in marks)
    fl = sum(b.elapsed_time(c) for _, b, c in marks)
    total, dec, fl = max_over_ranks([total, dec, fl], torch, dist, world, "cuda")
    return total, dec, fl


def time_e2e(arm, host, steps, torch, dist, world):
    """Same steps through the public calls with host buffers: every step
    copies each layer's inputs host->device from pinned memory, runs its
    window and copies every output back, the transfers overlapped with the
    kernels of the neighbouring layers (pipeline.HostIOPipeline)."""
    from linear_attention_recurrent_lq_b200.pipeline import HostIOPipeline, Layer
    layers = [Layer(arm.states[l], arm.inp[l], arm.out[l], host[l]["in"], host[l]["out"]) for l in range(arm.L)]
    pipe = HostIOPipeline(layers, arm.wl.window, flush=arm.has_flush)
    pipe.capture()
    h2d, d2h = pipe.bytes_per_step()
    pipe.fork()
    pipe.step()
    pipe.join()
    torch.cuda.synchronize()
    E = torch.cuda.Event
    start, end = E(enable_timing=True), E(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    pipe.fork()
    for _ in range(steps):
        pipe.step()
    pipe.join()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks([start.elapsed_time(end)], torch, dist, world, "cuda")[0]
    return ms, h2d, d2h


def make_layers(wl, L, torch, I):
    layers = []
    for l in range(L):
        s = I.InputStream(wl, stream=l)
        st = s.state()
        tk = s.tokens(wl.window)
        d = {**st, **tk}
        layers.append({"S0": torch.from_numpy(st["S0"]).cuda(), "dev": I.to_device(wl, d), "np": d})
    return layers


def cpu_baseline(wl, layer_np, seconds, oracle):
    """The oracle as it stands on this host's cores, on a sample of the same
    workload: heads of layer 0, its window of tokens repeated, sized to run
    for about `seconds`."""
    import numpy as np
    p = oracle.Params.of(wl)
    nh = wl.batch * wl.heads
    W = wl.window

    def run(nheads, nwin, threads=0):
        heads = np.arange(nheads)
        T = W * nwin
        tile = lambda x: np.tile(x, (nwin,) + (1,) * (x.ndim - 1))
        S0 = layer_np["S0"].reshape(nh, wl.dk, wl.dv)[heads]
        q = tile(layer_np["q"].reshape(W, nh, wl.dk)[:, heads])
        k = tile(layer_np["k"].reshape(W, nh, wl.dk)[:, heads])
        v = tile(layer_np["v"].reshape(W, nh, wl.dv)[:, heads])
        beta = tile(layer_np["beta"].reshape(W, nh)[:, heads])
        dshape = (W, nh, wl.dk) if wl.decay_kind == "kda" else (W, nh)
        decay = tile(layer_np["decay"].reshape(dshape)[:, heads])
        t0 = time.perf_counter()
        _, _, used = oracle.run(p, S0, q, k, v, beta, decay, threads=threads)
        return time.perf_counter() - t0, used, nheads * T

    dt, used, n = run(min(nh, 64), 1)
    rate = n / dt
    nheads = min(nh, max(1, int(rate * seconds / W)))
    nwin = max(1, int(round(rate * seconds / (nheads * W))))
    nwin = min(nwin, 64)
    dt, used, n = run(nheads, nwin)
    # one thread on a sample of about a second, for the per-core figure
    n1 = min(nh, max(1, int(rate / max(used, 1) / W)))
    dt1, _, m1 = run(n1, 1, threads=1)
    return {"value": n / dt, "unit": "head-tokens/s", "cores": used, "kind": "oracle",
            "sample": f"{nheads} heads of one layer x {W * nwin} tokens (its first window of "
                      f"{W} tokens repeated {nwin}x), FP64 C oracle, OpenMP over heads, "
                      f"{dt:.1f} s",
            "one_thread": {"value": m1 / dt1, "unit": "head-tokens/s",
                           "sample": f"{n1} heads x {W} tokens, {dt1:.2f} s"},
            "cpu_model": cpu_model()}


def cpu_model():
    """The host CPU's model name, as /proc/cpuinfo gives it."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def measure_config(name, args, torch, B, I, hbm, dist, world):
    """One more workload of the pages' setting, measured as the headline is:
    the step (W decode tokens over L layer-states, then the flushes) and the
    FP32-state kernel on the same inputs; L chosen so the rotated states are
    far larger than L2."""
    wl = rank_workload(I.WORKLOADS[name], int(os.environ.get("RANK", "0")))
    nh = wl.batch * wl.heads
    L = 4 if nh <= 4096 else 2
    layers = make_layers(wl, L, torch, I)
    arm = Arm(wl, layers, wl.bits, torch, B)
    arm.capture()
    ks = args.config_steps
    total, dec, fl = time_arm(arm, ks, 3, torch, dist, world)
    status = max(st.check() for st in arm.states)
    if status != 0:
        raise RuntimeError(f"device status after {name}: {B.STATUS_NAMES[status]}")
    W = wl.window
    value = whole_job_rate(ks * W * L * nh, world, total)
    dec_ms = dec / (ks * W * L)
    dbytes = nh * sum(decode_bytes(wl, c) for c in range(W)) / W
    achieved = dbytes / (dec_ms / 1e3) / 1e9
    step_bytes = nh * L * W * head_token_bytes(wl)
    out = {"value": value, "unit": "head-tokens/s", "steps": ks, "layers_rotated": L,
           "batch": wl.batch, "heads": wl.heads, "state_bits": wl.bits, "decay": wl.decay_kind,
           "window": W, "num_comp": wl.num_comp, "scales": wl.scale_dtype,
           "bytes_per_head_token": head_token_bytes(wl),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                        "frac": achieved / hbm, "kernel": f"decode_kernel<{wl.dk},{wl.bits}>",
                        "algorithmic_bytes_per_launch": dbytes, "avg_launch_us": dec_ms * 1e3},
           "step_frac": step_bytes / (total / ks / 1e3) / 1e9 / hbm,
           "flush_avg_launch_us": fl / (ks * L) * 1e3}
    del arm
    torch.cuda.empty_cache()
    arm32 = Arm(wl, layers, 32, torch, B)
    arm32.capture()
    t32, d32, _ = time_arm(arm32, max(4, ks // 2), 3, torch, dist, world)
    v32 = whole_job_rate(max(4, ks // 2) * W * L * nh, world, t32)
    a32 = nh * fp32_bytes(wl) / (d32 / (max(4, ks // 2) * W * L) / 1e3) / 1e9
    out["fp32_state"] = {"value": v32, "achieved_gbs": a32, "frac": a32 / hbm}
    out["vs_fp32_state_kernel"] = value / v32
    del arm32, layers
    torch.cuda.empty_cache()
    return out


class MixedLayer:
    """The prefix-cache-scale layer: 48 heads per sequence, held as a GDN state
    (36 heads) and a KDA state (12 heads), B live sequences, plus a pool of
    cached flushed sequences that are restored into live slots (prefix-cache
    hits, lq_copy_slots) at window boundaries, spread evenly over the run."""

    def __init__(self, wls, S0s, devs, pool_slots, torch, B, bits=8):
        self.wls, self.torch, self.B = wls, torch, B
        self.W = wls[0].window
        self.states, self.pools, self.inp, self.out, self.cfgs = [], [], [], [], []
        for wl, S0, dev in zip(wls, S0s, devs):
            cfg = B.config_for(wl, bits=bits)
            st = B.LQState(cfg)
            st.init(S0)
            pcfg = B.config_for(wl, bits=bits)
            pcfg.num_slots = pool_slots
            pool = B.LQState(pcfg)
            for h in range(0, pool_slots, wl.batch):   # the pool holds flushed entries
                n = min(wl.batch, pool_slots - h)
                sl = torch.arange(h, h + n, dtype=torch.int32, device="cuda")
                pool.init_slots(sl, S0[:n].contiguous())
            self.cfgs.append(cfg)
            self.states.append(st)
            self.pools.append(pool)
            self.inp.append({k: v[:self.W] for k, v in dev.items()})
            self.out.append(torch.empty((self.W, wl.batch, wl.heads, wl.dv), dtype=torch.float32,
                                        device="cuda"))
        self.flags = B.LQ_STEP_EARLY_STATE
        torch.cuda.synchronize()

    def decode_all(self):
        for t in range(self.W):
            for l, st in enumerate(self.states):
                x = self.inp[l]
                st.step(x["q"][t], x["k"][t], x["v"][t], x["beta"][t], x["decay"][t], self.out[l][t],
                        flags=self.flags)

    def flush_all(self):
        for st in self.states:
            st.flush()

    def restore(self, dst, src):
        """Cached pool entries src -> live slots dst (both int32 device lists),
        after the window's flushes; a plain launch, so the next step's early
        staging never overlaps it."""
        B = self.B
        for l, st in enumerate(self.states):
            pool = self.pools[l]
            B.lq_copy_slots(self.cfgs[l], st.buf, self.cfgs[l].num_slots, dst, pool.buf,
                            pool.cfg.num_slots, src)


def measure_sweep(args, torch, B, I, hbm, dist, world):
    """Config 4: W x r sweep of the mixed 3:1 GDN:KDA layer at 512 live
    sequences, with 1024 cached INT8 sequences restored once each over the
    run (one hit per four tokens)."""
    points = [tuple(int(x) for x in p.split("x")) for p in args.sweep.split(",") if p]
    if not points:
        return None
    rank = int(os.environ.get("RANK", "0"))
    base = [rank_workload(I.WORKLOADS[n], rank) for n in ("mix_gdn_b512h36", "mix_kda_b512h12")]
    Wmax = max(W for W, _ in points)
    S0s, devs = [], []
    for wl in base:
        s = I.InputStream(wl, stream=0)
        st = s.state()
        S0s.append(torch.from_numpy(st["S0"]).cuda())
        del st
        devs.append(I.to_device(wl, s.tokens(Wmax)))
    pool_slots = 1024
    live = base[0].batch
    nh = sum(wl.batch * wl.heads for wl in base)
    res = {"layer": "48 heads per sequence: 36 GDN + 12 KDA (two states)", "live_slots": live,
           "cached_sequences": pool_slots, "tokens_per_point": args.sweep_tokens,
           "hits": "one cached sequence restored per 4 tokens, cycling through the pool", "points": {}}
    E = torch.cuda.Event
    for W, r in points:
        wls = [wl.replace(window=W, num_comp=r) for wl in base]
        layer = MixedLayer(wls, S0s, devs, pool_slots, torch, B)
        steps = max(1, args.sweep_tokens // W)
        hits_per_step = max(1, W // 4)
        n_hits = steps * hits_per_step
        dst_all = torch.tensor([(i * 37) % live for i in range(n_hits)], dtype=torch.int32, device="cuda")
        src_all = torch.tensor([i % pool_slots for i in range(n_hits)], dtype=torch.int32, device="cuda")
        layer.decode_all()
        layer.flush_all()
        torch.cuda.synchronize()
        sgraph = torch.cuda.Stream()
        sgraph.wait_stream(torch.cuda.current_stream())
        g_dec, g_fl = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_dec, stream=sgraph):
            layer.decode_all()
        with torch.cuda.graph(g_fl, stream=sgraph):
            layer.flush_all()
        torch.cuda.synchronize()
        for x in range(2):  # warm-up windows (with restores of the first entries)
            g_dec.replay()
            g_fl.replay()
            layer.restore(dst_all[:hits_per_step], src_all[:hits_per_step])
        torch.cuda.synchronize()
        marks = [(E(enable_timing=True), E(enable_timing=True), E(enable_timing=True)) for _ in range(steps)]
        a, b = E(enable_timing=True), E(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a.record()
        for sidx in range(steps):
            m0, m1, m2 = marks[sidx]
            m0.record()
            g_dec.replay()
            m1.record()
            g_fl.replay()
            m2.record()
            h0 = sidx * hits_per_step
            layer.restore(dst_all[h0:h0 + hits_per_step], src_all[h0:h0 + hits_per_step])
        b.record()
        torch.cuda.synchronize()
        total = a.elapsed_time(b)
        dec = sum(x.elapsed_time(y) for x, y, _ in marks)
        fl = sum(y.elapsed_time(z) for _, y, z in marks)
        total, dec, fl = max_over_ranks([total, dec, fl], torch, dist, world, "cuda")
        status = max(st.check() for st in layer.states)
        if status != 0:
            raise RuntimeError(f"device status after sweep point W={W} r={r}: {B.STATUS_NAMES[status]}")
        tok = steps * W
        per_ht = sum(wl.batch * wl.heads * head_token_bytes(wl) for wl in wls) / nh
        per_ht += sum(n_hits * wl.heads * restore_bytes(wl) for wl in wls) / (nh * tok)
        dbytes = sum(wl.batch * wl.heads * sum(decode_bytes(wl, c) for c in range(W)) for wl in wls) / W
        dec_us = dec / (steps * W) * 1e3   # both states' decode launches of one token
        res["points"][f"W{W}_r{r}"] = {
            "value": whole_job_rate(tok * nh, world, total), "unit": "head-tokens/s",
            "steps": steps, "hits": n_hits, "bytes_per_head_token": per_ht,
            "step_frac": per_ht * tok * nh / (total / 1e3) / 1e9 / hbm,
            "decode_frac": dbytes / (dec_us / 1e6) / 1e9 / hbm,
            "decode_us_per_token": dec_us, "flush_us_per_window": fl / steps * 1e3}
        del layer, g_dec, g_fl
        torch.cuda.empty_cache()
    # the FP32-state kernel on the same 48-head layer (independent of W and r)
    v32 = None
    states32 = []
    for wl, S0 in zip(base, S0s):
        st = B.LQState(B.config_for(wl, bits=32))
        st.init(S0)
        states32.append(st)
    ins = [{k: v[:16] for k, v in d.items()} for d in devs]
    outs = [torch.empty((16, wl.batch, wl.heads, wl.dv), dtype=torch.float32, device="cuda") for wl in base]

    def fp32_window():
        for t in range(16):
            for l, st in enumerate(states32):
                x = ins[l]
                st.step(x["q"][t], x["k"][t], x["v"][t], x["beta"][t], x["decay"][t], outs[l][t])

    fp32_window()
    torch.cuda.synchronize()
    g32 = torch.cuda.CUDAGraph()
    sg = torch.cuda.Stream()
    sg.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g32, stream=sg):
        fp32_window()
    for _ in range(2):
        g32.replay()
    torch.cuda.synchronize()
    k32 = 8
    a, b = E(enable_timing=True), E(enable_timing=True)
    a.record()
    for _ in range(k32):
        g32.replay()
    b.record()
    torch.cuda.synchronize()
    ms32 = max_over_ranks([a.elapsed_time(b)], torch, dist, world, "cuda")[0]
    v32 = whole_job_rate(k32 * 16 * nh, world, ms32)
    res["fp32_state"] = {"value": v32, "unit": "head-tokens/s",
                         "frac": nh * fp32_bytes(base[0]) * k32 * 16 / (ms32 / 1e3) / 1e9 / hbm}
    for p in res["points"].values():
        p["vs_fp32_state_kernel"] = p["value"] / v32
    del states32, g32, S0s, devs
    torch.cuda.empty_cache()
    return res


def config_of(wl, args, world):
    return {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "dk": wl.dk, "dv": wl.dv,
            "window": wl.window, "num_comp": wl.num_comp, "state_bits": wl.bits,
            "decay": wl.decay_kind, "smoothing": wl.smoothing, "scales": wl.scale_dtype,
            "qkv_dtype": wl.in_dtype, "layers_rotated": args.layers,
            "step": f"one window: {wl.window} decode tokens x {args.layers} layers + {args.layers} flushes",
            "l2": "no flush: the rotated layer-states are larger than L2",
            "decode_call": ("lq_decode_step_ex(LQ_STEP_EARLY_STATE): the launch before each decode is "
                            "another layer-state's" if args.layers >= 2 else "lq_decode_step"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def main_ours(args):
    import numpy as np
    import torch
    world, rank, local = dist_setup()
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    import __graft_entry__
    __graft_entry__.build()
    from linear_attention_recurrent_lq_b200 import binding as B
    from linear_attention_recurrent_lq_b200 import inputs as I

    wl = rank_workload(I.WORKLOADS[args.workload], rank)
    L = args.layers
    layers = make_layers(wl, L, torch, I)
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    nh = wl.batch * wl.heads

    # ---- LeapQuant arm
    arm = Arm(wl, layers, wl.bits, torch, B)
    arm.capture()
    props = torch.cuda.get_device_properties(local)
    uuid = str(getattr(props, "uuid", "") or "")
    clocks = Clocks(uuid)
    clocks.start()
    total, dec, fl = time_arm(arm, args.steps, args.warmup, torch, dist, world)
    clk = clocks.stop()
    status = max(st.check() for st in arm.states)
    if status != 0:
        raise RuntimeError(f"device status after timing: {B.STATUS_NAMES[status]}")
    W = wl.window
    value = whole_job_rate(args.steps * W * L * nh, world, total)
    dec_launches = args.steps * W * L
    dec_bytes_per_launch = nh * sum(decode_bytes(wl, c) for c in range(W)) / W
    dec_ms = dec / dec_launches
    achieved = dec_bytes_per_launch / (dec_ms / 1e3) / 1e9
    traffic = profiled_traffic(f"decode_{wl.name}.md")
    fl_launches = args.steps * L
    fl_ms = fl / fl_launches
    step_bytes = nh * L * (sum(decode_bytes(wl, c) for c in range(W)) + flush_bytes(wl))
    line = {
        "metric": "decode head-tokens/s and achieved HBM GB/s (% of B200 peak) vs FP32-state kernel",
        "value": value, "unit": "head-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_of(wl, args, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "kernel": f"decode_kernel<{wl.dk},{wl.bits}>", "peak_source": f"{peak_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": dec_bytes_per_launch,
                     "avg_launch_us": dec_ms * 1e3,
                     "spec_gbs": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS},
        "step_hbm": {"algorithmic_bytes_per_step": step_bytes,
                     "achieved_gbs": step_bytes / (total / args.steps / 1e3) / 1e9 * world,
                     "frac": step_bytes / (total / args.steps / 1e3) / 1e9 / hbm,
                     "flush_avg_launch_us": fl_ms * 1e3,
                     "flush_algorithmic_bytes_per_launch": nh * flush_bytes(wl)},
        "gpu_launches": args.steps * arm.launches_per_step(),
        "state_memory": state_memory(wl, B),
        "clocks": clk,
    }

    # ---- FP32-state kernel on the same inputs (the comparison point)
    if not args.no_fp32:
        arm32 = Arm(wl, layers, 32, torch, B)
        arm32.capture()
        ks = args.fp32_steps or max(4, args.steps // 4)
        t32, d32, _ = time_arm(arm32, ks, max(3, args.warmup // 2), torch, dist, world)
        v32 = whole_job_rate(ks * W * L * nh, world, t32)
        b32 = nh * fp32_bytes(wl)
        a32 = b32 / (d32 / (ks * W * L) / 1e3) / 1e9
        line["fp32_state"] = {"value": v32, "unit": "head-tokens/s", "steps": ks,
                              "achieved_gbs": a32, "frac": a32 / hbm,
                              "algorithmic_bytes_per_launch": b32}
        line["vs_fp32_state_kernel"] = value / v32
        del arm32
        torch.cuda.empty_cache()

    # ---- the naive per-step baselines of the accuracy table on the same inputs:
    # BF16 and FP8 E4M3 states stored after every token, and INT8 per step
    # (LeapQuant's layout with W = 1, no compensators, no smoothing)
    if not args.no_baselines:
        base = {}
        kb = args.fp32_steps or max(4, args.steps // 4)
        wl1 = wl.replace(window=1, num_comp=0, smoothing=False)
        for name, arm_wl, bits, per_step, bytes_tok in (
                ("bf16", wl, 16, True, per_step_bytes(wl, "bf16")),
                ("fp8_e4m3", wl, 8, True, per_step_bytes(wl, "fp8")),
                ("int8", wl1, 8, False, decode_bytes(wl1, 0) + flush_bytes(wl1))):
            armb = Arm(arm_wl, layers, bits, torch, B, per_step=per_step)
            armb.capture()
            ksb = kb * (wl.window // arm_wl.window)
            tb, db, _ = time_arm(armb, ksb, max(3, args.warmup // 2), torch, dist, world)
            units = ksb * arm_wl.window * L * nh
            vb = whole_job_rate(units, world, tb)
            ab = nh * bytes_tok * ksb * arm_wl.window * L / (tb / 1e3) / 1e9
            base[name] = {"value": vb, "unit": "head-tokens/s", "steps": ksb,
                          "bytes_per_head_token": bytes_tok, "achieved_gbs": ab, "frac": ab / hbm,
                          "leapquant_speedup": value / vb}
            del armb
            torch.cuda.empty_cache()
        line["per_step_baselines"] = base

    # ---- multi-token decode: T tokens per launch, the compact state read once
    if args.mt_tokens > 1 and W % args.mt_tokens == 0:
        T = args.mt_tokens
        armm = MultiArm(wl, layers, torch, B, T)
        armm.capture()
        km = args.fp32_steps or max(4, args.steps // 4)
        tm, dm, fm = time_arm(armm, km, max(3, args.warmup // 2), torch, dist, world)
        status = max(st.check() for st in armm.states)
        if status != 0:
            raise RuntimeError(f"device status after the multi-token run: {B.STATUS_NAMES[status]}")
        n_launch = km * (W // T) * L
        mb = nh * sum(multi_decode_bytes(wl, c, T) for c in range(0, W, T)) / (W // T)
        dm_ms = dm / n_launch
        line["multi_token"] = {
            "tokens_per_launch": T, "value": whole_job_rate(km * W * L * nh, world, tm),
            "unit": "head-tokens/s", "steps": km, "decode_avg_launch_us": dm_ms * 1e3,
            "decode_us_per_token": dm_ms * 1e3 / T, "algorithmic_bytes_per_launch": mb,
            "achieved_gbs": mb / (dm_ms / 1e3) / 1e9, "frac": mb / (dm_ms / 1e3) / 1e9 / hbm,
            "flush_avg_launch_us": fm / (km * L) * 1e3}
        del armm
        torch.cuda.empty_cache()

    # ---- prompt handoff: the FP32 recurrence over a prompt, then compression
    if args.prefill_tokens > 0:
        Tp = args.prefill_tokens
        pin = I.InputStream(wl, stream=100)
        pst = pin.state()
        ptok = pin.tokens(Tp)
        pdev = I.to_device(wl, {**pst, **ptok})
        prompt = [pdev[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "beta", "decay")]
        del pdev
        S0p = torch.from_numpy(pst["S0"]).cuda()
        stp = B.LQState(B.config_for(wl))
        for _ in range(2):  # warm-up
            stp.prefill(Tp, *prompt, S0=S0p)
        torch.cuda.synchronize()
        kp = 3
        E = torch.cuda.Event
        a, b = E(enable_timing=True), E(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        a.record()
        for _ in range(kp):
            stp.prefill(Tp, *prompt, S0=S0p)
        b.record()
        torch.cuda.synchronize()
        pms = max_over_ranks([a.elapsed_time(b)], torch, dist, world, "cuda")[0] / kp
        status = stp.check()
        if status != 0:
            raise RuntimeError(f"device status after prefill: {B.STATUS_NAMES[status]}")
        # the chunkwise form on the tensor cores (dk = dv = 128): per chunk of
        # C = 64 tokens, TF32 MMAs [Kt;Qt] Kh^T (128x64x128), S'^T [Kt;Qt]^T
        # (128x128x128), U^T (128x64x64), O^T (128x64x64), S^T (128x128x64)
        C = 64
        mma = 2.0 * (128 * 64 * wl.dk + 128 * 128 * wl.dk + 128 * 64 * C + 128 * 64 * C + 128 * 128 * C)
        flops = mma * nh * math.ceil(Tp / C)
        tf32_peak = float(peaks.get("bf16_tflops", 1590.0)) * (1.1 / 2.25)
        # the token-recurrent count for comparison: decay (1), S'^T k and S'^T q
        # (2 x 2), update (2) flops per state entry and token
        rec = 7.0 * wl.dk * wl.dv * nh * Tp
        line["prefill"] = {
            "prompt_tokens": Tp, "value": whole_job_rate(nh * Tp, world, pms), "unit": "head-tokens/s",
            "ms_per_launch": pms, "bound": "tensor", "achieved_tflops": flops / (pms / 1e3) / 1e12,
            "peak_tflops": tf32_peak, "frac": flops / (pms / 1e3) / 1e12 / tf32_peak,
            "peak_source": f"{peak_kind} bf16_tflops x 1.1/2.25 (nominal TF32 / BF16 dense ratio)",
            "mma_flops_per_launch": flops, "recurrent_equivalent_tflops": rec / (pms / 1e3) / 1e12,
            "form": "chunkwise, 64-token chunks, TF32 tcgen05 MMAs"}
        del stp, prompt
        torch.cuda.empty_cache()

    # ---- the serving path: the same work through a slot list
    if not args.no_slots:
        arms = SlotArm(wl, layers, torch, B)
        arms.capture()
        kss = args.fp32_steps or max(4, args.steps // 4)
        ts, ds, fs = time_arm(arms, kss, max(3, args.warmup // 2), torch, dist, world)
        status = max(st.check() for st in arms.states)
        if status != 0:
            raise RuntimeError(f"device status after the slot-list run: {B.STATUS_NAMES[status]}")
        ds_ms = ds / (kss * W * L)
        line["serving_slots"] = {
            "value": whole_job_rate(kss * W * L * nh, world, ts), "unit": "head-tokens/s",
            "steps": kss, "slots": f"{wl.batch} rows on a shuffled subset of {2 * wl.batch} slots",
            "decode_avg_launch_us": ds_ms * 1e3,
            "decode_frac": dec_bytes_per_launch / (ds_ms / 1e3) / 1e9 / hbm,
            "flush_avg_launch_us": fs / (kss * L) * 1e3}
        del arms
        torch.cuda.empty_cache()

    # ---- the other workloads of the pages' setting, each on its own
    if not args.no_configs:
        pc = {}
        for name in ("kda_int8_b128h32", "gdn_6bit_b256h32", "gdn_4bit_b256h32"):
            pc[name] = measure_config(name, args, torch, B, I, hbm, dist, world)
        sweep = measure_sweep(args, torch, B, I, hbm, dist, world)
        if sweep is not None:
            pc["mix_b512h48_sweep"] = sweep
        line["per_config"] = pc

    # ---- end to end through the public calls with host buffers
    if not args.no_e2e:
        host = []
        for l in range(L):
            hin = {k: v.cpu().pin_memory() for k, v in layers[l]["dev"].items()}
            host.append({"in": hin, "out": torch.empty_like(arm.out[l], device="cpu").pin_memory()})
        ke = args.e2e_steps or max(3, args.steps // 10)
        ms, h2d, d2h = time_e2e(arm, host, ke, torch, dist, world)
        line["e2e"] = {"value": whole_job_rate(ke * W * L * nh, world, ms), "unit": "head-tokens/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": ke, "ms_per_step": ms / ke}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = cpu_baseline(wl, layers[0]["np"], args.cpu_seconds, oracle)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main_reference(args):
    """The oracle, as it stands, timed on the host cores on bounded samples of
    the same workload (rank 0 only)."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    from oracle import build as ob
    from linear_attention_recurrent_lq_b200 import inputs as I
    ob.build()
    wl = I.WORKLOADS[args.workload]
    s = I.InputStream(wl, stream=0)
    ld = {**s.state(), **s.tokens(wl.window)}
    p = oracle.Params.of(wl)
    nh = wl.batch * wl.heads
    W = wl.window

    def sample(nheads, h0):
        heads = (np.arange(nheads) + h0) % nh
        dshape = (W, nh, wl.dk) if wl.decay_kind == "kda" else (W, nh)
        return (ld["S0"].reshape(nh, wl.dk, wl.dv)[heads], ld["q"].reshape(W, nh, wl.dk)[:, heads],
                ld["k"].reshape(W, nh, wl.dk)[:, heads], ld["v"].reshape(W, nh, wl.dv)[:, heads],
                ld["beta"].reshape(W, nh)[:, heads], ld["decay"].reshape(dshape)[:, heads])

    t0 = time.perf_counter()
    _, _, used = oracle.run(p, *sample(64, 0))
    rate = 64 * W / (time.perf_counter() - t0)
    budget = 90.0 / max(1, args.steps + args.warmup)  # seconds per step
    nheads = int(min(nh, max(1, rate * budget / W)))
    for x in range(args.warmup):
        oracle.run(p, *sample(nheads, x * nheads))
    t0 = time.perf_counter()
    for x in range(args.steps):
        _, _, used = oracle.run(p, *sample(nheads, x * nheads))
    dt = time.perf_counter() - t0
    value = args.steps * nheads * W / dt
    desc = (f"per step: {nheads} heads x {W} tokens (one window incl. its flush) of one "
            f"{wl.name} layer, FP64 C oracle, OpenMP over heads")
    print(json.dumps({
        "metric": "decode head-tokens/s and achieved HBM GB/s (% of B200 peak) vs FP32-state kernel",
        "value": value, "unit": "head-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, args, world), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "head-tokens/s", "cores": used, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "head-tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


if __name__ == "__main__":
    a = parse_args()
    if a.impl == "reference":
        main_reference(a)
    else:
        main_ours(a)
