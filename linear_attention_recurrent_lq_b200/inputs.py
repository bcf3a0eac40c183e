"""Seeded synthetic inputs for the LeapQuant decode path.

This module draws the initial recurrent states and the per-token decode inputs
(q, k, v, beta, decay) for every workload the library is tested and measured
on.  It holds none of the method's arithmetic: no recurrence, no quantizer, no
compensator or smoothing rule.  Both the CUDA path and the CPU oracle consume
exactly the arrays produced here.

Workload shapes follow the pages' setting: decode in a hybrid model, where
every linear-attention head holds a dk x dv recurrent state that has to be read
from HBM and written back once per generated token (news post "Linear attention
has to move state every token it generates; LeapQuant compresses it to 8-bit
without losing accuracy", second paragraph), with Gated DeltaNet heads (scalar
decay) and Kimi Delta Attention heads (one decay per key channel) ("LeapQuant:
Efficient Linear Attention with Accurate Recurrent State Quantization",
original abstract).

Recipe (one numpy PCG64 stream per (seed, stream) pair, fixed draw order):
  1. S0 ~ N(0, 0.1) (0.1 is the standard deviation), shape [B, H, dk, dv],
     math convention: row i = key channel, column j = value channel.
  2. Outlier key rows, then outlier value columns, per head, drawn without
     replacement (random keys + argsort); the rows are multiplied by
     ``row_gain`` and the columns by ``col_gain`` (intersections get both).
  3. KDA only: ``slow_channels`` key channels per head, drawn the same way.
  4. Per token, in this order: q, k ~ N(0,1) of length dk; v ~ N(0,1) of
     length dv; beta-logit ~ N(0,1) per head; decay-logit ~ N(-4,1) per head
     (GDN) or per key channel (KDA); for KDA, slow-channel logits ~ N(-9, 0.5)
     clipped at <= -6.91 replace the drawn logits on the slow channels.
     q and k are L2-normalised per token, beta = sigmoid(logit),
     decay = exp(-softplus(logit)) (so decay in (0, 1); slow channels > 0.999).
  5. Inputs that the path reads in bf16 are rounded to bf16 (round to nearest
     even); the float32 values returned alongside are the rounded values, so
     both sides see identical numbers.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    """One decode workload: shapes, method parameters and input recipe."""

    name: str
    batch: int
    heads: int
    tokens: int
    window: int
    num_comp: int
    bits: int = 8
    decay_kind: str = "gdn"  # "gdn" (scalar decay) or "kda" (per key channel)
    smoothing: bool = True
    scale_dtype: str = "f32"  # storage dtype of quant and smoothing scales
    in_dtype: str = "bf16"  # dtype of q, k, v as read by the path
    dk: int = 128
    dv: int = 128
    outlier_rows: int = 4
    row_gain: float = 100.0
    outlier_cols: int = 2
    col_gain: float = 40.0
    slow_channels: int = 0
    seed: int = 0

    @property
    def num_heads_total(self) -> int:
        return self.batch * self.heads

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The decode workloads of the pages' setting, dk = dv = 128 throughout.
WORKLOADS = {
    # tiny GDN head: INT8, per-row symmetric quantization without smoothing
    "gdn_int8_b1h1": Workload(
        name="gdn_int8_b1h1", batch=1, heads=1, tokens=64, window=16,
        num_comp=2, bits=8, decay_kind="gdn", smoothing=False,
        scale_dtype="f32", in_dtype="f32", outlier_rows=2, row_gain=50.0,
        outlier_cols=1, col_gain=30.0, seed=0),
    # one GDN layer of a batch-64 decode: INT8 with smoothing, bf16 q/k/v
    "gdn_int8_b64h32": Workload(
        name="gdn_int8_b64h32", batch=64, heads=32, tokens=1024, window=16,
        num_comp=4, bits=8, decay_kind="gdn", smoothing=True, seed=1),
    # one KDA layer: per-key-channel decay with 8 slow channels per head
    "kda_int8_b128h32": Workload(
        name="kda_int8_b128h32", batch=128, heads=32, tokens=2048, window=16,
        num_comp=4, bits=8, decay_kind="kda", smoothing=True,
        slow_channels=8, seed=2),
    # packed low-bit GDN states with fp16 scales
    "gdn_6bit_b256h32": Workload(
        name="gdn_6bit_b256h32", batch=256, heads=32, tokens=1024, window=16,
        num_comp=8, bits=6, decay_kind="gdn", smoothing=True,
        scale_dtype="f16", seed=3),
    "gdn_4bit_b256h32": Workload(
        name="gdn_4bit_b256h32", batch=256, heads=32, tokens=1024, window=16,
        num_comp=8, bits=4, decay_kind="gdn", smoothing=True,
        scale_dtype="f16", seed=3),
    # prefix-cache-scale layer: 48 heads mixed 3:1 GDN:KDA, held as two states
    # (36 GDN heads and 12 KDA heads per sequence); W and r are swept
    "mix_gdn_b512h36": Workload(
        name="mix_gdn_b512h36", batch=512, heads=36, tokens=4096, window=16,
        num_comp=4, bits=8, decay_kind="gdn", smoothing=True, seed=4),
    "mix_kda_b512h12": Workload(
        name="mix_kda_b512h12", batch=512, heads=12, tokens=4096, window=16,
        num_comp=4, bits=8, decay_kind="kda", smoothing=True,
        slow_channels=8, seed=1004),
}


def rng_for(seed: int, stream: int = 0) -> np.random.Generator:
    """The numpy PCG64 stream used for (seed, stream)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _subset(rng: np.random.Generator, shape: tuple, n: int, count: int) -> np.ndarray:
    """`count` distinct indices in [0, n) per leading index, uniform."""
    if count == 0:
        return np.zeros(shape + (0,), dtype=np.int64)
    keys = rng.random(shape + (n,))
    return np.argsort(keys, axis=-1, kind="stable")[..., :count]


def _sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def _exp_neg_softplus(z):
    # exp(-log(1 + e^z)) = 1 / (1 + e^z)
    return 1.0 / (1.0 + np.exp(z))


class InputStream:
    """Draws one workload's initial state and then its tokens, in order.

    ``state()`` must be called before the first ``tokens()`` call; every
    ``tokens(n)`` call continues the same stream, so drawing 16 tokens twice
    gives the same values as drawing 32 tokens once.
    """

    def __init__(self, wl: Workload, stream: int = 0):
        self.wl = wl
        self.rng = rng_for(wl.seed, stream)
        self._state_drawn = False
        self.slow = None

    def state(self) -> dict:
        wl, rng = self.wl, self.rng
        B, H, dk, dv = wl.batch, wl.heads, wl.dk, wl.dv
        S0 = rng.normal(0.0, 0.1, size=(B, H, dk, dv))
        rows = _subset(rng, (B, H), dk, wl.outlier_rows)
        cols = _subset(rng, (B, H), dv, wl.outlier_cols)
        b_idx = np.arange(B)[:, None, None]
        h_idx = np.arange(H)[None, :, None]
        if wl.outlier_rows:
            S0[b_idx, h_idx, rows, :] *= wl.row_gain
        if wl.outlier_cols:
            S0[b_idx, h_idx, :, cols] *= wl.col_gain
        if wl.decay_kind == "kda":
            self.slow = _subset(rng, (B, H), dk, wl.slow_channels)
        self._state_drawn = True
        return {"S0": S0.astype(np.float32), "outlier_rows": rows, "outlier_cols": cols,
                "slow_channels": self.slow}

    def tokens(self, n: int) -> dict:
        """Draw the next n tokens: arrays with a leading token axis [n, B, H, ...]."""
        if not self._state_drawn:
            raise RuntimeError("draw the initial state before the tokens")
        wl, rng = self.wl, self.rng
        B, H, dk, dv = wl.batch, wl.heads, wl.dk, wl.dv
        q = np.empty((n, B, H, dk), np.float32)
        k = np.empty((n, B, H, dk), np.float32)
        v = np.empty((n, B, H, dv), np.float32)
        beta = np.empty((n, B, H), np.float32)
        if wl.decay_kind == "kda":
            decay = np.empty((n, B, H, dk), np.float32)
        else:
            decay = np.empty((n, B, H), np.float32)
        b_idx = np.arange(B)[:, None, None]
        h_idx = np.arange(H)[None, :, None]
        for t in range(n):
            qt = rng.standard_normal((B, H, dk))
            kt = rng.standard_normal((B, H, dk))
            vt = rng.standard_normal((B, H, dv))
            bl = rng.standard_normal((B, H))
            if wl.decay_kind == "kda":
                dl = rng.normal(-4.0, 1.0, size=(B, H, dk))
                if wl.slow_channels:
                    sl = np.minimum(rng.normal(-9.0, 0.5, size=(B, H, wl.slow_channels)), -6.91)
                    dl[b_idx, h_idx, self.slow] = sl
            else:
                dl = rng.normal(-4.0, 1.0, size=(B, H))
            q[t] = qt / np.linalg.norm(qt, axis=-1, keepdims=True)
            k[t] = kt / np.linalg.norm(kt, axis=-1, keepdims=True)
            v[t] = vt
            beta[t] = _sigmoid(bl)
            decay[t] = _exp_neg_softplus(dl)
        out = {"beta": beta, "decay": decay}
        if wl.in_dtype == "bf16":
            for name, x in (("q", q), ("k", k), ("v", v)):
                bits = bf16_bits(x)
                out[name + "_bits"] = bits
                out[name] = bf16_value(bits)
        else:
            out["q"], out["k"], out["v"] = q, k, v
        return out


def draw(wl: Workload, n_tokens: int | None = None, stream: int = 0) -> dict:
    """Initial state plus the first ``n_tokens`` tokens of a workload."""
    s = InputStream(wl, stream)
    st = s.state()
    st.update(s.tokens(wl.tokens if n_tokens is None else n_tokens))
    return st


def to_device(wl: Workload, d: dict, device="cuda") -> dict:
    """Upload drawn tokens as the tensors the library reads: q, k, v in the
    workload's input dtype (bf16 as its bit patterns), beta and decay f32."""
    import torch
    dev = {}
    for name in ("q", "k", "v"):
        if wl.in_dtype == "bf16":
            bits = np.ascontiguousarray(d[name + "_bits"]).view(np.int16)
            dev[name] = torch.from_numpy(bits).to(device).view(torch.bfloat16)
        else:
            dev[name] = torch.from_numpy(np.ascontiguousarray(d[name])).to(device)
    dev["beta"] = torch.from_numpy(np.ascontiguousarray(d["beta"])).to(device)
    dev["decay"] = torch.from_numpy(np.ascontiguousarray(d["decay"])).to(device)
    return dev
