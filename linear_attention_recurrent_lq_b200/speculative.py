"""Speculative verification on LeapQuant states, with exact rollback.

A verify step decodes T draft tokens of each running row in one multi-token
launch.  Each row then keeps only its accepted prefix of a <= T tokens.  The
pairs of the rejected tokens cannot simply be dropped: the window's decay
product (and, after a frame move, the stored scales) already include them.
So before the verify step the rows' blobs are snapshotted into a pool with
lq_copy_slots; a row that accepts every token keeps the result, and a row
that accepts a < T tokens gets its snapshot back and is decoded again for
its first a tokens.  Decode is deterministic and a multi-token launch equals
single-token calls bit for bit, so the re-run reproduces exactly the state
an a-token verify step would have left.
"""
from __future__ import annotations

NAMES = ("q", "k", "v", "beta", "decay")


class SpeculativeDecoder:
    """Verify / accept over the slots of one LQState (bits 8/6/4)."""

    def __init__(self, state, max_rows: int):
        import torch
        self.torch = torch
        self.state = state
        self.max_rows = max_rows
        cfg = state.cfg
        self.pool = torch.empty(max_rows * cfg.num_heads * state.blob_bytes, dtype=torch.uint8,
                                device=state.buf.device)
        self._slots = None

    def verify(self, slots, tokens: int, q, k, v, beta, decay, out):
        """Snapshot the rows' blobs, then decode `tokens` draft tokens per row.
        slots: int32 device tensor [rows]; inputs [rows, T, H, .]; out [rows, T, H, dv]."""
        from . import binding as B
        torch = self.torch
        n = int(slots.numel())
        if n > self.max_rows:
            raise ValueError(f"{n} rows exceed the snapshot pool of {self.max_rows}")
        cfg = self.state.cfg
        pool_slots = torch.arange(n, dtype=torch.int32, device=slots.device)
        B.lq_copy_slots(cfg, self.pool, self.max_rows, pool_slots, self.state.buf, cfg.num_slots, slots)
        B.lq_decode_steps_slots(cfg, self.state.buf, slots, tokens, q, k, v, beta, decay, out)
        self._slots, self._tokens, self._pool_slots = slots, tokens, pool_slots

    def accept(self, accepted, q, k, v, beta, decay, out=None):
        """Keep the first accepted[n] tokens of row n of the last verify step
        (host ints, 0 <= accepted[n] <= T).  The inputs are the verify step's;
        `out` (optional, [rows, T, H, dv]) receives the re-decoded rows' outputs
        again, which equal those of the verify step."""
        from . import binding as B
        torch = self.torch
        if self._slots is None:
            raise RuntimeError("accept() without a verify() before it")
        T = self._tokens
        acc = [int(a) for a in accepted]
        if len(acc) != int(self._slots.numel()) or any(a < 0 or a > T for a in acc):
            raise ValueError("accepted counts must be one per row, within [0, T]")
        cfg = self.state.cfg
        redo = [n for n, a in enumerate(acc) if a < T]
        if redo:
            rows = torch.tensor(redo, dtype=torch.int32, device=self._slots.device)
            dst = self._slots[rows.long()].contiguous()
            B.lq_copy_slots(cfg, self.state.buf, cfg.num_slots, dst, self.pool, self.max_rows,
                            self._pool_slots[rows.long()].contiguous())
            # one re-run per distinct accepted count
            for a in sorted({acc[n] for n in redo}):
                if a == 0:
                    continue
                sel = [n for n in redo if acc[n] == a]
                idx = torch.tensor(sel, dtype=torch.long, device=self._slots.device)
                ins = [x[idx, :a].contiguous() for x in (q, k, v, beta, decay)]
                o = torch.empty((len(sel), a) + tuple(out.shape[2:]) if out is not None else
                                (len(sel), a, cfg.num_heads, cfg.dv), dtype=torch.float32,
                                device=self._slots.device)
                B.lq_decode_steps_slots(cfg, self.state.buf, self._slots[idx].contiguous(), a, *ins, o)
                if out is not None:
                    out[idx, :a] = o
        self._slots = None
