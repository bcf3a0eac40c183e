"""Python binding of libleapquant.so: argument marshalling only.

Every function here has the name of the C entry point it calls (declared in
include/leapquant.h), takes torch tensors (or raw integer addresses) and the
current CUDA stream, and raises ``LQError`` on a non-zero status.  All
arithmetic runs in the library's sm_100a kernels; there is no fallback path:
if the library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libleapquant.so")

LQ_OK = 0
STATUS_NAMES = {0: "LQ_OK", 1: "LQ_ERR_INVALID_ARG", 2: "LQ_ERR_UNSUPPORTED", 3: "LQ_ERR_CUDA",
                4: "LQ_ERR_WINDOW_FULL", 5: "LQ_ERR_RANGE", 6: "LQ_ERR_MISALIGNED",
                7: "LQ_ERR_TIMEOUT", 8: "LQ_ERR_CORRUPT"}
(LQ_ERR_INVALID_ARG, LQ_ERR_UNSUPPORTED, LQ_ERR_CUDA, LQ_ERR_WINDOW_FULL, LQ_ERR_RANGE,
 LQ_ERR_MISALIGNED, LQ_ERR_TIMEOUT, LQ_ERR_CORRUPT) = range(1, 9)
ENTRY_POINTS = ("lq_validate_config", "lq_state_bytes", "lq_state_init", "lq_decode_step", "lq_decode_step_ex",
                "lq_decode_steps", "lq_window_flush", "lq_dequant_state", "lq_check_status",
                "lq_prefill", "lq_state_init_slots", "lq_decode_step_slots", "lq_decode_steps_slots",
                "lq_window_flush_slots", "lq_prefill_slots", "lq_copy_slots", "lq_selftest_wait",
                "lq_status_string")


class LQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({lq_status_string(status)})")


class lq_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_slots", "num_heads", "dk", "dv", "window", "num_comp", "bits", "decay_kind",
        "scale_dtype", "smoothing", "in_dtype", "per_step")]

    def __repr__(self):
        return "lq_config(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_config(num_slots, num_heads, dk=128, dv=128, window=16, num_comp=4, bits=8,
                decay_kind="gdn", scale_dtype="f32", smoothing=True, in_dtype="bf16",
                per_step=False) -> lq_config:
    """per_step=True selects the naive per-step baselines: bits 16 = BF16
    state, bits 8 = FP8 E4M3 state (window, num_comp, smoothing unused)."""
    return lq_config(int(num_slots), int(num_heads), int(dk), int(dv), int(window), int(num_comp),
                     int(bits), 1 if decay_kind == "kda" else 0, 1 if scale_dtype == "f16" else 0,
                     int(bool(smoothing)), 1 if in_dtype == "bf16" else 0, int(bool(per_step)))


def config_for(wl, bits: int | None = None, per_step: bool = False) -> lq_config:
    """The lq_config of a generator Workload (optionally another bit width, or
    one of the per-step baselines)."""
    return make_config(wl.batch, wl.heads, wl.dk, wl.dv, wl.window, wl.num_comp,
                       wl.bits if bits is None else bits, wl.decay_kind, wl.scale_dtype,
                       wl.smoothing, wl.in_dtype, per_step)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run linear_attention_recurrent_lq_b200/build.py "
                          "(or __graft_entry__.build())")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(lq_config)
    vp, st = ctypes.c_void_p, ctypes.c_int
    L.lq_validate_config.argtypes = [P]
    L.lq_validate_config.restype = st
    L.lq_state_bytes.argtypes = [P]
    L.lq_state_bytes.restype = ctypes.c_size_t
    L.lq_state_init.argtypes = [P, vp, vp, vp]
    L.lq_state_init.restype = st
    L.lq_decode_step.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
    L.lq_decode_step.restype = st
    L.lq_decode_step_ex.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_uint32, vp]
    L.lq_decode_step_ex.restype = st
    L.lq_window_flush.argtypes = [P, vp, vp]
    L.lq_window_flush.restype = st
    L.lq_dequant_state.argtypes = [P, vp, vp, vp]
    L.lq_dequant_state.restype = st
    L.lq_check_status.argtypes = [P, vp, vp]
    L.lq_check_status.restype = st
    i32 = ctypes.c_int
    L.lq_state_init_slots.argtypes = [P, vp, vp, i32, vp, vp]
    L.lq_state_init_slots.restype = st
    L.lq_decode_step_slots.argtypes = [P, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    L.lq_decode_step_slots.restype = st
    L.lq_window_flush_slots.argtypes = [P, vp, vp, i32, vp]
    L.lq_window_flush_slots.restype = st
    L.lq_copy_slots.argtypes = [P, vp, i32, vp, vp, i32, vp, i32, vp]
    L.lq_decode_steps.argtypes = [P, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    L.lq_decode_steps.restype = st
    L.lq_decode_steps_slots.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    L.lq_decode_steps_slots.restype = st
    L.lq_prefill.argtypes = [P, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.lq_prefill.restype = st
    L.lq_prefill_slots.argtypes = [P, vp, vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.lq_prefill_slots.restype = st
    L.lq_copy_slots.restype = st
    L.lq_selftest_wait.argtypes = [vp, vp]
    L.lq_selftest_wait.restype = st
    L.lq_status_string.argtypes = [st]
    L.lq_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return x.data_ptr()


# ---- tensor checks -------------------------------------------------------
# The C library trusts the shapes it is given: an undersized or mistyped
# buffer, or one on another device, would make a kernel read or write out of
# bounds.  Every torch tensor is therefore checked here, before the call, for
# its element type, its element count against cfg and its device (the GPU
# that is current, where the library launches).  Raw integer addresses are
# passed through unchecked: their owner vouches for them.

def _dt(name):
    import torch
    return {"f32": torch.float32, "bf16": torch.bfloat16, "i32": torch.int32, "u8": torch.uint8}[name]


def _in_dt(cfg) -> str:
    return "bf16" if cfg.in_dtype else "f32"


def _validate(*specs):
    """Check (tensor, what, dtype(s), numel, at_least) specs: first every
    element type and count, then that every tensor sits on the current CUDA
    device.  ValueError on the first mismatch; None and integer addresses
    pass."""
    import torch
    ts = [sp for sp in specs if sp[0] is not None and not isinstance(sp[0], int)]
    for x, what, dtype, numel, at_least in ts:
        want = dtype if isinstance(dtype, tuple) else (dtype,)
        if x.dtype not in tuple(_dt(d) for d in want):
            raise ValueError(f"{what}: dtype {x.dtype}, expected {' or '.join(want)}")
        if numel is not None:
            n = x.numel()
            if (n < numel) if at_least else (n != numel):
                raise ValueError(f"{what}: {n} elements, expected {'at least ' if at_least else ''}{numel}")
    for x, what, *_ in ts:
        if x.device.type != "cuda":
            raise ValueError(f"{what}: on {x.device}, expected a CUDA tensor")
        dev = torch.cuda.current_device()
        if x.device.index != dev:
            raise ValueError(f"{what}: on cuda:{x.device.index}, but the library launches on cuda:{dev}")


def _spec(x, what, dtype, numel=None, at_least=False):
    return (x, what, dtype, numel, at_least)


def _state_spec(cfg, state, num_slots=None, what="state"):
    n = cfg.num_slots if num_slots is None else num_slots
    bb = lib.lq_state_bytes(ctypes.byref(cfg))
    return _spec(state, what, "u8", n * cfg.num_heads * bb if bb else None, at_least=True)


def _rows_specs(cfg, rows: int, T: int, q, k, v, beta, decay, out):
    H, dk, dv = cfg.num_heads, cfg.dk, cfg.dv
    n = rows * T * H
    return [_spec(q, "q", _in_dt(cfg), n * dk), _spec(k, "k", _in_dt(cfg), n * dk),
            _spec(v, "v", _in_dt(cfg), n * dv), _spec(beta, "beta", "f32", n),
            _spec(decay, "decay", "f32", n * (dk if cfg.decay_kind == 1 else 1)),
            _spec(out, "out", "f32", n * dv)]


def _dense_spec(cfg, x, what, rows):
    return _spec(x, what, "f32", rows * cfg.num_heads * cfg.dk * cfg.dv)



def _stream(stream) -> int | None:
    if stream is None:
        import torch
        if not torch.cuda.is_available():
            return None
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != LQ_OK:
        raise LQError(status, where)


def lq_status_string(status: int) -> str:
    return lib.lq_status_string(int(status)).decode()


def lq_validate_config(cfg: lq_config) -> int:
    return lib.lq_validate_config(ctypes.byref(cfg))


def lq_state_bytes(cfg: lq_config) -> int:
    n = lib.lq_state_bytes(ctypes.byref(cfg))
    if n == 0:
        _check(lq_validate_config(cfg) or 1, "lq_state_bytes")
    return n


def lq_state_init(cfg, state, S0, stream=None):
    _validate(_state_spec(cfg, state), _dense_spec(cfg, S0, "S0", cfg.num_slots))
    _check(lib.lq_state_init(ctypes.byref(cfg), _ptr(state), _ptr(S0), _stream(stream)),
           "lq_state_init")


def lq_decode_step(cfg, state, q, k, v, beta, decay, out, stream=None):
    _validate(_state_spec(cfg, state), *_rows_specs(cfg, cfg.num_slots, 1, q, k, v, beta, decay, out))
    _check(lib.lq_decode_step(ctypes.byref(cfg), _ptr(state), _ptr(q), _ptr(k), _ptr(v),
                              _ptr(beta), _ptr(decay), _ptr(out), _stream(stream)),
           "lq_decode_step")


LQ_STEP_EARLY_STATE = 0x1


def lq_decode_step_ex(cfg, state, q, k, v, beta, decay, out, flags=0, stream=None):
    _validate(_state_spec(cfg, state), *_rows_specs(cfg, cfg.num_slots, 1, q, k, v, beta, decay, out))
    _check(lib.lq_decode_step_ex(ctypes.byref(cfg), _ptr(state), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(beta), _ptr(decay), _ptr(out), int(flags), _stream(stream)),
           "lq_decode_step_ex")


def lq_window_flush(cfg, state, stream=None):
    _validate(_state_spec(cfg, state))
    _check(lib.lq_window_flush(ctypes.byref(cfg), _ptr(state), _stream(stream)), "lq_window_flush")


def lq_dequant_state(cfg, state, S_out, stream=None):
    _validate(_state_spec(cfg, state), _dense_spec(cfg, S_out, "S_out", cfg.num_slots))
    _check(lib.lq_dequant_state(ctypes.byref(cfg), _ptr(state), _ptr(S_out), _stream(stream)),
           "lq_dequant_state")


def lq_check_status(cfg, state, stream=None) -> int:
    """Synchronizes the stream; returns the status code (does not raise)."""
    _validate(_state_spec(cfg, state))
    return lib.lq_check_status(ctypes.byref(cfg), _ptr(state), _stream(stream))


def _n(slots) -> int:
    return 0 if slots is None else int(slots.numel()) if hasattr(slots, "numel") else len(slots)


def _prefill_specs(cfg, rows, tokens, q, k, v, beta, decay, S0, lengths, out, S_final):
    T = max(int(tokens), 0)
    return _rows_specs(cfg, rows, T, q, k, v, beta, decay, out) + [
        _dense_spec(cfg, S0, "S0", rows), _dense_spec(cfg, S_final, "S_final", rows),
        _spec(lengths, "lengths", "i32", rows)]


def lq_state_init_slots(cfg, state, slots, S0, stream=None):
    _validate(_state_spec(cfg, state), _spec(slots, "slots", "i32"), _dense_spec(cfg, S0, "S0", _n(slots)))
    _check(lib.lq_state_init_slots(ctypes.byref(cfg), _ptr(state), _ptr(slots), _n(slots), _ptr(S0),
                                   _stream(stream)), "lq_state_init_slots")


def lq_decode_step_slots(cfg, state, slots, q, k, v, beta, decay, out, stream=None):
    _validate(_state_spec(cfg, state), _spec(slots, "slots", "i32"),
              *_rows_specs(cfg, _n(slots), 1, q, k, v, beta, decay, out))
    _check(lib.lq_decode_step_slots(ctypes.byref(cfg), _ptr(state), _ptr(slots), _n(slots), _ptr(q),
                                    _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(out),
                                    _stream(stream)), "lq_decode_step_slots")


def lq_decode_steps(cfg, state, tokens, q, k, v, beta, decay, out, stream=None):
    _validate(_state_spec(cfg, state),
              *_rows_specs(cfg, cfg.num_slots, max(int(tokens), 0), q, k, v, beta, decay, out))
    _check(lib.lq_decode_steps(ctypes.byref(cfg), _ptr(state), int(tokens), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(beta), _ptr(decay), _ptr(out), _stream(stream)), "lq_decode_steps")


def lq_decode_steps_slots(cfg, state, slots, tokens, q, k, v, beta, decay, out, stream=None):
    _validate(_state_spec(cfg, state), _spec(slots, "slots", "i32"),
              *_rows_specs(cfg, _n(slots), max(int(tokens), 0), q, k, v, beta, decay, out))
    _check(lib.lq_decode_steps_slots(ctypes.byref(cfg), _ptr(state), _ptr(slots), _n(slots), int(tokens),
                                     _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(out),
                                     _stream(stream)), "lq_decode_steps_slots")


def lq_prefill(cfg, state, tokens, q, k, v, beta, decay, S0=None, lengths=None, out=None, S_final=None,
               stream=None):
    _validate(_state_spec(cfg, state),
              *_prefill_specs(cfg, cfg.num_slots, tokens, q, k, v, beta, decay, S0, lengths, out, S_final))
    _check(lib.lq_prefill(ctypes.byref(cfg), _ptr(state), int(tokens), _ptr(lengths), _ptr(S0), _ptr(q),
                          _ptr(k), _ptr(v), _ptr(beta), _ptr(decay), _ptr(out), _ptr(S_final),
                          _stream(stream)), "lq_prefill")


def lq_prefill_slots(cfg, state, slots, tokens, q, k, v, beta, decay, S0=None, lengths=None, out=None,
                     S_final=None, stream=None):
    _validate(_state_spec(cfg, state), _spec(slots, "slots", "i32"),
              *_prefill_specs(cfg, _n(slots), tokens, q, k, v, beta, decay, S0, lengths, out, S_final))
    _check(lib.lq_prefill_slots(ctypes.byref(cfg), _ptr(state), _ptr(slots), _n(slots), int(tokens),
                                _ptr(lengths), _ptr(S0), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                _ptr(decay), _ptr(out), _ptr(S_final), _stream(stream)),
           "lq_prefill_slots")


def lq_window_flush_slots(cfg, state, slots, stream=None):
    _validate(_state_spec(cfg, state), _spec(slots, "slots", "i32"))
    _check(lib.lq_window_flush_slots(ctypes.byref(cfg), _ptr(state), _ptr(slots), _n(slots),
                                     _stream(stream)), "lq_window_flush_slots")


def lq_copy_slots(cfg, dst, dst_num_slots, dst_slots, src, src_num_slots, src_slots, stream=None):
    if _n(dst_slots) != _n(src_slots):
        raise ValueError("dst_slots and src_slots must have the same length")
    _validate(_state_spec(cfg, dst, int(dst_num_slots), "dst"), _state_spec(cfg, src, int(src_num_slots), "src"),
              _spec(dst_slots, "dst_slots", "i32"), _spec(src_slots, "src_slots", "i32"))
    _check(lib.lq_copy_slots(ctypes.byref(cfg), _ptr(dst), int(dst_num_slots), _ptr(dst_slots),
                             _ptr(src), int(src_num_slots), _ptr(src_slots), _n(src_slots),
                             _stream(stream)), "lq_copy_slots")


def lq_selftest_wait(status, stream=None):
    """Device diagnostic: a bounded wait that runs out writes LQ_DEV_TIMEOUT to status."""
    _validate(_spec(status, "status", "i32", 1, at_least=True))
    _check(lib.lq_selftest_wait(_ptr(status), _stream(stream)), "lq_selftest_wait")


class LQState:
    """N*H state blobs in one device buffer, with the library's calls bound."""

    def __init__(self, cfg: lq_config, device="cuda"):
        import torch
        self.cfg = cfg
        self.blob_bytes = lq_state_bytes(cfg)
        self.buf = torch.empty(cfg.num_slots * cfg.num_heads * self.blob_bytes, dtype=torch.uint8,
                               device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def blobs(self):
        """[N*H, blob_bytes] uint8 view."""
        return self.buf.view(-1, self.blob_bytes)

    def init(self, S0, stream=None):
        lq_state_init(self.cfg, self.buf, S0, stream)

    def step(self, q, k, v, beta, decay, out, stream=None, flags=0):
        if flags:
            lq_decode_step_ex(self.cfg, self.buf, q, k, v, beta, decay, out, flags, stream)
        else:
            lq_decode_step(self.cfg, self.buf, q, k, v, beta, decay, out, stream)

    def flush(self, stream=None):
        lq_window_flush(self.cfg, self.buf, stream)

    def prefill(self, tokens, q, k, v, beta, decay, S0=None, lengths=None, out=None, S_final=None,
                stream=None):
        """Prompt of T tokens per (slot, head) (inputs [N, T, H, .]), then compress."""
        lq_prefill(self.cfg, self.buf, tokens, q, k, v, beta, decay, S0, lengths, out, S_final, stream)

    def steps(self, tokens, q, k, v, beta, decay, out, stream=None):
        """T tokens per (slot, head): inputs [N, T, H, .], out [N, T, H, dv]."""
        lq_decode_steps(self.cfg, self.buf, tokens, q, k, v, beta, decay, out, stream)

    def dequant(self, S_out=None, stream=None):
        import torch
        c = self.cfg
        if S_out is None:
            S_out = torch.empty((c.num_slots, c.num_heads, c.dk, c.dv), dtype=torch.float32,
                                device=self.buf.device)
        lq_dequant_state(c, self.buf, S_out, stream)
        return S_out

    def check(self, stream=None) -> int:
        return lq_check_status(self.cfg, self.buf, stream)

    # slot lists: int32 device tensors of slot indices (one per active row)
    def init_slots(self, slots, S0, stream=None):
        lq_state_init_slots(self.cfg, self.buf, slots, S0, stream)

    def step_slots(self, slots, q, k, v, beta, decay, out, stream=None):
        lq_decode_step_slots(self.cfg, self.buf, slots, q, k, v, beta, decay, out, stream)

    def steps_slots(self, slots, tokens, q, k, v, beta, decay, out, stream=None):
        lq_decode_steps_slots(self.cfg, self.buf, slots, tokens, q, k, v, beta, decay, out, stream)

    def flush_slots(self, slots, stream=None):
        lq_window_flush_slots(self.cfg, self.buf, slots, stream)
