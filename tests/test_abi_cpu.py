"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/leapquant.h declares, sizes blobs as documented,
and rejects bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "leapquant.h")


@pytest.fixture(scope="module")
def B():
    from linear_attention_recurrent_lq_b200 import build
    build.build()
    from linear_attention_recurrent_lq_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^LQ_API\s+[\w\s\*]+?\b(lq_\w+)\s*\(", text, flags=re.M)


def test_library_exports_every_declared_entry_point(B):
    names = declared_functions()
    assert set(names) == set(B.ENTRY_POINTS)
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_state_bytes_follow_documented_layout(B):
    from tests import blob
    for bits in (8, 6, 4):
        for kda in (0, 1):
            for f16 in (0, 1):
                for d in (64, 128):
                    for w, r in ((16, 4), (1, 0), (64, 16)):
                        cfg = B.make_config(2, 3, d, d, w, r, bits, "kda" if kda else "gdn",
                                            "f16" if f16 else "f32")
                        L = blob.layout(d, d, w, r, bits, kda, f16)
                        assert B.lq_state_bytes(cfg) == L.blob
                        assert L.blob % 256 == 0
    cfg = B.make_config(64, 32, bits=32)
    assert B.lq_state_bytes(cfg) == blob.layout(128, 128, 16, 4, 32, 0, 0).blob
    # per-step baselines: header, then bf16 S; or f32 scales (128-aligned) and fp8 codes
    for d in (64, 128):
        bf16 = B.make_config(2, 3, d, d, bits=16, per_step=True)
        fp8 = B.make_config(2, 3, d, d, bits=8, per_step=True)
        assert B.lq_state_bytes(bf16) == (128 + 2 * d * d + 255) // 256 * 256
        assert B.lq_state_bytes(fp8) == (128 + (4 * d + 127) // 128 * 128 + d * d + 255) // 256 * 256


def test_headline_blob_size(B):
    # GDN, INT8, dk = dv = 128, W = 16, r = 4, f32 scales
    assert B.lq_state_bytes(B.make_config(64, 32)) == 36096


@pytest.mark.parametrize("field,value,expect", [
    ("num_slots", 0, 1), ("num_heads", -1, 1), ("window", 0, 1), ("bits", 5, 1),
    ("decay_kind", 2, 1), ("scale_dtype", 3, 1), ("num_comp", -1, 1),
    ("dk", 256, 2), ("dv", 64, 2), ("window", 65, 2), ("num_comp", 17, 2), ("per_step", 2, 1),
    ("bits", 16, 1)])
def test_config_validation(B, field, value, expect):
    cfg = B.make_config(4, 4)
    setattr(cfg, field, value)
    assert B.lq_validate_config(cfg) == expect
    assert B.lib.lq_state_bytes(ctypes.byref(cfg)) == 0


def test_per_step_formats_validate(B):
    assert B.lq_validate_config(B.make_config(4, 4, bits=16, per_step=True)) == 0
    assert B.lq_validate_config(B.make_config(4, 4, bits=8, per_step=True)) == 0
    for bits in (4, 6, 32):
        assert B.lq_validate_config(B.make_config(4, 4, bits=bits, per_step=True)) == 1


def test_null_and_misaligned_pointers_rejected_before_launch(B):
    cfg = B.make_config(4, 4)
    L = B.lib
    c = ctypes.byref(cfg)
    assert L.lq_decode_step(c, None, 16, 16, 16, 16, 16, 16, None) == 1
    assert L.lq_decode_step(c, 256, 16, 16, 16, 16, 16, None, None) == 1
    assert L.lq_decode_step(c, 128, 16, 16, 16, 16, 16, 16, None) == 6   # state needs 256 B
    assert L.lq_decode_step(c, 256, 8, 16, 16, 16, 16, 16, None) == 6    # q needs 16 B
    assert L.lq_decode_step(c, 256, 16, 16, 16, 2, 16, 16, None) == 6    # beta needs 4 B
    assert L.lq_state_init(c, 256, 4, None) == 6
    assert L.lq_state_init(c, None, 16, None) == 1
    assert L.lq_window_flush(c, 100, None) == 6
    assert L.lq_window_flush(c, None, None) == 1
    assert L.lq_dequant_state(c, 256, 12, None) == 6
    assert L.lq_check_status(c, None, None) == 1
    assert L.lq_decode_step(None, 256, 16, 16, 16, 16, 16, 16, None) == 1


def test_status_strings(B):
    for code in range(9):
        assert B.lq_status_string(code)
    assert B.lq_status_string(99) == "unknown status"


def test_slot_entry_points_rejected_before_launch(B):
    cfg = B.make_config(4, 4)
    L = B.lib
    c = ctypes.byref(cfg)
    # an empty slot list launches nothing
    assert L.lq_decode_step_slots(c, 256, None, 0, None, None, None, None, None, None, None) == 0
    assert L.lq_window_flush_slots(c, 256, None, 0, None) == 0
    assert L.lq_state_init_slots(c, 256, None, 0, None, None) == 0
    assert L.lq_copy_slots(c, 256, 2, None, 512, 3, None, 0, None) == 0
    # missing pointers, negative counts
    assert L.lq_decode_step_slots(c, 256, None, 2, 16, 16, 16, 16, 16, 16, None) == 1
    assert L.lq_decode_step_slots(c, 256, 64, 2, 16, 16, 16, 16, 16, None, None) == 1
    assert L.lq_decode_step_slots(c, 256, 64, -1, 16, 16, 16, 16, 16, 16, None) == 1
    assert L.lq_window_flush_slots(c, None, 64, 2, None) == 1
    assert L.lq_state_init_slots(c, 256, 64, 2, None, None) == 1
    assert L.lq_copy_slots(c, 256, 0, 64, 512, 3, 64, 1, None) == 1
    assert L.lq_copy_slots(c, 256, 2, None, 512, 3, 64, 1, None) == 1
    # alignment: slot list 4 B, state 256 B, S0 16 B
    assert L.lq_decode_step_slots(c, 256, 66, 2, 16, 16, 16, 16, 16, 16, None) == 6
    assert L.lq_window_flush_slots(c, 128, 64, 2, None) == 6
    assert L.lq_state_init_slots(c, 256, 64, 2, 8, None) == 6
    assert L.lq_copy_slots(c, 256, 2, 64, 384, 3, 64, 1, None) == 6
    # only the LeapQuant formats run through a slot list
    for other in (B.make_config(4, 4, bits=32), B.make_config(4, 4, bits=8, per_step=True)):
        o = ctypes.byref(other)
        assert L.lq_decode_step_slots(o, 256, 64, 2, 16, 16, 16, 16, 16, 16, None) == 2
        assert L.lq_window_flush_slots(o, 256, 64, 2, None) == 2
        assert L.lq_state_init_slots(o, 256, 64, 2, 16, None) == 2
    # a bad config is reported first
    bad = B.make_config(4, 4)
    bad.window = 0
    assert L.lq_copy_slots(ctypes.byref(bad), 256, 2, 64, 512, 3, 64, 1, None) == 1


def test_multi_token_arguments_rejected_before_launch(B):
    cfg = B.make_config(4, 4, window=16)
    L = B.lib
    c = ctypes.byref(cfg)
    ok = (16, 16, 16, 16, 16, 16)
    assert L.lq_decode_steps(c, 256, 0, *ok, None) == 1          # T >= 1
    assert L.lq_decode_steps(c, 256, 9, *ok, None) == 2          # T <= 8
    small = B.make_config(4, 4, window=4)
    assert L.lq_decode_steps(ctypes.byref(small), 256, 5, *ok, None) == 1  # T <= W
    assert L.lq_decode_steps(c, None, 2, *ok, None) == 1
    assert L.lq_decode_steps(c, 128, 2, *ok, None) == 6
    assert L.lq_decode_steps(c, 256, 2, 16, 16, 16, 16, 16, None, None) == 1
    assert L.lq_decode_steps(c, 256, 2, 8, 16, 16, 16, 16, 16, None) == 6
    for other in (B.make_config(4, 4, bits=32), B.make_config(4, 4, bits=16, per_step=True)):
        assert L.lq_decode_steps(ctypes.byref(other), 256, 2, *ok, None) == 2
    assert L.lq_decode_steps_slots(c, 256, 64, 0, 2, None, None, None, None, None, None, None) == 0
    assert L.lq_decode_steps_slots(c, 256, None, 2, 2, *ok, None) == 1
    assert L.lq_decode_steps_slots(c, 256, 64, 2, 9, *ok, None) == 2


def test_prefill_arguments_rejected_before_launch(B):
    cfg = B.make_config(4, 4)
    L = B.lib
    c = ctypes.byref(cfg)
    inp = (16, 16, 16, 16, 16)  # q, k, v, beta, decay
    assert L.lq_prefill(c, 256, -1, None, None, *inp, None, None, None) == 1
    assert L.lq_prefill(c, None, 4, None, None, *inp, None, None, None) == 1
    assert L.lq_prefill(c, 256, 4, None, None, 16, None, 16, 16, 16, None, None, None) == 1
    assert L.lq_prefill(c, 128, 4, None, None, *inp, None, None, None) == 6
    assert L.lq_prefill(c, 256, 4, 2, None, *inp, None, None, None) == 6      # lengths 4 B
    assert L.lq_prefill(c, 256, 4, None, 8, *inp, None, None, None) == 6      # S0 16 B
    assert L.lq_prefill(c, 256, 4, None, None, *inp, None, 8, None) == 6      # S_final 16 B
    for other in (B.make_config(4, 4, bits=32), B.make_config(4, 4, bits=8, per_step=True)):
        assert L.lq_prefill(ctypes.byref(other), 256, 4, None, None, *inp, None, None, None) == 2
    assert L.lq_prefill_slots(c, 256, 64, 0, 4, None, None, *inp, None, None, None) == 0
    assert L.lq_prefill_slots(c, 256, None, 2, 4, None, None, *inp, None, None, None) == 1


def test_selftest_wait_arguments(B):
    assert B.lib.lq_selftest_wait(None, None) == 1
    assert B.lib.lq_selftest_wait(2, None) == 6


def test_decode_step_ex_flags(B):
    cfg = B.make_config(4, 4)
    c = ctypes.byref(cfg)
    ok = (256, 16, 16, 16, 16, 16, 16)
    assert B.lib.lq_decode_step_ex(c, *ok, 2, None) == 1          # unknown flag bit
    assert B.lib.lq_decode_step_ex(c, 128, 16, 16, 16, 16, 16, 16, 1, None) == 6
    assert B.lib.lq_decode_step_ex(c, None, 16, 16, 16, 16, 16, 16, 1, None) == 1


def test_binding_checks_tensors_before_any_call(B, monkeypatch):
    """The binding refuses a tensor of the wrong dtype, the wrong element count
    or not on the current CUDA device, before the library is called (the C
    side trusts the shapes it is given, so a bad buffer would otherwise be
    read or written out of bounds on the GPU)."""
    torch = pytest.importorskip("torch")
    calls = []
    real_lib = B.lib

    class Spy:
        def __getattr__(self, name):
            real = getattr(real_lib, name)
            if name == "lq_state_bytes":
                return real
            def f(*a):
                calls.append(name)
                return 0
            return f

    monkeypatch.setattr(B, "lib", Spy())
    N, H, d = 2, 3, 64
    cfg = B.make_config(N, H, d, d, bits=8, in_dtype="bf16")
    nb = B.lq_state_bytes(cfg)
    f32, bf16 = torch.float32, torch.bfloat16
    good = dict(state=torch.zeros(N * H * nb, dtype=torch.uint8), q=torch.zeros(N, H, d, dtype=bf16),
                k=torch.zeros(N, H, d, dtype=bf16), v=torch.zeros(N, H, d, dtype=bf16),
                beta=torch.zeros(N, H, dtype=f32), decay=torch.zeros(N, H, dtype=f32),
                out=torch.zeros(N, H, d, dtype=f32))

    def step(**over):
        a = {**good, **over}
        B.lq_decode_step(cfg, a["state"], a["q"], a["k"], a["v"], a["beta"], a["decay"], a["out"], stream=0)

    bad = [
        ("dtype", dict(q=torch.zeros(N, H, d, dtype=f32))),
        ("elements", dict(out=torch.zeros(N, H, d - 1, dtype=f32))),
        ("elements", dict(decay=torch.zeros(N, H, d, dtype=f32))),   # KDA-sized decay on a GDN state
        ("at least", dict(state=torch.zeros(N * H * nb - 1, dtype=torch.uint8))),
    ]
    for why, over in bad:
        with pytest.raises(ValueError, match=why):
            step(**over)
    with pytest.raises(ValueError, match="CUDA tensor"):
        step()                                   # right shapes and types, but host memory
    with pytest.raises(ValueError, match="dtype"):
        B.lq_state_init(cfg, good["state"], torch.zeros(N, H, d, d, dtype=torch.float64), stream=0)
    with pytest.raises(ValueError, match="elements"):
        B.lq_dequant_state(cfg, good["state"], torch.zeros(N, H, d, d + 1, dtype=f32), stream=0)
    with pytest.raises(ValueError, match="dtype"):
        B.lq_window_flush_slots(cfg, good["state"], torch.zeros(2, dtype=torch.int64), stream=0)
    T = 3
    with pytest.raises(ValueError, match="elements"):   # per-token tensors need T rows
        B.lq_decode_steps(cfg, good["state"], T, good["q"], good["k"], good["v"], good["beta"],
                          good["decay"], good["out"], stream=0)
    with pytest.raises(ValueError, match="lengths"):
        B.lq_prefill(cfg, good["state"], 1, good["q"], good["k"], good["v"], good["beta"], good["decay"],
                     lengths=torch.zeros(N + 1, dtype=torch.int32), stream=0)
    assert calls == []
    # raw addresses are the caller's responsibility and pass through
    B.lq_window_flush(cfg, 256, stream=0)
    assert calls == ["lq_window_flush"]


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++11")])
def test_header_compiles_without_cuda_headers(lang, std):
    """include/leapquant.h stands alone: plain C99 and C++11, strict warnings,
    no CUDA header on the include path (the stream is an opaque type)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = '#include "leapquant.h"\nint main(void) { lq_config c; (void)c; return (int)LQ_OK; }\n'
    r = subprocess.run([cc, std, "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), "-x", lang, "-"],
                       input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
