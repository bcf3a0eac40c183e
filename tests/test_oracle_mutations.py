"""The oracle's pins have teeth: plant one plausible mistake at a time in a
copy of the oracle source (a dropped term, a wrong sign, a wrong index or
axis, a transposed operand, a wrong tie order or rounding), rebuild it, and
check that at least one pin in test_oracle_pins.py fails on it."""
import os
import subprocess

import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lq_oracle.c")

MUTATIONS = {
    "decay dropped from the step": (
        "for (int j = 0; j < dv; ++j) S[i * dv + j] *= a[i];",
        "for (int j = 0; j < dv; ++j) S[i * dv + j] *= 1.0;"),
    "sign of the delta flipped": ("u[j] = beta * (v[j] - s);", "u[j] = beta * (v[j] + s);"),
    "transposed read S k instead of S^T k": (
        "for (int i = 0; i < dk; ++i) s += S[i * dv + j] * k[i];",
        "for (int i = 0; i < dk; ++i) s += S[j * dv + i] * k[i];"),
    "output before the update": (
        "for (int i = 0; i < dk; ++i) s += S[i * dv + j] * q[i];\n        o[j] = s;",
        "for (int i = 0; i < dk; ++i) s += (S[i * dv + j] - k[i] * u[j]) * q[i];\n        o[j] = s;"),
    "beta dropped": ("u[j] = beta * (v[j] - s);", "u[j] = (v[j] - s);"),
    "column energy over the wrong axis": (
        "for (int i = 0; i < dk; ++i) e += R[i * dv + j] * R[i * dv + j];\n            colE[j] = e;",
        "for (int i = 0; i < dk; ++i) e += R[j * dv + i] * R[j * dv + i];\n            colE[j] = e;"),
    "column before row on ties": (
        "if (colE[j] > best) {", "if (colE[j] >= best) {"),
    "smoothing scale not a power of two": (
        "s = pow2_ceil(m);", "s = m;"),
    "quantization scale per key row": (
        "for (int i = 0; i < dk; ++i) m = fmax(m, fabs(R[i * dv + j]));\n        float s",
        "for (int i = 0; i < dk; ++i) m = fmax(m, fabs(R[j * dv + i]));\n        float s"),
    "round half away from zero": ("double n = nearbyint((double)t);", "double n = round((double)t);"),
    "quotient in FP64 instead of FP32": (
        "float t = (float)R[i * dv + j] / s;", "double t = R[i * dv + j] / (double)s;"),
    "compensator not added back": ("S[i0 * dv + j] += (double)w[j];", "S[i0 * dv + j] += 0.0;"),
    "window boundary off by one": ("++in_window == p->window", "++in_window == p->window + 1"),
    "buffered form misses the pair decay": (
        "for (int s = m + 1; s <= t; ++s) prod *= a[(size_t)s * dk + i];",
        "for (int s = m + 2; s <= t; ++s) prod *= a[(size_t)s * dk + i];"),
    "6-bit high code bits swapped": (
        "unsigned hi = (((unsigned)(uint8_t)cg[12 + b] & 0x3F) >> (2 * q)) & 0x3;",
        "unsigned hi = (((unsigned)(uint8_t)cg[12 + b] & 0x3F) >> (4 - 2 * q)) & 0x3;"),
    "f16 rounding truncates": ("double r = nearbyint(ax / quantum) * quantum;",
                               "double r = floor(ax / quantum) * quantum;"),
    "bf16 keeps one bit too many": ("double r = round_format(x, 8, -126);",
                                    "double r = round_format(x, 9, -126);"),
    "e4m3 does not saturate": ("if (r > 448.0) return 448.0;", "if (r > 480.0) return 448.0;"),
    "fp8 scale for the wrong format maximum": ("const float sc = (float)((double)m / 448.0);",
                                               "const float sc = (float)((double)m / 240.0);"),
    "fp8 scale per key row": ("for (int i = 0; i < dk; ++i) m = fmaxf(m, fabsf(S32[i * dv + j]));",
                              "for (int i = 0; i < dk; ++i) m = fmaxf(m, fabsf(S32[j * dv + i]));"),
    "prefill ignores the prompt length": (
        "const int n = len ? (len[h] < 0 ? 0 : (len[h] > T ? T : len[h])) : T;",
        "const int n = T;"),
    "prefill reads the decay of the wrong token": (
        "ad[i] = kda ? decay[th * dk + i] : decay[th];",
        "ad[i] = kda ? decay[(th % nh) * dk + i] : decay[th % nh];"),
    "prefill starts from a zero state": (
        "for (int x = 0; x < dk * dv; ++x) S[x] = (double)S0[(size_t)h * dk * dv + x];\n        for (int t = 0; t < T; ++t) {\n            size_t th = (size_t)t * nh + h;\n            if (t >= n) {",
        "for (int x = 0; x < dk * dv; ++x) S[x] = 0.0;\n        for (int t = 0; t < T; ++t) {\n            size_t th = (size_t)t * nh + h;\n            if (t >= n) {"),
    "per-step state not stored after the token": (
        "                per_step_store(p, S, buf32, qs, val);\n            } else",
        "                ;\n            } else"),
    "rebuild drops the decay": ("S[i * dv + j] = g[i] * acc;", "S[i * dv + j] = acc;"),
    "rebuild applies the decay per value column": ("S[i * dv + j] = g[i] * acc;",
                                                   "S[i * dv + j] = g[j] * acc;"),
    "rebuild adds a column compensator along a row": (
        "if ((int)(meta[c] & 0x7FFFFFFFu) == j) acc = acc + w[i];",
        "if ((int)(meta[c] & 0x7FFFFFFFu) == i) acc = acc + w[j];"),
    "rebuild drops the compensators": ("if ((int)meta[c] == i) acc = acc + w[j];",
                                       "if ((int)meta[c] == i) acc = acc + 0.0f;"),
    "rebuild takes the pairs in reverse order": (
        "acc = fmaf(pairs[(size_t)m * pd + i], pairs[(size_t)m * pd + dk + j], acc);",
        "acc = fmaf(pairs[(size_t)(count - 1 - m) * pd + i], pairs[(size_t)(count - 1 - m) * pd + dk + j], acc);"),
    "rebuild multiplies then adds the pair terms": (
        "acc = fmaf(pairs[(size_t)m * pd + i], pairs[(size_t)m * pd + dk + j], acc);",
        "acc = acc + pairs[(size_t)m * pd + i] * pairs[(size_t)m * pd + dk + j];"),
    "rebuild reads u at the wrong pair offset": (
        "pairs[(size_t)m * pd + dk + j], acc);", "pairs[(size_t)m * pd + dv + j], acc);"),
    "rebuild drops the last pair": ("for (int m = 0; m < count; ++m)\n                acc = fmaf(",
                                    "for (int m = 0; m + 1 < count; ++m)\n                acc = fmaf("),
    "rebuild adds the compensators in reverse round order": (
        "for (int c = 0; c < p->num_comp; ++c) {\n                if (meta[c] == LQO_NONE) continue;\n                const float *w = vec + (size_t)c * maxd;\n                if (meta[c] & LQO_KIND_COL) {\n                    if ((int)(meta[c] & 0x7FFFFFFFu) == j)",
        "for (int c = p->num_comp - 1; c >= 0; --c) {\n                if (meta[c] == LQO_NONE) continue;\n                const float *w = vec + (size_t)c * maxd;\n                if (meta[c] & LQO_KIND_COL) {\n                    if ((int)(meta[c] & 0x7FFFFFFFu) == j)"),
}

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _call(fn):
    import inspect
    params = inspect.signature(fn).parameters
    marks = getattr(fn, "pytestmark", [])
    cases = [{}]
    for m in marks:
        if m.name == "parametrize":
            names = [x.strip() for x in m.args[0].split(",")] if isinstance(m.args[0], str) else m.args[0]
            new = []
            for vals in m.args[1]:
                vals = vals if isinstance(vals, tuple) else (vals,)
                for c in cases:
                    new.append({**c, **dict(zip(names, vals))})
            cases = new
    for c in cases:
        kw = {k: v for k, v in c.items() if k in params}
        if "oracle_lib" in params:
            kw["oracle_lib"] = oracle
        fn(**kw)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {name}"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new, 1))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", *obuild.CFLAGS, "-o", str(so), str(mutated), "-lm"], check=True)
    prev = oracle.use(oracle.bind(str(so)))
    try:
        caught = []
        for fn in PIN_TESTS:
            try:
                _call(fn)
            except Exception as e:  # any failure of a pin counts as caught
                caught.append(fn.__name__)
        assert caught, f"no pin caught: {name}"
    finally:
        oracle.use(prev)
