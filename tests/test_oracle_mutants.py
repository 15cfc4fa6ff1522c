"""Plant plausible mistakes in copies of the oracle (on the CPU) and check the pins catch them.

Each mutant is one textual edit of ``oracle/kv4_oracle.c`` or ``oracle/gtq_oracle.c`` (a dropped
term, a wrong sign, rounding mode, index or constant).  It is compiled to a temporary library and the full pin
list runs against it in a child process; the mutant is "killed" when any pin fails (or the
child crashes).  A surviving mutant means the pins do not constrain that part of the oracle.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")
FILES = ("kv4_oracle.c", "gtq_oracle.c", "kv4_oracle.h", "gtq_oracle.h")

# (name, original text, replacement, occurrence index or None for all)
MUTANTS = [
    ("butterfly-sign", "x[j + st] = a - b;", "x[j + st] = b - a;", 0),
    ("butterfly-f64-sign", "x[j + st] = a - b;", "x[j + st] = b - a;", 1),
    ("zero-round-nearest", "orc_f32_to_f16(mn, ORC_RD)", "orc_f32_to_f16(mn, ORC_RN)", None),
    ("scale-round-nearest", "orc_f32_to_f16(sq, ORC_RU)", "orc_f32_to_f16(sq, ORC_RN)", None),
    ("int4-levels-16", "r / 15.0f", "r / 16.0f", None),
    ("int4-truncate", "const float rq = rintf(t);", "const float rq = truncf(t);", None),
    ("int8-levels-128", "a / 127.0f", "a / 128.0f", None),
    ("int8-scale-round-nearest", "orc_f32_to_f16(a / 127.0f, ORC_RU)", "orc_f32_to_f16(a / 127.0f, ORC_RN)", None),
    ("nibble-swap", "put_nibble(pool, orc_k4_byte(c, page, g, pp, e), orc_k4_high(c, pp, e), c4[e]);",
     "put_nibble(pool, orc_k4_byte(c, page, g, pp, e), orc_k4_high(c, pp, e) ^ 1, c4[e]);", None),
    ("k4-pair-row-no-swizzle", "(b / 16) ^ (D >= 128 ? (pr & 1) : 0)", "(b / 16)", None),
    ("v4-pair-index", "4 * j + 2 * (r & 1) + (k >> 1)", "4 * j + 2 * ((r >> 1) & 1) + (k >> 1)", None),
    ("k8-no-swizzle", "16 * ((e / 16) ^ (r & 1))", "16 * (e / 16)", None),
    ("route-ring-strict", "p >= lens_after[b] - w", "p > lens_after[b] - w", None),
    ("ring-row-no-offset", "row = s + p % w;", "row = p % w;", None),
    ("q-rot-sqrt-norm", "qr[e] *= 1.0 / (double)h;", "qr[e] *= 1.0 / sqrt((double)h);", None),
    ("q-not-rotated", "orc_fwht_f64(qr, D, h);", ";", None),
    ("q-signs-ignored", "if (orc_sign(c, e)) qr[e] = -qr[e];", ";", None),
    ("k-signs-ignored", "if (orc_sign(c, e)) x[e] = -x[e];", ";", None),
    ("v-rotation-not-undone", "if (c->rotate_values) {", "if (0) {", None),
    ("v-rotation-no-signs", "(orc_sign(c, e) ? -o[e] : o[e]) / (double)h", "o[e] / (double)h", None),
    ("tau-wrong", "1.0 / sqrt((double)D)", "1.0 / (double)D", None),
    ("merge-no-rescale-l", "l += parts[i].l * f;", "l += parts[i].l;", None),
    ("merge-no-rescale-o", "out[e] += parts[i].o[e] * f;", "out[e] += parts[i].o[e];", None),
    ("recent-begin-off-by-one", "const int r_begin = (L - w) > s ? (L - w) : s;",
     "const int r_begin = (L - w + 1) > s ? (L - w + 1) : s;", None),
    ("dequant-drop-zero", "kr[e] = kz + ks *", "kr[e] = ks *", None),
    ("gqa-map", "(size_t)(g * G + i)", "(size_t)(g + i * Hkv)", None),
    ("f16-no-subnormal", "if (E < -14) E = -14;", ";", None),
    ("f16-ties-away", "(frac == 0.5 && fmod(n, 2.0) == 1.0)", "(frac == 0.5)", None),
    ("int4-range-unreported", "  return out_of_range;\n}", "  return 0;\n}", 0),
    ("int8-range-unreported", "  return out_of_range;\n}", "  return 0;\n}", 1),
    ("bf16-truncate", "const uint32_t up = lo > 0x8000u || (lo == 0x8000u && (hi & 1u));",
     "const uint32_t up = 0;", None),
    ("bf16-ties-away", "const uint32_t up = lo > 0x8000u || (lo == 0x8000u && (hi & 1u));",
     "const uint32_t up = lo >= 0x8000u;", None),
    ("vbf-no-swizzle", "const int swz = units >= 4 ? ((pl & 2) | (gq & 1)) : (units >= 2 ? (gq & 1) : 0);",
     "const int swz = 0;", None),
    ("vbf-pair-rows", "return (size_t)(((half * 8 + gq) * 4 + pl) * (D / 2) + 16 * (u ^ swz) + within + 2 * (r & 1));",
     "return (size_t)(((half * 8 + gq) * 4 + pl) * (D / 2) + 16 * (u ^ swz) + within + 2 * ((r >> 1) & 1));", None),
    ("single-softmax-max", "if (logit[j] > ps->m) ps->m = logit[j];", "if (logit[j] < ps->m) ps->m = logit[j];", None),
]

# mutants of the mixed bit-width key cache (gtq_oracle.c)
GTQ_MUTANTS = [
    ("gtq-gain-2-per-bit", "ldexp(energy[b], -2 * (int)widths[b]); /* E * 4^-w, exact */",
     "ldexp(energy[b], -(int)widths[b]);", None),
    ("gtq-ties-to-highest", "if (best < 0 || gain > best_gain) {", "if (best < 0 || gain >= best_gain) {", None),
    ("gtq-cap-7", "if (widths[b] >= 8) continue;", "if (widths[b] >= 7) continue;", None),
    ("gtq-adjacent-pairs", "gtq_load(K, k_dtype, row + (size_t)(b + nb));", "gtq_load(K, k_dtype, row + (size_t)(b ^ 1));", None),
    ("gtq-energy-one-coordinate", "e = e + (x0 * x0 + x1 * x1);", "e = e + x0 * x0;", None),
    ("gtq-scale-mean-not-rms", "(float)sqrt(energy[b] / (2.0 * (double)T))", "(float)(energy[b] / (2.0 * (double)T))", None),
    ("gtq-key-scale-round-nearest", "const uint16_t sb = orc_f32_to_f16(m, ORC_RU);", "const uint16_t sb = orc_f32_to_f16(m, ORC_RN);", None),
    ("gtq-key-ignores-sigma", "const float a = fabsf(x[i]) / sc[i];", "const float a = fabsf(x[i]);", None),
    ("gtq-key-round-not-floor", "const float f = floorf(u);", "const float f = rintf(u);", None),
    ("gtq-key-levels-off", "(t + 1.0f) * (float)(1 << (w - 1))", "(t + 1.0f) * (float)(1 << w)", None),
    ("gtq-key-recon-midpoint", "(ldexp(2.0 * code + 1.0, -w) - 1.0)", "(ldexp(2.0 * code, -w) - 1.0)", None),
    ("gtq-w0-not-zero", "if (w == 0) return 0.0;", "if (w == 0) return (double)orc_f16_to_f32(scale) * (double)sigma;", None),
    ("gtq-value-levels-2w", "const int top = (1 << bits) - 1;", "const int top = (1 << bits);", 0),
    ("gtq-value-zero-round-nearest", "const uint16_t zb = orc_f32_to_f16(mn, ORC_RD);", "const uint16_t zb = orc_f32_to_f16(mn, ORC_RN);", None),
    ("gtq-pack-msb-first", "row[n >> 3] |= (uint8_t)(1u << (n & 7));", "row[n >> 3] |= (uint8_t)(0x80u >> (n & 7));", None),
    ("gtq-value-rows-after-params", "return slice_base(c, page, g, pp) + 16u * orc_gtq_key_row_bytes(c) + (size_t)(pp % 16) * orc_gtq_value_row_bytes(c);",
     "return slice_base(c, page, g, pp) + 16u * (orc_gtq_key_row_bytes(c) + 8u) + (size_t)(pp % 16) * orc_gtq_value_row_bytes(c);", None),
    ("gtq-page-major-not-slice-major", "(size_t)(pp / 16) * 16u * (orc_gtq_key_row_bytes(c) + orc_gtq_value_row_bytes(c) + 8u);",
     "0u; (void)pp;", None),
    ("gtq-param-order", "put16(pool + orc_gtq_param(c, page, g, pp) + 4, z);", "put16(pool + orc_gtq_param(c, page, g, pp) + 6, z);", None),
    ("gtq-block-of-coordinate", "wc[i] = widths[(size_t)g * (size_t)nb + (size_t)(i % nb)];", "wc[i] = widths[(size_t)g * (size_t)nb + (size_t)(i / 2)];", None),
    ("gtq-softmax-scale", "const double tau = 1.0 / sqrt((double)D);", "const double tau = 1.0 / (double)D;", None),
]

RUNNER = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
import oracle_pins as P
for i, pin in enumerate(P.ALL_PINS):
    try:
        pin()
    except Exception as e:
        print("KILLED by pin", i, type(e).__name__)
        sys.exit(3)
print("SURVIVED")
sys.exit(0)
"""


def _mutate(text: str, old: str, new: str, occ):
    assert old in text, f"mutation anchor not found: {old!r}"
    if occ is None:
        return text.replace(old, new)
    parts = text.split(old)
    assert len(parts) > occ + 1, f"occurrence {occ} of {old!r} missing"
    return old.join(parts[:occ + 1]) + new + old.join(parts[occ + 1:])


def _run_mutant(tmp: str, fname: str, name: str, old: str, new: str, occ) -> tuple[str, str]:
    d = os.path.join(tmp, name)
    os.makedirs(d)
    for f in FILES:
        text = open(os.path.join(ORACLE, f)).read()
        if f == fname:
            text = _mutate(text, old, new, occ)
        with open(os.path.join(d, f), "w") as out:
            out.write(text)
    so = os.path.join(d, "lib.so")
    from oracle.oracle import CFLAGS
    srcs = [os.path.join(d, f) for f in FILES if f.endswith(".c")]
    subprocess.run(["gcc", *[c for c in CFLAGS if c not in ("-Wall", "-Wextra")], "-o", so, *srcs, "-lm"],
                   check=True, capture_output=True)
    env = dict(os.environ, KV4_ORACLE_LIB=so, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, tests=os.path.join(ROOT, "tests"))],
                       env=env, capture_output=True, text=True, timeout=600)
    return name, (r.stdout.strip().splitlines() or ["(crashed: %d)" % r.returncode])[-1]


@pytest.mark.slow
def test_every_mutant_is_killed():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
            jobs = [("kv4_oracle.c", *m) for m in MUTANTS] + [("gtq_oracle.c", *m) for m in GTQ_MUTANTS]
            results = list(ex.map(lambda m: _run_mutant(tmp, *m), jobs))
    survivors = [(n, r) for n, r in results if "SURVIVED" in r]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
