"""The pins catch plausible mistakes: each case plants one mistake in a copy
of the oracle's C source (on the CPU), builds it, runs the pin suite against
the mutant and expects at least one pin to fail."""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qmv_oracle.c")

MUTANTS = {
    "e8m0 target exponent 2 -> 1": ("e = orc_floor_log2(amax) - 2;", "e = orc_floor_log2(amax) - 1;"),
    "nibble order swapped (fp4)": ("cb[i / 2] = (uint8_t)(c[0] | (c[1] << 4));", "cb[i / 2] = (uint8_t)(c[1] | (c[0] << 4));"),
    "E2M1 ties to odd": ("(c % 2 == 0) && (best % 2 == 1)", "(c % 2 == 1) && (best % 2 == 0)"),
    "int rounding half away from zero": ("float r = rintf(w[i] / s);", "float r = roundf(w[i] / s);"),
    "int4 offset 8 -> 7 in dequant": ("int q = ((k % 2) ? (byte >> 4) : (byte & 15)) - 8;",
                                      "int q = ((k % 2) ? (byte >> 4) : (byte & 15)) - 7;"),
    "clip: last minimum kept": ("if (!have || err < best_err) {", "if (!have || err <= best_err) {"),
    "matvec drops the batch index": ("acc += xd[b * K + k] *", "acc += xd[k] *"),
    "k-means ties to the higher index": ("    if (d < bd) {\n      bd = d;\n      best = k;",
                                         "    if (d <= bd) {\n      bd = d;\n      best = k;"),
    "k-means centre update skipped": ("if (cnt[k] > 0) c[k] = (double)(float)(sum[k] / (double)cnt[k]);",
                                      "if (cnt[k] > 0 && 0) c[k] = (double)(float)(sum[k] / (double)cnt[k]);"),
    "fp16 ties away from zero": ("double m = nearbyint(ldexp(a, 10 - E));", "double m = round(ldexp(a, 10 - E));"),
    "int8 clamp at 126": ("if (r > (float)qmax) r = (float)qmax;", "if (r > (float)qmax - 1) r = (float)qmax - 1;"),
    "int4aff zero point dropped in dequant": ("return (float)(q - z) * s;", "return (float)(q) * s;"),
    "int4aff range without zero": ("float lo = 0.0f, hi = 0.0f;", "float lo = w[0], hi = w[0];"),
    "int4aff zero-point nibble order": ("zp[b / 2] |= (uint8_t)(z << ((b % 2) * 4));",
                                        "zp[b / 2] |= (uint8_t)(z << ((1 - b % 2) * 4));"),
    "k-means start at the lower quantile edge": ("c[k] = (double)s[((2 * k + 1) * n) / (2 * nc)];",
                                                 "c[k] = (double)s[(k * n) / nc];"),
    "int8km indices against unrounded centres": ("(uint8_t)orc_nearest(cl, 256, (double)w[i]);",
                                                 "(uint8_t)orc_nearest(c, 256, (double)w[i]);"),
    "int8km last partial group dropped": ("return (N + ORC_KM8_GROUP - 1) / ORC_KM8_GROUP;",
                                          "return N / ORC_KM8_GROUP;"),
    "outlier columns by the smallest maximum": ("if (x->m != y->m) return (x->m > y->m) ? -1 : 1;",
                                                "if (x->m != y->m) return (x->m > y->m) ? 1 : -1;"),
    "outlier dequant with the first scale only": ("oscales[n * (C / 32) + jo / 32]", "oscales[n * (C / 32)]"),
    "int8km LUT shared by 16 rows in dequant": ("aux)[(n / ORC_KM8_GROUP) * 256 + j]", "aux)[(n / 16) * 256 + j]"),
    "mixed main-part nibbles swapped in dequant": ("int e = (jm % 2) ? (byte >> 4) : (byte & 15);\n        Wdq",
                                                   "int e = (jm % 2) ? (byte & 15) : (byte >> 4);\n        Wdq"),
    "outlier membership off by one column": ("return lo < C && cols[lo] == k;", "return lo < C && cols[lo] == k + 1;"),
}


def _compile(src_text, out):
    path = out + ".c"
    with open(path, "w") as f:
        f.write(src_text)
    for cc in ("/usr/bin/gcc", os.environ.get("CC") or "gcc", "gcc"):
        r = subprocess.run([cc, "-std=c11", "-O2", "-ffp-contract=off", "-fPIC", "-shared", path, "-o", out, "-lm"],
                           capture_output=True, text=True)
        if r.returncode == 0:
            return
    raise RuntimeError(r.stderr)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site not found: {name}"
    lib = str(tmp_path / "liboracle_mutant.so")
    _compile(src.replace(old, new, 1), lib)
    env = dict(os.environ, QMV_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")], env=env, capture_output=True,
                       text=True, cwd=ROOT, timeout=600)
    assert r.returncode != 0, f"mutant survived: {name}\n{r.stdout[-2000:]}"
