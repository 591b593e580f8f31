"""The oracle's pins have teeth: each plausible mistake planted into a copy
of the oracle source (on the CPU, never in the product) makes the pin suite
in test_oracle.py fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "bonsai_oracle.c")

MUTATIONS = {
    "dropped last product": ("for (int64_t k = 0; k < j->K; ++k) {", "for (int64_t k = 0; k < j->K - 1; ++k) {"),
    "group index along the wrong axis": ("double s = oracle_half_to_double(s_row[k / GROUP]);",
                                         "double s = oracle_half_to_double(s_row[k % (K / GROUP)]);"),
    "wrong sign of a ternary code": ("else if (field == 3u) t = -1;", "else if (field == 3u) t = 1;"),
    "weight row indexed by the token": ("const double* w = j->w + n * j->K;",
                                        "const double* w = j->w + (m % j->N) * j->K;"),
    "ties rounded away from zero": ("(rest == 0.5 && fmod(qi, 2.0) != 0.0)", "(rest == 0.5)"),
    "subnormal decode off by one binade": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "binary pair order swapped": ("static int binary_bit(int i) { return 16 * (i & 1) + 15 - (i >> 1); }",
                                  "static int binary_bit(int i) { return 16 * (1 - (i & 1)) + 15 - (i >> 1); }"),
    "scale row stride wrong": ("dequant_row(t + n * K, scales + n * (K / GROUP), K, w + n * K);",
                               "dequant_row(t + n * K, scales + n, K, w + n * K);"),
    "base-3 digits read least significant first": ("const int q = (value / kPow3[i]) % 3;",
                                                   "const int q = (value / kPow3[4 - i]) % 3;"),
    "base-3 trit decoded with the wrong sign": ("if (k < GROUP) t[k] = (int8_t)(q - 1);",
                                                "if (k < GROUP) t[k] = (int8_t)(1 - q);"),
    "base-3 value stored rounded down": ("out[j] = (uint8_t)((256 * value + 242) / 243);",
                                         "out[j] = (uint8_t)((256 * value) / 243);"),
    "4-bit halves swapped": ("static int hqq4_bit(int i) { return 16 * (i & 1) + 4 * (i >> 1); }",
                             "static int hqq4_bit(int i) { return 16 * (1 - (i & 1)) + 4 * (i >> 1); }"),
    "4-bit zero added": ("oracle_double_to_half((double)q[n * K + k] - z);",
                         "oracle_double_to_half((double)q[n * K + k] + z);"),
    "4-bit affine group of 128": ("#define HQQ_GROUP 64", "#define HQQ_GROUP 128"),
    "4-bit difference not rounded to FP16": (
        "w[n * K + k] = oracle_double_to_half(oracle_half_to_double(d) * s);",
        "w[n * K + k] = oracle_double_to_half(((double)q[n * K + k] - z) * s + 0.0 * d);"),
    "base-3 groups packed without blocks": (
        "return g / B3_BLOCK_GROUPS * B3_BLOCK_BYTES + g % B3_BLOCK_GROUPS * B3_GROUP_BYTES;",
        "return g * B3_GROUP_BYTES;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name!r} not found exactly once"
    mutated = tmp_path / "mutated.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutated.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(lib), str(mutated), "-lm"],
                   check=True)
    env = dict(os.environ, BONSAI_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch: {name}\n{r.stdout[-2000:]}"
