"""Mutation check of the oracle's pins.

Each case plants one plausible mistake (a wrong sign, a dropped term, a
transposed operand, a wrong normalisation, a different rounding rule...) in a
temporary copy of oracle/w4a4_oracle.c, compiles it, and runs
tests/test_oracle_pins.py against the mutated library.  The pins must fail for
every mutation; a mutation that survives means a gap in the pins.
Nothing here touches the committed oracle or any GPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "w4a4_oracle.c")

MUTATIONS = {
    "hadamard_sign": ("H[(int64_t)(i + n) * d + (j + n)] = -h;", "H[(int64_t)(i + n) * d + (j + n)] = h;"),
    "hadamard_quadrant": ("H[(int64_t)(i + n) * d + j] = h;", "H[(int64_t)(i + n) * d + j] = -h;"),
    "rotate_norm": ("1.0 / sqrt((double)d)", "1.0 / (double)d"),
    "rotate_drop_last_input": ("for (int32_t i = 0; i < d; ++i) {\n                    const double xi",
                               "for (int32_t i = 0; i < d - 1; ++i) {\n                    const double xi"),
    "smooth_exponent": ("pow(aw, 1.0 - alpha)", "pow(aw, alpha)"),
    "smooth_no_abs": ("ax = fmax(ax, fabs(Xt[i * K + j]));", "ax = fmax(ax, Xt[i * K + j]);"),
    "smooth_inverted": ("s[j] = pow(ax, alpha) / pow(aw, 1.0 - alpha);",
                        "s[j] = pow(aw, 1.0 - alpha) / pow(ax, alpha);"),
    "quant_round_away": ("nearbyint(y[j] / d)", "round(y[j] / d)"),
    "quant_qmax": ("const double qmax = (double)((1 << (bits - 1)) - 1);",
                   "const double qmax = (double)(1 << (bits - 1));"),
    # (the clamp itself cannot fire when delta = absmax / qmax, so a mutation of it is
    # behaviour-preserving and is not listed)
    "quant_absmax_signed": ("amax = fmax(amax, fabs(y[j]));", "amax = fmax(amax, y[j]);"),
    "pack_nibble_order": ("(uint8_t)(((unsigned)lo & 0xFu) | (((unsigned)hi & 0xFu) << 4))",
                          "(uint8_t)(((unsigned)hi & 0xFu) | (((unsigned)lo & 0xFu) << 4))"),
    "unpack_sign": ("(int8_t)(lo >= 8 ? lo - 16 : lo)", "(int8_t)(lo)"),
    "gemm_transposed_b": ("const int8_t *b = B + (int64_t)n * K;", "const int8_t *b = B + (int64_t)n;"),
    "dequant_drop_bias": ("+ (bias ? bias[n] : 0.0);\n    return 0;\n}\n\n/* Plain",
                          ";\n    return 0;\n}\n\n/* Plain"),
    "dequant_drop_channel_scale": ("(double)acc[m * N + n] * delta_tok[m] * delta_ch[n]",
                                   "(double)acc[m * N + n] * delta_tok[m]"),
    "gelu_no_sqrt2": ("erf(v / sqrt(2.0))", "erf(v)"),
    "bf16_round_truncate": ("double r = nearbyint(m * 256.0);", "double r = trunc(m * 256.0);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(lib), str(mutated), "-lm"], check=True)
    env = dict(os.environ, W4A4_ORACLE_LIB=str(lib), OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0, f"mutation {name} survived the pins:\n{r.stdout[-2000:]}"
