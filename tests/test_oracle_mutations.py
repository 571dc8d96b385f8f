"""The pins bite: plausible mistakes planted in a copy of the oracle must fail them.

Each case edits one spot of oracle/awq_oracle.c in a temporary copy (a wrong
rounding rule, a swapped index, a dropped term, a flipped sign, ...), builds
it, and runs the pin suite (tests/test_oracle_pins.py) against that library
in a subprocess.  The suite must fail for every mutant; the real oracle is
never modified.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "awq_oracle.c")

MUTANTS = {
    "codes round half away from zero": ("(int32_t)nearbyintf(w / sf) + z", "(int32_t)roundf(w / sf) + z"),
    "nibble order reversed": ("|= (int32_t)((uint32_t)q << (4 * (k % 8)))",
                              "|= (int32_t)((uint32_t)q << (4 * (7 - k % 8)))"),
    "s divides instead of multiplying": ("float w = h2f(W[k * N + n]) * h2f(s[k]);",
                                         "float w = h2f(W[k * N + n]) / h2f(s[k]);"),
    "zero point sign flipped": ("nearbyintf(-mn / sf)", "nearbyintf(mn / sf)"),
    "step from r/16": ("f2h(r / 15.0f)", "f2h(r / 16.0f)"),
    "statistic without absolute value": ("acc += fabs(awq_oracle_half_to_double(xcal[r * K + k]));",
                                         "acc += awq_oracle_half_to_double(xcal[r * K + k]);"),
    "scale normalised by the maximum": ("double c = sqrt(tmax * tmin);", "double c = tmax;"),
    "zero point dropped in dequant": ("return (int)(((uint32_t)zeros[g * (N / 8) + n / 8]",
                                      "return 0 * (int)(((uint32_t)zeros[g * (N / 8) + n / 8]"),
    "packed row/nibble index swapped": ("((uint32_t)Q[(k / 8) * N + n] >> (4 * (k % 8)))",
                                        "((uint32_t)Q[(k % 8) * N + n] >> (4 * ((k / 8) % 8)))"),
    "subnormal exponent off by one": ("v = ldexp((double)f, -24);", "v = ldexp((double)f, -25);"),
    "binary16 ties rounded away": ("double n = nearbyint(ldexp(a, -q));", "double n = round(ldexp(a, -q));"),
    "activation multiplied by s": ("xp = xp / ", "xp = xp * "),
    "symmetric step from max/8": ("f2h(amax / 7.0f)", "f2h(amax / 8.0f)"),
    "symmetric levels round half away": ("float level = nearbyintf(w / sf);", "float level = roundf(w / sf);"),
    "symmetric codes offset by 7": ("int32_t q = (int32_t)level + 8;", "int32_t q = (int32_t)level + 7;"),
    "symmetric range without absolute value": ("if (fabsf(w) > amax) amax = fabsf(w);", "if (w > amax) amax = w;"),
    "fold multiplies by s": ("f2h(h2f(a[r * K + k]) / h2f(s[k]))", "f2h(h2f(a[r * K + k]) * h2f(s[k]))"),
    "alpha chain: 1/8 power from the square root": ("r3 = sqrt(r2);", "r3 = sqrt(r1);"),
    "scale search keeps the largest loss": ("if (loss < best) {", "if (loss > best) {"),
    "clip ratio applied to the maximum only": ("group_params(c * mn, c * mx, &sh, &z);", "group_params(mn, c * mx, &sh, &z);"),
    "clip loss ignores the activations": ("y += xp[r * GROUP + kk] * e[kk];", "y += e[kk];"),
    "missing zeros read as zero": ("if (!zeros)\n        return 8;", "if (!zeros)\n        return 0;"),
}


@pytest.fixture(scope="module")
def source():
    return open(SRC).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_fail_on_planted_mistake(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, f"mutation site not found: {old!r}"
    mutated = source.replace(old, new)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(mutated)
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", "-pthread", str(c), "-o", str(so), "-lm"], check=True)
    env = dict(os.environ, AWQ_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch: {name}\n{r.stdout[-2000:]}"
