"""The pins must catch plausible mistakes in the oracle. Each case plants one
mistake in a copy of oracle/wp_oracle.c (on the CPU), builds it, and runs the
pin suite against it in a subprocess: at least one pin has to fail."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "wp_oracle.c")

MUTANTS = {
    "channel window off by one": ("if (dist > (int64_t)cut[c])", "if (dist >= (int64_t)cut[c])"),
    "group window off by one": ("if (dist > (int64_t)cut[g])", "if (dist >= (int64_t)cut[g])"),
    "rotation sign": ("yr[a] = xa * cs - xb * sn;", "yr[a] = xa * cs + xb * sn;"),
    "half-split pair": ("*b = c + d_h / 2;", "*b = c + 1;"),
    "half-split owner": ("return layout == WPO_INTERLEAVED ? k / 2 : k % (d_h / 2);",
                         "return layout == WPO_INTERLEAVED ? k / 2 : k / 2;"),
    "ceil instead of floor": ("double fl = floor(w);", "double fl = ceil(w);"),
    "frequency index": ("pow(theta, -2.0 * (double)c / (double)d_h)", "pow(theta, -2.0 * (double)(c + 1) / (double)d_h)"),
    "lse without max": ("double lse = m + log(s);", "double lse = log(s) + 0.0 * m;"),
    "gqa head map": ("int64_t hk = h / rep;", "int64_t hk = h % Hkv;"),
    "scale dropped": ("return scale * acc;", "return acc;"),
    "tile full rule": ("else if ((int64_t)cut[g] >= hi)", "else if ((int64_t)cut[g] > hi)"),
    "tile skip rule": ("else if ((int64_t)cut[g] < lo)", "else if ((int64_t)cut[g] <= lo)"),
    "causal diagonal dropped": ("for (int64_t j = 0; j <= i; ++j) {\n        L[j]", "for (int64_t j = 0; j < i; ++j) {\n        L[j]"),
    "group width": ("for (int t = 16 * g; t < 16 * g + 16; ++t)", "for (int t = 16 * g; t < 16 * g + 15; ++t)"),
    "backward: softmax correction dropped": ("double dl = p * (dp - D);", "double dl = p * dp;"),
    "backward: dV without the weight": ("dvb[j * ks + t] += p * doi[t];", "dvb[j * ks + t] += doi[t];"),
    "backward: dK from k": ("dk[t] += s * q[t];", "dk[t] += s * k[t];"),
    "backward: dQ channel partner dim": ("dq[b] += s * k[b];", "dq[b] += s * k[a];"),
    "backward: scale dropped": ("double s = scale * dl;", "double s = dl;"),
    "backward: mask ignored": ("            if (dist > (int64_t)cut[g])\n                continue;\n            for (int t = 16 * g; t < 16 * g + 16; ++t) {\n                dq[t]",
                               "            for (int t = 16 * g; t < 16 * g + 16; ++t) {\n                dq[t]"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "mutant.c"
    so = tmp_path / "libmutant.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", str(c),
                           "-o", str(so), "-lm"])
    env = dict(os.environ, WP_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught the planted mistake '{name}'"
