"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pins catch every one: each mutant must fail at least one pin.
Every mutation keeps all memory accesses in bounds, so the mutants run
in-process."""
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fa_oracle.c")

MUTANTS = {
    "unscaled-scores": ("s[j] = scale * acc;", "s[j] = acc;"),
    "causal-sign": ("return j <= i + (lk - lq);", "return j <= i + (lq - lk);"),
    "causal-strict": ("return j <= i + (lk - lq);", "return j < i + (lk - lq);"),
    "lse-missing-log": ("double lse = mx + log(sum);", "double lse = mx + sum;"),
    "dq-missing-scale": ("dqi[c] += scale * ds *", "dqi[c] += ds *"),
    "dk-transposed-operand": ("dk[koffs[j] + c] += scale * ds * load_in(q, qoff + c, dtype);",
                              "dk[koffs[j] + c] += scale * ds * load_in(k, koffs[j] + c, dtype);"),
    "dS-dropped-D": ("const double ds = p[j] * (dp[j] - D);", "const double ds = p[j] * dp[j];"),
    "dS-wrong-sign": ("const double ds = p[j] * (dp[j] - D);", "const double ds = p[j] * (D - dp[j]);"),
    "dv-uses-dS": ("dv[koffs[j] + c] += p[j] * load_in(dout", "dv[koffs[j] + c] += ds * load_in(dout"),
    "head-stride": ("(int64_t)h * d;", "(int64_t)h * H;"),
    "lse-row-index": ("lse[(int64_t)h * total_q + cu_q[b] + i] = l;", "lse[(int64_t)h * total_q + i] = l;"),
    "seqlen-off-by-one": ("len[b] = cu[b + 1] - cu[b];", "len[b] = cu[b + 1] - cu[b] - 1;"),
    "bf16-widen-shift": ("<< 16;", "<< 15;"),
    "gqa-interleaved-heads": ("const int hk = h / g;", "const int hk = h % Hk;"),
    "gqa-bwd-one-head-per-group": ("for (int h = hk * g; h < (hk + 1) * g; ++h)",
                                   "for (int h = hk * g; h < hk * g + 1; ++h)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    src = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as td:
        c_path = os.path.join(td, "mutant.c")
        so_path = os.path.join(td, "libmutant.so")
        with open(c_path, "w") as f:
            f.write(src)
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", c_path,
                               "-o", so_path, "-lm"])
        orc = oracle.OracleLib(so_path)
        failed = []
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(orc)
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
        assert failed, f"mutant {name} passed every pin"
