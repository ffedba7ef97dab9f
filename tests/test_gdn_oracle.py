"""The recurrent-scan oracle against its pins (tests/gdn_pins.py), and planted
mistakes in copies of it that the pins must catch.  Mutants are built from a
patched copy of oracle/gdn_oracle.c in a temporary directory."""
import os

import numpy as np
import pytest

import gdn_pins
import gen
import oracle.build as oracle_build
import oracle.gdn as G

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "gdn_oracle.c")


@pytest.mark.parametrize("check", gdn_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_gdn_oracle_pin(check):
    check(G.lib())


MUTANTS = {
    "recall before forgetting": ("row[j] = a * row[j];\n                        u += row[j] * kt[j];",
                                 "u += row[j] * kt[j];\n                        row[j] = a * row[j];"),
    "gate taken as the decay": ("const double a = exp((double)g[tv]);", "const double a = (double)g[tv];"),
    "write strength dropped": ("const double w = bt * (bf16_value(v[tv * dv + i]) - u);",
                               "const double w = (bf16_value(v[tv * dv + i]) - u);"),
    "correction sign": ("const double w = bt * (bf16_value(v[tv * dv + i]) - u);",
                        "const double w = bt * (bf16_value(v[tv * dv + i]) + u);"),
    "read before the write": ("row[j] = row[j] + w * kt[j];\n                        r += row[j] * qt[j];",
                              "r += row[j] * qt[j];\n                        row[j] = row[j] + w * kt[j];"),
    "read with the key": ("r += row[j] * qt[j];", "r += row[j] * kt[j];"),
    "key head by modulo": ("const int64_t hk = h / group;", "const int64_t hk = h % Hk;"),
    "output scale dropped": ("o[tv * dv + i] = scale * r;", "o[tv * dv + i] = r;"),
    "write along the query": ("row[j] = row[j] + w * kt[j];", "row[j] = row[j] + w * qt[j];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_gdn_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, "mutation site not found exactly once: %r" % old
    src = tmp_path / "gdn_oracle.c"
    src.write_text(text.replace(old, new))
    so = tmp_path / "libgdn_mutant.so"
    oracle_build.build_gdn(True, out=str(so), src=str(src))
    L = G.lib(str(so))
    caught = []
    for check in gdn_pins.ALL_CHECKS:
        try:
            check(L)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, "no pin catches the mutant %r" % name


def test_generator_scan_inputs():
    """The seeded scan inputs have the stated structure: unit q and k (to bf16
    rounding), the decay exp(g) in [0.9, 1), beta in [0.05, 0.95)."""
    d = gen.make_scan(gen.scan_config(0))
    for name in ("q", "k"):
        n = np.linalg.norm(gen.bf16_to_f32(d[name]).astype(np.float64), axis=-1)
        assert np.all(np.abs(n - 1.0) < 4e-3)
    a = np.exp(d["g"].astype(np.float64))
    assert a.min() >= 0.9 - 1e-7 and a.max() < 1.0
    assert d["beta"].min() >= 0.05 and d["beta"].max() < 0.95
    again = gen.make_scan(gen.scan_config(0))
    assert all(np.array_equal(d[n], again[n]) for n in ("q", "k", "v", "g", "beta", "S0"))
