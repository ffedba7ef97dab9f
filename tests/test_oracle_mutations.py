"""Plants plausible mistakes in copies of the CPU oracle and checks that the
pins catch every one of them (so the pins constrain each part of the oracle).

Mutants are built from a patched copy of oracle/moe_oracle.c in a temporary
directory; the real oracle is never touched.
"""
import os

import pytest

import oracle
import oracle.build as oracle_build
import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "moe_oracle.c")

MUTANTS = {
    "nibble order reversed": ("(word >> (4 * j))", "(word >> (28 - 4 * j))"),
    "scale and bias swapped": ("double scale = bf16_to_double(pair[0]);",
                               "double scale = bf16_to_double(pair[1]);"),
    "bias subtracted": ("scale * (double)moe_oracle_code(row, k) + bias",
                        "scale * (double)moe_oracle_code(row, k) - bias"),
    "group index from wrong axis": ("(n * (K / G) + k / G) * 2", "(n * (K / G) + (k / 8) % (K / G)) * 2"),
    "butterfly reversed": ("for (int off = 16; off >= 1; off /= 2)", "for (int off = 1; off <= 16; off *= 2)"),
    "chunk order reversed": ("int64_t h = 8 * c + j;", "int64_t h = 8 * c + (7 - j);"),
    "subnormal partial sums flushed": (
        "acc[s] = fmaf(bf16_to_float(xr[h]), bf16_to_float(wr[h]), acc[s]);",
        "acc[s] = fmaf(bf16_to_float(xr[h]), bf16_to_float(wr[h]), acc[s]);\n"
        "                if (fabsf(acc[s]) < 1.17549435e-38f) acc[s] = 0.0f;"),
    "router bias dropped": ("if (bias) l = l + bias[t * bias_stride + e];", "(void)bias_stride;"),
    "tie goes to higher index": ("if (best < 0 || l[e] > l[best]) best = e;",
                                 "if (best < 0 || l[e] >= l[best]) best = e;"),
    "no renormalisation": ("w[t * k + s] = p[idx[t * k + s]] / sel;", "w[t * k + s] = p[idx[t * k + s]];"),
    "gate and up swapped": ("h[j] = silu(g) * u;", "h[j] = silu(u) * g;"),
    "silu sign": ("return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    "down transposed": ("y += h[j] * Wd[o * I + j];", "y += h[j] * Wd[j * H + o];"),
    "weights paired with wrong slot": ("acc += w[i * k + s] * ys[(i * nslot + s) * H + o];",
                                       "acc += w[i * k + (k - 1 - s)] * ys[(i * nslot + s) * H + o];"),
    "shared expert dropped": ("if (has_shared) acc += ys[(i * nslot + k) * H + o];", "(void)has_shared;"),
    "permutation not stable by token": (
        "for (int64_t t = 0; t < T; ++t)\n            for (int64_t a = 0; a < k; ++a)\n                if (idx[t * k + a] == e) {",
        "for (int64_t t = T - 1; t >= 0; --t)\n            for (int64_t a = 0; a < k; ++a)\n                if (idx[t * k + a] == e) {"),
    "exclusive scan off by one": ("offsets[e + 1] = offsets[e] + counts[e];",
                                  "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, "mutation site not found exactly once: %r" % old
    src = tmp_path / "moe_oracle.c"
    src.write_text(text.replace(old, new))
    so = tmp_path / "libmutant.so"
    oracle_build.build(True, out=str(so), src=str(src))   # the oracle's own compiler flags
    L = oracle.lib(str(so))
    caught = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(L)
        except (AssertionError, oracle.OracleError):
            caught.append(check.__name__)
    assert caught, "no pin catches the mutant %r" % name
