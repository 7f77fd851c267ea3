"""Each plausible mistake planted in a copy of the oracle (on the CPU) must be
caught by at least one pin: this is what makes the pins worth trusting.

The planted mistakes cover a flipped sign, a dropped term, a wrong index, a
transposed operand, a missing mask and a wrong memory layout.  The copies are
built in a temporary directory; the oracle source itself is not touched.
"""
import os
import shutil

import pytest

import oracle
from tests import _pins

# (name, text to replace, replacement, which occurrence (0-based) or None = all)
MUTANTS = [
    ("bias-sign", "return alpha * s + bias;", "return alpha * s - bias;", None),
    ("sigmoid-sign", "return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));", None),
    ("sigmoid-grad-dropped-term", "return p * (1.0 - p);", "return p;", None),
    ("fwd-no-query-mask", "if (i >= n_q) continue;", "", 0),
    ("fwd-no-key-mask", "for (int64_t j = 0; j < n_k; ++j) {", "for (int64_t j = 0; j < Lk; ++j) {", 0),
    ("dq-no-key-mask", "for (int64_t j = 0; j < n_k; ++j) {", "for (int64_t j = 0; j < Lk; ++j) {", 1),
    ("dq-dropped-sigma-prime", "double ds = p * (1.0 - p) * dp;", "double ds = p * dp;", 0),
    ("dkdv-dropped-sigma-prime", "double ds = p * (1.0 - p) * dp;", "double ds = p * dp;", 1),
    ("dq-dropped-alpha", "for (int d = 0; d < D; ++d) g[d] *= alpha;", "", None),
    ("dk-dropped-alpha", "for (int d = 0; d < D; ++d) gk[d] *= alpha;", "", None),
    ("dv-wrong-operand", "gv[d] += p * load_elem(dout, dtype, qo + d);",
     "gv[d] += p * load_elem(q, dtype, qo + d);", None),
    ("dk-wrong-operand", "gk[d] += ds * load_elem(q, dtype, qo + d);",
     "gk[d] += ds * load_elem(k, dtype, qo + d);", None),
    ("dkdv-transposed-score",
     "double p = oracle_sigmoid(score(q, k, dtype, z, h, i, j, Lq, Lk, H, D, alpha, bias));",
     "double p = oracle_sigmoid(score(q, k, dtype, z, h, j, i, Lq, Lk, H, D, alpha, bias));", 2),
    ("dq-dp-wrong-operand", "double dp = dot_rows(dout, v, dtype, z, h, i, j, Lq, Lk, H, D);",
     "double dp = dot_rows(dout, k, dtype, z, h, i, j, Lq, Lk, H, D);", 0),
    ("dkdv-padded-queries-flow", "for (int64_t i = 0; i < n_q; ++i) {", "for (int64_t i = 0; i < Lq; ++i) {", None),
    ("key-rows-in-query-layout", "int64_t ko = offset_of(z, j, h, Lk, H, D);",
     "int64_t ko = offset_of(z, j, h, Lq, H, D);", None),
    ("dkdv-no-key-row-mask", "if (j >= n_k) continue;", "", None),
    ("layout-h-l-swapped", "return ((z * L + l) * H + h) * (int64_t)D;",
     "return ((z * H + h) * L + l) * (int64_t)D;", None),
    ("dbias-dropped-sigma-prime", "acc += p * (1.0 - p) * dp;", "acc += p * dp;", None),
    ("dbias-no-key-mask", "for (int64_t j = 0; j < n_k; ++j) {", "for (int64_t j = 0; j < Lk; ++j) {", 2),
    ("dbias-no-query-mask", "if (i < n_q) {", "if (i < Lq) {", None),
    ("bias-per-sample-wrong-index", "const double bias = bias_z[z];", "const double bias = bias_z[0];", None),
    ("bf16-widening", "uint32_t bits = ((uint32_t)b) << 16;", "uint32_t bits = ((uint32_t)b) << 15;", None),
    ("fwd-value-from-key", "for (int d = 0; d < D; ++d) o[d] += p * load_elem(v, dtype, vo + d);",
     "for (int d = 0; d < D; ++d) o[d] += p * load_elem(k, dtype, vo + d);", None),
]


def _mutate(src: str, old: str, new: str, occurrence):
    if old not in src:
        raise AssertionError(f"mutation anchor not found: {old!r}")
    if occurrence is None:
        return src.replace(old, new)
    pos = -1
    for _ in range(occurrence + 1):
        pos = src.index(old, pos + 1)
    return src[:pos] + new + src[pos + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, occ):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    with open(oracle.SOURCE) as f:
        src = f.read()
    mutated = _mutate(src, old, new, occ)
    assert mutated != src
    c = os.path.join(tmp_path, "mutant.c")
    so = os.path.join(tmp_path, "mutant.so")
    with open(c, "w") as f:
        f.write(mutated)
    oracle.build(force=True, src=c, out=so)
    orc = oracle.OracleLib(so)
    caught = []
    for pin in _pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError as e:
            caught.append(pin.__name__)
            break
    assert caught, f"mutant {name} passed every pin"


def test_real_oracle_passes_every_pin():
    orc = oracle.default()
    for pin in _pins.ALL_PINS:
        pin(orc)
