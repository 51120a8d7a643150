"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one. The planted copies live in a temporary directory; the
committed oracle is never modified. CPU only."""
import os
import shutil

import pytest

import oracle
import oracle_pins

# (name, text in grkan_oracle.c, replacement, which occurrence (0-based))
MUTANTS = [
    ("Q gets a constant term", "Q = (Q + b[j - 1]) * x;", "Q = Q * x + b[j - 1];", 0),
    ("P' drops the factor i", "dP = dP * x + (double)i * a[i];", "dP = dP * x + a[i];", 0),
    ("P' index off by one", "dP = dP * x + (double)i * a[i];",
     "dP = dP * x + (double)(i - 1) * a[i];", 0),
    ("Q' drops the factor j", "dQ = dQ * x + (double)j * b[j - 1];", "dQ = dQ * x + b[j - 1];", 0),
    ("denominator without abs", "o->D = 1.0 + fabs(Q);", "o->D = 1.0 + Q;", 0),
    ("sign(0) = +1", "((Q < 0.0) ? -1.0 : 0.0)", "((Q < 0.0) ? -1.0 : 1.0)", 0),
    ("dx sign flipped", "dx[k] = gv * (p.dP - p.y * p.s * p.dQ) / p.D;",
     "dx[k] = gv * (p.dP + p.y * p.s * p.dQ) / p.D;", 0),
    ("dx misses the 1/D", "dx[k] = gv * (p.dP - p.y * p.s * p.dQ) / p.D;",
     "dx[k] = gv * (p.dP - p.y * p.s * p.dQ);", 0),
    ("dA misses the 1/D", "double term = gv * xi / p.D;", "double term = gv * xi;", 0),
    ("dA power off by one", "        double xi = 1.0;\n        for (int i = 0; i <= m; ++i) {\n"
     "          double term", "        double xi = xv;\n        for (int i = 0; i <= m; ++i) {\n"
     "          double term", 0),
    ("dB sign flipped", "double term = -gv * p.y * p.s * xi / p.D;",
     "double term = gv * p.y * p.s * xi / p.D;", 0),
    ("dB power off by one", "        xi = xv;\n        for (int j = 1; j <= n; ++j) {\n"
     "          double term", "        xi = 1.0;\n        for (int j = 1; j <= n; ++j) {\n"
     "          double term", 0),
    ("dB uses P instead of y", "double term = -gv * p.y * p.s * xi / p.D;",
     "double term = -gv * p.P * p.s * xi / p.D;", 0),
    ("groups interleaved, not contiguous", "int g = (int)(col / dg);",
     "int g = (int)(col % n_g);", 0),
    ("elementwise groups interleaved", "int g = (int)((e % d) / dg);",
     "int g = (int)((e % d) % n_g);", 1),
    ("last reduction chunk dropped", "  for (int64_t c = 0; c < nchunks; ++c) {\n    const double* sum",
     "  for (int64_t c = 0; c + 1 < nchunks; ++c) {\n    const double* sum", 0),
    ("bf16 widened from the wrong half", "<< 16;", "<< 15;", 0),
    ("noise scale not squared", "qrow[i] += w * w;", "qrow[i] += w;", 0),
    ("dB noise scale drops kappa_p", "(kp + 2.0 * fabs(p.P) * kq / p.D)", "(2.0 * fabs(p.P) * kq / p.D)",
     0),
    ("forward groups interleaved", "int g = (int)((e % d) / dg);",
     "int g = (int)((e % d) % n_g);", 0),
    # the error scales that widen the y / dx tolerances and the sign-ambiguity test
    ("kappa_y drops the denominator term", "return (sa + fabs(p->y) * sb) / p->D;",
     "return sa / p->D;", 0),
    ("kappa_y misses the 1/D", "return (sa + fabs(p->y) * sb) / p->D;",
     "return sa + fabs(p->y) * sb;", 0),
    ("kappa_y uses the signed y", "return (sa + fabs(p->y) * sb) / p->D;",
     "return (sa + p->y * sb) / p->D;", 0),
    ("kappa_y doubled", "return (sa + fabs(p->y) * sb) / p->D;",
     "return 2.0 * (sa + fabs(p->y) * sb) / p->D;", 0),
    ("kappa_y denominator powers start at x^0", "  xi = ax;\n  for (int j = 1; j <= n; ++j) {",
     "  xi = 1.0;\n  for (int j = 1; j <= n; ++j) {", 0),
    ("kappa_q powers start at x^0", "double ax = fabs(x), sb = 0.0, xi = ax;",
     "double ax = fabs(x), sb = 0.0, xi = 1.0;", 0),
    ("kappa_q uses the signed x", "double ax = fabs(x), sb = 0.0, xi = ax;",
     "double ax = x, sb = 0.0, xi = ax;", 0),
    ("kappa_q doubled", "  return sb;\n}", "  return 2.0 * sb;\n}", 0),
    ("kappa_dx drops the kappa_y |Q'| term",
     "(sa + fabs(p.y) * sb + ky * fabs(p.dQ)) / p.D;", "(sa + fabs(p.y) * sb) / p.D;", 0),
    ("kappa_dx misses the 1/D", "(sa + fabs(p.y) * sb + ky * fabs(p.dQ)) / p.D;",
     "(sa + fabs(p.y) * sb + ky * fabs(p.dQ));", 0),
    ("kappa_dx doubled", "kappa_dx[k] = fabs(gv) * (", "kappa_dx[k] = 2.0 * fabs(gv) * (", 0),
    ("kappa_dx drops the factor i", "sa += (double)i * fabs(ga[i]) * xi;",
     "sa += fabs(ga[i]) * xi;", 0),
    ("kappa_dx uses the signed y", "(sa + fabs(p.y) * sb + ky * fabs(p.dQ)) / p.D;",
     "(sa + p.y * sb + ky * fabs(p.dQ)) / p.D;", 0),
    ("kappa_dx uses the signed Q'", "(sa + fabs(p.y) * sb + ky * fabs(p.dQ)) / p.D;",
     "(sa + fabs(p.y) * sb + ky * p.dQ) / p.D;", 0),
    ("dA noise weight drops kappa_q / D", "double w = fabs(term) * (1.0 + kq / p.D);",
     "double w = fabs(term);", 0),
    ("dB noise weight drops the 2|P| kappa_q / D part", "(kp + 2.0 * fabs(p.P) * kq / p.D)",
     "(kp)", 0),
]


def _replace_nth(text, old, new, k):
    pos = -1
    for _ in range(k + 1):
        pos = text.find(old, pos + 1)
        assert pos >= 0, "mutation anchor not found: %r (occurrence %d)" % (old, k)
    return text[:pos] + new + text[pos + len(old):]


@pytest.mark.parametrize("name,old,new,k", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, k):
    src = open(oracle.SRC).read()
    mutated = _replace_nth(src, old, new, k)
    assert mutated != src
    shutil.copy(os.path.join(os.path.dirname(oracle.SRC), "grkan_oracle.h"), tmp_path)
    msrc = tmp_path / "grkan_oracle.c"
    msrc.write_text(mutated)
    lib = oracle.build(str(msrc), str(tmp_path / "libmutant.so"), force=True)
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin caught the planted mistake: %s" % name
