"""Plant plausible mistakes in copies of the oracle and check that each one
trips at least one pin. The mutants are compiled from the oracle's C source
into a temporary directory on the CPU; the real oracle is not touched."""
import os

import pytest

import oracle
import pins
from oracle import build as obuild

# (name, text in parallax_oracle.c, replacement)
MUTANTS = [
    ("drop correction (definition)", "hv->o[d] += ws * (vi[d] - vbar[d]);",
     "hv->o[d] += 0.0 * ws * (vi[d] - vbar[d]);"),
    ("drop correction (expanded)", "hv->o[d] = vbar + C[d] / l - (bb / l) * vbar;",
     "hv->o[d] = vbar;"),
    ("wrong sign (expanded)", "hv->o[d] = vbar + C[d] / l - (bb / l) * vbar;",
     "hv->o[d] = vbar + C[d] / l + (bb / l) * vbar;"),
    ("wrong sign (streaming)",
     "hv->o[d] = vbar + total->C[d] / total->l - (total->b / total->l) * vbar;",
     "hv->o[d] = vbar - total->C[d] / total->l + (total->b / total->l) * vbar;"),
    # Centring either factor of the weighted covariance alone is exact (the
    # other factor's weighted mean is zero), so only the doubly uncentred
    # product, which drops the -(b/l) vbar term, is a mistake.
    ("uncentred covariance",
     "double ws = w[i] * (s[i] - sbar);\n        for (int d = 0; d < D; ++d) hv->o[d] += ws * (vi[d] - vbar[d]);",
     "double ws = w[i] * s[i];\n        for (int d = 0; d < D; ++d) hv->o[d] += ws * vi[d];"),
    ("scale applied to probe", "if (s) s[i] = hv->r ? dot(hv->r, ki, D) : 0.0;",
     "if (s) s[i] = hv->r ? scale * dot(hv->r, ki, D) : 0.0;"),
    ("probe used as query", "t[i] = scale * dot(hv->q, ki, D);",
     "t[i] = scale * dot(hv->r ? hv->r : hv->q, ki, D);"),
    ("GQA modulo mapping", "int g = h / G;", "int g = h % Hkv;"),
    ("last key dropped", "for (int i = 0; i < hv->n; ++i) {\n        const double* ki",
     "for (int i = 0; i + 1 < hv->n; ++i) {\n        const double* ki"),
    ("no rescale in online update", "double alpha = exp(a->m - m_new);",
     "double alpha = 1.0;"),
    ("merge without rescale", "into->l = ai * into->l + ap * part->l;",
     "into->l = into->l + part->l;"),
    ("C accumulates e v", "a->C[d] = alpha * a->C[d] + e * s * v[d];",
     "a->C[d] = alpha * a->C[d] + e * v[d];"),
    ("b accumulates e", "a->b = alpha * a->b + e * s;", "a->b = alpha * a->b + e;"),
    ("softmax without normalisation", "for (int i = 0; i < n; ++i) w[i] /= z;",
     "for (int i = 0; i < n; ++i) w[i] /= 1.0;"),
    ("prefill sees its own key only from row 1", "hv.n = causal ? i + 1 : L;",
     "hv.n = causal ? (i > 0 ? i : 1) : L;"),
    ("prefill GQA modulo mapping",
     "size_t ko = ((size_t)b * Hkv + (size_t)(h / G)) * (size_t)L * (size_t)D;",
     "size_t ko = ((size_t)b * Hkv + (size_t)(h % Hkv)) * (size_t)L * (size_t)D;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = obuild.compile_source(str(path), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    failed = []
    for pin in pins.PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError) as e:
            failed.append(pin.__name__)
    assert failed, f"mutant '{name}' passed every pin"
