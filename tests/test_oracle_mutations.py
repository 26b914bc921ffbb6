"""Plant plausible mistakes in a copy of the oracle and check the pins catch
each one (CPU only).  The mistakes are planted in a temporary copy of the C
source; the committed oracle is never modified."""
import os
import tempfile

import pytest

import oracle
from tests import pins

# (name, exact text in avq_oracle.c, replacement)
MUTANTS = [
    ("child-not-strict-vs-parent", "if (C > 0 && d_child < d_best) return c_star;",
     "if (C > 0 && d_child <= d_best) return c_star;"),
    ("child-tie-to-last", "if (dc < d_child) { /* where", "if (dc <= d_child) { /* where"),
    ("parent-tie-to-last", "if (dm < d_best) {", "if (dm <= d_best) {"),
    ("child-count-dropped", "ns[code] += 1;\n      }\n      assign", "\n      }\n      assign"),
    ("aggregate-child-count-dropped", "ns[code] += 1;\n      }\n    }\n  }\n}",
     "\n      }\n    }\n  }\n}"),
    ("aggregate-child-sum-to-parent",
     "vs[(size_t)code * d + t] += v[t];\n        ns[code] += 1;\n      }\n    }\n  }\n}",
     "vs[(size_t)a * d + t] += v[t];\n        ns[code] += 1;\n      }\n    }\n  }\n}"),
    ("aggregate-parent-of-child-wrong",
     "int32_t a = code < M0 ? code : (code - M0) / C;\n      const double* v",
     "int32_t a = code < M0 ? code : (code - M0) % C;\n      const double* v"),
    ("d3-grandchild-not-strict-vs-child", "if (d_g < d_child) return M0 + M0 * C + c * C + g_star;",
     "if (d_g <= d_child) return M0 + M0 * C + c * C + g_star;"),
    ("d3-grandchild-tie-to-last", "if (dg < d_g) { /* first strict minimum */",
     "if (dg <= d_g) { /* first strict minimum */"),
    ("d3-grandchild-count-dropped", "ns[code] += 1;\n      }\n      assign", "\n      }\n      assign"),
    ("d3-child-of-grandchild-wrong", "else { child = M0 + (code - M0 - M1) / C; a = (child - M0) / C; }",
     "else { child = M0 + (code - M0 - M1) % C; a = (child - M0) / C; }"),
    ("d3-grandchild-index-transposed", "gc_h + ((size_t)cc * C + g) * d", "gc_h + ((size_t)g * M1 + cc) * d"),
    ("d3-child-importance-no-count", "w2[u] += exp(sc[(size_t)r * nc + u] - m[r]) * n_u / z[r];",
     "w2[u] += exp(sc[(size_t)r * nc + u] - m[r]) / z[r];"),
    ("d3-grandchild-dA-sign", "double dA = ns[x_g] > 0 ? exp(sg[g] - m[r]) - Ac : 0.0;",
     "double dA = ns[x_g] > 0 ? Ac - exp(sg[g] - m[r]) : 0.0;"),
    ("d3-child-mean-divisor", "scm /= C;", "scm /= (C + 1);"),
    ("d3-top-p2-tie-to-higher-code", "(w[j] == w[best] && code[j] < code[best])",
     "(w[j] == w[best] && code[j] > code[best])"),
    ("d3-no-rescale-grandchildren", "      double f = exp(m[r] - mp);\n      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] *= f;\n      z[r] *= f;\n      m[r] = mp;\n      /* the child's logit",
     "      double f = 1.0;\n      for (int t = 0; t < d; ++t) x[(size_t)r * d + t] *= f;\n      z[r] *= f;\n      m[r] = mp;\n      /* the child's logit"),
    ("child-index-transposed", "ch_h + ((size_t)a * C + c) * d", "ch_h + ((size_t)c * M0 + a) * d"),
    ("dA-sign", "exp(sc[c] - m[r]) - Ap", "Ap - exp(sc[c] - m[r])"),
    ("no-rescale", "double f = exp(m[r] - mp);", "double f = 1.0;"),
    ("max-includes-empty-child", "if (nc[c] > 0 && sc[c] > mp) mp = sc[c];", "if (sc[c] > mp) mp = sc[c];"),
    ("dA-not-masked", "double dA = nc[c] > 0 ? exp(sc[c] - m[r]) - Ap : 0.0;",
     "double dA = exp(sc[c] - m[r]) - Ap;"),
    ("A-not-masked", "ns[j] > 0 ? exp(s[(size_t)r * M0 + j] - m[r]) : 0.0;",
     "exp(s[(size_t)r * M0 + j] - m[r]);"),
    ("importance-no-denominator", "w[j] += A[(size_t)r * M0 + j] * ns[j] / z[r];",
     "w[j] += A[(size_t)r * M0 + j] * ns[j];"),
    ("importance-no-count", "w[j] += A[(size_t)r * M0 + j] * ns[j] / z[r];",
     "w[j] += A[(size_t)r * M0 + j] / z[r];"),
    ("topp-tie-to-higher", "if (best < 0 || w[j] > w[best]) best = j;",
     "if (best < 0 || w[j] >= w[best]) best = j;"),
    ("child-logit-unscaled", "sc[c] = scale * dot(q, ch_p + (size_t)c * d, d);",
     "sc[c] = dot(q, ch_p + (size_t)c * d, d);"),
    ("parent-mean-wrong-divisor", "sp /= C;", "sp /= (C + 1);"),
    ("z-missing-count", "z[r] += a * ns[j];", "z[r] += a;"),
    ("child-z-missing-count", "z[r] += dA * nc[c];", "z[r] += dA;"),
    ("tiled-seen-codes-not-keys", "nseen += ns[j];", "nseen += 1.0;"),
    ("tiled-extrapolation-inverted", "ns[j] / (ntot / nseen * zpart[r]);",
     "ns[j] / (nseen / ntot * zpart[r]);"),
    ("tiled-exact-denominator", "ns[j] / (ntot / nseen * zpart[r]);", "ns[j] / z[r];"),
    ("tiled-partial-z-unweighted", "zpart[r] += A[(size_t)r * M0 + j] * ns[j];",
     "zpart[r] += A[(size_t)r * M0 + j];"),
    ("ema-weights-swapped", "lambda * Nst[(size_t)h * Mt + x] + (1.0 - lambda) * n;",
     "(1.0 - lambda) * Nst[(size_t)h * Mt + x] + lambda * n;"),
    ("projection-not-mass-weighted", "shift = nc > 0.0 ? delta / (nc * sigma) : 0.0;",
     "shift = nc > 0.0 ? delta / massive : 0.0;"),
    ("projection-residual-sign", "double delta = -C * cp[t];", "double delta = C * cp[t];"),
    ("massless-child-moves", "shift = nc > 0.0 ? delta / (nc * sigma) : 0.0;",
     "shift = nc > 0.0 ? delta / (nc * sigma) : delta / C;"),
]


# The depth-3 functions sit after this line of the oracle; "d3-" mistakes are
# planted there, the others before it (some statements appear in both).
DEPTH3_MARK = " * Depth-3 tree: the"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    src = open(oracle.SRC).read()
    cut = src.index(DEPTH3_MARK)
    head, tail = src[:cut], src[cut:]
    if name.startswith("d3-"):
        assert tail.count(old) == 1, f"mutation site not unique or missing: {name}"
        mutated = head + tail.replace(old, new)
    else:
        assert head.count(old) == 1, f"mutation site not unique or missing: {name}"
        mutated = head.replace(old, new) + tail
    with tempfile.TemporaryDirectory() as tmp:
        msrc = os.path.join(tmp, "mutant.c")
        with open(msrc, "w") as f:
            f.write(mutated)
        lib = oracle.build(src=msrc, out=os.path.join(tmp, "libmutant.so"), force=True)
        orc = oracle.Oracle(lib)
        caught = []
        # the pins of the mutant's section; the first one that fails is enough
        section = [p for p in pins.ALL_PINS if p.__name__.startswith("pin3_") == name.startswith("d3-")]
        for pin in section:
            try:
                with __import__("numpy").errstate(all="ignore"):
                    pin(orc)
            except (AssertionError, ValueError, IndexError, FloatingPointError) as e:  # noqa: PERF203
                caught.append((pin.__name__, type(e).__name__))
                break
        assert caught, f"no pin caught mutant {name}"
