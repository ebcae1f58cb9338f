"""Plant plausible mistakes in a scratch copy of the oracle's C source (on the CPU) and
check that every one of them fails at least one pin.  The real oracle is untouched."""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "csa_oracle.c")

# (name, text in csa_oracle.c, replacement)
MUTATIONS = [
    ("rope_sign", "x[a + 1] = xa * s + xb * c;", "x[a + 1] = -xa * s + xb * c;"),
    ("rope_pair_index", "int64_t a = D - R + 2 * i;", "int64_t a = D - R + i;"),
    ("rope_theta", "pow(base, -2.0 * (double)i / (double)R)", "pow(base, -1.0 * (double)i / (double)R)"),
    ("no_derotation", "rope_rotate(o, -tq, D, R, base);", "(void)0;"),
    ("compress_no_overlap", "int64_t lo = overlap ? (j - 1) * m : j * m;", "int64_t lo = j * m;"),
    ("compress_window_end", "int64_t hi = (j + 1) * m;", "int64_t hi = (j + 1) * m - 1;"),
    ("compress_unweighted_den", "den += e;", "den += 1.0;"),
    ("visibility_off_by_one", "int64_t n = (t + 1) / m;", "int64_t n = (t + 2) / m;"),
    ("indexer_no_relu", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    ("indexer_no_weight", "acc += w[(b * n + i) * HI + h] * relu;", "acc += relu;"),
    ("topk_ascending", "if (a->s > b->s) return -1;\n    if (a->s < b->s) return 1;",
     "if (a->s < b->s) return -1;\n    if (a->s > b->s) return 1;"),
    ("topk_tie_order", "return (a->j < b->j) ? -1 : (a->j > b->j);", "return (a->j > b->j) ? -1 : (a->j < b->j);"),
    ("sink_dropped", "double Z = (sink[h] == -INFINITY) ? 0.0 : exp(sink[h] - M);", "double Z = 0.0;"),
    ("no_scale", "logit[x] = scale * dot;", "logit[x] = dot;"),
    ("window_short", "if (s > t - W && s <= t) {", "if (s > t - W + 1 && s <= t) {"),
    ("entry_position", "kpos[nk] = (double)j * (double)m;\n                        ++nk;\n                    }\n                } else {",
     "kpos[nk] = (double)(j + 1) * (double)m;\n                        ++nk;\n                    }\n                } else {"),
    ("hca_entry_position", "kpos[nk] = (double)j * (double)m;\n                        ++nk;\n                    }\n                }\n                attend_query",
     "kpos[nk] = (double)(j + 1) * (double)m - 1.0;\n                        ++nk;\n                    }\n                }\n                attend_query"),
    ("value_unrotated", "o[d] += p * krot[x * D + d];", "o[d] += p * keys[x][d];"),
    ("step_closes_early", "if (fill + 1 < m) continue;", "if (fill + 2 < m) continue;"),
    ("step_overlap_not_kept", "n_ovl[b] = m;", "n_ovl[b] = 0;"),
    ("step_overlap_not_pooled", "n = n_ovl[b];\n", "n = 0;\n"),
    ("step_unweighted_norm", "z += wgt;", "z += 1.0;"),
]

# Entry-position readings are choices the pages do not fix; the pins cannot catch them.
UNPINNED = {"entry_position", "hca_entry_position"}


def _build_mutant(tmpdir, name, old, new):
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, "mutation anchor for %s must occur exactly once" % name
    path_c = os.path.join(tmpdir, name + ".c")
    path_so = os.path.join(tmpdir, name + ".so")
    with open(path_c, "w") as f:
        f.write(text.replace(old, new))
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o",
                           path_so, path_c, "-lm"])
    return path_so


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, old, new):
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, name, old, new)
        failed = []
        with oracle.using(so):
            for pin in ALL_PINS:
                try:
                    pin()
                except (AssertionError, ValueError):
                    failed.append(pin.__name__)
        if name in UNPINNED:
            pytest.skip("reading not fixed by the pages (parity unpinned); pins failing: %s" % failed)
        assert failed, "mutation %s passed every pin" % name
