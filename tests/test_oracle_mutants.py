"""Plant plausible mistakes in copies of the oracle's C file (on the CPU) and
check that the pins catch every one of them."""
import os
import shutil

import pytest

import oracle
import pins

# (description, exact text in kda_oracle.c, replacement)
MUTANTS = [
    ("decay not applied", "row[j] *= a;", "row[j] *= 1.0;"),
    ("decay on value axis", "const double a = exp(gt[i]);", "const double a = exp(gt[i < dv ? i : 0]);\n            (void)0;"),
    ("recall from undecayed state (decay after recall)",
     "            for (int j = 0; j < dv; ++j) row[j] *= a;\n        }\n        /* recall p = S^T k */",
     "        }\n        /* recall p = S^T k */"),
    ("beta dropped", "u[j] = bt * (vt[j] - p[j]);", "u[j] = (vt[j] - p[j]);"),
    ("sign of the erase flipped", "u[j] = bt * (vt[j] - p[j]);", "u[j] = bt * (vt[j] + p[j]);"),
    ("erase dropped (plain linear attention)", "u[j] = bt * (vt[j] - p[j]);", "u[j] = bt * vt[j];"),
    ("recall with q instead of k", "const double ki = kt[i];\n            const double* row = S + (size_t)i * dv;\n            for (int j = 0; j < dv; ++j) p[j] += row[j] * ki;",
     "const double ki = qt[i];\n            const double* row = S + (size_t)i * dv;\n            for (int j = 0; j < dv; ++j) p[j] += row[j] * ki;"),
    ("output read before the write", "        /* read the updated state */", "        for (int i = 0; i < dk; ++i) for (int j = 0; j < dv; ++j) S[(size_t)i*dv+j] -= kt[i]*u[j];\n        /* read the updated state */"),
    ("transposed state index in the read", "for (int j = 0; j < dv; ++j) ot[j] += row[j] * qi;",
     "for (int j = 0; j < dv; ++j) ot[j] += S[(size_t)j * dv + (i % dv)] * qi;"),
    ("h0 ignored", "if (h0 != S) memcpy(S, h0, sizeof(double) * (size_t)dk * dv);",
     "memset(S, 0, sizeof(double) * (size_t)dk * dv);"),
    ("off-by-one token in g", "const double* gt = g + t * dk;", "const double* gt = g + (t > 0 ? t - 1 : 0) * dk;"),
]


@pytest.mark.parametrize("desc,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, desc, old, new):
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not unique/found: {desc}"
    mutated = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = oracle.compile_c(str(path), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for name, (fn, tol) in pins.ALL_PINS.items():
        try:
            err = fn(orc)
        except Exception:  # a crash or shape error also counts as caught
            err = float("inf")
        if not (err <= tol):
            caught.append(name)
    assert caught, f"no pin caught the planted mistake: {desc}"
