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


# (description, exact text in kda_oracle_bwd.c, replacement)
BWD_MUTANTS = [
    ("dq read from the decayed state, not the updated one",
     "const double* row = S + (size_t)i * dv;\n                    for (int j = 0; j < dv; ++j) acc += row[j] * dO[t * dv + j];",
     "const double* row = Sd + (size_t)i * dv;\n                    for (int j = 0; j < dv; ++j) acc += row[j] * dO[t * dv + j];"),
    ("read not added to the state adjoint", "row[j] += qt[i] * dO[t * dv + j];",
     "row[j] += 0.0 * qt[i] * dO[t * dv + j];"),
    ("dk misses the write term", "dkt[i] = acc;", "dkt[i] = 0.0 * acc;"),
    ("dk misses the recall term", "dkt[i] += acc;", "dkt[i] += 0.0 * acc;"),
    ("dbeta from v instead of v - p", "db += du[j] * (vt[j] - p[j]);", "db += du[j] * vt[j];"),
    ("sign of dp flipped", "dp[j] = -bt * du[j];", "dp[j] = bt * du[j];"),
    ("dv without beta", "dvt[j] = bt * du[j];", "dvt[j] = du[j];"),
    ("recall's state term dropped", "row[j] += kt[i] * dp[j];", "(void)row;"),
    ("dg from the undecayed state",
     "const double* srow = Sd + (size_t)i * dv;",
     "const double* srow = seg + (size_t)(t - t0) * st + (size_t)i * dv;"),
    ("state adjoint not decayed",
     "                const double a = exp(gt[i]);\n                for (int j = 0; j < dv; ++j) row[j] *= a;",
     "                const double a = 1.0;\n                for (int j = 0; j < dv; ++j) row[j] *= a;"),
    ("segment recomputed from the previous checkpoint",
     "memcpy(S, ck + (size_t)c * st, sizeof(double) * st);",
     "memcpy(S, ck + (size_t)(c > 0 ? c - 1 : 0) * st, sizeof(double) * st);"),
    ("dhT ignored", "if (dhT) memcpy(dS, dhT, sizeof(double) * st);",
     "if (0) memcpy(dS, dhT, sizeof(double) * st);"),
    ("transposed state index in dq",
     "for (int j = 0; j < dv; ++j) acc += row[j] * dO[t * dv + j];",
     "for (int j = 0; j < dv; ++j) acc += S[(size_t)(j % dk) * dv + (i % dv)] * dO[t * dv + j];"),
]


@pytest.mark.parametrize("desc,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_bwd_mutant_is_caught(tmp_path, desc, old, new):
    import pins_bwd
    with open(oracle.SOURCE_BWD) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation site not unique/found: {desc}"
    path = tmp_path / "mutant_bwd.c"
    path.write_text(src.replace(old, new))
    lib = oracle.compile_c(str(path), str(tmp_path / "libmutant_bwd.so"))
    orc = oracle.Oracle(oracle.build(), lib)
    caught = []
    for name, (fn, tol) in pins_bwd.ALL_PINS.items():
        try:
            err = fn(orc)
        except Exception:  # a crash or shape error also counts as caught
            err = float("inf")
        if not (err <= tol):
            caught.append(name)
    assert caught, f"no pin caught the planted mistake: {desc}"
