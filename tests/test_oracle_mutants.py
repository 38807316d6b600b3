"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of the oracle (oracle/ssa_oracle.c, or
the Case-2 plan routine of oracle/oracle.py): a dropped term, a wrong comparison, a
swapped index or operand, an off-by-one bound.  The copy is built with the oracle's own
flags and the pin file of that routine runs against it: at least one pin must fail.  An unmutated copy run the same way must pass, which checks the harness.  The
mistakes are planted in the oracle on the CPU only; nothing here touches the library.
"""

import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "ssa_oracle.c")
PY_SRC = os.path.join(ROOT, "oracle", "oracle.py")

CAP, PLAN, ATTN, MAPS, CASE2 = ("tests/test_oracle_capture.py", "tests/test_oracle_plan.py",
                                "tests/test_oracle_attn.py", "tests/test_oracle_maps.py",
                                "tests/test_oracle_case2.py")

# (name, text in ssa_oracle.c (exactly one occurrence), replacement, pin files)
MUTANTS = [
    ("box-cox: eps dropped", "double z = v + eps;", "double z = v;", CAP),
    ("true mask: t > tau instead of t >= tau", "bit = (t >= tau) ? 1 : 0;", "bit = (t > tau) ? 1 : 0;", CAP),
    ("true mask: constant row scores 0", "t = 1.0;\n", "t = 0.0;\n", CAP),
    ("true mask: row min / max over the whole row, not its causal part",
     "        for (int j = 0; j <= i; ++j) {\n            double x = (double)row[j];",
     "        for (int j = 0; j < L; ++j) {\n            double x = (double)row[j];", CAP),
    ("true mask: per-map scaling ignored", "if (scaling == 1) {\n            mn = map_mn;",
     "if (scaling == 2) {\n            mn = map_mn;", CAP),
    ("gamma: mask transposed", "num += M[(size_t)i * L + (i - r)];", "num += M[(size_t)(i - r) * L + i];", CAP),
    ("gamma: denominator off by one", "gamma_diag[r] = (double)num / (double)den;",
     "gamma_diag[r] = (double)num / (double)(den + 1);", CAP),
    ("select: diagonal ties dropped", "if (gamma_diag[r] >= mu)", "if (gamma_diag[r] > mu)", CAP),
    ("select: column ties dropped", "if (gamma_vert[c] >= mu)", "if (gamma_vert[c] > mu)", CAP),
    ("extend: diagonal r = S kept", "if (D[k] < S) ext_diag_offsets[od++] = D[k];",
     "if (D[k] <= S) ext_diag_offsets[od++] = D[k];", PLAN),
    ("extend: column c = S kept", "if (C[k] < S) ext_vert_cols[oc++] = C[k];",
     "if (C[k] <= S) ext_vert_cols[oc++] = C[k];", PLAN),
    ("plan (interval): FULL ignores the columns",
     "            int full = ((long)T * (qb + 1) <= S) && popcount256(dm) == 2 * T - 1 && cm[0] == 0 &&\n"
     "                       cm[1] == 0;",
     "            int full = ((long)T * (qb + 1) <= S) && popcount256(dm) == 2 * T - 1;", PLAN),
    ("plan (brute): FULL without the whole-block condition",
     "                int full = ((long)T * (qb + 1) <= S) && popcount256(dm)",
     "                int full = 1 && popcount256(dm)", PLAN),
    ("plan (interval): stripe count one short", "stripe_cnt[h * nqb + qb] = count_le(C, nc, (int32_t)hi_i);",
     "stripe_cnt[h * nqb + qb] = count_le(C, nc, (int32_t)hi_i - 1);", PLAN),
    # (a run boundary at a gap of exactly 128 changes nothing: the two runs' key ranges
    # touch, so the windows are the same; a gap of 129 leaves an unneeded key between them)
    ("plan (interval): offsets 129 apart taken as one run", "D[k] - D[k - 1] <= ORA_TILE",
     "D[k] - D[k - 1] <= ORA_TILE + 1", PLAN),
    ("nnz: a cell on a diagonal and a column counted twice", "total += own - shared;", "total += own;", PLAN),
    ("attention: LSE in log2", "*lse = m + log(l);", "*lse = m + log2(l);", ATTN),
    ("attention: GQA heads interleaved instead of grouped", "return kv_map ? kv_map[h] : h / (Hq / Hkv);",
     "return kv_map ? kv_map[h] : h % Hkv;", ATTN),
    ("attention: exponentials not shifted by the row max", "double p = exp(s[a] - m);",
     "double p = exp(s[a]);", ATTN),
    ("attention (rows): diagonal r = i skipped", "if (D[k] > i) continue;", "if (D[k] >= i) continue;", ATTN),
    ("attention (dense): a column's first cell missing",
     "for (long i = C[k]; i < S; ++i) Mt[(size_t)i * S + C[k]] = 1;",
     "for (long i = C[k] + 1; i < S; ++i) Mt[(size_t)i * S + C[k]] = 1;", ATTN),
    ("case 2: the true-mask block added to the patterns instead of replacing them",
     "Mt[(size_t)i * S + j] = Bh[(size_t)i * Lb + j] ? 1 : 0;",
     "Mt[(size_t)i * S + j] |= Bh[(size_t)i * Lb + j] ? 1 : 0;", CASE2),
    ("maps: scale dropped", "s[j] = scale * dot;", "s[j] = dot;", MAPS),
    ("maps: query and key rows swapped",
     "bf16_bits_to_double(q[(size_t)i * d + c]) * bf16_bits_to_double(k[(size_t)j * d + c])",
     "bf16_bits_to_double(q[(size_t)j * d + c]) * bf16_bits_to_double(k[(size_t)i * d + c])", MAPS),
    ("maps: exponentials not shifted by the row max", "s[j] = exp(s[j] - mx);", "s[j] = exp(s[j]);", MAPS),
    ("maps: mean over samples without 1/B", "row[j] += s[j] / sum / B;", "row[j] += s[j] / sum;", MAPS),
    ("maps: softmax sum starts at 1", "double sum = 0.0;", "double sum = 1.0;", MAPS),
    ("box-cox: general lambda takes the reciprocal power", "return (pow(z, lambda) - 1.0) / lambda;",
     "return (pow(z, 1.0 / lambda) - 1.0) / lambda;", CAP),
    ("true mask: map min / max over the whole map, not its causal part",
     "    for (int i = 0; i < L; ++i)\n        for (int j = 0; j <= i; ++j) {\n            double x = (double)map[",
     "    for (int i = 0; i < L; ++i)\n        for (int j = 0; j < L; ++j) {\n            double x = (double)map[", CAP),
    ("gamma: column mask transposed", "num += M[(size_t)i * L + c];", "num += M[(size_t)c * L + i];", CAP),
    ("capture: diagonal offsets advanced by the column count", "diag_ptr[m + 1] = diag_ptr[m] + cnt_d[m];",
     "diag_ptr[m + 1] = diag_ptr[m] + cnt_v[m];", CAP),
    ("plan (brute): a window of column cells only is listed", "if (j <= i && isD[i - j] && !isC[j])",
     "if (j <= i && isD[i - j])", PLAN),
    ("plan (interval): rows past S make a window listed", "if (nrows - 1 < il_hi) il_hi = nrows - 1;", "", PLAN),
    ("plan (brute): stripe count one long", "count_le(C, nc, last_row)", "count_le(C, nc, last_row + 1)", PLAN),
    ("plan (interval): diagonal mask shifted by one", "long base = lo - key0 - (T - 1);",
     "long base = lo - key0 - T;", PLAN),
    ("nnz: shared cells counted up to S", "if ((long long)C[k] + D[q] < S) ++shared;",
     "if ((long long)C[k] + D[q] <= S) ++shared;", PLAN),
    ("attention (rows): column c = i skipped", "if (C[k] > i) continue;", "if (C[k] >= i) continue;", ATTN),
    ("attention (dense): a diagonal's first cell missing", "for (long i = D[k]; i < S; ++i)",
     "for (long i = D[k] + 1; i < S; ++i)", ATTN),
    ("attention: scale dropped", "s[a] = scale * dot;", "s[a] = dot;", ATTN),
    ("attention: output not normalised", "for (int k = 0; k < d; ++k) o[k] /= l;", "", ATTN),
    ("attention: empty row gives LSE 0", "*lse = -INFINITY;", "*lse = 0.0;", ATTN),
    ("case 2: the block's diagonal cells kept from the patterns",
     "for (int j = 0; j <= i; ++j) Mt[(size_t)i * S + j] = Bh", "for (int j = 0; j < i; ++j) Mt[(size_t)i * S + j] = Bh",
     CASE2),
    ("plan items: stripe count one short", "if (stripe_cnt) stripe_cnt[a] = count_le(C, nc, (int32_t)hi_i);",
     "if (stripe_cnt) stripe_cnt[a] = count_le(C, nc, (int32_t)hi_i - 1);", PLAN),
    ("true mask: a constant map under per-map scaling not scored 1", "if (mx == mn) {",
     "if (mx == mn && scaling == 0) {", CAP),
    ("attention (rows): a cell on a diagonal and a column taken twice", "if (!mark[C[k]]) {", "if (1) {", ATTN),
    ("extend: duplicate offsets accepted", "if (k > 0 && a[k] <= a[k - 1]) return 0;",
     "if (k > 0 && a[k] < a[k - 1]) return 0;", PLAN),
    ("extend: negative offsets accepted", "if (a[k] < 0) return 0;", "", PLAN),
    ("maps: row max never taken", "if (s[j] > mx) mx = s[j];", "if (s[j] > mx) mx = 0.0;", MAPS),
    ("attention: an explicit GQA map ignored", "return kv_map ? kv_map[h] : h / (Hq / Hkv);",
     "return h / (Hq / Hkv);", ATTN),
    ("attention: LSE without the row max", "*lse = m + log(l);", "*lse = log(l);", ATTN),
    ("select: the one-cell diagonal r = L - 1 never considered",
     "    for (int r = 0; r < L; ++r)\n        if (gamma_diag[r] >= mu)",
     "    for (int r = 0; r < L - 1; ++r)\n        if (gamma_diag[r] >= mu)", CAP),
    ("select: the one-cell column c = L - 1 never considered",
     "    for (int c = 0; c < L; ++c)\n        if (gamma_vert[c] >= mu)",
     "    for (int c = 0; c < L - 1; ++c)\n        if (gamma_vert[c] >= mu)", CAP),
    ("gamma: a diagonal's first cell skipped", "for (int i = r; i < L; ++i) {", "for (int i = r + 1; i < L; ++i) {", CAP),
    ("maps: the diagonal entry left out of the mean", "for (int j = 0; j <= i; ++j) row[j] += s[j] / sum / B;",
     "for (int j = 0; j < i; ++j) row[j] += s[j] / sum / B;", MAPS),
    ("attention: keys taken for values", "const uint16_t *vj = V + (size_t)J[a] * d;",
     "const uint16_t *vj = K + (size_t)J[a] * d;", ATTN),
    ("gamma: column denominator off by one", "gamma_vert[c] = (double)num / (double)den;",
     "gamma_vert[c] = (double)num / (double)(den + 1);", CAP),
]

# Mistakes in the Case-2 plan routine (Python, over the C routines' lists).
PY_MUTANTS = [
    ("case 2 plan: past row L the columns are dropped", "cell[il, c] = (i - j) in D or j in Cs",
     "cell[il, c] = (i - j) in D", CASE2),
    ("case 2 plan: bitmap blocks keep their stripe counts", "                stripe[it] = 0\n", "", CASE2),
    ("case 2 plan: slots of a head overlap", "slot = h * slots + qb * (qb + 1) // 2 + kb",
     "slot = h * slots + qb * qb // 2 + kb", CASE2),
    ("case 2 plan: bitmap blocks counted from L even when S < L",
     "nL = (min(L, S) + TILE - 1) // TILE", "nL = (L + TILE - 1) // TILE", CASE2),
    ("wrapper: capture passes mu for tau and tau for mu",
     "lib().ora_capture(_p(maps), n, Ln, lam, tau, mu, eps,", "lib().ora_capture(_p(maps), n, Ln, lam, mu, tau, eps,",
     CAP),
    ("wrapper: true mask passes tau for eps and eps for tau",
     "lib().ora_true_mask(_p(amap), Ln, lam, eps, tau, _p(M))", "lib().ora_true_mask(_p(amap), Ln, lam, tau, eps, _p(M))",
     CAP),
    ("wrapper: capture under per-map scaling scales per row", "mu, eps, SCALINGS[scaling], _p(dp)", "mu, eps, 0, _p(dp)",
     CAP),
    ("case 2 plan: empty bitmap tiles listed", "                    if not cell.any():\n                        continue\n",
     "", CASE2),
]

# The copy is a package of its own (oracle/__init__.py, oracle.py, the built C library)
# placed first on the path, so the pins import it instead of the repository's oracle.
_DRIVER = (
    "import sys\n"
    "sys.path.insert(0, sys.argv[1])\n"
    "sys.path.insert(0, sys.argv[2])\n"
    "from oracle import oracle as o\n"
    "assert o.__file__.startswith(sys.argv[2])\n"
    "o.LIB = sys.argv[3]\n"
    "o.build = lambda force=False: o.LIB\n"
    "import pytest\n"
    "sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', '-m', 'not gpu'] + sys.argv[4].split(',')))\n"
)


def _build_and_run(c_text, py_text, workdir, tests):
    pkg = os.path.join(workdir, "oracle")
    os.makedirs(pkg, exist_ok=True)
    for name, text in (("ssa_oracle.c", c_text), ("oracle.py", py_text), ("__init__.py", "")):
        with open(os.path.join(pkg, name), "w") as f:
            f.write(text)
    so_path = os.path.join(pkg, "libssa_oracle.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                    "-o", so_path, os.path.join(pkg, "ssa_oracle.c"), "-lm"], check=True)
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run([sys.executable, "-c", _DRIVER, ROOT, workdir, so_path, tests], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return p.returncode, p.stdout[-1500:] + p.stderr[-1500:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = tmp_path_factory.mktemp("mutants")
    src, py = open(SRC).read(), open(PY_SRC).read()
    jobs = {"unmutated": (src, py, ",".join((CAP, PLAN, ATTN, MAPS, CASE2)))}
    for name, old, new, tests in MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
        jobs[name] = (src.replace(old, new), py, tests)
    for name, old, new, tests in PY_MUTANTS:
        assert py.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
        jobs[name] = (src, py.replace(old, new), tests)
    with cf.ThreadPoolExecutor(max_workers=8) as ex:
        futs = {name: ex.submit(_build_and_run, c, p, str(base / f"m{k}"), tests)
                for k, (name, (c, p, tests)) in enumerate(jobs.items())}
        return {name: f.result() for name, f in futs.items()}


def test_unmutated_copy_passes_every_pin(outcomes):
    rc, log = outcomes["unmutated"]
    assert rc == 0, log


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS + PY_MUTANTS])
def test_planted_mistake_fails_a_pin(outcomes, name):
    rc, log = outcomes[name]
    assert rc == 1, f"{name}: pins {'passed' if rc == 0 else f'ended with code {rc}'}\n{log}"
