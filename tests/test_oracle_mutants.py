"""The oracle's pins must catch plausible mistakes in the oracle itself.

C side: each case plants one mistake in a copy of the oracle's C sources (on the CPU, in a
temporary directory), builds the copy with the oracle's own compiler flags, and runs the
pin suite (tests/test_oracle_pins.py) against it through FK_ORACLE_LIB.

Python side: each case plants one mistake in a copy of the oracle package (the steps it
strings together: rounding between iterations, the tie window, the bf16 cast) and runs a
copy of the pin suite that imports it.

The pin suite must fail for every mistake.  The unchanged copies must pass: that shows the
harness itself works.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")
SOURCES = ("lloyd_oracle.c", "ivf_search_oracle.c")

# (name, source file, text to replace (exactly once), replacement)
MUTANTS = [
    ("assign_tie_to_highest_index", "lloyd_oracle.c",
     "if (s < best) {", "if (s <= best) {"),
    ("distance_sign", "lloyd_oracle.c",
     "double t = x[j] - c[j];", "double t = x[j] + c[j];"),
    ("second_distance_not_tracked", "lloyd_oracle.c",
     "} else if (s < second) {", "} else if (s < best) {"),
    ("objective_not_squared", "lloyd_oracle.c",
     "per[i] = sqdist(X + i * (int64_t)d, C + (int64_t)labels[i] * d, d);",
     "per[i] = sqrt(sqdist(X + i * (int64_t)d, C + (int64_t)labels[i] * d, d));"),
    ("mean_count_off_by_one", "lloyd_oracle.c",
     "sums[o] / (double)cnt[k]", "sums[o] / (double)(cnt[k] + 1)"),
    ("empty_cluster_zeroed", "lloyd_oracle.c",
     ": C_old[o];", ": 0.0;"),
    ("csr_unstable_order", "lloyd_oracle.c",
     "for (int64_t i = 0; i < n; ++i) perm[cursor[labels[i]]++] = (int32_t)i;",
     "for (int64_t i = n - 1; i >= 0; --i) perm[cursor[labels[i]]++] = (int32_t)i;"),
    ("normalize_by_squared_norm", "lloyd_oracle.c",
     "x[j] = x[j] / nrm;", "x[j] = x[j] / s;"),
    ("normalize_no_zero_guard", "lloyd_oracle.c",
     "if (nrm == 0.0) nrm = 1.0;", ""),
    ("search_tie_to_higher_index", "ivf_search_oracle.c",
     "return da < db || (da == db && ia < ib);", "return da < db || (da == db && ia > ib);"),
    ("search_probes_farthest_cells", "ivf_search_oracle.c",
     "keep_smallest(pd, pi, &plen, nprobe, sq_dist(qv, C + (int64_t)c * d, d), c);",
     "keep_smallest(pd, pi, &plen, nprobe, -sq_dist(qv, C + (int64_t)c * d, d), c);"),
    ("search_scans_unprobed_cells", "ivf_search_oracle.c",
     "if (probed[labels[i]])", "if (!probed[labels[i]])"),
    ("search_pads_with_zero_distance", "ivf_search_oracle.c",
     "dist[q * k + t] = t < klen ? kd[t] : INFINITY;",
     "dist[q * k + t] = t < klen ? kd[t] : 0.0;"),
    ("search_pads_ids_with_zero", "ivf_search_oracle.c",
     "ids[q * k + t] = t < klen ? ki[t] : -1;", "ids[q * k + t] = t < klen ? ki[t] : 0;"),
    ("csr_offsets_not_accumulated", "lloyd_oracle.c",
     "offsets[k + 1] = offsets[k] + counts[k];", "offsets[k + 1] = counts[k];"),
    ("distance_in_expanded_form", "lloyd_oracle.c",
     "        double t = x[j] - c[j];\n        s += t * t;\n",
     "        s += x[j] * x[j] + c[j] * c[j] - 2.0 * x[j] * c[j];\n"),
    ("assign_skips_last_centroid", "lloyd_oracle.c",
     "for (int k = 0; k < K; ++k) {\n            double s = sqdist(",
     "for (int k = 0; k < K - 1; ++k) {\n            double s = sqdist("),
    ("objective_against_first_centroid", "lloyd_oracle.c",
     "per[i] = sqdist(X + i * (int64_t)d, C + (int64_t)labels[i] * d, d);",
     "per[i] = sqdist(X + i * (int64_t)d, C, d);"),
    ("normalize_skips_last_column", "lloyd_oracle.c",
     "for (int j = 0; j < d; ++j) s += x[j] * x[j];",
     "for (int j = 0; j < d - 1; ++j) s += x[j] * x[j];"),
    ("search_drops_last_probed_cell", "ivf_search_oracle.c",
     "for (int t = 0; t < plen; ++t) probed[pi[t]] = 1;",
     "for (int t = 0; t + 1 < plen; ++t) probed[pi[t]] = 1;"),
    ("search_distance_in_expanded_form", "ivf_search_oracle.c",
     "        const double t = a[j] - b[j];\n        s += t * t;\n",
     "        s += a[j] * a[j] + b[j] * b[j] - 2.0 * a[j] * b[j];\n"),
]


def _build_copy(tmp_path, mutant=None):
    srcs = []
    for name in SOURCES:
        with open(os.path.join(ORACLE, name)) as f:
            text = f.read()
        if mutant is not None and mutant[1] == name:
            assert text.count(mutant[2]) == 1, f"{mutant[0]}: the planted text must occur once"
            text = text.replace(mutant[2], mutant[3])
        path = tmp_path / name
        path.write_text(text)
        srcs.append(str(path))
    lib = tmp_path / "liboracle_copy.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                    "-fno-fast-math", "-ffp-contract=off", *srcs, "-o", str(lib), "-lm"],
                   check=True)
    return str(lib)


def _run_pins(lib):
    env = dict(os.environ, FK_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x",
                           "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def _run_all(cases, job):
    """Run job(case) for every case at once (each is its own subprocess); map name ->
    result, the unchanged copy under None."""
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        futs = {(c[0] if c else None): ex.submit(job, c) for c in [None, *cases]}
        return {name: f.result() for name, f in futs.items()}


@pytest.fixture(scope="module")
def c_results(tmp_path_factory):
    return _run_all(MUTANTS, lambda m: _run_pins(_build_copy(tmp_path_factory.mktemp("c"), m)))


def test_unchanged_copy_passes_the_pins(c_results):
    r = c_results[None]
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(c_results, mutant):
    r = c_results[mutant[0]]
    # 1: tests ran and at least one failed (not a collection or usage error)
    assert r.returncode == 1, f"{mutant[0]} survived the pins:\n{r.stdout[-2000:]}"


# (name, text in oracle/__init__.py to replace (exactly once), replacement)
PY_MUTANTS = [
    ("lloyd_means_not_rounded_to_fp32",
     "Cnew = round_f32(update(Xd, labels, Cm))", "Cnew = update(Xd, labels, Cm)"),
    ("lloyd_bf16_assign_unrounded",
     'Cu = round_bf16(Cm) if precision == "bf16" else Cm', "Cu = Cm"),
    ("lloyd_objective_against_master",
     "J = objective(Xd, Cu, labels)", "J = objective(Xd, Cm, labels)"),
    ("lloyd_cosine_leaves_centroids", "        Cm = normalize_rows(Cm)\n", ""),
    ("tie_window_uses_smallest_centroid",
     "(C * C).sum(axis=1).max()", "(C * C).sum(axis=1).min()"),
    ("bf16_rounding_truncates",
     "return t.to(torch.bfloat16).double().numpy()",
     "return (t.view(torch.int32) & -65536).view(torch.float32).double().numpy()"),
]


def _python_copy(tmp_path, mutant=None):
    shutil.copytree(ORACLE, tmp_path / "oracle",
                    ignore=shutil.ignore_patterns("_build", "__pycache__"))
    tests = tmp_path / "tests"
    tests.mkdir()
    for name in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), tests / name)
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), tests / "golden")
    if mutant is not None:
        init = tmp_path / "oracle" / "__init__.py"
        text = init.read_text()
        assert text.count(mutant[1]) == 1, f"{mutant[0]}: the planted text must occur once"
        init.write_text(text.replace(mutant[1], mutant[2]))
    return str(tmp_path)


def _run_copied_pins(cwd):
    import oracle
    env = dict(os.environ, FK_ORACLE_LIB=oracle.build.build(), OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x",
                           "-q", "-p", "no:cacheprovider", "-m", "not gpu"],
                          cwd=cwd, env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def py_results(tmp_path_factory):
    return _run_all(PY_MUTANTS,
                    lambda m: _run_copied_pins(_python_copy(tmp_path_factory.mktemp("py"), m)))


def test_unchanged_python_copy_passes_the_pins(py_results):
    r = py_results[None]
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_planted_python_mistake_fails_a_pin(py_results, mutant):
    r = py_results[mutant[0]]
    assert r.returncode == 1, f"{mutant[0]} survived the pins:\n{r.stdout[-2000:]}"
