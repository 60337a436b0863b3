"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case plants one mistake in a copy of the oracle's C sources (on the CPU, in a temporary
directory), builds the copy with the oracle's own compiler flags, and runs the pin suite
(tests/test_oracle_pins.py) against it through FK_ORACLE_LIB.  The pin suite must fail.
The unchanged copy, built the same way, must pass: that shows the harness itself works.
"""
import os
import subprocess
import sys

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


def test_unchanged_copy_passes_the_pins(tmp_path):
    r = _run_pins(_build_copy(tmp_path))
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(tmp_path, mutant):
    r = _run_pins(_build_copy(tmp_path, mutant))
    # 1: tests ran and at least one failed (not a collection or usage error)
    assert r.returncode == 1, f"{mutant[0]} survived the pins:\n{r.stdout[-2000:]}"
