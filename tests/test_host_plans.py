"""Host-side planning of the library, checked on the CPU: the radix sort's digits and
tiles, the update's chunks, and the Lloyd and IVF-Flat search workspace layouts
(exact_lloyd_means_b200/csrc/fk_common.cuh).  A small host-only program includes the
header, is built with nvcc (no GPU needed) and checks the invariants the kernels rely on
over a grid of shapes."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_lloyd_means_b200", "csrc")

PROGRAM = r"""
#include "fk_common.cuh"
#include <cstdio>
using namespace fk;

static int fails = 0;
#define CHECK(c)                                                                       \
    do {                                                                               \
        if (!(c)) {                                                                    \
            if (fails < 20)                                                            \
                std::printf("FAIL %s: N=%lld K=%d d=%d\n", #c, (long long)N, K, d);    \
            ++fails;                                                                   \
        }                                                                              \
    } while (0)

int main() {
    const long long Ns[] = {1, 2, 255, 256, 1023, 1024, 1025, 65536, 150001, 1 << 20,
                            4194304, 4194305, 10000000, 16000000, 100000000, 2147483646LL};
    const int Ks[] = {1, 2, 3, 255, 256, 257, 300, 1024, 4096, 32768, 65535, 65536, 65537,
                      1 << 20};
    const int ds[] = {4, 8, 64, 100, 128, 129, 256, 768, 1032};
    int cases = 0;
    for (long long N : Ns) {
        for (int K : Ks) {
            if (K > N) continue;
            int d = 0;
            const SortPlan p = sort_plan(N, K);
            // digits cover exactly the bits of the largest key, with no empty pass
            CHECK(K == 1 ? p.nbits == 0 : (1LL << p.nbits) >= K && (1LL << (p.nbits - 1)) < K);
            CHECK(p.bits <= kSortMaxBits && p.passes * p.bits >= p.nbits);
            CHECK(p.passes == 0 || (p.passes - 1) * p.bits < p.nbits);
            // tiles cover [0, N) with no empty block; the last tile's end fits 32 bits
            const long long tile = (long long)kSortThreads * p.items;
            CHECK(p.items == (N <= kSortSmallN ? kSortItemsSmall : kSortItems));
            CHECK(p.nblocks * tile >= N && (p.nblocks - 1) * tile < N);
            CHECK(p.nblocks * tile <= 0xffffffffLL);
            for (int dd : ds) {
                d = dd;
                const UpdPlan u = upd_plan(N, d);
                CHECK(u.rows >= kUpdMinRows && u.rows <= kUpdMaxRows);
                CHECK((u.rows & (u.rows - 1)) == 0);  // combine spans stay powers of two
                CHECK(u.nwarps * u.rows >= N && (u.nwarps - 1) * u.rows < N);
                CHECK(u.ncolblk * 128 >= d && (u.ncolblk - 1) * 128 < d);
                CHECK(u.dcov == u.ncolblk * 128);
                if (N > 20000000 && d > 128) continue;  // layouts beyond any real device
                for (int dt = 0; dt < 2; ++dt) {
                    const fk_dtype dtype = dt ? FK_BF16 : FK_F32;
                    const WsLayout L = ws_layout(N, d, K, dtype, FK_COSINE);
                    const size_t offs[] = {L.err, L.obj, L.xn, L.xs, L.xnorm, L.cs, L.cn,
                                           L.caug, L.cused, L.calt, L.keys0, L.keys1,
                                           L.vals0, L.vals1, L.hist, L.dtot, L.pieces,
                                           L.pkeys, L.piecesb, L.pkeysb, L.jpart, L.jdev,
                                           L.cnt, L.off, L.cand, L.nfb, L.fbrows, L.fblab,
                                           L.xsfb, L.cmax2};
                    const int n = sizeof(offs) / sizeof(offs[0]);
                    for (int i = 0; i < n; ++i) CHECK(offs[i] % 256 == 0);
                    for (int i = 1; i < n; ++i) CHECK(offs[i] > offs[i - 1]);
                    CHECK(L.total > offs[n - 1]);
                    // the sort's histogram and keys, and the combine's buffers, fit
                    const long long bins = 1LL << (p.bits > 0 ? p.bits : 1);
                    CHECK(L.dtot - L.hist >= sizeof(uint32_t) * bins * p.nblocks);
                    CHECK(L.keys1 - L.keys0 >= sizeof(int32_t) * N);
                    CHECK(L.pkeys - L.pieces >= sizeof(double) * u.nwarps * 2 * u.dcov);
                    CHECK(L.dp % kBK == 0 && L.dp >= d && L.Kp % kBN == 0 && L.Kp >= K);
                    ++cases;
                }
            }
        }
    }
    // IVF-Flat search: the workspace for every (queries, cells, probes, k) shape
    const long long nqs[] = {1, 31, 32, 1000, 10000, 100000};
    const int nlists[] = {1, 7, 256, 1024, 4096, 16384};
    const int probes[] = {1, 4, 32, 128, 256, 1024};
    const int kk[] = {1, 10, 16, 32};
    for (long long nq : nqs) {
        for (int nlist : nlists) {
            for (int nprobe : probes) {
                if (nprobe > nlist) continue;
                for (int k : kk) {
                    long long N = nq;
                    int K = nlist, d = 768;
                    const SearchLayout S = search_layout(nq, d, nlist, nprobe, k);
                    const size_t offs[] = {S.err, S.qn, S.cn, S.D, S.probes, S.keys0, S.keys1,
                                           S.vals0, S.vals1, S.hist, S.dtot, S.psorted, S.poff,
                                           S.items, S.nitems, S.Ld, S.Li, S.qplanes, S.qxn,
                                           S.cplanes, S.ccn, S.cused, S.caug, S.cmax2, S.Sv,
                                           S.Sp, S.Slost, S.fb};
                    const int n = sizeof(offs) / sizeof(offs[0]);
                    for (int i = 0; i < n; ++i) CHECK(offs[i] % 256 == 0);
                    for (int i = 1; i < n; ++i) CHECK(offs[i] > offs[i - 1]);
                    CHECK(S.total > offs[n - 1]);
                    CHECK(S.P == nq * nprobe);
                    // a coarse batch is a multiple of 32 queries or all of them, and its
                    // distances (fp64) or screened values (fp32 rows of Kp) fit
                    CHECK(S.qbatch == nq || S.qbatch % 32 == 0);
                    CHECK(S.qbatch >= 1 && S.qbatch <= nq);
                    CHECK(S.probes - S.D >= sizeof(double) * S.qbatch * nlist);
                    CHECK(S.probes - S.D >= sizeof(float) * S.qbatch * S.Kp);
                    const long long bins = 1LL << (S.sp.bits > 0 ? S.sp.bits : 1);
                    CHECK(S.dtot - S.hist >= sizeof(uint32_t) * bins * S.sp.nblocks);
                    // every pair fits the items: at most one partial item per cell
                    CHECK(S.max_items >= nlist + (S.P + kSearchPairsPerItem - 1) /
                                                     kSearchPairsPerItem);
                    CHECK(S.nitems - S.items >= sizeof(int32_t) * 2 * S.max_items);
                    CHECK(S.Li - S.Ld >= sizeof(double) * S.P * k);
                    ++cases;
                }
            }
        }
    }
    // the one-launch combine: for every cluster range of level-1 units [a0, a1], each level
    // it does not finish at writes its partials into a buffer large enough (level 2 into
    // the first, then alternating), and its shared memory fits an SM
    {
        long long N = 0;
        int K = 0, d = 128;
        CHECK(upd_wide_smem(kUpdWideUnits) + 3 * 1024 <= 228 * 1024);
        const long long units[] = {1, 2, 15, 16, 17, 255, 256, 257, 1000, 1024, 2047, 2048};
        for (long long U : units) {
            N = U;
            const int l2 = upd_wide_l2cap(U), l3 = upd_wide_l3cap(U);
            for (long long lo = 0; lo < U; ++lo) {
                for (long long hi = lo; hi < U; hi += (U > 300 ? 7 : 1)) {
                    long long a0 = lo, a1 = hi;
                    bool first = true;
                    while (a0 != a1) {
                        const long long g0 = a0 / kUpdGroup, g1 = a1 / kUpdGroup;
                        if (g0 == g1) break;  // finished at this level: nothing stored
                        CHECK(g1 - g0 + 1 <= (first ? l2 : l3));
                        a0 = g0;
                        a1 = g1;
                        first = !first;
                    }
                }
            }
            ++cases;
        }
    }
    std::printf("%d layouts checked, %d failures\n", cases, fails);
    return fails == 0 ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc is needed to build the check")
def test_sort_update_and_workspace_plans(tmp_path):
    src = tmp_path / "plans.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "plans"
    subprocess.run(["nvcc", "-std=c++17", "-O1", f"-I{CSRC}", str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    print(r.stdout)
    assert r.returncode == 0, r.stdout
