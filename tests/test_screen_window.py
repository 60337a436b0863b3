"""The screened route's window, checked on the CPU against emulated arithmetic.

The single-product screening pass accumulates v~ = ||c||^2 - 2 RN_bf16(x) . RN_bf16(c) in
fp32 (the squared norm folded in as an exact three-part bf16 split of its fp32 rounding),
and screen_window() promises E = W / 2 >= |v~ - v| for the exact v = ||c||^2 - 2 x.c.  The
tensor core's internal accumulation order and rounding are not documented, so a host
program (built with nvcc, no GPU needed) emulates several: one rounding per 16-product
MMA step, one per product, round-to-nearest or toward zero, the norm step first or last.
Every emulation must stay inside E, on random, scaled, aligned, unit-norm and adversarial
data at the dimensions the route serves (the adversarial case, where every operand rounds
the same way, must come within a factor 2 of E, so the bound is not loose by more); and
the exact argmin, and every column of the exact top m (the search's coarse pass, m = 1, 8,
32), must lie within W of the m-th smallest screened value."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "exact_lloyd_means_b200", "csrc")

PROGRAM = r"""
#include "fk_common.cuh"
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <random>
#include <vector>
using namespace fk;

static float bf16_rn(float f) {  // round to nearest even, 8 significant bits
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}
static float to_f32(double v, bool rz) {  // one rounding of an exact value to fp32
    float f = static_cast<float>(v);
    if (rz && std::fabs(static_cast<double>(f)) > std::fabs(v))
        f = std::nextafter(f, 0.0f);
    return f;
}

int main() {
    std::mt19937_64 rng(12345);
    std::normal_distribution<double> nd(0.0, 1.0);
    std::uniform_real_distribution<double> ud(-1.0, 1.0);
    const int dims[] = {256, 384, 768, 1024};
    const double scales[] = {1e-3, 1.0, 37.0, 1e3};
    long long checked = 0, bad = 0, argmin_bad = 0;
    double worst = 0.0, worst_adv = 0.0;  // largest |v~ - v| / E: all kinds, adversarial
    for (int d : dims) {
        const int dp = static_cast<int>(round_up(d, kBK));
        for (double scale : scales) {
            // kinds: normal, uniform, nearly parallel, unit norm, and adversarial: every
            // operand just under a bf16 half-unit above a power of two, so all roundings
            // shrink it by 0.98 u and, with the centroids parallel to x, every product
            // errs the same way (the operand term of the bound is nearly reached)
            for (int kind = 0; kind < 5; ++kind) {
                const int K = 48;
                std::vector<float> x(d), C(static_cast<size_t>(K) * d);
                const double p2 = std::ldexp(1.0, std::ilogb(scale));
                for (int j = 0; j < d; ++j) {
                    if (kind == 4) {
                        const double m = (1.0 + 0.49 * std::ldexp(1.0, -7)) *
                                         std::ldexp(1.0, static_cast<int>(rng() % 5) - 2);
                        x[j] = static_cast<float>(p2 * ((rng() & 1) ? m : -m));
                    } else {
                        x[j] = static_cast<float>(scale * (kind == 1 ? ud(rng) : nd(rng)));
                    }
                }
                for (int k = 0; k < K; ++k)
                    for (int j = 0; j < d; ++j) {
                        float &cv = C[static_cast<size_t>(k) * d + j];
                        if (kind == 4) {
                            cv = x[j] * static_cast<float>(1 << (k % 4));
                            continue;
                        }
                        double v = kind == 1 ? ud(rng) : nd(rng);
                        if (kind == 2) v = x[j] / scale + 0.01 * v;  // nearly parallel to x
                        cv = static_cast<float>(scale * v);
                    }
                if (kind == 3) {  // cosine data: unit rows
                    auto unit = [&](float *r) {
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) s += double(r[j]) * r[j];
                        const double n = std::sqrt(s);
                        for (int j = 0; j < d; ++j) r[j] = static_cast<float>(r[j] / n);
                    };
                    unit(x.data());
                    for (int k = 0; k < K; ++k) unit(&C[static_cast<size_t>(k) * d]);
                }
                double xs = 0.0;
                for (int j = 0; j < d; ++j) xs += double(x[j]) * x[j];
                const float xnorm2 = static_cast<float>(xs);
                std::vector<float> cn(K);
                float cmax2 = 0.f;
                for (int k = 0; k < K; ++k) {
                    double s = 0.0;
                    for (int j = 0; j < d; ++j) {
                        const double c = C[static_cast<size_t>(k) * d + j];
                        s += c * c;
                    }
                    cn[k] = static_cast<float>(s);
                    cmax2 = std::fmax(cmax2, cn[k]);
                }
                const float W = screen_window(xnorm2, cmax2, dp);
                const double E = 0.5 * W;
                for (int mode = 0; mode < 8; ++mode) {
                    const bool per_product = mode & 1, rz = (mode >> 1) & 1,
                               norm_last = (mode >> 2) & 1;
                    std::vector<double> vt(K), ve(K);
                    for (int k = 0; k < K; ++k) {
                        const float *c = &C[static_cast<size_t>(k) * d];
                        double dot = 0.0, exact_n = 0.0;
                        for (int j = 0; j < d; ++j) {
                            dot += double(x[j]) * c[j];
                            exact_n += double(c[j]) * c[j];
                        }
                        ve[k] = exact_n - 2.0 * dot;
                        // the norm step: exact bf16 split of the fp32 norm, added exactly
                        const float h = bf16_rn(cn[k]), m = bf16_rn(cn[k] - h),
                                    l = bf16_rn(cn[k] - h - m);
                        const double nstep = double(h) + m + l;
                        float acc = 0.f;
                        if (!norm_last) acc = to_f32(double(acc) + nstep, rz);
                        for (int j0 = 0; j0 < dp; j0 += 16) {
                            double chunk = 0.0;
                            for (int j = j0; j < j0 + 16; ++j) {
                                const double p = j < d ? double(bf16_rn(x[j])) *
                                                             (-2.0 * bf16_rn(c[j]))
                                                       : 0.0;
                                if (per_product) acc = to_f32(double(acc) + p, rz);
                                else chunk += p;  // 16 bf16 products: exact in fp64
                            }
                            if (!per_product) acc = to_f32(double(acc) + chunk, rz);
                        }
                        if (norm_last) acc = to_f32(double(acc) + nstep, rz);
                        vt[k] = acc;
                        const double err = std::fabs(vt[k] - ve[k]);
                        worst = std::fmax(worst, err / E);
                        if (kind == 4) worst_adv = std::fmax(worst_adv, err / E);
                        ++checked;
                        if (err > E) {
                            if (bad < 10)
                                std::printf("FAIL d=%d scale=%g kind=%d mode=%d k=%d: |v~-v|=%g"
                                            " E=%g\n", d, scale, kind, mode, k, err, E);
                            ++bad;
                        }
                    }
                    int ke = 0, kt = 0;
                    for (int k = 1; k < K; ++k) {
                        if (ve[k] < ve[ke]) ke = k;
                        if (vt[k] < vt[kt]) kt = k;
                    }
                    if (vt[ke] > vt[kt] + W) ++argmin_bad;
                    // the search's coarse pass: every column of the exact top m lies within
                    // W of the m-th smallest screened value
                    for (int m : {1, 8, 32}) {
                        std::vector<int> ord(K);
                        for (int t = 0; t < K; ++t) ord[t] = t;
                        std::stable_sort(ord.begin(), ord.end(),
                                         [&](int a, int b) { return ve[a] < ve[b]; });
                        std::vector<double> srt(vt);
                        std::sort(srt.begin(), srt.end());
                        for (int r = 0; r < m; ++r)
                            if (vt[ord[r]] > srt[m - 1] + W) ++argmin_bad;
                    }
                }
            }
        }
    }
    std::printf("%lld screened values, worst |v~ - v| / E = %.3f (adversarial %.3f), "
                "%lld outside E, %lld argmin / top-m columns outside W\n", checked, worst, worst_adv, bad,
                argmin_bad);
    // the adversarial inputs come close to the bound: a bound half as wide would fail
    return (bad == 0 && argmin_bad == 0 && worst_adv > 0.5) ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc is needed to build the check")
def test_screen_window_bounds_emulated_screening(tmp_path):
    src = tmp_path / "window.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "window"
    subprocess.run(["nvcc", "-std=c++17", "-O2", f"-I{CSRC}", str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    print(r.stdout)
    assert r.returncode == 0, r.stdout


FINE_PROGRAM = r"""
#include "fk_common.cuh"
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <random>
#include <vector>
using namespace fk;

static float bf16_rn(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}
static float to_f32(double v, bool rz) {
    float f = static_cast<float>(v);
    if (rz && std::fabs(static_cast<double>(f)) > std::fabs(v)) f = std::nextafter(f, 0.0f);
    return f;
}

int main() {
    std::mt19937_64 rng(777);
    std::normal_distribution<double> nd(0.0, 1.0);
    std::uniform_real_distribution<double> pos(0.0, 1.0);
    const int dims[] = {64, 128, 768, 1024};
    const double scales[] = {1e-3, 1.0, 1e3};
    long long checked = 0, bad = 0, topk_bad = 0;
    double worst = 0.0, worst_adv = 0.0;
    for (int d : dims) {
        const int dp = static_cast<int>(round_up(d, kBK));
        float ce_dot, ce_round;
        fine_window_coeffs(dp, &ce_dot, &ce_round);
        for (double scale : scales) {
            // kinds: normal; near duplicates of the query; adversarial: every coordinate
            // positive, so all partial sums grow and one-sided roundings pile up
            for (int kind = 0; kind < 3; ++kind) {
                const int M = 64, k = 10;
                std::vector<float> q(d), X(static_cast<size_t>(M) * d);
                for (int j = 0; j < d; ++j)
                    q[j] = static_cast<float>(scale * (kind == 2 ? pos(rng) : nd(rng)));
                for (int i = 0; i < M; ++i)
                    for (int j = 0; j < d; ++j) {
                        double v = kind == 2 ? pos(rng) * scale : nd(rng) * scale;
                        if (kind == 1) v = q[j] + 1e-3 * scale * nd(rng);
                        X[static_cast<size_t>(i) * d + j] = static_cast<float>(v);
                    }
                double qn = 0.0;
                for (int j = 0; j < d; ++j) qn += double(q[j]) * q[j];
                std::vector<double> xn(M, 0.0);
                double xmax2 = 0.0;
                for (int i = 0; i < M; ++i) {
                    for (int j = 0; j < d; ++j) {
                        const double x = X[static_cast<size_t>(i) * d + j];
                        xn[i] += x * x;
                    }
                    xmax2 = std::max(xmax2, xn[i]);
                }
                for (int mode = 0; mode < 4; ++mode) {
                    const bool per_product = mode & 1, rz = (mode >> 1) & 1;
                    std::vector<double> st(M), se(M);
                    for (int i = 0; i < M; ++i) {
                        const float *x = &X[static_cast<size_t>(i) * d];
                        double s = 0.0;
                        for (int j = 0; j < d; ++j) {
                            const double t = double(q[j]) - x[j];
                            s += t * t;
                        }
                        se[i] = s;
                        float acc = 0.f;
                        for (int j0 = 0; j0 < dp; j0 += 16) {
                            for (int prod = 0; prod < 3; ++prod) {  // hi.hi, hi.lo, lo.hi
                                double chunk = 0.0;
                                for (int j = j0; j < j0 + 16 && j < d; ++j) {
                                    const float qh = bf16_rn(q[j]), ql = bf16_rn(q[j] - qh);
                                    const float xh = bf16_rn(x[j]), xl = bf16_rn(x[j] - xh);
                                    const double p = prod == 0 ? double(qh) * xh
                                                     : prod == 1 ? double(qh) * xl
                                                                 : double(ql) * xh;
                                    if (per_product) acc = to_f32(double(acc) + p, rz);
                                    else chunk += p;
                                }
                                if (!per_product) acc = to_f32(double(acc) + chunk, rz);
                            }
                        }
                        st[i] = static_cast<float>(std::fma(-2.0, double(acc), qn + xn[i]));
                        const double E = ce_dot * std::sqrt(qn * xn[i]) + ce_round * (qn + xn[i]);
                        const double err = std::fabs(st[i] - se[i]);
                        worst = std::max(worst, err / E);
                        if (kind == 2) worst_adv = std::max(worst_adv, err / E);
                        ++checked;
                        if (err > E) {
                            if (bad < 10)
                                std::printf("FAIL d=%d scale=%g kind=%d mode=%d: |s~-s|=%g E=%g\n",
                                            d, scale, kind, mode, err, E);
                            ++bad;
                        }
                    }
                    // every point of the exact top-k lies within 2E (E at the largest
                    // point norm) of the k-th smallest screened value
                    std::vector<int> ord(M);
                    for (int i = 0; i < M; ++i) ord[i] = i;
                    std::stable_sort(ord.begin(), ord.end(),
                                     [&](int a, int b) { return se[a] < se[b]; });
                    std::vector<double> sorted_t(st);
                    std::sort(sorted_t.begin(), sorted_t.end());
                    const double Eq = ce_dot * std::sqrt(qn * xmax2) + ce_round * (qn + xmax2);
                    for (int r = 0; r < k; ++r)
                        if (st[ord[r]] > sorted_t[k - 1] + 2.0 * Eq) ++topk_bad;
                }
            }
        }
    }
    std::printf("%lld screened distances, worst |s~ - s| / E = %.3f (adversarial %.3f), "
                "%lld outside E, %lld top-k points outside 2E\n", checked, worst, worst_adv,
                bad, topk_bad);
    return (bad == 0 && topk_bad == 0) ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc is needed to build the check")
def test_search_fine_window_bounds_emulated_three_product_screening(tmp_path):
    """The IVF-Flat search's fine window (fine_window_coeffs): s~ = ||q||^2 + ||x||^2 - 2 q.x~
    rounded to fp32, with q.x~ the three bf16 products of the hi/lo splits accumulated in
    fp32 (per MMA step or per product, to nearest or toward zero), stays within E of the
    exact squared distance, and the exact top-k lies within 2E of the k-th screened value."""
    src = tmp_path / "fine_window.cu"
    src.write_text(FINE_PROGRAM)
    exe = tmp_path / "fine_window"
    subprocess.run(["nvcc", "-std=c++17", "-O2", f"-I{CSRC}", str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    print(r.stdout)
    assert r.returncode == 0, r.stdout


THREE_PROGRAM = r"""
#include "fk_common.cuh"
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <random>
#include <vector>
using namespace fk;

static float bf16_rn(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    u &= 0xffff0000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}
static float to_f32(double v, bool rz) {
    float f = static_cast<float>(v);
    if (rz && std::fabs(static_cast<double>(f)) > std::fabs(v)) f = std::nextafter(f, 0.0f);
    return f;
}

int main() {
    std::mt19937_64 rng(4242);
    std::normal_distribution<double> nd(0.0, 1.0);
    const int dims[] = {8, 64, 128, 768, 1024};
    const double scales[] = {1e-3, 1.0, 1e3};
    const double tau = 1e-4;  // the parity rule's tie window: tau * (||x||^2 + max ||c||^2)
    long long checked = 0, bad = 0;
    double worst = 0.0, worst_open = 0.0;  // asserted models; per-product truncation, d > 768
    for (int d : dims) {
        const int dp = static_cast<int>(round_up(d, kBK));
        for (double scale : scales) {
            // kinds: normal; nearly parallel to x; adversarial: every coordinate a value
            // whose hi/lo split leaves the largest residual, centroids parallel to x
            for (int kind = 0; kind < 3; ++kind) {
                const int K = 32;
                std::vector<float> x(d), C(static_cast<size_t>(K) * d);
                const double p2 = std::ldexp(1.0, std::ilogb(scale));
                for (int j = 0; j < d; ++j) {
                    if (kind == 2) {
                        // 1 + 0.49 2^-7 + 0.49 2^-15: RN keeps 1 in hi, 0.49 2^-7 in lo,
                        // and 0.49 2^-15 (about 2^-16 relative) is left over
                        const double m = 1.0 + 0.49 * std::ldexp(1.0, -7) +
                                         0.49 * std::ldexp(1.0, -15);
                        x[j] = static_cast<float>(p2 * m * ((rng() & 1) ? 1.0 : -1.0));
                    } else {
                        x[j] = static_cast<float>(scale * nd(rng));
                    }
                }
                for (int k = 0; k < K; ++k)
                    for (int j = 0; j < d; ++j) {
                        float &cv = C[static_cast<size_t>(k) * d + j];
                        if (kind == 2) cv = x[j] * static_cast<float>(1 << (k % 4));
                        else if (kind == 1) cv = static_cast<float>(x[j] + 0.01 * scale * nd(rng));
                        else cv = static_cast<float>(scale * nd(rng));
                    }
                double xs = 0.0;
                for (int j = 0; j < d; ++j) xs += double(x[j]) * x[j];
                std::vector<float> cn(K);
                double cmax2 = 0.0;
                for (int k = 0; k < K; ++k) {
                    double s = 0.0;
                    for (int j = 0; j < d; ++j) {
                        const double c = C[static_cast<size_t>(k) * d + j];
                        s += c * c;
                    }
                    cn[k] = static_cast<float>(s);
                    cmax2 = std::max(cmax2, s);
                }
                const double half_window = 0.5 * tau * (xs + cmax2);
                for (int mode = 0; mode < 4; ++mode) {
                    const bool per_product = mode & 1, rz = (mode >> 1) & 1;
                    for (int k = 0; k < K; ++k) {
                        const float *c = &C[static_cast<size_t>(k) * d];
                        double dot = 0.0, exact_n = 0.0;
                        for (int j = 0; j < d; ++j) {
                            dot += double(x[j]) * c[j];
                            exact_n += double(c[j]) * c[j];
                        }
                        const double v = exact_n - 2.0 * dot;
                        const float h = bf16_rn(cn[k]), m = bf16_rn(cn[k] - h),
                                    l = bf16_rn(cn[k] - h - m);
                        float acc = to_f32(double(h) + m + l, rz);
                        for (int j0 = 0; j0 < dp; j0 += 16) {
                            for (int prod = 0; prod < 3; ++prod) {  // xh.ch, xl.ch, xh.cl
                                double chunk = 0.0;
                                for (int j = j0; j < j0 + 16 && j < d; ++j) {
                                    const float xh = bf16_rn(x[j]), xl = bf16_rn(x[j] - xh);
                                    const float ch = bf16_rn(c[j]), cl = bf16_rn(c[j] - ch);
                                    const double p = prod == 0 ? double(xh) * (-2.0 * ch)
                                                     : prod == 1 ? double(xl) * (-2.0 * ch)
                                                                 : double(xh) * (-2.0 * cl);
                                    if (per_product) acc = to_f32(double(acc) + p, rz);
                                    else chunk += p;
                                }
                                if (!per_product) acc = to_f32(double(acc) + chunk, rz);
                            }
                        }
                        const double err = std::fabs(double(acc) - v);
                        // every model is asserted wherever the library lets the three
                        // products decide a label (padded depth <= kThreeProductMaxDp);
                        // beyond it the library never does, so the error is only printed
                        if (dp > kThreeProductMaxDp) {
                            worst_open = std::max(worst_open, err / half_window);
                            continue;
                        }
                        worst = std::max(worst, err / half_window);
                        ++checked;
                        if (err >= half_window) {
                            if (bad < 10)
                                std::printf("FAIL d=%d scale=%g kind=%d mode=%d: err=%g "
                                            "half window=%g\n", d, scale, kind, mode, err,
                                            half_window);
                            ++bad;
                        }
                    }
                }
            }
        }
    }
    std::printf("%lld three-product values up to d_p = %d, worst error / half tie window = "
                "%.3f, %lld at or beyond it; beyond d_p = %d (never used there) the worst model "
                "reaches %.3f\n", checked, kThreeProductMaxDp, worst, bad, kThreeProductMaxDp,
                worst_open);
    return bad == 0 ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc is needed to build the check")
def test_three_product_assignment_stays_inside_half_the_tie_window(tmp_path):
    """The three-product route (fp32 points on bf16 tensor cores: xh.ch + xl.ch + xh.cl,
    the norm folded in first, as the kernel does) has an error below half the parity
    rule's tie window, so every point outside the window keeps its exact label.  Emulated
    as above, with normal, nearly parallel and adversarial data (split residuals as large
    as they get).  Every model (one rounding per MMA step or per product, to nearest or
    toward zero) is asserted at every depth up to the library's kThreeProductMaxDp (768),
    the deepest at which the three products still decide labels.  Beyond it (d = 1024
    here) truncation after every single product leaves the half window (about 1.5x); the
    library then sends every row to the screened route with exact fp64 re-ranking and an
    exact scan for overflowing rows, so that figure is printed, not asserted."""
    src = tmp_path / "three.cu"
    src.write_text(THREE_PROGRAM)
    exe = tmp_path / "three"
    subprocess.run(["nvcc", "-std=c++17", "-O2", f"-I{CSRC}", str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    print(r.stdout)
    assert r.returncode == 0, r.stdout
