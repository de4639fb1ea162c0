// Lloyd-Max codebook of the Lemma-1 coordinate law, on the host in fp64.
//
// TurboQuant review (Jump2Paper, arXiv 2504.19874):
//   Lemma 1: a coordinate of a uniform point on S^{d-1} has density
//            f_X(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1 - x^2)^((d-3)/2).
//   Theorem 1 (MSE): the MSE problem splits into d copies of 1-D continuous k-means on
//            f_X, D_mse = d C(f_X, b); codebooks for b = 1..8 are precomputed by
//            Max-Lloyd optimisation (experiment setup table).
//
// Method here: the Lloyd-Max conditions (boundaries at midpoints of neighbouring
// centroids, centroids at the conditional means of their cells) are solved by Lloyd
// iteration from a spread start and then polished with Newton's method on the
// boundary equations t_k = (c_k + c_{k+1})/2, whose Jacobian is tridiagonal. Cell
// integrals use the substitution x = sin(theta), under which
//     f_X(x) dx = C_d cos(theta)^(d-2) d(theta),
// a smooth integrand for every d >= 2, integrated by composite Gauss-Legendre
// quadrature. The first moment uses its antiderivative -C_d (1-x^2)^((d-1)/2)/(d-1).
#include <algorithm>
#include <cmath>
#include <vector>

#include "internal.h"

namespace tq {
namespace {

constexpr int kGL = 20;  // Gauss-Legendre nodes per panel

struct GaussLegendre {
    double x[kGL], w[kGL];
    GaussLegendre() {
        // Nodes are the roots of P_n, found by Newton's method from Chebyshev guesses.
        const int n = kGL;
        for (int i = 0; i < n; ++i) {
            double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
            double dp = 1.0;
            for (int it = 0; it < 100; ++it) {
                double p0 = 1.0, p1 = z;
                for (int k = 2; k <= n; ++k) {
                    double pk = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = pk;
                }
                dp = n * (z * p1 - p0) / (z * z - 1.0);
                double dz = p1 / dp;
                z -= dz;
                if (std::fabs(dz) < 1e-16) break;
            }
            {
                double p0 = 1.0, p1 = z;
                for (int k = 2; k <= n; ++k) {
                    double pk = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = pk;
                }
                dp = n * (z * p1 - p0) / (z * z - 1.0);
            }
            x[i] = z;
            w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
        }
    }
};

const GaussLegendre& gl() {
    static GaussLegendre g;
    return g;
}

struct Law {
    int d;
    double logC;     // log C_d
    double panel;    // theta panel width
    explicit Law(int dim) : d(dim) {
        logC = std::lgamma(d / 2.0) - std::lgamma((d - 1) / 2.0) - 0.5 * std::log(M_PI);
        panel = std::min(0.05, 0.3 / std::sqrt((double)d));
    }
    double pdf(double x) const {
        double u = 1.0 - x * x;
        if (u <= 0.0) return (d == 3) ? std::exp(logC) : 0.0;
        return std::exp(logC + 0.5 * (d - 3) * std::log(u));
    }
    // integrals over [a, b] of x^k f_X(x) for k = 0 and 2 (theta substitution)
    void moments02(double a, double b, double* m0, double* m2) const {
        double ta = std::asin(std::max(-1.0, std::min(1.0, a)));
        double tb = std::asin(std::max(-1.0, std::min(1.0, b)));
        double s0 = 0.0, s2 = 0.0;
        if (tb > ta) {
            int np = std::max(1, (int)std::ceil((tb - ta) / panel));
            double h = (tb - ta) / np;
            const GaussLegendre& g = gl();
            for (int p = 0; p < np; ++p) {
                double mid = ta + (p + 0.5) * h;
                for (int i = 0; i < kGL; ++i) {
                    double th = mid + 0.5 * h * g.x[i];
                    double cth = std::cos(th);
                    double wgt = (d == 2) ? 1.0 : (cth > 0.0 ? std::exp((d - 2) * std::log(cth)) : 0.0);
                    wgt *= 0.5 * h * g.w[i];
                    double sn = std::sin(th);
                    s0 += wgt;
                    s2 += wgt * sn * sn;
                }
            }
        }
        double C = std::exp(logC);
        *m0 = C * s0;
        *m2 = C * s2;
    }
    double m1(double a, double b) const {
        auto G = [&](double x) {
            double u = std::max(0.0, 1.0 - x * x);
            return -std::exp(logC + 0.5 * (d - 1) * std::log(u)) / (d - 1);
        };
        return G(b) - G(a);
    }
};

// Centroids of the cells given by L-1 boundaries; also cell masses.
void centroids_from_bounds(const Law& law, int L, const double* t, double* c, double* mass) {
    for (int i = 0; i < L; ++i) {
        double a = (i == 0) ? -1.0 : t[i - 1];
        double b = (i == L - 1) ? 1.0 : t[i];
        double m0, m2;
        law.moments02(a, b, &m0, &m2);
        mass[i] = m0;
        c[i] = (m0 > 0.0) ? law.m1(a, b) / m0 : 0.5 * (a + b);
    }
}

}  // namespace

int build_codebook(int d, int b, double* c_out, double* t_out, double* dmse_out) {
    if (d < 2 || b < 0 || b > 8) return TQ_EINVAL;
    const int L = 1 << b;
    Law law(d);
    std::vector<double> c(L), t(std::max(1, L - 1)), mass(L);
    if (L == 1) {
        c[0] = 0.0;
    } else {
        // Spread start: centroids evenly over +-2.5 standard deviations (sd = 1/sqrt(d)).
        const double sd = 1.0 / std::sqrt((double)d);
        for (int i = 0; i < L; ++i) c[i] = std::min(0.999, 2.5 * sd) * (2.0 * (i + 0.5) / L - 1.0);
        // Lloyd iterations until the centroids move little.
        for (int it = 0; it < 20000; ++it) {
            for (int k = 0; k < L - 1; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
            std::vector<double> cn(L);
            centroids_from_bounds(law, L, t.data(), cn.data(), mass.data());
            double mv = 0.0;
            for (int i = 0; i < L; ++i) mv = std::max(mv, std::fabs(cn[i] - c[i]));
            c.swap(cn);
            if (mv < 1e-9 * sd) break;
        }
        // Newton on G_k(t) = t_k - (c_k(t) + c_{k+1}(t))/2 = 0, k = 0..L-2.
        const int n = L - 1;
        std::vector<double> lo(n), di(n), up(n), rhs(n);
        for (int it = 0; it < 60; ++it) {
            for (int k = 0; k < n; ++k) t[k] = (it == 0) ? 0.5 * (c[k] + c[k + 1]) : t[k];
            centroids_from_bounds(law, L, t.data(), c.data(), mass.data());
            double gmax = 0.0;
            for (int k = 0; k < n; ++k) {
                // cell k = [t_{k-1}, t_k], cell k+1 = [t_k, t_{k+1}]
                double fk = law.pdf(t[k]);
                double dck_dtk = fk * (t[k] - c[k]) / mass[k];            // upper edge of cell k
                double dck1_dtk = fk * (c[k + 1] - t[k]) / mass[k + 1];   // lower edge of cell k+1
                di[k] = 1.0 - 0.5 * (dck_dtk + dck1_dtk);
                lo[k] = (k > 0) ? -0.5 * law.pdf(t[k - 1]) * (c[k] - t[k - 1]) / mass[k] : 0.0;
                up[k] = (k < n - 1) ? -0.5 * law.pdf(t[k + 1]) * (t[k + 1] - c[k + 1]) / mass[k + 1] : 0.0;
                rhs[k] = -(t[k] - 0.5 * (c[k] + c[k + 1]));
                gmax = std::max(gmax, std::fabs(rhs[k]));
            }
            if (gmax < 1e-17) break;
            // Thomas algorithm for the tridiagonal system.
            for (int k = 1; k < n; ++k) {
                double m = lo[k] / di[k - 1];
                di[k] -= m * up[k - 1];
                rhs[k] -= m * rhs[k - 1];
            }
            rhs[n - 1] /= di[n - 1];
            for (int k = n - 2; k >= 0; --k) rhs[k] = (rhs[k] - up[k] * rhs[k + 1]) / di[k];
            double step = 0.0;
            for (int k = 0; k < n; ++k) {
                t[k] += rhs[k];
                step = std::max(step, std::fabs(rhs[k]));
            }
            if (step < 1e-16) {
                centroids_from_bounds(law, L, t.data(), c.data(), mass.data());
                break;
            }
        }
        // f_X is even: store the antisymmetric part so that 0 is exactly a boundary.
        for (int i = 0; i < L / 2; ++i) {
            double v = 0.5 * (c[L - 1 - i] - c[i]);
            c[i] = -v;
            c[L - 1 - i] = v;
        }
        for (int k = 0; k < L - 1; ++k) t[k] = 0.5 * (c[k] + c[k + 1]);
    }
    // D_mse = d * sum over cells of the integral of (x - c_i)^2 f_X.
    double D = 0.0;
    for (int i = 0; i < L; ++i) {
        double a = (i == 0) ? -1.0 : t[i - 1];
        double bb = (i == L - 1) ? 1.0 : t[i];
        double m0, m2;
        law.moments02(a, bb, &m0, &m2);
        D += m2 - 2.0 * c[i] * law.m1(a, bb) + c[i] * c[i] * m0;
    }
    if (c_out) std::copy(c.begin(), c.end(), c_out);
    if (t_out && L > 1) std::copy(t.begin(), t.begin() + (L - 1), t_out);
    if (dmse_out) *dmse_out = d * D;
    return TQ_OK;
}

// Probabilities of the L cells of the boundaries t[0..L-2] under f_X (Lemma 1), computed for
// the lower half and mirrored (the law is even).
void index_law(int d, int L, const double* t, double* p) {
    Law law(d);
    for (int i = 0; i < L / 2; ++i) {
        double a = (i == 0) ? -1.0 : t[i - 1];
        double b = t[i];
        double m0, m2;
        law.moments02(a, b, &m0, &m2);
        p[i] = m0;
        p[L - 1 - i] = m0;
    }
    if (L == 1) p[0] = 1.0;
}

}  // namespace tq
