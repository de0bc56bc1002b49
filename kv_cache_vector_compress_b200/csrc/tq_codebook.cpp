// tq_codebook.cpp -- host-side Lloyd-Max codebook for the N(0, 1/dim) coordinate law.
//
// The pages build the codebook with build_lloyd_max_codebook(dim, bits), returning
// (boundaries, centroids), by numerical integration of the coordinate law of a rotated
// unit vector, which they give as N(0, 1/d) ("turboquant-pytorch", nav.superapi.store,
// 核心 API and 限制与注意事项; atskills.one, "Why Random Rotation?").  For a Gaussian the
// centroid condition has a closed form, so this solves Lloyd's conditions directly:
//   t_k = (c_{k-1} + c_k) / 2                     (cell edges: nearest neighbour)
//   c_k = (phi(t_k) - phi(t_{k+1})) / (Phi(t_{k+1}) - Phi(t_k))   (cell means)
// Because the law is symmetric only the positive half is iterated (the middle edge is 0).
//
// lloyd_max_beta: the same conditions under the exact law of one coordinate of a random unit
// vector in R^dim, density proportional to (1 - y^2)^a with a = (dim - 3) / 2 ("TurboQuant er nå
// tilgjengelig som Python-bibliotek", jansverre.net, "Hva er TurboQuant, kort fortalt?": a
// concentrated Beta law).  The first moment of a cell has a closed form,
//   int_l^h y (1 - y^2)^a dy = ((1 - l^2)^(a+1) - (1 - h^2)^(a+1)) / (2 (a + 1)),
// and the mass comes from a table of F(y) = int_0^y (1 - s^2)^a ds on 2^16 steps of [0, 1]
// (two-point Gauss rule per step), read with cubic Hermite interpolation (F' is the density).
#include <cmath>
#include <cstring>
#include <vector>

#include "tq_internal.cuh"

namespace tq {

namespace {

double gauss_density(double t) { return std::exp(-0.5 * t * t) * 0.3989422804014327; }
// P(Z > t) for t >= 0, from erfc (no cancellation in the tail)
double gauss_tail(double t) { return 0.5 * std::erfc(t * 0.7071067811865476); }

}  // namespace

int lloyd_max_gaussian(int dim, int bits, double *bounds, double *cents) {
    if (dim < 1 || bits < 1 || bits > 4) return -1;
    const int K = 1 << bits, H = K / 2;  // H positive centroids
    double pos[8], edge[9];
    // start from the means of H equal-probability slices of the positive half-line
    for (int k = 0; k < H; ++k) pos[k] = 0.4 + 2.4 * k / (H > 1 ? H - 1 : 1);
    if (H == 1) pos[0] = 1.0;
    int it = 0;
    for (; it < 100000; ++it) {
        edge[0] = 0.0;
        for (int k = 1; k < H; ++k) edge[k] = 0.5 * (pos[k - 1] + pos[k]);
        edge[H] = INFINITY;
        double moved = 0.0;
        for (int k = 0; k < H; ++k) {
            double a = edge[k], b = edge[k + 1];
            double pa = gauss_density(a), pb = std::isinf(b) ? 0.0 : gauss_density(b);
            double mass = gauss_tail(a) - (std::isinf(b) ? 0.0 : gauss_tail(b));
            double c = (pa - pb) / mass;
            moved = std::fmax(moved, std::fabs(c - pos[k]));
            pos[k] = c;
        }
        if (moved < 1e-15) break;
    }
    const double sd = 1.0 / std::sqrt((double)dim);
    for (int k = 0; k < H; ++k) {
        cents[H + k] = pos[k] * sd;
        cents[H - 1 - k] = -pos[k] * sd;
    }
    bounds[H - 1] = 0.0;
    for (int k = 1; k < H; ++k) {
        double e = 0.5 * (pos[k - 1] + pos[k]) * sd;
        bounds[H - 1 + k] = e;
        bounds[H - 1 - k] = -e;
    }
    return it;
}

int lloyd_max_beta(int dim, int bits, double *bounds, double *cents) {
    if (dim < 3 || bits < 1 || bits > 4) return -1;
    const int K = 1 << bits, H = K / 2;
    const double a = 0.5 * (dim - 3);
    const int NSTEP = 1 << 16;
    const double h = 1.0 / NSTEP;
    auto dens = [&](double y) { return std::pow(std::fmax(0.0, 1.0 - y * y), a); };
    std::vector<double> F(NSTEP + 1);
    F[0] = 0.0;
    const double g = h / (2.0 * std::sqrt(3.0));
    for (int i = 0; i < NSTEP; ++i) {
        const double mid = (i + 0.5) * h;
        F[i + 1] = F[i] + 0.5 * h * (dens(mid - g) + dens(mid + g));
    }
    auto Fat = [&](double y) {
        if (y <= 0.0) return 0.0;
        if (y >= 1.0) return F[NSTEP];
        int i = (int)(y / h);
        if (i >= NSTEP) i = NSTEP - 1;
        const double y0 = i * h, t = (y - y0) / h;
        const double f0 = dens(y0) * h, f1 = dens(y0 + h) * h;
        const double t2 = t * t, t3 = t2 * t;
        return (2 * t3 - 3 * t2 + 1) * F[i] + (t3 - 2 * t2 + t) * f0 + (-2 * t3 + 3 * t2) * F[i + 1] +
               (t3 - t2) * f1;
    };
    auto moment = [&](double l, double u) {
        return (std::pow(1.0 - l * l, a + 1.0) - std::pow(std::fmax(0.0, 1.0 - u * u), a + 1.0)) / (2.0 * (a + 1.0));
    };
    double pos[8], edge[9];
    const double sd = 1.0 / std::sqrt((double)dim);
    for (int k = 0; k < H; ++k) pos[k] = sd * (0.4 + 2.4 * k / (H > 1 ? H - 1 : 1));
    if (H == 1) pos[0] = sd;
    int it = 0;
    for (; it < 100000; ++it) {
        edge[0] = 0.0;
        for (int k = 1; k < H; ++k) edge[k] = 0.5 * (pos[k - 1] + pos[k]);
        edge[H] = 1.0;
        double moved = 0.0;
        for (int k = 0; k < H; ++k) {
            const double mass = Fat(edge[k + 1]) - Fat(edge[k]);
            const double c = moment(edge[k], edge[k + 1]) / mass;
            moved = std::fmax(moved, std::fabs(c - pos[k]));
            pos[k] = c;
        }
        if (moved < 1e-15 * sd) break;
    }
    for (int k = 0; k < H; ++k) {
        cents[H + k] = pos[k];
        cents[H - 1 - k] = -pos[k];
    }
    bounds[H - 1] = 0.0;
    for (int k = 1; k < H; ++k) {
        const double e = 0.5 * (pos[k - 1] + pos[k]);
        bounds[H - 1 + k] = e;
        bounds[H - 1 - k] = -e;
    }
    return it;
}

}  // namespace tq
