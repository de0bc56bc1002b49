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
#include <cmath>
#include <cstring>

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

}  // namespace tq
