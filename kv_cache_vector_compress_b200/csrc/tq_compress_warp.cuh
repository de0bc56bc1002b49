// tq_compress_warp.cuh -- one vector compressed by one warp on the CUDA cores.
//
// Steps (TurboQuantMSE.quantize for values, TurboQuantProd.compress for keys;
// "turboquant-pytorch", nav.superapi.store, 核心 API; atskills.one, "What It Does"):
//   n = ||x||, u = x / n, y = R u, idx_j = #{k : b_k < y_j}, planar bit-pack of idx;
//   keys: e = y - c[idx] (the residual on rotated coordinates, r = R^T e), rho = ||e||,
//         p = S' e with S' = S R^T (so p = S r), sign_i = [p_i >= 0].
// All arithmetic is fp32 with fp32 accumulation; the codebook decisions are taken on the
// fp32 rotated values.  Lane l holds coordinates l, l+32, ..., so coordinate 32g+l of every
// 32-group sits in lane l and a warp ballot produces each planar code word directly.
// Used by the CUDA-core compress kernel and by the decode step that appends one token per
// (batch, KV head) before attending.
#pragma once

#include "tq_common.cuh"
#include "tq_internal.cuh"

namespace tq {

// Compress row `row` of x (D = 32 NPL coordinates, fp16 or fp32) with the whole warp.
// bnd / cen: the codebook (shared memory); us: D floats of scratch (shared memory, this warp's);
// out_codes: the vector's beta * NPL code words; out_signs: its m / 32 sign words (keys).
template <int NPL, bool IS_KEY, bool X_F16>
__device__ __forceinline__ void compress_vector_warp(const Prepared &P, const void *__restrict__ x, int64_t row,
                                                     const float *bnd, const float *cen, float *us, int lane,
                                                     uint32_t *out_codes, uint32_t *out_signs, uint16_t *out_norm,
                                                     uint16_t *out_rnorm) {
    constexpr int D = NPL * 32;
    const int beta = IS_KEY ? P.kbeta : P.vbeta;
    const int nb = (1 << beta) - 1;
    const int m = P.m, mpl = m >> 5;
    // 1. norm and unit vector
    float xv[NPL];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const int64_t e = row * D + 32 * k + lane;
        float t;
        if (X_F16) t = __half2float(((const __half *)x)[e]);
        else t = ((const float *)x)[e];
        xv[k] = t;
        ss = fmaf(t, t, ss);
    }
    ss = warp_sum(ss);
    const float nv = sqrtf(ss);
    const float inv = nv > 0.f ? 1.0f / nv : 0.f;
    __syncwarp();
#pragma unroll
    for (int k = 0; k < NPL; ++k) us[32 * k + lane] = xv[k] * inv;
    __syncwarp();
    // 2. rotate: y_i = sum_j R[i][j] u_j, with R^T read row by row (coalesced over i)
    float y[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) y[k] = 0.f;
    for (int j = 0; j < D; ++j) {
        const float uj = us[j];
        const float *rt = P.RT + (int64_t)j * D + lane;
#pragma unroll
        for (int k = 0; k < NPL; ++k) y[k] = fmaf(__ldg(rt + 32 * k), uj, y[k]);
    }
    // 3./4. quantize and pack: word (g, p) = ballot of bit p over the 32 lanes
    int ci[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const int c = bucketize(bnd, nb, y[k]);
        ci[k] = c;
        uint32_t mine = 0;
        for (int p = 0; p < beta; ++p) {
            const uint32_t w = __ballot_sync(kFull, (c >> p) & 1);
            if (lane == p) mine = w;
        }
        if (lane < beta) out_codes[k * beta + lane] = mine;
    }
    if (lane == 0) *out_norm = f32_to_f16_bits(nv);
    if (!IS_KEY) return;
    // 5./6. residual on rotated coordinates and its norm
    __syncwarp();
    float ee = 0.f;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const float e = y[k] - cen[ci[k]];
        us[32 * k + lane] = e;
        ee = fmaf(e, e, ee);
    }
    ee = warp_sum(ee);
    if (lane == 0) *out_rnorm = f32_to_f16_bits(sqrtf(ee));
    __syncwarp();
    // 7. QJL signs: p_a = sum_i S'[a][i] e_i, four sign words at a time
    for (int kc = 0; kc < mpl; kc += 4) {
        float pa[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = 0; i < D; ++i) {
            const float ei = us[i];
            const float *sp = P.SpT + (int64_t)i * m + 32 * kc + lane;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (kc + q < mpl) pa[q] = fmaf(__ldg(sp + 32 * q), ei, pa[q]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (kc + q < mpl) {
                const uint32_t w = __ballot_sync(kFull, pa[q] >= 0.f);
                if (lane == 0) out_signs[kc + q] = w;
            }
    }
    __syncwarp();
}

}  // namespace tq
