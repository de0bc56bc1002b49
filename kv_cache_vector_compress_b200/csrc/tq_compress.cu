// tq_compress.cu -- key / value compression, warp-per-vector CUDA-core version.
//
// Steps per vector (TurboQuantMSE.quantize for values, TurboQuantProd.compress for keys;
// "turboquant-pytorch", nav.superapi.store, 核心 API; atskills.one, "What It Does"):
//   n = ||x||, u = x / n, y = R u, idx_j = #{k : b_k < y_j}, planar bit-pack of idx;
//   keys: e = y - c[idx] (the residual on rotated coordinates, r = R^T e), rho = ||e||,
//         p = S' e with S' = S R^T (so p = S r), sign_i = [p_i >= 0].
// All arithmetic is fp32 with fp32 accumulation; the codebook decisions are taken on the
// fp32 rotated values.  One warp owns one vector: lane l holds coordinates l, l+32, ...,
// so coordinate 32g+l of every 32-group sits in lane l and a warp ballot produces each
// planar code word directly.
#include "tq_common.cuh"
#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kWarps = 8;

template <int NPL, bool IS_KEY, bool X_F16>
__global__ void __launch_bounds__(kWarps * 32)
    compress_simt_kernel(Prepared P, const void *__restrict__ x, int64_t n, uint32_t *__restrict__ codes,
                         uint32_t *__restrict__ signs, uint16_t *__restrict__ norm,
                         uint16_t *__restrict__ rnorm) {
    constexpr int D = NPL * 32;
    __shared__ float bnd[kMaxLevels], cen[kMaxLevels];
    __shared__ float vec[kWarps][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int beta = IS_KEY ? P.kbeta : P.vbeta;
    const int nb = (1 << beta) - 1;
    if (threadIdx.x < kMaxLevels) {
        bnd[threadIdx.x] = IS_KEY ? P.cb->kb[threadIdx.x] : P.cb->vb[threadIdx.x];
        cen[threadIdx.x] = IS_KEY ? P.cb->kc[threadIdx.x] : P.cb->vc[threadIdx.x];
    }
    __syncthreads();
    float *us = vec[warp];
    const int wpv = beta * NPL;
    const int m = P.m, mpl = m >> 5;

    for (int64_t v = (int64_t)blockIdx.x * kWarps + warp; v < n; v += (int64_t)gridDim.x * kWarps) {
        // 1. norm and unit vector
        float xv[NPL];
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
            const int64_t e = v * D + 32 * k + lane;
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
            if (lane < beta) codes[v * wpv + k * beta + lane] = mine;
        }
        if (lane == 0) norm[v] = f32_to_f16_bits(nv);
        if (!IS_KEY) continue;
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
        if (lane == 0) rnorm[v] = f32_to_f16_bits(sqrtf(ee));
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
                    if (lane == 0) signs[v * mpl + kc + q] = w;
                }
        }
    }
}

template <int NPL>
cudaError_t launch_npl(const Prepared &P, bool is_key, const void *x, bool x_f16, int64_t n,
                       uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                       cudaStream_t s) {
    int64_t blocks64 = (n + kWarps - 1) / kWarps;
    int blocks = (int)(blocks64 < 148 * 16 ? blocks64 : 148 * 16);
    if (is_key) {
        if (x_f16)
            compress_simt_kernel<NPL, true, true><<<blocks, kWarps * 32, 0, s>>>(P, x, n, codes, signs, norm, rnorm);
        else
            compress_simt_kernel<NPL, true, false><<<blocks, kWarps * 32, 0, s>>>(P, x, n, codes, signs, norm, rnorm);
    } else {
        if (x_f16)
            compress_simt_kernel<NPL, false, true><<<blocks, kWarps * 32, 0, s>>>(P, x, n, codes, signs, norm, rnorm);
        else
            compress_simt_kernel<NPL, false, false><<<blocks, kWarps * 32, 0, s>>>(P, x, n, codes, signs, norm, rnorm);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress(const Prepared &P, bool is_key, const void *x, bool x_f16, int64_t n,
                            uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                            int32_t *dev_status, cudaStream_t s) {
    if (compress_tc_supported(P, is_key, x_f16) && n <= (int64_t)INT32_MAX)
        return launch_compress_tc(P, is_key, x, n, codes, signs, norm, rnorm, dev_status, s);
    if (compress_big_supported(P, is_key))
        return launch_compress_big(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, dev_status, s);
    switch (P.d) {
        case 32: return launch_npl<1>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        case 64: return launch_npl<2>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        case 128: return launch_npl<4>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        case 256: return launch_npl<8>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        case 512: return launch_npl<16>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        case 1024: return launch_npl<32>(P, is_key, x, x_f16, n, codes, signs, norm, rnorm, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
