// tq_compress.cu -- key / value compression, warp-per-vector CUDA-core version (the steps are in
// tq_compress_warp.cuh), and the dispatch between the compress kernels.
#include "tq_common.cuh"
#include "tq_compress_warp.cuh"
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
    if (threadIdx.x < kMaxLevels) {
        bnd[threadIdx.x] = IS_KEY ? P.cb->kb[threadIdx.x] : P.cb->vb[threadIdx.x];
        cen[threadIdx.x] = IS_KEY ? P.cb->kc[threadIdx.x] : P.cb->vc[threadIdx.x];
    }
    __syncthreads();
    float *us = vec[warp];
    const int wpv = beta * NPL;
    const int m = P.m, mpl = m >> 5;

    for (int64_t v = (int64_t)blockIdx.x * kWarps + warp; v < n; v += (int64_t)gridDim.x * kWarps)
        compress_vector_warp<NPL, IS_KEY, X_F16>(P, x, v, bnd, cen, us, lane, codes + v * wpv,
                                                 IS_KEY ? signs + v * mpl : nullptr, norm + v,
                                                 IS_KEY ? rnorm + v : nullptr);
}

// Decode-step append for shapes outside the tensor-core attention kernel: warp 2s compresses the
// new key of slice s, warp 2s+1 its new value, into record s * Ts + tnew of the caches.
template <int NPL, bool X_F16>
__global__ void __launch_bounds__(kWarps * 32) append_kernel(Prepared P, ScoreProblem sp) {
    constexpr int D = NPL * 32;
    __shared__ float vec[kWarps][D];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t nsl = (int64_t)sp.B * sp.Hkv;
    const int64_t job = (int64_t)blockIdx.x * kWarps + warp;
    if (job >= 2 * nsl) return;
    const int64_t sl = job >> 1;
    const int64_t rec = sl * sp.Ts + sp.tnew;
    if ((job & 1) == 0) {
        const int mpl = P.m >> 5;
        compress_vector_warp<NPL, true, X_F16>(P, sp.knew, sl, P.cb->kb, P.cb->kc, vec[warp], lane,
                                               sp.kcodes_w + rec * (P.kbeta * NPL), sp.ksigns_w + rec * mpl,
                                               sp.knorm_w + rec, sp.krnorm_w + rec);
    } else {
        compress_vector_warp<NPL, false, X_F16>(P, sp.vnew, sl, P.cb->vb, P.cb->vc, vec[warp], lane,
                                                sp.vcodes_w + rec * (P.vbeta * NPL), nullptr, sp.vnorm_w + rec,
                                                nullptr);
    }
}

template <int NPL>
cudaError_t launch_append_npl(const Prepared &P, const ScoreProblem &sp, cudaStream_t s) {
    const int64_t jobs = 2 * (int64_t)sp.B * sp.Hkv;
    const unsigned blocks = (unsigned)((jobs + kWarps - 1) / kWarps);
    if (sp.new_f16) append_kernel<NPL, true><<<blocks, kWarps * 32, 0, s>>>(P, sp);
    else append_kernel<NPL, false><<<blocks, kWarps * 32, 0, s>>>(P, sp);
    return cudaGetLastError();
}

// Records i of the staging arrays (the new rows, compressed contiguously) to record i * Ts + tnew
// of the caches: one thread per word of a record, the norms by the record's first thread.
__global__ void scatter_new_kernel(ScoreProblem sp, int kw, int sw, int vw, const uint32_t *__restrict__ skc,
                                   const uint32_t *__restrict__ sks, const uint32_t *__restrict__ svc,
                                   const uint16_t *__restrict__ skn, const uint16_t *__restrict__ skr,
                                   const uint16_t *__restrict__ svn) {
    const int64_t nsl = (int64_t)sp.B * sp.Hkv;
    const int per = kw + sw + vw;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < nsl * per;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / per;
        const int w = (int)(e % per);
        const int64_t rec = i * sp.Ts + sp.tnew;
        if (w < kw) {
            sp.kcodes_w[rec * kw + w] = skc[i * kw + w];
        } else if (w < kw + sw) {
            sp.ksigns_w[rec * sw + (w - kw)] = sks[i * sw + (w - kw)];
        } else {
            sp.vcodes_w[rec * vw + (w - kw - sw)] = svc[i * vw + (w - kw - sw)];
        }
        if (w == 0) {
            sp.knorm_w[rec] = skn[i];
            sp.krnorm_w[rec] = skr[i];
            sp.vnorm_w[rec] = svn[i];
        }
    }
}

struct AppendStage {
    size_t kc, ks, vc, kn, kr, vn, total;
};
AppendStage append_stage_layout(const Prepared &P, const ScoreProblem &sp) {
    const size_t nsl = (size_t)sp.B * sp.Hkv;
    AppendStage L;
    size_t o = 0;
    L.kc = o;
    o = align_up(o + nsl * P.kbeta * (P.d / 32) * 4, 256);
    L.ks = o;
    o = align_up(o + nsl * (P.m / 32) * 4, 256);
    L.vc = o;
    o = align_up(o + nsl * P.vbeta * (P.d / 32) * 4, 256);
    L.kn = o;
    o = align_up(o + nsl * 2, 256);
    L.kr = o;
    o = align_up(o + nsl * 2, 256);
    L.vn = o;
    o = align_up(o + nsl * 2, 256);
    L.total = o;
    return L;
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

cudaError_t launch_append(const Prepared &P, const ScoreProblem &sp, cudaStream_t s) {
    switch (P.d) {
        case 32: return launch_append_npl<1>(P, sp, s);
        case 64: return launch_append_npl<2>(P, sp, s);
        case 128: return launch_append_npl<4>(P, sp, s);
        case 256: return launch_append_npl<8>(P, sp, s);
        case 512: return launch_append_npl<16>(P, sp, s);
        case 1024: return launch_append_npl<32>(P, sp, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t append_stage_bytes(const Prepared &P, const ScoreProblem &sp) { return append_stage_layout(P, sp).total; }

cudaError_t launch_append_staged(const Prepared &P, const ScoreProblem &sp, void *stage, int32_t *dev_status,
                                 cudaStream_t s) {
    const AppendStage L = append_stage_layout(P, sp);
    char *b = (char *)stage;
    uint32_t *skc = (uint32_t *)(b + L.kc), *sks = (uint32_t *)(b + L.ks), *svc = (uint32_t *)(b + L.vc);
    uint16_t *skn = (uint16_t *)(b + L.kn), *skr = (uint16_t *)(b + L.kr), *svn = (uint16_t *)(b + L.vn);
    const int64_t nsl = (int64_t)sp.B * sp.Hkv;
    cudaError_t e = launch_compress(P, true, sp.knew, sp.new_f16, nsl, skc, sks, skn, skr, dev_status, s);
    if (e == cudaSuccess) e = launch_compress(P, false, sp.vnew, sp.new_f16, nsl, svc, nullptr, svn, nullptr, dev_status, s);
    if (e != cudaSuccess) return e;
    const int kw = P.kbeta * (P.d / 32), sw = P.m / 32, vw = P.vbeta * (P.d / 32);
    const int64_t work = nsl * (kw + sw + vw);
    const unsigned blocks = (unsigned)((work + 255) / 256 < 148 * 8 ? (work + 255) / 256 : 148 * 8);
    scatter_new_kernel<<<blocks, 256, 0, s>>>(sp, kw, sw, vw, skc, sks, svc, skn, skr, svn);
    return cudaGetLastError();
}

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
