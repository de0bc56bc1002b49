// tq_api.cu -- the extern "C" entry points of libtq: argument checks, then launches.
#include <cmath>
#include <cstring>

#include "tq_internal.cuh"

using namespace tq;

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool dim_supported(int d) {
    return d == 32 || d == 64 || d == 128 || d == 256 || d == 512 || d == 1024;
}

// Common checks on a parameter set; `need_keys` requires the QJL part.
tq_status check_params(const tq_params *p, bool need_keys) {
    if (!p) return TQ_ERR_INVALID_ARG;
    if (p->dim < 32 || p->dim > kMaxDim || p->dim % 32) return TQ_ERR_INVALID_ARG;
    if (p->bits < 1 || p->bits > 4) return TQ_ERR_INVALID_ARG;
    if (p->proj_dim < 0 || p->proj_dim > kMaxProj || p->proj_dim % 32) return TQ_ERR_INVALID_ARG;
    if (need_keys && (p->bits < 2 || p->proj_dim < 32)) return TQ_ERR_INVALID_ARG;
    if (!p->workspace || !aligned16(p->workspace)) return TQ_ERR_INVALID_ARG;
    if (p->workspace_bytes < ws_layout(p->dim, p->proj_dim).total) return TQ_ERR_INVALID_ARG;
    if (!dim_supported(p->dim)) return TQ_ERR_UNSUPPORTED;
    return TQ_OK;
}

tq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

tq_status check_problem(const tq_params *p, int B, int Hq, int Hkv, int Nq, int64_t T, const float *q,
                        const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                        const uint16_t *krnorm) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || T < 1 || Hq % Hkv) return TQ_ERR_INVALID_ARG;
    if (T > (int64_t)INT32_MAX) return TQ_ERR_UNSUPPORTED;
    // every index used by the kernels must fit in int64 comfortably
    const double recs = (double)B * Hkv * (double)T, rows = (double)B * Hq * Nq;
    if (recs * p->dim > 9e18 || rows * (double)T > 9e18) return TQ_ERR_INVALID_ARG;
    const void *ptrs[] = {q, kcodes, ksigns, knorm, krnorm};
    for (const void *x : ptrs)
        if (!x || !aligned16(x)) return TQ_ERR_INVALID_ARG;
    return TQ_OK;
}

ScoreProblem make_problem(int B, int Hq, int Hkv, int Nq, int64_t T, const float *q, const uint32_t *kcodes,
                          const uint32_t *ksigns, const uint16_t *knorm, const uint16_t *krnorm,
                          const uint32_t *vcodes, const uint16_t *vnorm) {
    ScoreProblem sp;
    memset(&sp, 0, sizeof(sp));
    sp.B = B;
    sp.Hq = Hq;
    sp.Hkv = Hkv;
    sp.Nq = Nq;
    sp.T = T;
    sp.Ts = T;
    sp.q = q;
    sp.kcodes = kcodes;
    sp.ksigns = ksigns;
    sp.knorm = knorm;
    sp.krnorm = krnorm;
    sp.vcodes = vcodes;
    sp.vnorm = vnorm;
    return sp;
}

}  // namespace

extern "C" {

const char *tq_status_string(int status) {
    switch (status) {
        case TQ_OK: return "TQ_OK";
        case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
        case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
        case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
        case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
        default: return "TQ_ERR_UNKNOWN";
    }
}

int tq_version(void) { return 100; }

tq_status tq_codebook(int dim, int bits, float *boundaries, float *centroids) {
    if (dim < 1 || bits < 1 || bits > 4 || !boundaries || !centroids) return TQ_ERR_INVALID_ARG;
    double b[kMaxLevels], c[kMaxLevels];
    if (lloyd_max_gaussian(dim, bits, b, c) < 0) return TQ_ERR_INVALID_ARG;
    const int K = 1 << bits;
    for (int k = 0; k < K - 1; ++k) boundaries[k] = (float)b[k];
    for (int k = 0; k < K; ++k) centroids[k] = (float)c[k];
    return TQ_OK;
}

tq_status tq_codebook_beta(int dim, int bits, float *boundaries, float *centroids) {
    if (dim < 3 || bits < 1 || bits > 4 || !boundaries || !centroids) return TQ_ERR_INVALID_ARG;
    double b[kMaxLevels], c[kMaxLevels];
    if (lloyd_max_beta(dim, bits, b, c) < 0) return TQ_ERR_INVALID_ARG;
    const int K = 1 << bits;
    for (int k = 0; k < K - 1; ++k) boundaries[k] = (float)b[k];
    for (int k = 0; k < K; ++k) centroids[k] = (float)c[k];
    return TQ_OK;
}

size_t tq_workspace_bytes(int dim, int bits, int proj_dim) {
    if (dim < 32 || dim > kMaxDim || dim % 32 || bits < 1 || bits > 4) return 0;
    if (proj_dim < 0 || proj_dim > kMaxProj || proj_dim % 32) return 0;
    return ws_layout(dim, proj_dim).total;
}

tq_status tq_prepare(const tq_params *p, int32_t *dev_status, tq_stream_t stream) {
    return tq_prepare_law(p, TQ_LAW_GAUSSIAN, dev_status, stream);
}

tq_status tq_prepare_law(const tq_params *p, int law, int32_t *dev_status, tq_stream_t stream) {
    (void)dev_status;
    tq_status st = check_params(p, false);
    if (st != TQ_OK) return st;
    if (law != TQ_LAW_GAUSSIAN && law != TQ_LAW_BETA) return TQ_ERR_INVALID_ARG;
    if (!p->R || !aligned16(p->R)) return TQ_ERR_INVALID_ARG;
    if (p->proj_dim > 0 && (!p->S || !aligned16(p->S))) return TQ_ERR_INVALID_ARG;
    auto solve = law == TQ_LAW_BETA ? lloyd_max_beta : lloyd_max_gaussian;
    Codebooks cb;
    memset(&cb, 0, sizeof(cb));
    double b[kMaxLevels], c[kMaxLevels];
    const int K = 1 << p->bits;
    if (solve(p->dim, p->bits, b, c) < 0) return TQ_ERR_INVALID_ARG;
    for (int k = 0; k < K; ++k) {
        cb.vc[k] = (float)c[k];
        if (k < K - 1) cb.vb[k] = (float)b[k];
    }
    // unused boundary slots never count: +inf is never below a finite value
    for (int k = K - 1; k < kMaxLevels; ++k) cb.vb[k] = INFINITY;
    if (p->bits >= 2) {
        const int Kk = K / 2;
        if (solve(p->dim, p->bits - 1, b, c) < 0) return TQ_ERR_INVALID_ARG;
        for (int k = 0; k < Kk; ++k) {
            cb.kc[k] = (float)c[k];
            if (k < Kk - 1) cb.kb[k] = (float)b[k];
        }
        for (int k = Kk - 1; k < kMaxLevels; ++k) cb.kb[k] = INFINITY;
    } else {
        for (int k = 0; k < kMaxLevels; ++k) cb.kb[k] = INFINITY;
    }
    return from_cuda(launch_prepare(p, cb, (cudaStream_t)stream));
}

tq_status tq_compress_keys(const tq_params *p, const void *x, tq_dtype dtype, int64_t n, uint32_t *codes,
                           uint32_t *signs, uint16_t *norm, uint16_t *rnorm, int32_t *dev_status,
                           tq_stream_t stream) {
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    if (dtype != TQ_F16 && dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
    if (n < 0) return TQ_ERR_INVALID_ARG;
    if (n == 0) return TQ_OK;
    const void *ptrs[] = {x, codes, signs, norm, rnorm};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    return from_cuda(launch_compress(P, true, x, dtype == TQ_F16, n, codes, signs, norm, rnorm, dev_status,
                                     (cudaStream_t)stream));
}

tq_status tq_compress_values(const tq_params *p, const void *x, tq_dtype dtype, int64_t n, uint32_t *codes,
                             uint16_t *norm, int32_t *dev_status, tq_stream_t stream) {
    tq_status st = check_params(p, false);
    if (st != TQ_OK) return st;
    if (dtype != TQ_F16 && dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
    if (n < 0) return TQ_ERR_INVALID_ARG;
    if (n == 0) return TQ_OK;
    const void *ptrs[] = {x, codes, norm};
    for (const void *q : ptrs)
        if (!q || !aligned16(q)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    return from_cuda(launch_compress(P, false, x, dtype == TQ_F16, n, codes, nullptr, norm, nullptr,
                                     dev_status, (cudaStream_t)stream));
}

size_t tq_scores_scratch_bytes(const tq_params *p, int B, int Hq, int Hkv, int Nq, int64_t T, int topk) {
    if (check_params(p, true) != TQ_OK) return 0;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || T < 1 || Hq % Hkv) return 0;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, T, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                   nullptr);
    const ScoresPlan plan = plan_scores(P, sp, topk);
    size_t bytes = qprep_bytes(P, sp);
    if (plan.search) bytes += search_scratch_bytes(P, sp, plan.fused_topk ? topk : 0);
    if (plan.planes) bytes += planes_frag_bytes(P, sp);
    if (topk > 0 && !plan.fused_topk) bytes += topk_scratch_bytes(P, sp, topk);
    return bytes;
}

namespace {
tq_status scores_impl(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                      const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                      const uint16_t *krnorm, float *scores, int topk, int32_t *topk_idx, float *topk_val,
                      void *scratch, size_t scratch_bytes, int32_t *dev_status, tq_stream_t stream,
                      bool fp16) {
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    st = check_problem(p, B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm);
    if (st != TQ_OK) return st;
    if (topk < 0 || topk > kMaxTopk || topk > T) return TQ_ERR_INVALID_ARG;
    if (topk == 0 && !scores) return TQ_ERR_INVALID_ARG;
    if (scores && !aligned16(scores)) return TQ_ERR_INVALID_ARG;
    if (topk > 0 && (!topk_idx || !topk_val || !aligned16(topk_idx) || !aligned16(topk_val)))
        return TQ_ERR_INVALID_ARG;
    if (!scratch || !aligned16(scratch)) return TQ_ERR_INVALID_ARG;
    if (scratch_bytes < tq_scores_scratch_bytes(p, B, Hq, Hkv, Nq, T, topk)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm, nullptr, nullptr);
    cudaStream_t s = (cudaStream_t)stream;
    const ScoresPlan plan = plan_scores(P, sp, topk);
    char *cur = (char *)scratch;
    float *qprep = (float *)cur;
    cur += qprep_bytes(P, sp);
    void *search_scratch = cur;
    if (plan.search) cur += search_scratch_bytes(P, sp, plan.fused_topk ? topk : 0);
    uint32_t *frag = (uint32_t *)cur;
    if (plan.planes) cur += planes_frag_bytes(P, sp);
    float *sbuf = scores;
    if (!sbuf && !plan.fused_topk) sbuf = (float *)cur;
    cudaError_t e = plan.planes ? cudaSuccess : launch_qprep(P, sp, qprep, s);
    if (e != cudaSuccess) return from_cuda(e);
    if (plan.fused_topk) {
        e = launch_search(P, sp, qprep, search_scratch, scores, topk, topk_idx, topk_val, dev_status, s, fp16);
        return from_cuda(e);
    }
    if (plan.search)
        e = launch_search(P, sp, qprep, search_scratch, sbuf, 0, nullptr, nullptr, dev_status, s, fp16);
    else if (plan.planes)
        e = launch_planes(P, sp, 1.0f, frag, plan_planes(sp), false, sbuf, nullptr, s);
    else if (plan.mma)
        e = launch_decode_mma(P, sp, qprep, 1.0f, sbuf, decode_mma_splits(sp), false, s);
    else
        e = launch_scores(P, sp, qprep, sbuf, s);
    if (e == cudaSuccess && topk > 0) e = launch_topk(sp, sbuf, topk, topk_idx, topk_val, s);
    return from_cuda(e);
}
}  // namespace

tq_status tq_scores(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, float *scores, int topk, int32_t *topk_idx, float *topk_val,
                    void *scratch, size_t scratch_bytes, int32_t *dev_status, tq_stream_t stream) {
    return scores_impl(p, q, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, scores, topk, topk_idx, topk_val,
                       scratch, scratch_bytes, dev_status, stream, false);
}

tq_status tq_search(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, float *scores, int topk, int32_t *topk_idx, float *topk_val,
                    void *scratch, size_t scratch_bytes, int32_t *dev_status, tq_stream_t stream) {
    return scores_impl(p, q, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, scores, topk, topk_idx, topk_val,
                       scratch, scratch_bytes, dev_status, stream, true);
}

size_t tq_attend_scratch_bytes(const tq_params *p, int B, int Hq, int Hkv, int Nq, int64_t T) {
    if (check_params(p, true) != TQ_OK) return 0;
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || T < 1 || Hq % Hkv) return 0;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, T, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                   nullptr);
    const AttendPlan plan = plan_attend(P, sp);
    // bit-plane path: query operands, then the staging of tq_append_attend's new records
    return qprep_bytes(P, sp) + attend_partials_bytes(P, sp, plan.splits) +
           (plan.planes ? planes_frag_bytes(P, sp) + append_stage_bytes(P, sp) : 0);
}

tq_status tq_attend(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, const uint32_t *vcodes, const uint16_t *vnorm, float scale,
                    float *out, void *scratch, size_t scratch_bytes, int32_t *dev_status,
                    tq_stream_t stream) {
    (void)dev_status;
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    st = check_problem(p, B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm);
    if (st != TQ_OK) return st;
    if (!vcodes || !vnorm || !out || !aligned16(vcodes) || !aligned16(vnorm) || !aligned16(out))
        return TQ_ERR_INVALID_ARG;
    if (!(scale == scale)) return TQ_ERR_INVALID_ARG;  // NaN
    if (!scratch || !aligned16(scratch)) return TQ_ERR_INVALID_ARG;
    if (scratch_bytes < tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm, vcodes, vnorm);
    if (scale <= 0.f) scale = 1.0f / sqrtf((float)p->dim);
    cudaStream_t s = (cudaStream_t)stream;
    float *qprep = (float *)scratch;
    const AttendPlan plan = plan_attend(P, sp);
    float *partials = (float *)((char *)scratch + qprep_bytes(P, sp));
    uint32_t *frag = (uint32_t *)((char *)partials + attend_partials_bytes(P, sp, plan.splits));
    cudaError_t e = plan.planes ? cudaSuccess : launch_qprep(P, sp, qprep, s);
    if (e == cudaSuccess) {
        if (plan.planes) {
            e = launch_planes(P, sp, scale, frag, plan.pp, true, out, partials, s);
        } else if (plan.mma) {
            e = launch_decode_mma(P, sp, qprep, scale, partials, plan.splits, true, s);
            if (e == cudaSuccess) e = launch_attend_combine(P, sp, partials, plan.splits, out, s);
        } else {
            e = launch_attend(P, sp, qprep, scale, partials, plan.splits, out, s);
        }
    }
    return from_cuda(e);
}

namespace {
struct HostStepScratch {
    size_t k, v, q, o, att, total;
};
HostStepScratch host_step_layout(const tq_params *p, tq_dtype dtype, int B, int Hq, int Hkv, int Nq, int64_t T) {
    HostStepScratch L;
    const size_t es = dtype == TQ_F16 ? 2 : 4;
    const size_t kv = (size_t)B * Hkv * (size_t)T * p->dim * es;
    const size_t qo = (size_t)B * Hq * (size_t)Nq * p->dim * 4;
    size_t o = 0;
    L.k = o;
    o = align_up(o + kv, 256);
    L.v = o;
    o = align_up(o + kv, 256);
    L.q = o;
    o = align_up(o + qo, 256);
    L.o = o;
    o = align_up(o + qo, 256);
    L.att = o;
    o += tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T);
    L.total = o;
    return L;
}
}  // namespace

size_t tq_compress_attend_host_scratch_bytes(const tq_params *p, tq_dtype dtype, int B, int Hq, int Hkv, int Nq,
                                             int64_t T) {
    if (check_params(p, true) != TQ_OK) return 0;
    if (dtype != TQ_F16 && dtype != TQ_F32) return 0;
    if (tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T) == 0) return 0;
    return host_step_layout(p, dtype, B, Hq, Hkv, Nq, T).total;
}

tq_status tq_compress_attend_host(const tq_params *p, const void *k_host, const void *v_host, tq_dtype dtype,
                                  const float *q_host, int B, int Hq, int Hkv, int Nq, int64_t T, uint32_t *kcodes,
                                  uint32_t *ksigns, uint16_t *knorm, uint16_t *krnorm, uint32_t *vcodes,
                                  uint16_t *vnorm, float scale, float *out_host, void *scratch, size_t scratch_bytes,
                                  int32_t *dev_status, tq_stream_t stream) {
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    if (!k_host || !v_host || !q_host || !out_host) return TQ_ERR_INVALID_ARG;
    if (dtype != TQ_F16 && dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
    const size_t need = tq_compress_attend_host_scratch_bytes(p, dtype, B, Hq, Hkv, Nq, T);
    if (need == 0) return TQ_ERR_INVALID_ARG;
    if (!scratch || !aligned16(scratch) || scratch_bytes < need) return TQ_ERR_INVALID_ARG;
    const HostStepScratch L = host_step_layout(p, dtype, B, Hq, Hkv, Nq, T);
    char *base = (char *)scratch;
    const int64_t n = (int64_t)B * Hkv * T;
    const size_t es = dtype == TQ_F16 ? 2 : 4;
    const size_t kvb = (size_t)n * p->dim * es, qob = (size_t)B * Hq * (size_t)Nq * p->dim * 4;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(base + L.k, k_host, kvb, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + L.v, v_host, kvb, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + L.q, q_host, qob, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return from_cuda(e);
    st = tq_compress_keys(p, base + L.k, dtype, n, kcodes, ksigns, knorm, krnorm, dev_status, stream);
    if (st != TQ_OK) return st;
    st = tq_compress_values(p, base + L.v, dtype, n, vcodes, vnorm, dev_status, stream);
    if (st != TQ_OK) return st;
    st = tq_attend(p, (const float *)(base + L.q), B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, vcodes, vnorm,
                   scale, (float *)(base + L.o), base + L.att, scratch_bytes - L.att, dev_status, stream);
    if (st != TQ_OK) return st;
    return from_cuda(cudaMemcpyAsync(out_host, base + L.o, qob, cudaMemcpyDeviceToHost, s));
}

tq_status tq_attend_partial(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                            const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                            const uint16_t *krnorm, const uint32_t *vcodes, const uint16_t *vnorm, float scale,
                            float *partial, void *scratch, size_t scratch_bytes, int32_t *dev_status,
                            tq_stream_t stream) {
    (void)dev_status;
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    st = check_problem(p, B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm);
    if (st != TQ_OK) return st;
    if (!vcodes || !vnorm || !partial || !aligned16(vcodes) || !aligned16(vnorm) || !aligned16(partial))
        return TQ_ERR_INVALID_ARG;
    if (!(scale == scale)) return TQ_ERR_INVALID_ARG;  // NaN
    if (!scratch || !aligned16(scratch)) return TQ_ERR_INVALID_ARG;
    if (scratch_bytes < tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, T, q, kcodes, ksigns, knorm, krnorm, vcodes, vnorm);
    if (scale <= 0.f) scale = 1.0f / sqrtf((float)p->dim);
    cudaStream_t s = (cudaStream_t)stream;
    float *qprep = (float *)scratch;
    const AttendPlan plan = plan_attend(P, sp);
    float *partials = (float *)((char *)scratch + qprep_bytes(P, sp));
    uint32_t *frag = (uint32_t *)((char *)partials + attend_partials_bytes(P, sp, plan.splits));
    cudaError_t e = plan.planes ? cudaSuccess : launch_qprep(P, sp, qprep, s);
    if (e == cudaSuccess) {
        if (plan.planes) {
            e = launch_planes(P, sp, scale, frag, plan.pp, true, partial, partials, s, true);
        } else if (plan.mma) {
            e = launch_decode_mma(P, sp, qprep, scale, partials, plan.splits, true, s);
            if (e == cudaSuccess)
                e = launch_merge_partials(P, (int64_t)B * Hq * Nq, plan.splits, partials,
                                          (int64_t)plan.splits * (p->dim + 2), p->dim + 2, false, partial, s);
        } else {
            e = launch_attend(P, sp, qprep, scale, partials, plan.splits, partial, s, false);
        }
    }
    return from_cuda(e);
}

tq_status tq_attend_merge(const tq_params *p, const float *partials, int parts, int64_t rows, float *out,
                          int32_t *dev_status, tq_stream_t stream) {
    (void)dev_status;
    tq_status st = check_params(p, false);
    if (st != TQ_OK) return st;
    if (parts < 1 || rows < 1) return TQ_ERR_INVALID_ARG;
    if (!partials || !out || !aligned16(partials) || !aligned16(out)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    return from_cuda(launch_merge_partials(P, rows, parts, partials, p->dim + 2, rows * (int64_t)(p->dim + 2), true,
                                           out, (cudaStream_t)stream));
}

tq_status tq_append_attend(const tq_params *p, const float *q, const void *k_new, const void *v_new,
                           tq_dtype dtype, int B, int Hq, int Hkv, int Nq, int64_t t, int64_t t_cap,
                           uint32_t *kcodes, uint32_t *ksigns, uint16_t *knorm, uint16_t *krnorm,
                           uint32_t *vcodes, uint16_t *vnorm, float scale, float *out, void *scratch,
                           size_t scratch_bytes, int32_t *dev_status, tq_stream_t stream) {
    tq_status st = check_params(p, true);
    if (st != TQ_OK) return st;
    if (t < 0 || t_cap < 1 || t >= t_cap) return TQ_ERR_INVALID_ARG;
    if (dtype != TQ_F16 && dtype != TQ_F32) return TQ_ERR_INVALID_ARG;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return TQ_ERR_INVALID_ARG;
    // the checks of tq_attend, over the whole cache extent
    st = check_problem(p, B, Hq, Hkv, Nq, t_cap, q, kcodes, ksigns, knorm, krnorm);
    if (st != TQ_OK) return st;
    if (!vcodes || !vnorm || !out || !aligned16(vcodes) || !aligned16(vnorm) || !aligned16(out))
        return TQ_ERR_INVALID_ARG;
    if (!(scale == scale)) return TQ_ERR_INVALID_ARG;  // NaN
    if (!scratch || !aligned16(scratch)) return TQ_ERR_INVALID_ARG;
    if (scratch_bytes < tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, t + 1)) return TQ_ERR_INVALID_ARG;
    Prepared P = prepared_view(p);
    ScoreProblem sp = make_problem(B, Hq, Hkv, Nq, t + 1, q, kcodes, ksigns, knorm, krnorm, vcodes, vnorm);
    sp.Ts = t_cap;
    sp.knew = k_new;
    sp.vnew = v_new;
    sp.new_f16 = dtype == TQ_F16;
    sp.tnew = t;
    sp.kcodes_w = kcodes;
    sp.ksigns_w = ksigns;
    sp.knorm_w = knorm;
    sp.krnorm_w = krnorm;
    sp.vcodes_w = vcodes;
    sp.vnorm_w = vnorm;
    const AttendPlan plan = plan_attend(P, sp);
    if (scale <= 0.f) scale = 1.0f / sqrtf((float)p->dim);
    cudaStream_t s = (cudaStream_t)stream;
    float *qprep = (float *)scratch;
    float *partials = (float *)((char *)scratch + qprep_bytes(P, sp));
    uint32_t *frag = (uint32_t *)((char *)partials + attend_partials_bytes(P, sp, plan.splits));
    cudaError_t e = plan.planes ? cudaSuccess : launch_qprep(P, sp, qprep, s);
    if (plan.planes) {
        // the new rows through the compress kernels into a staging area, scattered to slot t; then
        // the bit-plane attention over slots 0..t of the strided cache
        if (e == cudaSuccess) e = launch_append_staged(P, sp, (char *)frag + planes_frag_bytes(P, sp), dev_status, s);
        ScoreProblem rd = sp;
        rd.knew = rd.vnew = nullptr;
        if (e == cudaSuccess) e = launch_planes(P, rd, scale, frag, plan.pp, true, out, partials, s);
    } else if (plan.mma) {
        // the append runs inside the attention kernel
        if (e == cudaSuccess) e = launch_decode_mma(P, sp, qprep, scale, partials, plan.splits, true, s);
        if (e == cudaSuccess) e = launch_attend_combine(P, sp, partials, plan.splits, out, s);
    } else {
        // other shapes: the append kernel, then the CUDA-core attention over the strided cache
        if (e == cudaSuccess) e = launch_append(P, sp, s);
        ScoreProblem rd = sp;
        rd.knew = rd.vnew = nullptr;
        if (e == cudaSuccess) e = launch_attend(P, rd, qprep, scale, partials, plan.splits, out, s);
    }
    return from_cuda(e);
}

}  // extern "C"
