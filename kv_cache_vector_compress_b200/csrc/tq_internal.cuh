// tq_internal.cuh -- definitions shared by the host code and the kernels of libtq.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxDim = 1024;
constexpr int kMaxProj = 1024;
constexpr int kMaxLevels = 16;  // 4 bits
constexpr int kMaxTopk = 64;
constexpr uint32_t kWsMagic = 0x54513031u;  // "TQ01"

// Codebooks of one prepared parameter set, as the kernels read them.
struct Codebooks {
    float kb[kMaxLevels];  // key boundaries (K-1 used)
    float kc[kMaxLevels];  // key centroids
    float vb[kMaxLevels];  // value boundaries
    float vc[kMaxLevels];  // value centroids
};

// Byte offsets of the prepared arrays inside the caller's workspace.
struct WsLayout {
    size_t header;     // WsHeader
    size_t codebooks;  // Codebooks
    size_t R;          // fp32 [d, d]      copy of R
    size_t RT;         // fp32 [d, d]      R transposed
    size_t ST;         // fp32 [d, m]      S transposed
    size_t SpT;        // fp32 [d, m]      (S R^T) transposed
    size_t Rsw;        // fp16 hi | lo of R * 2^kRScaleLog2, tensor-core operand layout
    size_t Ssw;        // fp16 hi | lo of (S R^T) * 2^kSScaleLog2, same layout
    size_t RSsw;       // fp16 hi | lo of [R; S] * 2^kRScaleLog2 (d + m rows), same layout
    size_t S;          // fp32 [m, d]      copy of S
    size_t Sp;         // fp32 [m, d]      S R^T
    size_t total;
};

// Split-precision scales: R (entries <= 1) and S' = S R^T (entries ~N(0,1)) are scaled
// by a power of two before the fp16 hi/lo split so that the lo parts stay normal numbers.
constexpr int kRScaleLog2 = 8;
constexpr int kSScaleLog2 = 4;

// Byte offset of element (r, k) of a K-major fp16 operand with `rows` rows in the
// 128-byte-swizzled layout the tensor cores read: K is cut into blocks of 64 elements
// (128 bytes); each block holds `rows` rows of 128 bytes; the 16-byte chunk index of a
// row is XORed with (row mod 8).  Blocks start on 1024-byte boundaries when rows % 8 == 0.
__host__ __device__ inline size_t sw128_offset(int rows, int r, int k) {
    const int kb = k >> 6, kk = k & 63;
    const int chunk = (kk * 2) >> 4, within = (kk * 2) & 15;
    return (size_t)kb * rows * 128 + (size_t)r * 128 + (size_t)(((chunk ^ (r & 7)) << 4) + within);
}

struct WsHeader {
    uint32_t magic;
    int32_t dim, bits, proj_dim;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(int d, int m) {
    WsLayout L;
    size_t o = 0;
    L.header = o;
    o = align_up(o + sizeof(WsHeader), 256);
    L.codebooks = o;
    o = align_up(o + sizeof(Codebooks), 256);
    L.R = o;
    o = align_up(o + sizeof(float) * (size_t)d * d, 256);
    L.RT = o;
    o = align_up(o + sizeof(float) * (size_t)d * d, 256);
    L.ST = o;
    o = align_up(o + sizeof(float) * (size_t)d * (m > 0 ? m : 1), 256);
    L.SpT = o;
    o = align_up(o + sizeof(float) * (size_t)d * (m > 0 ? m : 1), 1024);
    L.Rsw = o;
    o = align_up(o + 2 * sizeof(uint16_t) * (size_t)d * d, 1024);
    L.Ssw = o;
    o = align_up(o + 2 * sizeof(uint16_t) * (size_t)d * (m > 0 ? m : 1), 1024);
    L.RSsw = o;
    o = align_up(o + 2 * sizeof(uint16_t) * (size_t)d * (d + m), 1024);
    L.S = o;
    o = align_up(o + sizeof(float) * (size_t)d * (m > 0 ? m : 1), 256);
    L.Sp = o;
    o = align_up(o + sizeof(float) * (size_t)d * (m > 0 ? m : 1), 256);
    L.total = o;
    return L;
}

// Device views of a prepared parameter set.
struct Prepared {
    int d, m, kbeta, vbeta;
    const Codebooks *cb;
    const float *R, *RT, *ST, *SpT, *S, *Sp;
    const uint16_t *Rsw, *Ssw, *RSsw;
};

inline Prepared prepared_view(const tq_params *p) {
    WsLayout L = ws_layout(p->dim, p->proj_dim);
    const char *w = (const char *)p->workspace;
    Prepared v;
    v.d = p->dim;
    v.m = p->proj_dim;
    v.kbeta = p->bits - 1;
    v.vbeta = p->bits;
    v.cb = (const Codebooks *)(w + L.codebooks);
    v.R = (const float *)(w + L.R);
    v.RT = (const float *)(w + L.RT);
    v.ST = (const float *)(w + L.ST);
    v.SpT = (const float *)(w + L.SpT);
    v.Rsw = (const uint16_t *)(w + L.Rsw);
    v.Ssw = (const uint16_t *)(w + L.Ssw);
    v.RSsw = (const uint16_t *)(w + L.RSsw);
    v.S = (const float *)(w + L.S);
    v.Sp = (const float *)(w + L.Sp);
    return v;
}

// Host-side Lloyd-Max (tq_codebook.cpp).
int lloyd_max_gaussian(int dim, int bits, double *bounds, double *cents);
int lloyd_max_beta(int dim, int bits, double *bounds, double *cents);

// Kernel launchers (tq_*.cu).  All return a cudaError_t from cudaGetLastError.
cudaError_t launch_prepare(const tq_params *p, const Codebooks &cb, cudaStream_t s);
bool compress_tc_supported(const Prepared &P, bool is_key, bool x_f16);
cudaError_t launch_compress_tc(const Prepared &P, bool is_key, const void *x, int64_t n, uint32_t *codes,
                               uint32_t *signs, uint16_t *norm, uint16_t *rnorm, int32_t *dev_status,
                               cudaStream_t s);
bool compress_big_supported(const Prepared &P, bool is_key);
cudaError_t launch_compress_big(const Prepared &P, bool is_key, const void *x, bool x_f16, int64_t n,
                                uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                                int32_t *dev_status, cudaStream_t s);
cudaError_t launch_compress(const Prepared &P, bool is_key, const void *x, bool x_f16, int64_t n,
                            uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                            int32_t *dev_status, cudaStream_t s);

struct ScoreProblem {
    int B, Hq, Hkv, Nq;
    int64_t T;   // tokens scored / attended per (batch, KV head)
    int64_t Ts;  // record stride of the caches: slice s holds records s * Ts .. s * Ts + T - 1
    const float *q;
    const uint32_t *kcodes, *ksigns;
    const uint16_t *knorm, *krnorm;
    const uint32_t *vcodes;
    const uint16_t *vnorm;
    // decode-step append: when knew is set, the attention kernel first compresses row s of knew
    // and vnew ([B * Hkv, d], fp16 or fp32) into record s * Ts + tnew of the caches below (the
    // same arrays as the read-only pointers above)
    const void *knew, *vnew;
    int new_f16;
    int64_t tnew;
    uint32_t *kcodes_w, *ksigns_w, *vcodes_w;
    uint16_t *knorm_w, *krnorm_w, *vnorm_w;
};

// Compress the new key / value of every slice into record s * Ts + tnew (sp.knew, sp.vnew set).
cudaError_t launch_append(const Prepared &P, const ScoreProblem &sp, cudaStream_t s);
// The same append through the compress kernels: the new rows are compressed contiguously into
// `stage` (append_stage_bytes), then scattered to record s * Ts + tnew.
size_t append_stage_bytes(const Prepared &P, const ScoreProblem &sp);
cudaError_t launch_append_staged(const Prepared &P, const ScoreProblem &sp, void *stage, int32_t *dev_status,
                                 cudaStream_t s);
size_t qprep_bytes(const Prepared &P, const ScoreProblem &sp);
int attend_splits(const ScoreProblem &sp);
size_t attend_partials_bytes(const Prepared &P, const ScoreProblem &sp, int splits);
cudaError_t launch_attend_combine(const Prepared &P, const ScoreProblem &sp, const float *partials, int splits,
                                  float *out, cudaStream_t s);
// Merge partials (M, l, o_rot) of `parts` context pieces per row: element (row, part) at
// row * row_stride + part * part_stride.  final: out = R^T o / l [rows, d]; else the merged
// partial [rows, d + 2].
cudaError_t launch_merge_partials(const Prepared &P, int64_t rows, int parts, const float *partials,
                                  int64_t row_stride, int64_t part_stride, bool final, float *out, cudaStream_t s);
bool decode_mma_supported(const Prepared &P, const ScoreProblem &sp, bool attend);
int decode_mma_splits(const ScoreProblem &sp);
cudaError_t launch_decode_mma(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale,
                              float *out, int splits, bool attend, cudaStream_t s);

// Bit-plane integer tensor-core attention and scores (tq_attend_planes.cu): up to four query
// rows per KV head, head_dim 64/128/256 with proj_dim = head_dim / 2.
struct PlanesPlan {
    int range;   // tokens per CTA
    int splits;  // CTAs per (batch, KV head)
};
bool planes_supported(const Prepared &P, const ScoreProblem &sp, bool attend);
PlanesPlan plan_planes(const ScoreProblem &sp);
size_t planes_frag_bytes(const Prepared &P, const ScoreProblem &sp);
// Query operands (rotation and projection of the queries included), then scores (attend =
// false: out = scores [B, Hq, Nq, T]) or the attention output (attend = true: out = [B, Hq, Nq, d],
// through per-range partials [rows, splits, d + 2] that the last CTA of each slice merges).
cudaError_t launch_planes(const Prepared &P, const ScoreProblem &sp, float scale, uint32_t *frag,
                          const PlanesPlan &pl, bool attend, float *out, float *partials, cudaStream_t s,
                          bool merged_partial = false);

// Which attention kernel a problem uses and how many context splits it takes.
struct AttendPlan {
    bool planes;
    bool mma;
    int splits;
    PlanesPlan pp;
};
inline AttendPlan plan_attend(const Prepared &P, const ScoreProblem &sp) {
    AttendPlan a;
    a.planes = planes_supported(P, sp, true);
    a.mma = !a.planes && decode_mma_supported(P, sp, true);
    a.pp = plan_planes(sp);
    a.splits = a.planes ? a.pp.splits : a.mma ? decode_mma_splits(sp) : attend_splits(sp);
    return a;
}
size_t topk_scratch_bytes(const Prepared &P, const ScoreProblem &sp, int topk);

// Many query rows per (batch, KV head): tensor-core scores with an optional fused top-k.
bool search_tc_supported(const Prepared &P, const ScoreProblem &sp, int topk);
size_t search_scratch_bytes(const Prepared &P, const ScoreProblem &sp, int topk);
// fp16: single fp16 operand products (tq_search) instead of the hi + lo splits (tq_scores)
cudaError_t launch_search(const Prepared &P, const ScoreProblem &sp, const float *qprep, void *scratch,
                          float *scores, int topk, int32_t *topk_idx, float *topk_val, int32_t *dev_status,
                          cudaStream_t s, bool fp16 = false);

// Which kernels tq_scores runs: the tensor-core search (top-k fused when short enough), the
// register-MMA decode kernel (few rows), or the plain kernel; a separate top-k pass otherwise.
struct ScoresPlan {
    bool search;      // launch_search
    bool fused_topk;  // the search keeps the top-k itself
    bool planes;      // launch_planes in scores mode
    bool mma;         // launch_decode_mma in scores mode
};
inline ScoresPlan plan_scores(const Prepared &P, const ScoreProblem &sp, int topk) {
    ScoresPlan a;
    a.fused_topk = topk > 0 && search_tc_supported(P, sp, topk);
    a.search = a.fused_topk || search_tc_supported(P, sp, 0);
    a.planes = !a.search && planes_supported(P, sp, false);
    a.mma = !a.search && !a.planes && decode_mma_supported(P, sp, false);
    return a;
}

cudaError_t launch_qprep(const Prepared &P, const ScoreProblem &sp, float *qprep, cudaStream_t s);
cudaError_t launch_scores(const Prepared &P, const ScoreProblem &sp, const float *qprep,
                          float *scores, cudaStream_t s);
cudaError_t launch_topk(const ScoreProblem &sp, const float *scores, int topk, int32_t *idx,
                        float *val, cudaStream_t s);
// final = false: out is the merged partial [rows, d + 2] (max, sum, o_rot) instead of [rows, d]
cudaError_t launch_attend(const Prepared &P, const ScoreProblem &sp, const float *qprep,
                          float scale, float *partials, int splits, float *out, cudaStream_t s, bool final = true);

}  // namespace tq
