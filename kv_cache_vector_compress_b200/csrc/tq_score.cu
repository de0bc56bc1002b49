// tq_score.cu -- query preparation, asymmetric scores, top-k and fused decode attention.
//
// Scores straight from packed keys (TurboQuantProd.inner_product / asymmetric attention
// scores; "turboquant-pytorch", nav.superapi.store, 核心 API and 常见使用模式):
//   s = ||k|| * ( <R q, c[idx]> + rho * sqrt(pi/2)/m * <S q, 2*sign - 1> )
// which equals <q, R^T c[idx]> + ... because R is orthogonal: the query is rotated once
// (q_rot = R q, sq = S q) instead of dequantizing every key.
// Attention: softmax(scale * s) over the tokens, then the weighted sum of the values'
// centroids in the rotated domain, o_rot = sum_t a_t ||v_t|| c[vidx_t], rotated back once
// per query (o = R^T o_rot).  Long contexts are split across CTAs (partial max, sum and
// o_rot per split) and combined with the usual log-sum-exp rescaling.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kTile = 128;     // tokens per CTA tile (one per thread)
constexpr int kMaxRows = 16;   // query rows handled per pass

inline int rows_per_pass(int d, int m, int cap_regs) {
    int by_smem = (int)((40 * 1024 / sizeof(float)) / (size_t)(d + m));
    int r = kMaxRows;
    if (by_smem < r) r = by_smem;
    if (cap_regs < r) r = cap_regs;
    return r < 1 ? 1 : r;
}

// ------------------------------------------------------------------ query prep

constexpr int kQpR = 64;    // query rows per block tile
constexpr int kQpC = 128;   // output coordinates per block tile
constexpr int kQpK = 16;    // input coordinates per shared-memory step

// q_rot = R q and sq = S q as one fp32 GEMM, out[r][i] = sum_j q[r][j] W[j][i] with
// W = [R^T | S^T]: 64 x 128 output tiles, 4 x 8 per thread (columns tx * 4 and 64 + tx * 4), the
// next step's operands loaded into registers while the current step computes.  Every output is
// accumulated by fmaf in ascending j, so the result does not depend on the tiling.
__global__ void __launch_bounds__(256) qprep_kernel(Prepared P, const float *__restrict__ q, int64_t rows,
                                                    float *__restrict__ out) {
    __shared__ __align__(16) float qs[kQpK][kQpR + 4];  // q tile, transposed
    __shared__ __align__(16) float ws[kQpK][kQpC];
    const int d = P.d, m = P.m, n = d + m;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int c0 = blockIdx.x * kQpC;
    // this thread's loads of a step: one float4 of q (row lr, k 4 lk4..) and two of W (k lw, columns
    // lc and lc + 64)
    const int lr = tid >> 2, lk4 = 4 * (tid & 3), lw = tid >> 4, lc = 4 * (tid & 15);
    auto wload = [&](int j, int c) -> float4 {
        const int i = c0 + c;
        if (i < d) return *(const float4 *)(P.RT + (int64_t)j * d + i);
        if (i < n) return *(const float4 *)(P.ST + (int64_t)j * m + (i - d));
        return make_float4(0.f, 0.f, 0.f, 0.f);
    };
    for (int64_t r0 = (int64_t)blockIdx.y * kQpR; r0 < rows; r0 += (int64_t)gridDim.y * kQpR) {
        float acc[4][8];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
        const bool qok = r0 + lr < rows;
        float4 gq = qok ? *(const float4 *)(q + (r0 + lr) * d + lk4) : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 gw0 = wload(lw, lc), gw1 = wload(lw, lc + 64);
        for (int k0 = 0; k0 < d; k0 += kQpK) {
            __syncthreads();  // the previous step's tiles are consumed
            qs[lk4 + 0][lr] = gq.x;
            qs[lk4 + 1][lr] = gq.y;
            qs[lk4 + 2][lr] = gq.z;
            qs[lk4 + 3][lr] = gq.w;
            *(float4 *)&ws[lw][lc] = gw0;
            *(float4 *)&ws[lw][lc + 64] = gw1;
            __syncthreads();
            if (k0 + kQpK < d) {
                const int k1 = k0 + kQpK;
                gq = qok ? *(const float4 *)(q + (r0 + lr) * d + k1 + lk4) : make_float4(0.f, 0.f, 0.f, 0.f);
                gw0 = wload(k1 + lw, lc);
                gw1 = wload(k1 + lw, lc + 64);
            }
#pragma unroll
            for (int k = 0; k < kQpK; ++k) {
                const float4 a4 = *(const float4 *)&qs[k][ty * 4];
                const float a[4] = {a4.x, a4.y, a4.z, a4.w};
                const float4 b0 = *(const float4 *)&ws[k][tx * 4];
                const float4 b1 = *(const float4 *)&ws[k][64 + tx * 4];
                const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int u = 0; u < 8; ++u) acc[t][u] = fmaf(b[u], a[t], acc[t][u]);
            }
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t r = r0 + ty * 4 + t;
            if (r >= rows) continue;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = c0 + (u < 4 ? tx * 4 + u : 64 + tx * 4 + (u - 4));
                if (i < n) out[r * n + i] = acc[t][u];
            }
        }
    }
}

// Accumulate, for one packed key and `rch` query rows, the MSE dot <q_rot, c[idx]>
// (acc) and the sign dot <sq, 2*sign-1> (acc2).
template <int RM>
__device__ __forceinline__ void key_dots(const Prepared &P, const float *cen, const float *qs,
                                         int rch, const uint32_t *kc, const uint32_t *ks,
                                         float *acc, float *acc2) {
    const int d = P.d, m = P.m, beta = P.kbeta, stride = d + m;
    for (int g = 0; g < (d >> 5); ++g) {
        uint32_t w[4] = {0, 0, 0, 0};
        for (int p = 0; p < beta; ++p) w[p] = kc[g * beta + p];
        for (int l = 0; l < 32; ++l) {
            int idx = 0;
            for (int p = 0; p < beta; ++p) idx |= ((w[p] >> l) & 1u) << p;
            const float c = cen[idx];
            const int j = 32 * g + l;
#pragma unroll
            for (int r = 0; r < RM; ++r)
                if (r < rch) acc[r] = fmaf(qs[r * stride + j], c, acc[r]);
        }
    }
    for (int g = 0; g < (m >> 5); ++g) {
        const uint32_t w = ks[g];
        for (int l = 0; l < 32; ++l) {
            const int a = 32 * g + l;
            const bool pos = (w >> l) & 1u;
#pragma unroll
            for (int r = 0; r < RM; ++r)
                if (r < rch) {
                    const float s = qs[r * stride + d + a];
                    acc2[r] += pos ? s : -s;
                }
        }
    }
}

__device__ __forceinline__ int64_t query_row(const ScoreProblem &sp, int b, int kv, int r) {
    const int G = sp.Hq / sp.Hkv;
    const int g = r / sp.Nq, i = r % sp.Nq;
    return ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
}

// --------------------------------------------------------------------- scores

__global__ void __launch_bounds__(kTile) scores_kernel(Prepared P, ScoreProblem sp,
                                                       const float *__restrict__ qprep, int rpp,
                                                       float *__restrict__ scores) {
    extern __shared__ float qs[];
    __shared__ float cen[kMaxLevels];
    const int d = P.d, m = P.m, stride = d + m;
    if (threadIdx.x < kMaxLevels) cen[threadIdx.x] = P.cb->kc[threadIdx.x];
    const int64_t sl = blockIdx.y;
    const int b = (int)(sl / sp.Hkv), kv = (int)(sl % sp.Hkv);
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int64_t t = (int64_t)blockIdx.x * kTile + threadIdx.x;
    const bool valid = t < sp.T;
    const int64_t rec = sl * sp.Ts + t;
    const float gamma = sqrtf(1.5707963267948966f) / (float)m;
    const int wpk = P.kbeta * (d >> 5), spk = m >> 5;
    float kn = 0.f, rn = 0.f;
    if (valid) {
        kn = f16_bits_to_f32(sp.knorm[rec]);
        rn = f16_bits_to_f32(sp.krnorm[rec]);
    }
    for (int r0 = 0; r0 < rows; r0 += rpp) {
        const int rch = min(rpp, rows - r0);
        __syncthreads();
        for (int e = threadIdx.x; e < rch * stride; e += blockDim.x) {
            const int r = e / stride, c = e % stride;
            qs[e] = qprep[query_row(sp, b, kv, r0 + r) * stride + c];
        }
        __syncthreads();
        if (valid) {
            float acc[kMaxRows], acc2[kMaxRows];
#pragma unroll
            for (int r = 0; r < kMaxRows; ++r) acc[r] = acc2[r] = 0.f;
            key_dots<kMaxRows>(P, cen, qs, rch, sp.kcodes + rec * wpk, sp.ksigns + rec * spk, acc, acc2);
#pragma unroll
            for (int r = 0; r < kMaxRows; ++r)
                if (r < rch)
                    scores[query_row(sp, b, kv, r0 + r) * sp.T + t] = kn * fmaf(rn * gamma, acc2[r], acc[r]);
        }
    }
}

// ---------------------------------------------------------------------- top-k

struct Cand {
    float v;
    int32_t i;
};

__device__ __forceinline__ bool better(float va, int32_t ia, float vb, int32_t ib) {
    return va > vb || (va == vb && ia < ib);
}

constexpr int kTopkThreads = 256;

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float *__restrict__ scores, int64_t T,
                                                            int k, int32_t *__restrict__ oidx,
                                                            float *__restrict__ oval) {
    const int64_t row = blockIdx.x;
    const float *s = scores + row * T;
    float lv[kMaxTopk];
    int32_t li[kMaxTopk];
    int cnt = 0;
    for (int64_t t = threadIdx.x; t < T; t += kTopkThreads) {
        const float v = s[t];
        const int32_t ti = (int32_t)t;
        if (cnt == k && !better(v, ti, lv[k - 1], li[k - 1])) continue;
        int pos = cnt < k ? cnt : k - 1;
        while (pos > 0 && better(v, ti, lv[pos - 1], li[pos - 1])) {
            lv[pos] = lv[pos - 1];
            li[pos] = li[pos - 1];
            --pos;
        }
        lv[pos] = v;
        li[pos] = ti;
        if (cnt < k) ++cnt;
    }
    // k rounds of a block-wide arg-max over the heads of the per-thread sorted lists
    __shared__ float wv[kTopkThreads / 32];
    __shared__ int32_t wi[kTopkThreads / 32];
    int head = 0;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int round = 0; round < k; ++round) {
        float v = head < cnt ? lv[head] : -INFINITY;
        int32_t i = head < cnt ? li[head] : INT32_MAX;
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, v, o);
            const int32_t oi = __shfl_xor_sync(kFull, i, o);
            if (better(ov, oi, v, i)) { v = ov; i = oi; }
        }
        if (lane == 0) { wv[warp] = v; wi[warp] = i; }
        __syncthreads();
        if (warp == 0) {
            v = lane < kTopkThreads / 32 ? wv[lane] : -INFINITY;
            i = lane < kTopkThreads / 32 ? wi[lane] : INT32_MAX;
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(kFull, v, o);
                const int32_t oi = __shfl_xor_sync(kFull, i, o);
                if (better(ov, oi, v, i)) { v = ov; i = oi; }
            }
            if (lane == 0) { wv[0] = v; wi[0] = i; oidx[row * k + round] = i; oval[row * k + round] = v; }
        }
        __syncthreads();
        if (head < cnt && li[head] == wi[0]) ++head;
        __syncthreads();
    }
}

// ------------------------------------------------------------------ attention

template <int CPT, int RM = (64 / CPT < kMaxRows ? 64 / CPT : kMaxRows)>
__global__ void __launch_bounds__(kTile) attend_kernel(Prepared P, ScoreProblem sp,
                                                       const float *__restrict__ qprep, int rpp,
                                                       float scale, float *__restrict__ partials,
                                                       int splits) {
    extern __shared__ float smem[];
    __shared__ float kcen[kMaxLevels], vcen[kMaxLevels];
    __shared__ float rowM[kMaxRows], rowL[kMaxRows], rowA[kMaxRows];
    const int d = P.d, m = P.m, stride = d + m;
    float *qs = smem;
    float *ps = smem + rpp * stride;
    if (threadIdx.x < kMaxLevels) {
        kcen[threadIdx.x] = P.cb->kc[threadIdx.x];
        vcen[threadIdx.x] = P.cb->vc[threadIdx.x];
    }
    const int split = blockIdx.x;
    const int64_t sl = blockIdx.y;
    const int b = (int)(sl / sp.Hkv), kv = (int)(sl % sp.Hkv);
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int64_t chunk = (sp.T + splits - 1) / splits;
    const int64_t t0 = (int64_t)split * chunk;
    const int64_t t1 = min(sp.T, t0 + chunk);
    const float gamma = sqrtf(1.5707963267948966f) / (float)m;
    const int wpk = P.kbeta * (d >> 5), spk = m >> 5, vwpv = P.vbeta * (d >> 5), vbeta = P.vbeta;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t rows_total = (int64_t)sp.B * sp.Hq * sp.Nq;

    for (int r0 = 0; r0 < rows; r0 += rpp) {
        const int rch = min(rpp, rows - r0);
        __syncthreads();
        for (int e = threadIdx.x; e < rch * stride; e += blockDim.x) {
            const int r = e / stride, c = e % stride;
            qs[e] = qprep[query_row(sp, b, kv, r0 + r) * stride + c];
        }
        if (threadIdx.x < kMaxRows) {
            rowM[threadIdx.x] = -INFINITY;
            rowL[threadIdx.x] = 0.f;
        }
        float o[RM][CPT];
#pragma unroll
        for (int r = 0; r < RM; ++r)
#pragma unroll
            for (int c = 0; c < CPT; ++c) o[r][c] = 0.f;
        __syncthreads();
        for (int64_t tb = t0; tb < t1; tb += kTile) {
            // scores of this tile, one token per thread
            const int64_t t = tb + threadIdx.x;
            const bool valid = t < t1;
            {
                float acc[RM], acc2[RM];
#pragma unroll
                for (int r = 0; r < RM; ++r) acc[r] = acc2[r] = 0.f;
                float kn = 0.f, rn = 0.f;
                if (valid) {
                    const int64_t rec = sl * sp.Ts + t;
                    kn = f16_bits_to_f32(sp.knorm[rec]);
                    rn = f16_bits_to_f32(sp.krnorm[rec]);
                    key_dots<RM>(P, kcen, qs, rch, sp.kcodes + rec * wpk, sp.ksigns + rec * spk, acc, acc2);
                }
#pragma unroll
                for (int r = 0; r < RM; ++r)
                    if (r < rch)
                        ps[r * kTile + threadIdx.x] =
                            valid ? scale * (kn * fmaf(rn * gamma, acc2[r], acc[r])) : -INFINITY;
            }
            __syncthreads();
            // online softmax bookkeeping: one warp per row
            for (int r = warp; r < rch; r += kTile / 32) {
                float mx = -INFINITY;
                for (int q = lane; q < kTile; q += 32) mx = fmaxf(mx, ps[r * kTile + q]);
                mx = warp_max(mx);
                const float oldM = rowM[r];
                const float newM = fmaxf(oldM, mx);
                const float alpha = (oldM == -INFINITY) ? 0.f : expf(oldM - newM);
                float sum = 0.f;
                for (int q = lane; q < kTile; q += 32) {
                    const float sv = ps[r * kTile + q];
                    const float e = (sv == -INFINITY) ? 0.f : expf(sv - newM);
                    ps[r * kTile + q] = e;
                    sum += e;
                }
                sum = warp_sum(sum);
                if (lane == 0) {
                    rowL[r] = rowL[r] * alpha + sum;
                    rowM[r] = newM;
                    rowA[r] = alpha;
                }
            }
            __syncthreads();
            // weighted value sum in the rotated domain; thread owns coordinates tid + 128c
#pragma unroll
            for (int r = 0; r < RM; ++r)
                if (r < rch) {
                    const float a = rowA[r];
#pragma unroll
                    for (int c = 0; c < CPT; ++c) o[r][c] *= a;
                }
            const int ntok = (int)min((int64_t)kTile, t1 - tb);
            for (int tt = 0; tt < ntok; ++tt) {
                const int64_t rec = sl * sp.Ts + tb + tt;
                const float vn = f16_bits_to_f32(sp.vnorm[rec]);
                const uint32_t *vw = sp.vcodes + rec * vwpv;
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int j = threadIdx.x + kTile * c;
                    if (j < d) {
                        const int g = j >> 5, l = j & 31;
                        int idx = 0;
                        for (int p = 0; p < vbeta; ++p) idx |= ((vw[g * vbeta + p] >> l) & 1u) << p;
                        const float w = vn * vcen[idx];
#pragma unroll
                        for (int r = 0; r < RM; ++r)
                            if (r < rch) o[r][c] = fmaf(ps[r * kTile + tt], w, o[r][c]);
                    }
                }
            }
            __syncthreads();
        }
        // partials[row][split] = (M, L, o_rot[d])
#pragma unroll
        for (int r = 0; r < RM; ++r)
            if (r < rch) {
                float *pp = partials + (query_row(sp, b, kv, r0 + r) * splits + split) * (int64_t)(d + 2);
                if (threadIdx.x == 0) {
                    pp[0] = rowM[r];
                    pp[1] = rowL[r];
                }
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int j = threadIdx.x + kTile * c;
                    if (j < d) pp[2 + j] = o[r][c];
                }
            }
    }
    (void)rows_total;
}

// Merge partials (max M_s, sum l_s, o_s) of each query row: element (row, s) starts at
// row * row_stride + s * part_stride.  final = true writes out = R^T (sum_s e^{M_s - M} o_s) /
// (sum_s e^{M_s - M} l_s) [rows, d]; final = false writes the merged partial (M, sum_s e^{M_s - M} l_s,
// sum_s e^{M_s - M} o_s) [rows, d + 2] in the rotated domain.  One block per row; the loads of a
// coordinate over the parts are issued eight at a time.
__global__ void __launch_bounds__(128) attend_combine_kernel(Prepared P, int64_t rows, int parts,
                                                             const float *__restrict__ partials,
                                                             int64_t row_stride, int64_t part_stride, int final,
                                                             float *__restrict__ out) {
    extern __shared__ float csm[];
    const int d = P.d;
    float *orot = csm;     // [d]
    float *wts = csm + d;  // [parts]
    __shared__ float lsum, mrow;
    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
        const float *pp = partials + row * row_stride;
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            float M = -INFINITY;
            for (int s = lane; s < parts; s += 32) M = fmaxf(M, pp[(int64_t)s * part_stride]);
            for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
            float L = 0.f;
            for (int s = lane; s < parts; s += 32) {
                const float *ps = pp + (int64_t)s * part_stride;
                const float w = (ps[0] == -INFINITY) ? 0.f : expf(ps[0] - M);
                wts[s] = w;
                L = fmaf(w, ps[1], L);
            }
            for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
            if (lane == 0) {
                lsum = L;
                mrow = M;
            }
        }
        __syncthreads();
        const float scl = final ? 1.f / lsum : 1.f;
        for (int j = threadIdx.x; j < d; j += blockDim.x) {
            const float *pj = pp + 2 + j;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            int s = 0;
            for (; s + 8 <= parts; s += 8) {
                float v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = pj[(int64_t)(s + u) * part_stride];
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[u] = fmaf(wts[s + u], v[u], acc[u]);
            }
            for (; s < parts; ++s) acc[0] = fmaf(wts[s], pj[(int64_t)s * part_stride], acc[0]);
            orot[j] = (((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]))) * scl;
        }
        __syncthreads();
        if (final) {
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int i = 0; i < d; i += 4) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) acc[u] = fmaf(P.R[(int64_t)(i + u) * d + j], orot[i + u], acc[u]);
                }
                out[row * d + j] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            }
        } else {
            float *po = out + row * (int64_t)(d + 2);
            if (threadIdx.x == 0) {
                po[0] = mrow;
                po[1] = lsum;
            }
            for (int j = threadIdx.x; j < d; j += blockDim.x) po[2 + j] = orot[j];
        }
        __syncthreads();
    }
}

}  // namespace

int attend_splits(const ScoreProblem &sp) {
    const int64_t slices = (int64_t)sp.B * sp.Hkv;
    int64_t want = (148 * 4 + slices - 1) / slices;
    int64_t cap = (sp.T + 255) / 256;
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return (int)want;
}

size_t qprep_bytes(const Prepared &P, const ScoreProblem &sp) {
    return align_up(sizeof(float) * (size_t)sp.B * sp.Hq * sp.Nq * (P.d + P.m), 256);
}

size_t attend_partials_bytes(const Prepared &P, const ScoreProblem &sp, int splits) {
    return align_up(sizeof(float) * (size_t)sp.B * sp.Hq * sp.Nq * splits * (P.d + 2), 256);
}

size_t topk_scratch_bytes(const Prepared &P, const ScoreProblem &sp, int topk) {
    (void)P;
    (void)topk;
    return align_up(sizeof(float) * (size_t)sp.B * sp.Hq * sp.Nq * (size_t)sp.T, 256);
}

cudaError_t launch_qprep(const Prepared &P, const ScoreProblem &sp, float *qprep, cudaStream_t s) {
    const int64_t rows = (int64_t)sp.B * sp.Hq * sp.Nq;
    const int64_t rtiles = (rows + kQpR - 1) / kQpR;
    dim3 grid((unsigned)((P.d + P.m + kQpC - 1) / kQpC), (unsigned)(rtiles < 65535 ? rtiles : 65535));
    qprep_kernel<<<grid, 256, 0, s>>>(P, sp.q, rows, qprep);
    return cudaGetLastError();
}

cudaError_t launch_scores(const Prepared &P, const ScoreProblem &sp, const float *qprep, float *scores,
                          cudaStream_t s) {
    const int rpp = rows_per_pass(P.d, P.m, kMaxRows);
    const size_t smem = sizeof(float) * (size_t)rpp * (P.d + P.m);
    dim3 grid((unsigned)((sp.T + kTile - 1) / kTile), (unsigned)(sp.B * sp.Hkv));
    cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    scores_kernel<<<grid, kTile, smem, s>>>(P, sp, qprep, rpp, scores);
    return cudaGetLastError();
}

cudaError_t launch_topk(const ScoreProblem &sp, const float *scores, int topk, int32_t *idx, float *val,
                        cudaStream_t s) {
    const int64_t rows = (int64_t)sp.B * sp.Hq * sp.Nq;
    topk_kernel<<<(unsigned)rows, kTopkThreads, 0, s>>>(scores, sp.T, topk, idx, val);
    return cudaGetLastError();
}

template <int CPT>
static cudaError_t launch_attend_cpt(const Prepared &P, const ScoreProblem &sp, const float *qprep,
                                     float scale, float *partials, int splits, cudaStream_t s) {
    const int rpp = rows_per_pass(P.d, P.m, 64 / CPT < kMaxRows ? 64 / CPT : kMaxRows);
    const size_t smem = sizeof(float) * ((size_t)rpp * (P.d + P.m) + (size_t)rpp * kTile);
    cudaFuncSetAttribute(attend_kernel<CPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((unsigned)splits, (unsigned)(sp.B * sp.Hkv));
    attend_kernel<CPT><<<grid, kTile, smem, s>>>(P, sp, qprep, rpp, scale, partials, splits);
    return cudaGetLastError();
}

cudaError_t launch_attend(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale,
                          float *partials, int splits, float *out, cudaStream_t s, bool final) {
    cudaError_t e;
    const int cpt = (P.d + kTile - 1) / kTile;
    switch (cpt) {
        case 1: e = launch_attend_cpt<1>(P, sp, qprep, scale, partials, splits, s); break;
        case 2: e = launch_attend_cpt<2>(P, sp, qprep, scale, partials, splits, s); break;
        case 4: e = launch_attend_cpt<4>(P, sp, qprep, scale, partials, splits, s); break;
        case 8: e = launch_attend_cpt<8>(P, sp, qprep, scale, partials, splits, s); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (!final)
        return launch_merge_partials(P, (int64_t)sp.B * sp.Hq * sp.Nq, splits, partials, (int64_t)splits * (P.d + 2),
                                     P.d + 2, false, out, s);
    return launch_attend_combine(P, sp, partials, splits, out, s);
}

cudaError_t launch_merge_partials(const Prepared &P, int64_t rows, int parts, const float *partials,
                                  int64_t row_stride, int64_t part_stride, bool final, float *out, cudaStream_t s) {
    const int blocks = (int)(rows < 148 * 16 ? rows : 148 * 16);
    const size_t smem = sizeof(float) * ((size_t)P.d + (size_t)parts);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(attend_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    attend_combine_kernel<<<blocks, 128, smem, s>>>(P, rows, parts, partials, row_stride, part_stride, final ? 1 : 0,
                                                    out);
    return cudaGetLastError();
}

cudaError_t launch_attend_combine(const Prepared &P, const ScoreProblem &sp, const float *partials, int splits,
                                  float *out, cudaStream_t s) {
    const int64_t rows = (int64_t)sp.B * sp.Hq * sp.Nq;
    return launch_merge_partials(P, rows, splits, partials, (int64_t)splits * (P.d + 2), P.d + 2, true, out, s);
}

}  // namespace tq
