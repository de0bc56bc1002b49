// tq_decode_mma.cu -- scores and fused decode attention over packed keys/values with
// warp-level tensor-core MMAs whose operands are decoded straight into registers.
//
// Math (asymmetric scores from the compressed keys, softmax, weighted sum over the MSE-
// dequantized values; "turboquant-pytorch", nav.superapi.store, 常见使用模式 and 核心 API):
//   s_tr = ||k_t|| ( <q_rot_r, c[kidx_t]> + rho_t sqrt(pi/2)/m <sq_r, 2 sign_t - 1> )
//   o_rot_r = sum_t softmax_t(scale s_tr) ||v_t|| c[vidx_t],   out_r = R^T o_rot_r
// Per warp and 16-token block, three kinds of m16n8k16 products (fp16 operands, fp32 accumulate):
//   C1[t, r] = Khat[t, :] . Qrot[r, :]      A = decoded key centroids, B = rotated queries
//   C2[t, r] = Sgn[t, :]  . SQ[r, :]        A = +-1 sign matrix,        B = S q
//   O[j, r] += Vhat[j, t] . P[t, r]         A = decoded value centroids, B = probabilities
// A fragments come from the planar code words with shifts, masks and small pair look-up tables
// in shared memory (two fp16 centroids per 32-bit entry; keys carry centroid hi + lo in one
// 64-bit entry); the queries stay in registers.  Scores are carried at split precision (centroid
// hi + lo, query hi + lo): with large key norms a single fp16 product moves the softmax logits by
// more than the output tolerance allows.  When a KV head has at most four query rows (decode with
// GQA group <= 4), the queries' hi and lo parts fill the eight MMA columns, so one product per
// centroid part carries both, and the halves are summed with one shuffle.
//
// Each warp streams its own contiguous token range through a two-stage cp.async ring (no block
// barrier in the main loop); the four warps' softmax states are merged at the end and written as
// one split-context partial (max, sum, o_rot) per row for attend_combine_kernel.
#include <math.h>

#include "tq_common.cuh"
#include "tq_compress_warp.cuh"
#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kThreadsMma = 128;
constexpr int kWarpStage = 32;  // tokens per warp stage (two 16-token blocks)
constexpr int kRowsPerCta = 8;

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int BYTES>
__device__ __forceinline__ void cp_async(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src), "n"(BYTES)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t lut32(const uint32_t *lut, uint32_t byte_offset) {
    return *(const uint32_t *)((const char *)lut + byte_offset);
}
__device__ __forceinline__ uint2 lut64(const uint2 *lut, uint32_t byte_offset) {
    return *(const uint2 *)((const char *)lut + byte_offset);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    return (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
}
__device__ __forceinline__ float hi_part(float x) { return __half2float(__float2half_rn(x)); }

// power-of-two scale that brings max|x| into [2^9, 2^10)
__device__ __forceinline__ int scale_exp(float maxabs) {
    if (!(maxabs > 0.f) || !isfinite(maxabs)) return 0;
    int e;
    frexpf(maxabs, &e);
    return 10 - e;
}

// Copy N consecutive 32-bit words (16-byte aligned when N % 4 == 0) into registers.
template <int N>
__device__ __forceinline__ void load_words(const uint32_t *p, uint32_t (&w)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const uint4 v = *(const uint4 *)(p + i);
            w[i] = v.x;
            w[i + 1] = v.y;
            w[i + 2] = v.z;
            w[i + 3] = v.w;
        }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            const uint2 v = *(const uint2 *)(p + i);
            w[i] = v.x;
            w[i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) w[i] = p[i];
    }
}

// Copy `words` 32-bit words from global to shared memory with the widest cp.async the
// per-record word count allows (records are 16/8/4-byte multiples and so is every offset).
template <int RECW>
__device__ __forceinline__ void stage_copy(uint32_t *dst, const uint32_t *src, int words, int lane) {
    constexpr int G = (RECW % 4 == 0) ? 4 : (RECW % 2 == 0) ? 2 : 1;
    for (int i = lane * G; i < words; i += 32 * G) cp_async<4 * G>(dst + i, src + i);
}

struct MmaSmem {
    uint32_t klut, slut, vlut, rowsc, ptile, stage, total;
    uint32_t stage_bytes, kc, ks, vc, kn, kr, vn;
    int nst;  // stages in each warp's ring
};

__host__ __device__ inline MmaSmem mma_smem_layout(int D, int KB, int VB, int m) {
    MmaSmem L;
    uint32_t o = 0;
    // 64-entry pair tables get one copy per lane (entry e of lane l at e * 256 + 8 l), so a
    // warp's random look-ups never conflict; smaller tables fit one bank row and the 256-entry
    // one stays shared
    L.klut = o;
    o += KB == 3 ? 64 * 32 * 8 : 64 * 8;
    L.slut = o;
    o += 16 * 4;
    L.vlut = o;
    o += VB == 3 ? 64 * 32 * 8 : 256 * 8;
    L.rowsc = o;
    o += 2 * kRowsPerCta * 4;
    L.ptile = o;
    o += 2 * 4 * kRowsPerCta * 16 * 2;  // per warp: P hi tile and P lo tile
    o = (o + 15) & ~15u;
    const uint32_t g32 = D / 32;
    L.kc = 0;
    L.ks = L.kc + kWarpStage * KB * g32 * 4;
    L.vc = L.ks + kWarpStage * (m / 32) * 4;
    // per-token fp16 norms: key, key residual, value; copied in 4-byte words from an even
    // record index, so one extra element on each side
    const uint32_t nb = ((kWarpStage + 2) * 2 + 15) & ~15u;
    L.kn = (L.vc + kWarpStage * VB * g32 * 4 + 15) & ~15u;
    L.kr = L.kn + nb;
    L.vn = L.kr + nb;
    L.stage_bytes = L.vn + nb;
    L.nst = 4 * 4 * L.stage_bytes <= 64u * 1024 ? 4 : 2;
    L.stage = o;
    o += 4 * L.nst * L.stage_bytes;  // 4 warps x nst stages
    const uint32_t comb = 4u * kRowsPerCta * (D + 2) * 4;
    if (o < L.stage + comb) o = L.stage + comb;
    L.total = o;
    return L;
}

template <int D, int KB, int VB, bool ATTEND, bool PACK4>
__global__ void __launch_bounds__(kThreadsMma) decode_mma_kernel(Prepared P, ScoreProblem sp,
                                                                 const float *__restrict__ qprep, float scale,
                                                                 float *__restrict__ out, int splits,
                                                                 int row_groups) {
    constexpr int G32 = D / 32;
    constexpr int KSTEP = D / 16;
    constexpr int MSTEP = KSTEP / 2;  // proj_dim = head_dim / 2
    constexpr int SW = MSTEP / 2;     // sign words per key
    constexpr int KWPT = KB * G32;
    constexpr int VWPT = VB * G32;
    constexpr int KSH = (KB <= 2) ? 3 : 2;  // key pair index scaled by 8 (or 4, then doubled)
    const int m = P.m;
    const MmaSmem L = mma_smem_layout(D, KB, ATTEND ? VB : 0, m);

    extern __shared__ __align__(16) uint8_t smem[];
    uint2 *klut = (uint2 *)(smem + L.klut);
    uint32_t *slut = (uint32_t *)(smem + L.slut);
    uint2 *vlut = (uint2 *)(smem + L.vlut);
    float *rowsc = (float *)(smem + L.rowsc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, t4 = lane & 3;
    const int split = blockIdx.x;
    const int64_t sl = blockIdx.y / row_groups;
    const int rg = blockIdx.y % row_groups;
    const int b = (int)(sl / sp.Hkv), kv = (int)(sl % sp.Hkv);
    const int G = sp.Hq / sp.Hkv;
    const int rows = G * sp.Nq;
    const int r0 = rg * kRowsPerCta;
    const int nrows = min(kRowsPerCta, rows - r0);
    const int64_t chunk = (sp.T + splits - 1) / splits;
    const int64_t t0 = min(sp.T, (int64_t)split * chunk);
    const int64_t t1 = min(sp.T, t0 + chunk);
    const int stride = P.d + m;
    const float gamma = sqrtf(1.5707963267948966f) / (float)m;
    auto qrow_of = [&](int rr) {
        const int row = r0 + rr;
        const int g = row / sp.Nq, i = row % sp.Nq;
        return ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
    };

    // ---- pair look-up tables and per-row query scales
    float kmax = 0.f, vmax = 0.f;
    for (int k = 0; k < (1 << KB); ++k) kmax = fmaxf(kmax, fabsf(P.cb->kc[k]));
    if (ATTEND)
        for (int k = 0; k < (1 << VB); ++k) vmax = fmaxf(vmax, fabsf(P.cb->vc[k]));
    const int ek = scale_exp(kmax), ev = scale_exp(vmax);
    const float ksc = ldexpf(1.f, ek), vsc = ldexpf(1.f, ev);
    constexpr int KCOPIES = KB == 3 ? 32 : 1, VCOPIES = VB == 3 ? 32 : 1;
    for (int ec = tid; ec < (1 << (2 * KB)) * KCOPIES; ec += kThreadsMma) {
        // index bits: plane p of (coordinate j, coordinate j+1) at bits (2p, 2p+1)
        const int e = ec / KCOPIES;
        int i0 = 0, i1 = 0;
        for (int p = 0; p < KB; ++p) {
            i0 |= ((e >> (2 * p)) & 1) << p;
            i1 |= ((e >> (2 * p + 1)) & 1) << p;
        }
        const float a0 = P.cb->kc[i0] * ksc, a1 = P.cb->kc[i1] * ksc;
        klut[ec] = make_uint2(pack_h2(a0, a1), pack_h2(a0 - hi_part(a0), a1 - hi_part(a1)));
    }
    if (tid < 4) slut[tid] = pack_h2((tid & 1) ? 1.f : -1.f, (tid & 2) ? 1.f : -1.f);
    if (ATTEND) {
        for (int ec = tid; ec < (1 << (2 * VB)) * VCOPIES; ec += kThreadsMma) {
            // low VB bits: token 2i, next VB bits: token 2i+1 (same coordinate); hi and lo fp16 parts
            const int e = ec / VCOPIES;
            const float a0 = P.cb->vc[e & ((1 << VB) - 1)] * vsc, a1 = P.cb->vc[e >> VB] * vsc;
            vlut[ec] = make_uint2(pack_h2(a0, a1), pack_h2(a0 - hi_part(a0), a1 - hi_part(a1)));
        }
    }
    if (tid < kRowsPerCta) {
        float qm = 0.f, smx = 0.f;
        if (tid < nrows) {
            const float *qp = qprep + qrow_of(tid) * stride;
            for (int j = 0; j < D; ++j) qm = fmaxf(qm, fabsf(qp[j]));
            for (int a = 0; a < m; ++a) smx = fmaxf(smx, fabsf(qp[D + a]));
        }
        rowsc[tid] = (float)scale_exp(qm);
        rowsc[kRowsPerCta + tid] = (float)scale_exp(smx);
    }
    uint16_t *ptile = (uint16_t *)(smem + L.ptile) + warp * (2 * kRowsPerCta * 16);
    uint16_t *ptile_lo = ptile + kRowsPerCta * 16;
    for (int e = lane; e < 2 * kRowsPerCta * 16; e += 32) ptile[e] = 0;
    // ---- decode-step append: a CTA whose token range holds record tnew first compresses the
    // slice's new key (warp 0) and value (warp 1) into the caches, then reads it back with the
    // rest of its range.  Every CTA of the slice that holds the record (one per row group)
    // writes the same bytes.  Scratch: the per-warp stage area, not yet in use.
    if constexpr (ATTEND) {
        if (sp.knew != nullptr && sp.tnew >= t0 && sp.tnew < t1 && warp < 2) {
            float *us = (float *)(smem + L.stage) + warp * D;
            const int64_t rec = sl * sp.Ts + sp.tnew;
            if (warp == 0) {
                if (sp.new_f16)
                    compress_vector_warp<G32, true, true>(P, sp.knew, sl, P.cb->kb, P.cb->kc, us, lane,
                                                          sp.kcodes_w + rec * KWPT, sp.ksigns_w + rec * SW,
                                                          sp.knorm_w + rec, sp.krnorm_w + rec);
                else
                    compress_vector_warp<G32, true, false>(P, sp.knew, sl, P.cb->kb, P.cb->kc, us, lane,
                                                           sp.kcodes_w + rec * KWPT, sp.ksigns_w + rec * SW,
                                                           sp.knorm_w + rec, sp.krnorm_w + rec);
            } else {
                if (sp.new_f16)
                    compress_vector_warp<G32, false, true>(P, sp.vnew, sl, P.cb->vb, P.cb->vc, us, lane,
                                                           sp.vcodes_w + rec * VWPT, nullptr, sp.vnorm_w + rec,
                                                           nullptr);
                else
                    compress_vector_warp<G32, false, false>(P, sp.vnew, sl, P.cb->vb, P.cb->vc, us, lane,
                                                            sp.vcodes_w + rec * VWPT, nullptr, sp.vnorm_w + rec,
                                                            nullptr);
            }
            __threadfence();
        }
    }
    __syncthreads();

    // ---- B fragments (queries) in registers
    // PACK4: column n = gid holds row (gid & 3), hi part for gid < 4 and lo part for gid >= 4.
    uint32_t bq[KSTEP][2], bql[PACK4 ? 1 : KSTEP][2], bs[MSTEP][2], bsl[PACK4 ? 1 : MSTEP][2];
    {
        const int brow = PACK4 ? (gid & 3) : gid;
        const bool lo_col = PACK4 && gid >= 4;
        const bool real = brow < nrows;
        const float *qp = real ? qprep + qrow_of(brow) * stride : nullptr;
        const float qs = ldexpf(1.f, (int)rowsc[brow]), ss = ldexpf(1.f, (int)rowsc[kRowsPerCta + brow]);
#pragma unroll
        for (int s = 0; s < KSTEP; ++s) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 16 * s + 8 * h + 2 * t4;
                const float x0 = real ? qp[j] * qs : 0.f, x1 = real ? qp[j + 1] * qs : 0.f;
                const float l0 = x0 - hi_part(x0), l1 = x1 - hi_part(x1);
                bq[s][h] = lo_col ? pack_h2(l0, l1) : pack_h2(x0, x1);
                if constexpr (!PACK4) bql[s][h] = pack_h2(l0, l1);
                if (s < MSTEP) {
                    const float y0 = real ? qp[D + j] * ss : 0.f, y1 = real ? qp[D + j + 1] * ss : 0.f;
                    const float m0 = y0 - hi_part(y0), m1 = y1 - hi_part(y1);
                    bs[s < MSTEP ? s : 0][h] = lo_col ? pack_h2(m0, m1) : pack_h2(y0, y1);
                    if constexpr (!PACK4) bsl[s < MSTEP ? s : 0][h] = pack_h2(m0, m1);
                }
            }
        }
    }
    // accumulator rows of this thread: (2*t4, 2*t4+1), or (2*(t4&1), +1) once PACK4 halves are summed
    const int ra = PACK4 ? 2 * (t4 & 1) : 2 * t4;
    const float qun0 = ldexpf(1.f, -(int)rowsc[ra] - ek), qun1 = ldexpf(1.f, -(int)rowsc[ra + 1] - ek);
    const float sun0 = ldexpf(1.f, -(int)rowsc[kRowsPerCta + ra]);
    const float sun1 = ldexpf(1.f, -(int)rowsc[kRowsPerCta + ra + 1]);
    const bool writes_p = !PACK4 || t4 < 2;

    // ---- this warp's token range and stage ring
    const int64_t wlen = (((t1 - t0) + 4 * 16 - 1) / (4 * 16)) * 16;
    const int64_t wt0 = min(t1, t0 + warp * wlen);
    const int64_t wt1 = min(t1, wt0 + wlen);
    const int NST = L.nst;
    uint8_t *wstage = smem + L.stage + (size_t)warp * NST * L.stage_bytes;
    const int64_t rec_base = sl * sp.Ts;
    const int64_t nrec = (int64_t)sp.B * sp.Hkv * sp.Ts;
    // fp16 norms of records [rec0, rec0 + ntok): 4-byte words from the even index below rec0; an
    // odd last element that would take its word past the end of the arrays is copied directly
    auto stage_norms = [&](uint16_t *dst, const uint16_t *src, int64_t rec0, int ntok) {
        const int64_t e0 = rec0 & ~(int64_t)1;
        const int64_t e1 = rec0 + ntok;
        const int words = (int)((e1 - e0) >> 1);
        for (int i = lane; i < words; i += 32) cp_async<4>((uint32_t *)dst + i, (const uint32_t *)(src + e0) + i);
        if (((e1 - e0) & 1) && lane == 0) {
            if (e1 + 1 <= nrec) cp_async<4>((uint32_t *)dst + words, (const uint32_t *)(src + e0) + words);
            else dst[2 * words] = src[e1 - 1];
        }
    };
    auto issue = [&](int s) {
        const int64_t tb = wt0 + (int64_t)s * kWarpStage;
        if (tb < wt1) {
            const int ntok = (int)min((int64_t)kWarpStage, wt1 - tb);
            uint8_t *st = wstage + (s % NST) * L.stage_bytes;
            const int64_t rec0 = rec_base + tb;
            stage_copy<KWPT>((uint32_t *)(st + L.kc), sp.kcodes + rec0 * KWPT, ntok * KWPT, lane);
            stage_copy<SW>((uint32_t *)(st + L.ks), sp.ksigns + rec0 * SW, ntok * SW, lane);
            if (ATTEND) stage_copy<VWPT>((uint32_t *)(st + L.vc), sp.vcodes + rec0 * VWPT, ntok * VWPT, lane);
            stage_norms((uint16_t *)(st + L.kn), sp.knorm, rec0, ntok);
            stage_norms((uint16_t *)(st + L.kr), sp.krnorm, rec0, ntok);
            if (ATTEND) stage_norms((uint16_t *)(st + L.vn), sp.vnorm, rec0, ntok);
        }
        cp_async_commit();
    };
    float oacc[ATTEND ? KSTEP : 1][4];
#pragma unroll
    for (int c = 0; c < (ATTEND ? KSTEP : 1); ++c) oacc[c][0] = oacc[c][1] = oacc[c][2] = oacc[c][3] = 0.f;
    float M0 = -INFINITY, M1 = -INFINITY, l0 = 0.f, l1 = 0.f;

    const int nstages = (int)((wt1 - wt0 + kWarpStage - 1) / kWarpStage);
    for (int k = 0; k < NST - 1; ++k) issue(k);
    for (int s = 0; s < nstages; ++s) {
        // the slot of stage s + NST - 1 was last read in iteration s - 1 (synchronised below)
        issue(s + NST - 1);
        if (NST == 4) cp_async_wait<3>();
        else cp_async_wait<1>();
        __syncwarp();
        const uint8_t *st = wstage + (s % NST) * L.stage_bytes;
        const int noff = (int)((rec_base + wt0 + (int64_t)s * kWarpStage) & 1);
        const uint16_t *skn = (const uint16_t *)(st + L.kn) + noff;
        const uint16_t *skr = (const uint16_t *)(st + L.kr) + noff;
        const uint16_t *svn = (const uint16_t *)(st + L.vn) + noff;
        const uint32_t *skc = (const uint32_t *)(st + L.kc);
        const uint32_t *sks = (const uint32_t *)(st + L.ks);
        const uint32_t *svc = (const uint32_t *)(st + L.vc);
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            const int ob = 16 * half;
            const int64_t gtb = wt0 + (int64_t)s * kWarpStage + ob;
            if (gtb >= wt1) break;
            const int ta = ob + gid, tb8 = ob + gid + 8;
            const bool va = gtb + gid < wt1, vb = gtb + gid + 8 < wt1;
            const float kna = va ? f16_bits_to_f32(skn[ta]) : 0.f, knb = vb ? f16_bits_to_f32(skn[tb8]) : 0.f;
            const float rna = va ? f16_bits_to_f32(skr[ta]) * gamma : 0.f;
            const float rnb = vb ? f16_bits_to_f32(skr[tb8]) * gamma : 0.f;
            const float vna = (ATTEND && va) ? f16_bits_to_f32(svn[ta]) : 0.f;
            const float vnb = (ATTEND && vb) ? f16_bits_to_f32(svn[tb8]) : 0.f;
            // ---------------- scores
            float cs[4] = {0.f, 0.f, 0.f, 0.f}, cd[4] = {0.f, 0.f, 0.f, 0.f};
            {
                uint32_t wa[KWPT], wb[KWPT];
                load_words<KWPT>(skc + ta * KWPT, wa);
                load_words<KWPT>(skc + tb8 * KWPT, wb);
#pragma unroll
                for (int g = 0; g < G32; ++g) {
                    uint32_t ya = 0, yb = 0;
#pragma unroll
                    for (int p = 0; p < KB; ++p) {
                        ya |= ((wa[g * KB + p] >> (2 * t4)) & 0x03030303u) << (2 * p + KSH);
                        yb |= ((wb[g * KB + p] >> (2 * t4)) & 0x03030303u) << (2 * p + KSH);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int sh0 = 16 * h, sh1 = 16 * h + 8;
                        uint32_t o[4] = {(ya >> sh0) & 0xFFu, (yb >> sh0) & 0xFFu, (ya >> sh1) & 0xFFu,
                                         (yb >> sh1) & 0xFFu};
                        uint32_t ah[4], al[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint2 e = KCOPIES > 1 ? lut64(klut, (o[u] << 6) + 8 * lane)
                                                        : lut64(klut, KSH == 3 ? o[u] : (o[u] << 1));
                            ah[u] = e.x;
                            al[u] = e.y;
                        }
                        mma16816(cs, ah, bq[2 * g + h][0], bq[2 * g + h][1]);
                        if constexpr (PACK4) {
                            mma16816(cs, al, bq[2 * g + h][0], bq[2 * g + h][1]);
                        } else {
                            mma16816(cs, ah, bql[2 * g + h][0], bql[2 * g + h][1]);
                            mma16816(cs, al, bq[2 * g + h][0], bq[2 * g + h][1]);
                        }
                    }
                }
                uint32_t sa[SW], sb[SW];
                load_words<SW>(sks + ta * SW, sa);
                load_words<SW>(sks + tb8 * SW, sb);
#pragma unroll
                for (int g = 0; g < SW; ++g) {
                    const uint32_t ya = ((sa[g] >> (2 * t4)) & 0x03030303u) << 2;
                    const uint32_t yb = ((sb[g] >> (2 * t4)) & 0x03030303u) << 2;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int sh0 = 16 * h, sh1 = 16 * h + 8;
                        uint32_t a[4];
                        a[0] = lut32(slut, (ya >> sh0) & 0xFFu);
                        a[1] = lut32(slut, (yb >> sh0) & 0xFFu);
                        a[2] = lut32(slut, (ya >> sh1) & 0xFFu);
                        a[3] = lut32(slut, (yb >> sh1) & 0xFFu);
                        mma16816(cd, a, bs[2 * g + h][0], bs[2 * g + h][1]);
                        if constexpr (!PACK4) mma16816(cd, a, bsl[2 * g + h][0], bsl[2 * g + h][1]);
                    }
                }
            }
            if constexpr (PACK4) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    cs[e] += __shfl_xor_sync(kFull, cs[e], 2);
                    cd[e] += __shfl_xor_sync(kFull, cd[e], 2);
                }
            }
            float sc[4];
            sc[0] = kna * fmaf(rna, cd[0] * sun0, cs[0] * qun0);
            sc[1] = kna * fmaf(rna, cd[1] * sun1, cs[1] * qun1);
            sc[2] = knb * fmaf(rnb, cd[2] * sun0, cs[2] * qun0);
            sc[3] = knb * fmaf(rnb, cd[3] * sun1, cs[3] * qun1);
            if constexpr (!ATTEND) {
                if (writes_p) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int rr = ra + (e & 1);
                        const bool v = (e < 2) ? va : vb;
                        if (v && rr < nrows) out[qrow_of(rr) * sp.T + gtb + ((e < 2) ? gid : gid + 8)] = sc[e];
                    }
                }
                continue;
            }
            // ---------------- online softmax (rows ra, ra+1)
            const float z0 = va ? scale * sc[0] : -INFINITY, z1 = va ? scale * sc[1] : -INFINITY;
            const float z2 = vb ? scale * sc[2] : -INFINITY, z3 = vb ? scale * sc[3] : -INFINITY;
            float bm0 = fmaxf(z0, z2), bm1 = fmaxf(z1, z3);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                bm0 = fmaxf(bm0, __shfl_xor_sync(kFull, bm0, o));
                bm1 = fmaxf(bm1, __shfl_xor_sync(kFull, bm1, o));
            }
            const float n0 = fmaxf(M0, bm0), n1 = fmaxf(M1, bm1);
            const float al0 = (M0 == -INFINITY) ? 0.f : __expf(M0 - n0);
            const float al1 = (M1 == -INFINITY) ? 0.f : __expf(M1 - n1);
            M0 = n0;
            M1 = n1;
            const float p0 = va ? __expf(z0 - n0) : 0.f, p1 = va ? __expf(z1 - n1) : 0.f;
            const float p2 = vb ? __expf(z2 - n0) : 0.f, p3 = vb ? __expf(z3 - n1) : 0.f;
            l0 = fmaf(l0, al0, p0 + p2);
            l1 = fmaf(l1, al1, p1 + p3);
            if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
                for (int c = 0; c < KSTEP; ++c) {
                    oacc[c][0] *= al0;
                    oacc[c][1] *= al1;
                    oacc[c][2] *= al0;
                    oacc[c][3] *= al1;
                }
            }
            // probabilities times value norms, split into fp16 hi + lo and transposed through shared
            // memory.  PACK4: tile rows 0..3 carry the hi parts (written by t4 < 2) and rows 4..7 the
            // lo parts of the same rows (written by t4 >= 2, which hold the same row values).
            {
                const float pa = va ? vna : 0.f, pb = vb ? vnb : 0.f;
                const float w[4] = {p0 * pa, p1 * pa, p2 * pb, p3 * pb};
                uint16_t hb[4], lb[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __half h = __float2half_rn(w[e]);
                    hb[e] = __half_as_ushort(h);
                    lb[e] = __half_as_ushort(__float2half_rn(w[e] - __half2float(h)));
                }
                if constexpr (PACK4) {
                    const int row = t4 < 2 ? ra : ra + 4;
                    const uint16_t *src = t4 < 2 ? hb : lb;
                    ptile[row * 16 + gid] = src[0];
                    ptile[(row + 1) * 16 + gid] = src[1];
                    ptile[row * 16 + gid + 8] = src[2];
                    ptile[(row + 1) * 16 + gid + 8] = src[3];
                } else {
                    ptile[ra * 16 + gid] = hb[0];
                    ptile[(ra + 1) * 16 + gid] = hb[1];
                    ptile[ra * 16 + gid + 8] = hb[2];
                    ptile[(ra + 1) * 16 + gid + 8] = hb[3];
                    ptile_lo[ra * 16 + gid] = lb[0];
                    ptile_lo[(ra + 1) * 16 + gid] = lb[1];
                    ptile_lo[ra * 16 + gid + 8] = lb[2];
                    ptile_lo[(ra + 1) * 16 + gid + 8] = lb[3];
                }
            }
            __syncwarp();
            const uint32_t bp0 = *(const uint32_t *)(ptile + gid * 16 + 2 * t4);
            const uint32_t bp1 = *(const uint32_t *)(ptile + gid * 16 + 2 * t4 + 8);
            uint32_t bl0 = 0, bl1 = 0;
            if constexpr (!PACK4) {
                bl0 = *(const uint32_t *)(ptile_lo + gid * 16 + 2 * t4);
                bl1 = *(const uint32_t *)(ptile_lo + gid * 16 + 2 * t4 + 8);
            }
            __syncwarp();
            // ---------------- values: A = Vhat^T (coordinates x tokens), pairs along tokens
            {
                const int tk = ob + 2 * t4;
                // pair index of (token 2i, token 2i+1) for one coordinate: 2*VB bits; for VB <= 3
                // the byte holds index*4 (the table offset), for VB == 4 the index itself
                constexpr int VSH = (VB <= 3) ? 2 : 0;
                auto value_group = [&](int g, const uint32_t *w0, const uint32_t *w1, const uint32_t *w8,
                                       const uint32_t *w9) {
                    uint32_t z0w = 0, z1w = 0, z8w = 0, z9w = 0;
#pragma unroll
                    for (int p = 0; p < VB; ++p) {
                        z0w |= ((w0[p] >> gid) & 0x01010101u) << p;
                        z1w |= ((w1[p] >> gid) & 0x01010101u) << p;
                        z8w |= ((w8[p] >> gid) & 0x01010101u) << p;
                        z9w |= ((w9[p] >> gid) & 0x01010101u) << p;
                    }
                    const uint32_t zz01 = (z0w << VSH) | (z1w << (VB + VSH));
                    const uint32_t zz89 = (z8w << VSH) | (z9w << (VB + VSH));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t o4[4] = {(zz01 >> (16 * h)) & 0xFFu, (zz01 >> (16 * h + 8)) & 0xFFu,
                                          (zz89 >> (16 * h)) & 0xFFu, (zz89 >> (16 * h + 8)) & 0xFFu};
                        uint32_t a[4];
                        uint32_t al[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const uint2 e = VCOPIES > 1 ? lut64(vlut, (o4[u] << 6) + 8 * lane)
                                                        : lut64(vlut, VSH ? (o4[u] << 1) : (o4[u] << 3));
                            a[u] = e.x;
                            al[u] = e.y;
                        }
                        mma16816(oacc[2 * g + h], a, bp0, bp1);
                        mma16816(oacc[2 * g + h], al, bp0, bp1);
                        if constexpr (!PACK4) mma16816(oacc[2 * g + h], a, bl0, bl1);
                    }
                };
                if constexpr (VB <= 3) {
                    uint32_t v0[VWPT], v1[VWPT], v8[VWPT], v9[VWPT];
                    load_words<VWPT>(svc + tk * VWPT, v0);
                    load_words<VWPT>(svc + (tk + 1) * VWPT, v1);
                    load_words<VWPT>(svc + (tk + 8) * VWPT, v8);
                    load_words<VWPT>(svc + (tk + 9) * VWPT, v9);
#pragma unroll
                    for (int g = 0; g < G32; ++g) value_group(g, v0 + g * VB, v1 + g * VB, v8 + g * VB, v9 + g * VB);
                } else {
#pragma unroll
                    for (int g = 0; g < G32; ++g) {
                        uint32_t v0[VB], v1[VB], v8[VB], v9[VB];
                        load_words<VB>(svc + tk * VWPT + g * VB, v0);
                        load_words<VB>(svc + (tk + 1) * VWPT + g * VB, v1);
                        load_words<VB>(svc + (tk + 8) * VWPT + g * VB, v8);
                        load_words<VB>(svc + (tk + 9) * VWPT + g * VB, v9);
                        value_group(g, v0, v1, v8, v9);
                    }
                }
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    if constexpr (!ATTEND) return;

    // ---- merge the four warps' softmax states, write (M, L, o_rot) per row
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, o);
        l1 += __shfl_xor_sync(kFull, l1, o);
    }
    if constexpr (PACK4) {
        // columns 4..7 (threads t4 >= 2) hold the lo-part products of rows 0..3
#pragma unroll
        for (int c = 0; c < KSTEP; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) oacc[c][e] += __shfl_xor_sync(kFull, oacc[c][e], 2);
    }
    __syncthreads();
    float *comb = (float *)(smem + L.stage);  // [warp][row][D + 2]
    const float ounsc = ldexpf(1.f, -ev);
    {
        float *cw = comb + (size_t)warp * kRowsPerCta * (D + 2);
        if (gid == 0 && writes_p) {
            cw[ra * (D + 2)] = M0;
            cw[ra * (D + 2) + 1] = l0;
            cw[(ra + 1) * (D + 2)] = M1;
            cw[(ra + 1) * (D + 2) + 1] = l1;
        }
        if (writes_p) {
#pragma unroll
            for (int c = 0; c < KSTEP; ++c) {
                const int j0 = 16 * c + gid, j1 = j0 + 8;
                cw[(2 * t4) * (D + 2) + 2 + j0] = oacc[c][0] * ounsc;
                cw[(2 * t4 + 1) * (D + 2) + 2 + j0] = oacc[c][1] * ounsc;
                cw[(2 * t4) * (D + 2) + 2 + j1] = oacc[c][2] * ounsc;
                cw[(2 * t4 + 1) * (D + 2) + 2 + j1] = oacc[c][3] * ounsc;
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < nrows * (D + 2); e += kThreadsMma) {
        const int rr = e / (D + 2), col = e % (D + 2);
        float Mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) Mx = fmaxf(Mx, comb[(w * kRowsPerCta + rr) * (D + 2)]);
        float v;
        if (col == 0) {
            v = Mx;
        } else {
            v = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float Mw = comb[(w * kRowsPerCta + rr) * (D + 2)];
                const float f = (Mw == -INFINITY) ? 0.f : __expf(Mw - Mx);
                v = fmaf(f, comb[(w * kRowsPerCta + rr) * (D + 2) + col], v);
            }
        }
        out[(qrow_of(rr) * splits + split) * (int64_t)(D + 2) + col] = v;
    }
}

template <int D, int KB, int VB, bool ATTEND, bool PACK4>
cudaError_t launch_dm(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale, float *out,
                      int splits, cudaStream_t s) {
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int row_groups = (rows + kRowsPerCta - 1) / kRowsPerCta;
    const MmaSmem L = mma_smem_layout(D, KB, ATTEND ? VB : 0, P.m);
    auto kern = decode_mma_kernel<D, KB, VB, ATTEND, PACK4>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)splits, (unsigned)((int64_t)sp.B * sp.Hkv * row_groups));
    kern<<<grid, kThreadsMma, L.total, s>>>(P, sp, qprep, scale, out, splits, row_groups);
    return cudaGetLastError();
}

template <int D, int KB, int VB, bool ATTEND>
cudaError_t launch_dm_pack(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale, float *out,
                           int splits, cudaStream_t s) {
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    if (rows <= 4) return launch_dm<D, KB, VB, ATTEND, true>(P, sp, qprep, scale, out, splits, s);
    return launch_dm<D, KB, VB, ATTEND, false>(P, sp, qprep, scale, out, splits, s);
}

template <int D, bool ATTEND>
cudaError_t launch_dm_bits(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale, float *out,
                           int splits, cudaStream_t s) {
    const int kb = P.kbeta, vb = P.vbeta;
    if constexpr (ATTEND) {
        if (kb == 1 && vb == 2) return launch_dm_pack<D, 1, 2, true>(P, sp, qprep, scale, out, splits, s);
        if (kb == 2 && vb == 3) return launch_dm_pack<D, 2, 3, true>(P, sp, qprep, scale, out, splits, s);
        if (kb == 3 && vb == 4) return launch_dm_pack<D, 3, 4, true>(P, sp, qprep, scale, out, splits, s);
    } else {
        // scores only: the value bit width is irrelevant
        if (kb == 1) return launch_dm_pack<D, 1, 1, false>(P, sp, qprep, scale, out, splits, s);
        if (kb == 2) return launch_dm_pack<D, 2, 1, false>(P, sp, qprep, scale, out, splits, s);
        if (kb == 3) return launch_dm_pack<D, 3, 1, false>(P, sp, qprep, scale, out, splits, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool decode_mma_supported(const Prepared &P, const ScoreProblem &sp, bool attend) {
    if (P.d != 64 && P.d != 128 && P.d != 256) return false;
    if (P.m * 2 != P.d) return false;  // proj_dim = head_dim / 2
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    if (!attend && rows > 64) return false;
    const int kb = P.kbeta, vb = P.vbeta;
    if (attend) return vb == kb + 1 && kb >= 1 && kb <= 3;
    return kb >= 1 && kb <= 3;
}

int decode_mma_splits(const ScoreProblem &sp) {
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int64_t ctas = (int64_t)sp.B * sp.Hkv * ((rows + kRowsPerCta - 1) / kRowsPerCta);
    int64_t want = (148 * 8 + ctas - 1) / ctas;
    int64_t cap = (sp.T + 4 * 2 * kWarpStage - 1) / (4 * 2 * kWarpStage);
    if (want > cap) want = cap;
    if (want < 1) want = 1;
    return (int)want;
}

cudaError_t launch_decode_mma(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale,
                              float *out, int splits, bool attend, cudaStream_t s) {
    switch (P.d) {
        case 64:
            return attend ? launch_dm_bits<64, true>(P, sp, qprep, scale, out, splits, s)
                          : launch_dm_bits<64, false>(P, sp, qprep, scale, out, splits, s);
        case 128:
            return attend ? launch_dm_bits<128, true>(P, sp, qprep, scale, out, splits, s)
                          : launch_dm_bits<128, false>(P, sp, qprep, scale, out, splits, s);
        case 256:
            return attend ? launch_dm_bits<256, true>(P, sp, qprep, scale, out, splits, s)
                          : launch_dm_bits<256, false>(P, sp, qprep, scale, out, splits, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
