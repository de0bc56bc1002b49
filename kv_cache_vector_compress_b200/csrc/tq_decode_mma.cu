// tq_decode_mma.cu -- scores and fused decode attention over packed keys/values with
// warp-level tensor-core MMAs whose operands are decoded straight into registers.
//
// Math (asymmetric scores from the compressed keys, softmax, weighted sum over the MSE-
// dequantized values; "turboquant-pytorch", nav.superapi.store, 常见使用模式 and 核心 API):
//   s_tr = ||k_t|| ( <q_rot_r, c[kidx_t]> + rho_t sqrt(pi/2)/m <sq_r, 2 sign_t - 1> )
//   o_rot_r = sum_t softmax_t(scale s_tr) ||v_t|| c[vidx_t],   out_r = R^T o_rot_r
// Per warp and 16-token block, three m16n8k16 products (fp16 operands, fp32 accumulate):
//   C1[t, r] = Khat[t, :] . Qrot[r, :]      A = decoded key centroids, B = rotated queries
//   C2[t, r] = Sgn[t, :]  . SQ[r, :]        A = +-1 sign matrix,        B = S q
//   O[j, r] += Vhat[j, t] . P[t, r]         A = decoded value centroids, B = probabilities
// The A fragments come from the planar code words with shifts, masks and a small pair
// look-up table in shared memory (two fp16 centroids per 32-bit entry); the queries stay in
// registers.  With SPLIT the centroids and queries are carried as fp16 hi + lo pairs (three
// products), which keeps the raw scores at fp32-level accuracy; fused attention uses the
// single product, whose error is far below the output tolerance after the softmax average.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kThreadsMma = 128;
constexpr int kStageTok = 128;
constexpr int kRowsPerCta = 8;

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t lut_at(const uint32_t *lut, uint32_t byte_offset) {
    return *(const uint32_t *)((const char *)lut + byte_offset);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    return (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
}

// power-of-two scale that brings max|x| into [2^9, 2^10)
__device__ __forceinline__ int scale_exp(float maxabs) {
    if (!(maxabs > 0.f) || !isfinite(maxabs)) return 0;
    int e;
    frexpf(maxabs, &e);  // maxabs = f * 2^e, f in [0.5, 1)
    return 10 - e;
}

struct MmaSmem {
    uint32_t klut, klut_lo, slut, vlut, rowsc, stage, ptile, total;
    uint32_t stage_bytes, kc, ks, vc, kn, kr, vn;
};

__host__ __device__ inline MmaSmem mma_smem_layout(int D, int KB, int VB, int m) {
    MmaSmem L;
    uint32_t o = 0;
    L.klut = o;
    o += 64 * 4;
    L.klut_lo = o;
    o += 64 * 4;
    L.slut = o;
    o += 16 * 4;
    L.vlut = o;
    o += 64 * 4;
    L.rowsc = o;
    o += 4 * kRowsPerCta * 4;
    L.ptile = o;
    o += 4 * kRowsPerCta * 16 * 2;
    o = (o + 15) & ~15u;
    const uint32_t g32 = D / 32;
    L.kc = 0;
    L.ks = L.kc + kStageTok * KB * g32 * 4;
    L.vc = L.ks + kStageTok * (m / 32) * 4;
    L.kn = L.vc + kStageTok * VB * g32 * 4;
    L.kr = L.kn + kStageTok * 2;
    L.vn = L.kr + kStageTok * 2;
    L.stage_bytes = (L.vn + kStageTok * 2 + 15) & ~15u;
    L.stage = o;
    o += 2 * L.stage_bytes;
    // the cross-warp combine reuses the stage buffers: 4 warps x 8 rows x (D + 2) floats
    const uint32_t comb = 4u * kRowsPerCta * (D + 2) * 4;
    if (o < L.stage + comb) o = L.stage + comb;
    L.total = o;
    return L;
}

template <int D, int KB, int VB, bool ATTEND>
__global__ void __launch_bounds__(kThreadsMma) decode_mma_kernel(Prepared P, ScoreProblem sp,
                                                                 const float *__restrict__ qprep, float scale,
                                                                 float *__restrict__ out, int splits,
                                                                 int row_groups) {
    constexpr int G32 = D / 32;
    constexpr int KSTEP = D / 16;
    constexpr int KWPT = KB * G32;
    constexpr int VWPT = VB * G32;
    // Scores are always carried at split precision: with large key norms (outlier channels) a
    // single fp16 product moves the softmax logits by more than the output tolerance allows.
    constexpr bool SPLIT = true;
    constexpr int MSTEP = KSTEP / 2;  // proj_dim = head_dim / 2
    const int m = P.m;
    constexpr int SW = MSTEP / 2;
    const MmaSmem L = mma_smem_layout(D, KB, ATTEND ? VB : 0, m);

    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *klut = (uint32_t *)(smem + L.klut);
    uint32_t *klut_lo = (uint32_t *)(smem + L.klut_lo);
    uint32_t *slut = (uint32_t *)(smem + L.slut);
    uint32_t *vlut = (uint32_t *)(smem + L.vlut);
    float *rowsc = (float *)(smem + L.rowsc);  // [4][8]: q scale, sq scale, real row flag, spare

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
    const int64_t t0 = (int64_t)split * chunk;
    const int64_t t1 = min(sp.T, t0 + chunk);
    const int stride = P.d + m;
    const float gamma = sqrtf(1.5707963267948966f) / (float)m;

    // ---- codebook scales and pair look-up tables
    float kmax = 0.f, vmax = 0.f;
    for (int k = 0; k < (1 << KB); ++k) kmax = fmaxf(kmax, fabsf(P.cb->kc[k]));
    if (ATTEND)
        for (int k = 0; k < (1 << VB); ++k) vmax = fmaxf(vmax, fabsf(P.cb->vc[k]));
    const int ek = scale_exp(kmax), ev = scale_exp(vmax);
    const float ksc = ldexpf(1.f, ek), vsc = ldexpf(1.f, ev);
    for (int e = tid; e < (1 << (2 * KB)); e += kThreadsMma) {
        // index bits: plane p of (coord j, coord j+1) at bits (2p, 2p+1)
        int i0 = 0, i1 = 0;
        for (int p = 0; p < KB; ++p) {
            i0 |= ((e >> (2 * p)) & 1) << p;
            i1 |= ((e >> (2 * p + 1)) & 1) << p;
        }
        const float a0 = P.cb->kc[i0] * ksc, a1 = P.cb->kc[i1] * ksc;
        klut[e] = pack_h2(a0, a1);
        const float h0 = __half2float(__float2half_rn(a0)), h1 = __half2float(__float2half_rn(a1));
        klut_lo[e] = pack_h2(a0 - h0, a1 - h1);
    }
    if (tid < 4) {
        // sign pair: bit0 -> projection j, bit1 -> projection j+1; 1 -> +1, 0 -> -1
        slut[tid] = pack_h2((tid & 1) ? 1.f : -1.f, (tid & 2) ? 1.f : -1.f);
    }
    if (ATTEND) {
        for (int e = tid; e < (1 << (2 * VB)); e += kThreadsMma) {
            // low VB bits: token 2i, next VB bits: token 2i+1 (same coordinate)
            const float a0 = P.cb->vc[e & ((1 << VB) - 1)] * vsc, a1 = P.cb->vc[e >> VB] * vsc;
            vlut[e] = pack_h2(a0, a1);
        }
    }
    // ---- per-row query scales and B fragments (row gid of this CTA's group)
    if (tid < kRowsPerCta) {
        float qm = 0.f, sm_ = 0.f;
        if (tid < nrows) {
            const int rr = r0 + tid;
            const int g = rr / sp.Nq, i = rr % sp.Nq;
            const int64_t qrow = ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
            const float *qp = qprep + qrow * stride;
            for (int j = 0; j < D; ++j) qm = fmaxf(qm, fabsf(qp[j]));
            for (int a = 0; a < m; ++a) sm_ = fmaxf(sm_, fabsf(qp[D + a]));
        }
        rowsc[tid] = (float)scale_exp(qm);
        rowsc[kRowsPerCta + tid] = (float)scale_exp(sm_);
    }
    __syncthreads();
    uint32_t bq[KSTEP][2], bql[KSTEP][2], bs[MSTEP][2], bsl[MSTEP][2];
    {
        const bool real = gid < nrows;
        const float *qp = nullptr;
        if (real) {
            const int rr = r0 + gid;
            const int g = rr / sp.Nq, i = rr % sp.Nq;
            const int64_t qrow = ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
            qp = qprep + qrow * stride;
        }
        const float qs = ldexpf(1.f, (int)rowsc[gid]), ss = ldexpf(1.f, (int)rowsc[kRowsPerCta + gid]);
#pragma unroll
        for (int s = 0; s < KSTEP; ++s) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 16 * s + 8 * h + 2 * t4;
                float x0 = real ? qp[j] * qs : 0.f, x1 = real ? qp[j + 1] * qs : 0.f;
                bq[s][h] = pack_h2(x0, x1);
                bql[s][h] = pack_h2(x0 - __half2float(__float2half_rn(x0)), x1 - __half2float(__float2half_rn(x1)));
                if (s < MSTEP) {
                    const float y0 = real ? qp[D + j] * ss : 0.f, y1 = real ? qp[D + j + 1] * ss : 0.f;
                    bs[s < MSTEP ? s : 0][h] = pack_h2(y0, y1);
                    bsl[s < MSTEP ? s : 0][h] =
                        pack_h2(y0 - __half2float(__float2half_rn(y0)), y1 - __half2float(__float2half_rn(y1)));
                }
            }
        }
    }
    // unscale factors of the thread's two accumulator rows (2*t4, 2*t4+1)
    const float qun0 = ldexpf(1.f, -(int)rowsc[2 * t4] - ek), qun1 = ldexpf(1.f, -(int)rowsc[2 * t4 + 1] - ek);
    const float sun0 = ldexpf(1.f, -(int)rowsc[kRowsPerCta + 2 * t4]);
    const float sun1 = ldexpf(1.f, -(int)rowsc[kRowsPerCta + 2 * t4 + 1]);

    // ---- token stages
    uint8_t *stage0 = smem + L.stage;
    auto stage_ptr = [&](int s) { return stage0 + (s & 1) * L.stage_bytes; };
    const int64_t rec_base = sl * sp.T;
    uint16_t nk_reg = 0, nr_reg = 0, nv_reg = 0;
    auto issue = [&](int s, int64_t tb) {
        if (tb < t1) {
            const int ntok = (int)min((int64_t)kStageTok, t1 - tb);
            uint8_t *st = stage_ptr(s);
            const int64_t rec0 = rec_base + tb;
            uint32_t *dkc = (uint32_t *)(st + L.kc);
            const uint32_t *gkc = sp.kcodes + rec0 * KWPT;
            for (int i = tid; i < ntok * KWPT; i += kThreadsMma) cp_async4(dkc + i, gkc + i);
            uint32_t *dks = (uint32_t *)(st + L.ks);
            const uint32_t *gks = sp.ksigns + rec0 * SW;
            for (int i = tid; i < ntok * SW; i += kThreadsMma) cp_async4(dks + i, gks + i);
            if (ATTEND) {
                uint32_t *dvc = (uint32_t *)(st + L.vc);
                const uint32_t *gvc = sp.vcodes + rec0 * VWPT;
                for (int i = tid; i < ntok * VWPT; i += kThreadsMma) cp_async4(dvc + i, gvc + i);
            }
        }
        cp_async_commit();
    };
    auto load_norms = [&](int64_t tb) {
        if (tb < t1 && tid < min((int64_t)kStageTok, t1 - tb)) {
            const int64_t rec = rec_base + tb + tid;
            nk_reg = sp.knorm[rec];
            nr_reg = sp.krnorm[rec];
            if (ATTEND) nv_reg = sp.vnorm[rec];
        }
    };

    float oacc[ATTEND ? KSTEP : 1][4];
#pragma unroll
    for (int c = 0; c < (ATTEND ? KSTEP : 1); ++c) oacc[c][0] = oacc[c][1] = oacc[c][2] = oacc[c][3] = 0.f;
    float M0 = -INFINITY, M1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    uint16_t *ptile = (uint16_t *)(smem + L.ptile) + warp * (kRowsPerCta * 16);

    issue(0, t0);
    issue(1, t0 + kStageTok);
    load_norms(t0);
    int s = 0;
    for (int64_t tb = t0; tb < t1; tb += kStageTok, ++s) {
        uint8_t *st = stage_ptr(s);
        cp_async_wait<1>();
        {
            uint16_t *kn_s = (uint16_t *)(st + L.kn), *kr_s = (uint16_t *)(st + L.kr), *vn_s = (uint16_t *)(st + L.vn);
            kn_s[tid] = nk_reg;
            kr_s[tid] = nr_reg;
            if (ATTEND) vn_s[tid] = nv_reg;
        }
        __syncthreads();
        load_norms(tb + kStageTok);
        const int ntok = (int)min((int64_t)kStageTok, t1 - tb);
        const uint32_t *skc = (const uint32_t *)(st + L.kc);
        const uint32_t *sks = (const uint32_t *)(st + L.ks);
        const uint32_t *svc = (const uint32_t *)(st + L.vc);
        const uint16_t *skn = (const uint16_t *)(st + L.kn);
        const uint16_t *skr = (const uint16_t *)(st + L.kr);
        const uint16_t *svn = (const uint16_t *)(st + L.vn);
        for (int blk = warp; blk * 16 < ntok; blk += 4) {
            const int ob = blk * 16;
            const int ta = ob + gid, tb8 = ob + gid + 8;
            const bool va = ta < ntok, vb = tb8 < ntok;
            // ---------------- scores
            float cs[4] = {0.f, 0.f, 0.f, 0.f}, cd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int g = 0; g < G32; ++g) {
                uint32_t ya = 0, yb = 0;
#pragma unroll
                for (int p = 0; p < KB; ++p) {
                    ya |= ((skc[ta * KWPT + g * KB + p] >> (2 * t4)) & 0x03030303u) << (2 * p + 2);
                    yb |= ((skc[tb8 * KWPT + g * KB + p] >> (2 * t4)) & 0x03030303u) << (2 * p + 2);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int sh0 = 16 * h, sh1 = 16 * h + 8;
                    uint32_t a[4];
                    a[0] = lut_at(klut, (ya >> sh0) & 0xFFu);
                    a[1] = lut_at(klut, (yb >> sh0) & 0xFFu);
                    a[2] = lut_at(klut, (ya >> sh1) & 0xFFu);
                    a[3] = lut_at(klut, (yb >> sh1) & 0xFFu);
                    mma16816(cs, a, bq[2 * g + h][0], bq[2 * g + h][1]);
                    if (SPLIT) {
                        uint32_t al[4];
                        al[0] = lut_at(klut_lo, (ya >> sh0) & 0xFFu);
                        al[1] = lut_at(klut_lo, (yb >> sh0) & 0xFFu);
                        al[2] = lut_at(klut_lo, (ya >> sh1) & 0xFFu);
                        al[3] = lut_at(klut_lo, (yb >> sh1) & 0xFFu);
                        mma16816(cs, a, bql[2 * g + h][0], bql[2 * g + h][1]);
                        mma16816(cs, al, bq[2 * g + h][0], bq[2 * g + h][1]);
                    }
                }
            }
#pragma unroll
            for (int g = 0; g < SW; ++g) {
                {
                    const uint32_t ya = ((sks[ta * SW + g] >> (2 * t4)) & 0x03030303u) << 2;
                    const uint32_t yb = ((sks[tb8 * SW + g] >> (2 * t4)) & 0x03030303u) << 2;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int sh0 = 16 * h, sh1 = 16 * h + 8;
                        uint32_t a[4];
                        a[0] = lut_at(slut, (ya >> sh0) & 0xFFu);
                        a[1] = lut_at(slut, (yb >> sh0) & 0xFFu);
                        a[2] = lut_at(slut, (ya >> sh1) & 0xFFu);
                        a[3] = lut_at(slut, (yb >> sh1) & 0xFFu);
                        mma16816(cd, a, bs[2 * g + h][0], bs[2 * g + h][1]);
                        if (SPLIT) mma16816(cd, a, bsl[2 * g + h][0], bsl[2 * g + h][1]);
                    }
                }
            }
            const float kna = f16_bits_to_f32(skn[ta]), knb = f16_bits_to_f32(skn[tb8]);
            const float rna = f16_bits_to_f32(skr[ta]) * gamma, rnb = f16_bits_to_f32(skr[tb8]) * gamma;
            float sc[4];
            sc[0] = kna * fmaf(rna, cd[0] * sun0, cs[0] * qun0);
            sc[1] = kna * fmaf(rna, cd[1] * sun1, cs[1] * qun1);
            sc[2] = knb * fmaf(rnb, cd[2] * sun0, cs[2] * qun0);
            sc[3] = knb * fmaf(rnb, cd[3] * sun1, cs[3] * qun1);
            if (!ATTEND) {
                // raw scores out: rows 2*t4, 2*t4+1 of this group, tokens ta, tb8
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int rr = 2 * t4 + (e & 1);
                    const bool v = (e < 2) ? va : vb;
                    if (v && rr < nrows) {
                        const int row = r0 + rr;
                        const int g = row / sp.Nq, i = row % sp.Nq;
                        const int64_t qrow = ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
                        out[qrow * sp.T + tb + ((e < 2) ? ta : tb8)] = sc[e];
                    }
                }
                continue;
            }
            // ---------------- online softmax (rows 2*t4, 2*t4+1)
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
            // probabilities times value norms, transposed through shared memory
            const float vna = va ? f16_bits_to_f32(svn[ta]) : 0.f, vnb = vb ? f16_bits_to_f32(svn[tb8]) : 0.f;
            ptile[(2 * t4) * 16 + gid] = __half_as_ushort(__float2half_rn(p0 * vna));
            ptile[(2 * t4 + 1) * 16 + gid] = __half_as_ushort(__float2half_rn(p1 * vna));
            ptile[(2 * t4) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(p2 * vnb));
            ptile[(2 * t4 + 1) * 16 + gid + 8] = __half_as_ushort(__float2half_rn(p3 * vnb));
            __syncwarp();
            const uint32_t bp0 = *(const uint32_t *)(ptile + gid * 16 + 2 * t4);
            const uint32_t bp1 = *(const uint32_t *)(ptile + gid * 16 + 2 * t4 + 8);
            __syncwarp();
            // ---------------- values: A = Vhat^T (coords x tokens), pairs along tokens
            const int tk0 = ob + 2 * t4, tk8 = ob + 2 * t4 + 8;
#pragma unroll
            for (int g = 0; g < G32; ++g) {
                uint32_t z[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int tt = ((u & 2) ? tk8 : tk0) + (u & 1);
                    uint32_t acc = 0;
#pragma unroll
                    for (int p = 0; p < VB; ++p) acc |= ((svc[tt * VWPT + g * VB + p] >> gid) & 0x01010101u) << p;
                    z[u] = acc;
                }
                const uint32_t zz01 = (z[0] << 2) | (z[1] << (VB + 2));
                const uint32_t zz89 = (z[2] << 2) | (z[3] << (VB + 2));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t a[4];
                    a[0] = lut_at(vlut, (zz01 >> (16 * h)) & 0xFFu);
                    a[1] = lut_at(vlut, (zz01 >> (16 * h + 8)) & 0xFFu);
                    a[2] = lut_at(vlut, (zz89 >> (16 * h)) & 0xFFu);
                    a[3] = lut_at(vlut, (zz89 >> (16 * h + 8)) & 0xFFu);
                    mma16816(oacc[2 * g + h], a, bp0, bp1);
                }
            }
        }
        __syncthreads();
        issue(s + 2, tb + 2 * kStageTok);
    }
    cp_async_wait<0>();
    if (!ATTEND) return;

    // ---- combine the four warps' partial softmax states, write (M, L, o_rot) per row
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, o);
        l1 += __shfl_xor_sync(kFull, l1, o);
    }
    __syncthreads();
    float *comb = (float *)(smem + L.stage);  // [warp][row][D + 2]
    const float ounsc = ldexpf(1.f, -ev);
    {
        float *cw = comb + (size_t)warp * kRowsPerCta * (D + 2);
        if (gid == 0) {
            cw[(2 * t4) * (D + 2)] = M0;
            cw[(2 * t4) * (D + 2) + 1] = l0;
            cw[(2 * t4 + 1) * (D + 2)] = M1;
            cw[(2 * t4 + 1) * (D + 2) + 1] = l1;
        }
#pragma unroll
        for (int c = 0; c < KSTEP; ++c) {
            const int j0 = 16 * c + gid, j1 = j0 + 8;
            cw[(2 * t4) * (D + 2) + 2 + j0] = oacc[c][0] * ounsc;
            cw[(2 * t4 + 1) * (D + 2) + 2 + j0] = oacc[c][1] * ounsc;
            cw[(2 * t4) * (D + 2) + 2 + j1] = oacc[c][2] * ounsc;
            cw[(2 * t4 + 1) * (D + 2) + 2 + j1] = oacc[c][3] * ounsc;
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
        const int row = r0 + rr;
        const int g = row / sp.Nq, i = row % sp.Nq;
        const int64_t qrow = ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
        out[(qrow * splits + split) * (int64_t)(D + 2) + col] = v;
    }
}

template <int D, int KB, int VB, bool ATTEND>
cudaError_t launch_dm(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale, float *out,
                      int splits, cudaStream_t s) {
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int row_groups = (rows + kRowsPerCta - 1) / kRowsPerCta;
    const MmaSmem L = mma_smem_layout(D, KB, ATTEND ? VB : 0, P.m);
    auto kern = decode_mma_kernel<D, KB, VB, ATTEND>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)splits, (unsigned)((int64_t)sp.B * sp.Hkv * row_groups));
    kern<<<grid, kThreadsMma, L.total, s>>>(P, sp, qprep, scale, out, splits, row_groups);
    return cudaGetLastError();
}

template <int D, bool ATTEND>
cudaError_t launch_dm_bits(const Prepared &P, const ScoreProblem &sp, const float *qprep, float scale, float *out,
                           int splits, cudaStream_t s) {
    const int kb = P.kbeta, vb = P.vbeta;
    if constexpr (ATTEND) {
        if (kb == 1 && vb == 2) return launch_dm<D, 1, 2, true>(P, sp, qprep, scale, out, splits, s);
        if (kb == 2 && vb == 3) return launch_dm<D, 2, 3, true>(P, sp, qprep, scale, out, splits, s);
    } else {
        // scores only: the value bit width is irrelevant
        if (kb == 1) return launch_dm<D, 1, 1, false>(P, sp, qprep, scale, out, splits, s);
        if (kb == 2) return launch_dm<D, 2, 1, false>(P, sp, qprep, scale, out, splits, s);
        if (kb == 3) return launch_dm<D, 3, 1, false>(P, sp, qprep, scale, out, splits, s);
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
    if (attend) {
        const bool ok = (kb == 1 && vb == 2) || (kb == 2 && vb == 3);
        if (!ok) return false;
    } else {
        if (kb < 1 || kb > 3) return false;
    }
    return true;
}

int decode_mma_splits(const ScoreProblem &sp) {
    const int rows = (sp.Hq / sp.Hkv) * sp.Nq;
    const int64_t ctas = (int64_t)sp.B * sp.Hkv * ((rows + kRowsPerCta - 1) / kRowsPerCta);
    int64_t want = (148 * 8 + ctas - 1) / ctas;
    int64_t cap = (sp.T + 2 * kStageTok - 1) / (2 * kStageTok);
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
