// tq_search_tc.cu -- many queries against packed keys on the tensor cores, with a fused top-k.
//
// Nearest-neighbour search by estimated inner product (TurboQuantProd for vector databases:
// "TurboQuant er nå tilgjengelig som Python-bibliotek", jansverre.net, "Hva gjør
// Python-implementasjonen?"; the score is the asymmetric estimator of "turboquant-pytorch",
// nav.superapi.store, 核心 API):
//   s[r, t] = ||k_t|| ( <q_rot_r, c[idx_t]> + rho_t sqrt(pi/2)/m <sq_r, 2 sign_t - 1> )
// computed as two GEMMs per tile of 128 keys x 128 query rows, K streamed in 64-wide blocks:
//   ACC1 = C (centroids, fp16 hi + lo) x Qrot^T (fp16 hi + lo)    three products per block
//   ACC2 = Sgn (+-1, exact) x SQ^T (fp16 hi + lo)                  two products per block
// Decoder warps write the keys' A tiles straight into the 128-byte-swizzled shared-memory layout
// from the packed codes; the queries' B tiles (split and swizzled once per call) arrive by bulk
// copy; tcgen05 accumulates into one of two TMEM slots while the epilogue turns the other slot
// into scores, transposes them through shared memory and keeps each query row's running top-k.
// A merge kernel combines the per-CTA lists.  Every operand product is exact in fp32 up to the
// dropped lo x lo terms (relative 2^-22), so the result matches fp32 evaluation of the formula.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {

namespace {

using namespace sm100;

constexpr int kSTile = 128;                    // keys per tile (MMA M) and query rows per tile (MMA N)
constexpr int kSThreads = 448;                 // 14 warps
constexpr int kDecWarp0 = 2;                   // warps 2..9 decode key tiles
constexpr int kEpiWarp0 = 10;                  // warps 10..13 epilogue
constexpr int kSStages = 2;                    // shared-memory operand stages
constexpr uint32_t kOpTile = kSTile * 128;     // one 128 x 64 fp16 operand tile (16 KB)
constexpr uint32_t kStageBytes = 4 * kOpTile;  // A hi, A lo, B hi, B lo
constexpr int kScStride = kSTile + 1;          // transposed score tile row stride (floats)
constexpr int kSearchSms = 148;                // grid sizing (fixed so scratch sizes do not vary)
constexpr int kMaxFusedTopk = 16;              // longest per-row list kept in shared memory

struct SearchSmem {
    uint32_t stage, sc, lv, li, rowoff, klut, bars, misc, total;
};

__host__ __device__ inline SearchSmem search_smem_layout(int K) {
    SearchSmem L;
    uint32_t o = 0;
    L.stage = o;
    o += kSStages * kStageBytes;
    L.sc = o;
    o += kSTile * kScStride * 4;
    L.lv = o;
    o += kSTile * (K > 0 ? K : 1) * 4;
    L.li = o;
    o += kSTile * (K > 0 ? K : 1) * 4;
    o = (o + 15) & ~15u;
    L.rowoff = o;
    o += kSTile * 8;
    L.klut = o;
    o += 64 * 8;
    L.bars = o;
    o += 16 * 8;
    L.misc = o;
    o += 64;
    L.total = o;
    return L;
}

enum SBar { kBFull = 0, kAFull = 2, kSEmpty = 4, kAccFull = 6, kAccEmpty = 8 };

struct SearchGeom {
    int d, m;
    int R;        // query rows per (batch, KV head) slice: G * Nq
    int nrb;      // row blocks per slice
    int64_t nkt;  // key tiles per slice
    int units;    // slices * nrb
    int kc;       // CTAs per unit, each taking every kc-th key tile
    int nkb;      // K-blocks per tile: d/64 (centroids) + m/64 (signs)
};

inline SearchGeom search_geom(const Prepared &P, const ScoreProblem &sp) {
    SearchGeom g;
    g.d = P.d;
    g.m = P.m;
    g.R = (sp.Hq / sp.Hkv) * sp.Nq;
    g.nrb = (g.R + kSTile - 1) / kSTile;
    g.nkt = (sp.T + kSTile - 1) / kSTile;
    g.units = sp.B * sp.Hkv * g.nrb;
    int64_t kc = kSearchSms / g.units;
    if (kc < 1) kc = 1;
    if (kc > g.nkt) kc = g.nkt;
    g.kc = (int)kc;
    g.nkb = P.d / 64 + P.m / 64;
    return g;
}

// Global query row (b, kv * G + g, i) of row r of unit `unit`, or -1 past the slice's rows.
__device__ __forceinline__ int64_t search_qrow(const ScoreProblem &sp, const SearchGeom &g, int unit, int r) {
    const int sl = unit / g.nrb, rb = unit % g.nrb;
    const int rr = rb * kSTile + r;
    if (rr >= g.R) return -1;
    const int b = sl / sp.Hkv, kv = sl % sp.Hkv, G = sp.Hq / sp.Hkv;
    const int gi = rr / sp.Nq, i = rr % sp.Nq;
    return ((int64_t)b * sp.Hq + (int64_t)kv * G + gi) * sp.Nq + i;
}

__device__ __forceinline__ uint32_t pack_h2s(float lo, float hi) {
    return (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
}
__device__ __forceinline__ float hi16(float x) { return __half2float(__float2half_rn(x)); }
// Exponent e with maxabs * 2^e in [512, 1024): the fp16 operands stay far from overflow and
// their lo halves far from the subnormal range.
__device__ __forceinline__ int pow2_exp(float maxabs) {
    if (!(maxabs > 0.f) || !isfinite(maxabs)) return 0;
    int e;
    frexpf(maxabs, &e);
    return 10 - e;
}

// ------------------------------------------------------------------ query operands

// Per unit (slice, block of 128 query rows): one scale exponent for the rotated-query columns and
// one for the projected-query columns, and the B operand tiles -- fp16 hi | lo of the scaled
// values -- in the 128-byte-swizzled K-major layout, K-block by K-block.
__global__ void search_prep_kernel(ScoreProblem sp, SearchGeom g, const float *__restrict__ qprep,
                                   uint8_t *__restrict__ qsw, int *__restrict__ uexp) {
    __shared__ float red[2][32];
    __shared__ int ex[2];
    const int unit = blockIdx.x;
    const int d = g.d, m = g.m, stride = d + m;
    float qm = 0.f, sm = 0.f;
    for (int e = threadIdx.x; e < kSTile * stride; e += blockDim.x) {
        const int r = e / stride, col = e % stride;
        const int64_t qr = search_qrow(sp, g, unit, r);
        if (qr < 0) continue;
        const float v = fabsf(qprep[qr * stride + col]);
        if (col < d) qm = fmaxf(qm, v);
        else sm = fmaxf(sm, v);
    }
    qm = warp_max(qm);
    sm = warp_max(sm);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = qm;
        red[1][warp] = sm;
    }
    __syncthreads();
    if (threadIdx.x < 2) {
        float mx = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[threadIdx.x][w]);
        ex[threadIdx.x] = pow2_exp(mx);
        uexp[unit * 2 + threadIdx.x] = ex[threadIdx.x];
    }
    __syncthreads();
    const float s0 = ldexpf(1.f, ex[0]), s1 = ldexpf(1.f, ex[1]);
    uint8_t *base = qsw + (size_t)unit * g.nkb * 2 * kOpTile;
    for (int e = threadIdx.x; e < kSTile * stride; e += blockDim.x) {
        const int r = e / stride, col = e % stride;
        const int64_t qr = search_qrow(sp, g, unit, r);
        const bool sgn = col >= d;
        const float v = qr >= 0 ? qprep[qr * stride + col] * (sgn ? s1 : s0) : 0.f;
        const int kb = sgn ? d / 64 + (col - d) / 64 : col / 64;
        const int kk = (sgn ? col - d : col) & 63;
        const uint32_t off = (uint32_t)r * 128 + ((((uint32_t)kk >> 3) ^ (r & 7)) << 4) + (kk & 7) * 2;
        const __half h = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(h));
        *(__half *)(base + (size_t)kb * 2 * kOpTile + off) = h;
        *(__half *)(base + (size_t)kb * 2 * kOpTile + kOpTile + off) = lo;
    }
}

// ------------------------------------------------------------------------ GEMM

template <int KB>
__global__ void __launch_bounds__(kSThreads, 1)
    search_gemm_kernel(Prepared P, ScoreProblem sp, SearchGeom g, const uint8_t *__restrict__ qsw,
                       const int *__restrict__ uexp, float *__restrict__ scores, int K, float *__restrict__ cand_v,
                       int32_t *__restrict__ cand_i, int32_t *__restrict__ dev_status) {
    const int DKB = g.d / 64;          // centroid K-blocks
    const int KWPT = KB * (g.d / 32);  // code words per key
    const int SWPT = g.m / 32;         // sign words per key
    const int NKB = g.nkb;
    const SearchSmem L = search_smem_layout(K);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    float *sc = (float *)(sm + L.sc);
    float *lv = (float *)(sm + L.lv);
    int32_t *li = (int32_t *)(sm + L.li);
    int64_t *rowoff = (int64_t *)(sm + L.rowoff);
    uint2 *klut = (uint2 *)(sm + L.klut);
    uint32_t *tmem_s = (uint32_t *)(sm + L.misc);
    volatile int *abort_s = (volatile int *)(sm + L.misc + 4);
    int *kexp_s = (int *)(sm + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x / g.kc, cidx = blockIdx.x % g.kc;
    const int sl = unit / g.nrb;
    const int my_tiles = (int)((g.nkt - cidx + g.kc - 1) / g.kc);
    const int64_t rec_base = (int64_t)sl * sp.T;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&bars[kBFull + s], 1);
            mbar_init(&bars[kAFull + s], 8);
            mbar_init(&bars[kSEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kAccFull + s], 1);
            mbar_init(&bars[kAccEmpty + s], 4);
        }
        *abort_s = 0;
        float kmax = 0.f;
        for (int k = 0; k < (1 << KB); ++k) kmax = fmaxf(kmax, fabsf(P.cb->kc[k]));
        *kexp_s = pow2_exp(kmax);
        fence_mbar_init();
    }
    __syncthreads();
    {
        // centroid pair table (hi, lo) for two coordinates whose plane bits interleave in idx
        const float ksc = ldexpf(1.f, *kexp_s);
        for (int e = threadIdx.x; e < (1 << (2 * KB)); e += blockDim.x) {
            int i0 = 0, i1 = 0;
            for (int p = 0; p < KB; ++p) {
                i0 |= ((e >> (2 * p)) & 1) << p;
                i1 |= ((e >> (2 * p + 1)) & 1) << p;
            }
            const float a0 = P.cb->kc[i0] * ksc, a1 = P.cb->kc[i1] * ksc;
            klut[e] = make_uint2(pack_h2s(a0, a1), pack_h2s(a0 - hi16(a0), a1 - hi16(a1)));
        }
        for (int r = threadIdx.x; r < kSTile; r += blockDim.x) {
            const int64_t qr = search_qrow(sp, g, unit, r);
            rowoff[r] = qr < 0 ? -1 : qr * sp.T;
        }
        for (int e = threadIdx.x; e < kSTile * K; e += blockDim.x) {
            lv[e] = -INFINITY;
            li[e] = INT32_MAX;
        }
    }
    if (warp == 0) {
        tmem_alloc(tmem_s, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_s;
    const uint8_t *qsw_u = qsw + (size_t)unit * NKB * 2 * kOpTile;

    if (warp == 0) {
        // -------------------------------------------------------- query tiles (bulk copies)
        if (lane == 0) {
            const int total = my_tiles * NKB;
            int issued = 0;
            for (int gk = 0; gk < total; ++gk) {
                const int st = gk % kSStages;
                if (gk >= kSStages && !mbar_wait(&bars[kSEmpty + st], ((gk / kSStages) - 1) & 1, abort_s)) break;
                const int kbi = gk % NKB;
                mbar_arrive_expect_tx(&bars[kBFull + st], 2 * kOpTile);
                bulk_load(sm + L.stage + st * kStageBytes + 2 * kOpTile, qsw_u + (size_t)kbi * 2 * kOpTile,
                          2 * kOpTile, &bars[kBFull + st]);
                issued = gk + 1;
            }
            // every copy must land before the CTA can exit (bounded waits)
            int dummy = 0;
            for (int gk = issued > kSStages ? issued - kSStages : 0; gk < issued; ++gk)
                mbar_wait(&bars[kBFull + gk % kSStages], (gk / kSStages) & 1, (volatile int *)&dummy);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(kSTile, kSTile);
            const uint32_t sbase = smem_u32(sm + L.stage);
            bool ok = true;
            for (int i = 0; ok && i < my_tiles; ++i) {
                const int slot = i & 1;
                if (i >= 2 && !mbar_wait(&bars[kAccEmpty + slot], ((i >> 1) - 1) & 1, abort_s)) break;
                tc_fence_after();
                const uint32_t acc1 = tmem + slot * 256, acc2 = acc1 + kSTile;
                for (int kbi = 0; kbi < NKB; ++kbi) {
                    const int gk = i * NKB + kbi, st = gk % kSStages;
                    if (!mbar_wait(&bars[kAFull + st], (gk / kSStages) & 1, abort_s) ||
                        !mbar_wait(&bars[kBFull + st], (gk / kSStages) & 1, abort_s)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_hi = sbase + st * kStageBytes, a_lo = a_hi + kOpTile;
                    const uint32_t b_hi = a_hi + 2 * kOpTile, b_lo = a_hi + 3 * kOpTile;
                    if (kbi < DKB) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t o = k * 32;
                            mma_ss(acc1, sdesc_sw128(a_hi + o), sdesc_sw128(b_hi + o), idesc, (kbi | k) ? 1u : 0u);
                            mma_ss(acc1, sdesc_sw128(a_hi + o), sdesc_sw128(b_lo + o), idesc, 1u);
                            mma_ss(acc1, sdesc_sw128(a_lo + o), sdesc_sw128(b_hi + o), idesc, 1u);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t o = k * 32;
                            mma_ss(acc2, sdesc_sw128(a_hi + o), sdesc_sw128(b_hi + o), idesc,
                                   ((kbi - DKB) | k) ? 1u : 0u);
                            mma_ss(acc2, sdesc_sw128(a_hi + o), sdesc_sw128(b_lo + o), idesc, 1u);
                        }
                    }
                    mma_commit(&bars[kSEmpty + st]);
                }
                if (ok) mma_commit(&bars[kAccFull + slot]);
            }
        }
    } else if (warp < kEpiWarp0) {
        // -------------------------------------------------------- key tile decode
        const int dt = threadIdx.x - kDecWarp0 * 32;  // 0..255
        const int kr = dt & (kSTile - 1), half = dt >> 7;
        const int total = my_tiles * NKB;
        for (int gk = 0; gk < total; ++gk) {
            const int st = gk % kSStages, kbi = gk % NKB, i = gk / NKB;
            const int64_t t = (int64_t)(cidx + (int64_t)i * g.kc) * kSTile + kr;
            const bool valid = t < sp.T;
            // fetch the packed words before waiting for the stage to free up
            uint32_t w[KB];
            if (kbi < DKB) {
                const uint32_t *src = sp.kcodes + (rec_base + t) * KWPT + (2 * kbi + half) * KB;
#pragma unroll
                for (int p = 0; p < KB; ++p) w[p] = valid ? __ldg(src + p) : 0u;
            } else {
                w[0] = valid ? __ldg(sp.ksigns + (rec_base + t) * SWPT + 2 * (kbi - DKB) + half) : 0u;
            }
            if (gk >= kSStages && !mbar_wait(&bars[kSEmpty + st], ((gk / kSStages) - 1) & 1, abort_s)) break;
            uint8_t *a_hi = sm + L.stage + st * kStageBytes;
            uint8_t *a_lo = a_hi + kOpTile;
            const uint32_t rowb = (uint32_t)kr * 128;
            if (kbi < DKB) {
                // coordinates 64 kbi + 32 half + (0..31): one group of KB plane words
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t hv[4], lo4[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int bpos = 8 * cc + 2 * q;
                        uint32_t idx = 0;
#pragma unroll
                        for (int p = 0; p < KB; ++p) idx |= ((w[p] >> bpos) & 3u) << (2 * p);
                        const uint2 e = klut[idx];
                        hv[q] = valid ? e.x : 0u;
                        lo4[q] = valid ? e.y : 0u;
                    }
                    const uint32_t off = rowb + (((uint32_t)(4 * half + cc) ^ (kr & 7)) << 4);
                    *(uint4 *)(a_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                    *(uint4 *)(a_lo + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                }
            } else {
                // projections 64 (kbi - DKB) + 32 half + (0..31): one sign word, bit set = +1
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t hv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t b2 = w[0] >> (8 * cc + 2 * q);
                        // fp16 +1 is 0x3C00 and -1 is 0xBC00: the sign bit is the inverted code bit
                        const uint32_t v = 0x3C003C00u | ((~b2 & 1u) << 15) | ((~b2 & 2u) << 30);
                        hv[q] = valid ? v : 0u;
                    }
                    const uint32_t off = rowb + (((uint32_t)(4 * half + cc) ^ (kr & 7)) << 4);
                    *(uint4 *)(a_hi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                }
            }
            // generic-proxy stores must be visible to the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kAFull + st]);
        }
    } else {
        // -------------------------------------------------------- scores and top-k
        const int q4 = warp & 3;                      // TMEM lane quarter this warp may read
        const int row = 32 * q4 + lane;               // key within the tile
        const int et = threadIdx.x - kEpiWarp0 * 32;  // query row whose top-k this thread keeps
        const bool et_live = rowoff[et] >= 0;
        const float gamma = sqrtf(1.5707963267948966f) / (float)g.m;
        const float u1 = ldexpf(1.f, -(uexp[unit * 2] + *kexp_s));
        const float u2 = ldexpf(1.f, -uexp[unit * 2 + 1]);
        float *mv = lv + et * (K > 0 ? K : 1);
        int32_t *mi = li + et * (K > 0 ? K : 1);
        float thv = -INFINITY;
        int cnt = 0;
        for (int i = 0; i < my_tiles; ++i) {
            const int slot = i & 1;
            const int64_t t0 = (int64_t)(cidx + (int64_t)i * g.kc) * kSTile;
            const int64_t t = t0 + row;
            const bool valid = t < sp.T;
            float c1 = 0.f, c2 = 0.f, bias = -INFINITY;
            if (valid) {
                const float kn = f16_bits_to_f32(sp.knorm[rec_base + t]);
                c1 = kn * u1;
                c2 = kn * f16_bits_to_f32(sp.krnorm[rec_base + t]) * gamma * u2;
                bias = 0.f;
            }
            if (!mbar_wait(&bars[kAccFull + slot], (i >> 1) & 1, abort_s)) break;
            tc_fence_after();
            const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16) + slot * 256;
#pragma unroll 1
            for (int c = 0; c < kSTile / 32; ++c) {
                uint32_t a1[32], a2[32];
                tmem_ld32(tl + 32 * c, a1);
                tmem_ld32(tl + kSTile + 32 * c, a2);
                tmem_ld_wait();
#pragma unroll
                for (int l = 0; l < 32; ++l) {
                    const float s = fmaf(c2, __uint_as_float(a2[l]), fmaf(c1, __uint_as_float(a1[l]), bias));
                    sc[(32 * c + l) * kScStride + row] = s;
                }
                if (scores && valid) {
#pragma unroll 4
                    for (int l = 0; l < 32; ++l) {
                        const int64_t ro = rowoff[32 * c + l];
                        if (ro >= 0) scores[ro + t] = sc[(32 * c + l) * kScStride + row];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kAccEmpty + slot]);
            if (K > 0) {
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et_live) {
                    // keys arrive in increasing index order, so a tie never displaces an entry
                    const float *srow = sc + et * kScStride;
#pragma unroll 8
                    for (int kk = 0; kk < kSTile; ++kk) {
                        const float s = srow[kk];
                        if (s > thv) {
                            int pos = cnt < K ? cnt : K - 1;
                            while (pos > 0 && s > mv[pos - 1]) {
                                mv[pos] = mv[pos - 1];
                                mi[pos] = mi[pos - 1];
                                --pos;
                            }
                            mv[pos] = s;
                            mi[pos] = (int32_t)(t0 + kk);
                            if (cnt < K) ++cnt;
                            if (cnt == K) thv = mv[K - 1];
                        }
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
        }
        if (K > 0) {
            const size_t base = ((size_t)blockIdx.x * kSTile + et) * K;
            for (int j = 0; j < K; ++j) {
                cand_v[base + j] = mv[j];
                cand_i[base + j] = mi[j];
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_s && dev_status) atomicExch(dev_status, (int)TQ_ERR_TIMEOUT);
}

__device__ __forceinline__ bool search_better(float va, int32_t ia, float vb, int32_t ib) {
    return va > vb || (va == vb && ia < ib);
}

// Per query row (one warp): the best K of the kc per-CTA lists, score descending, ties to the
// smaller key index.
__global__ void search_merge_kernel(ScoreProblem sp, SearchGeom g, int K, const float *__restrict__ cand_v,
                                    const int32_t *__restrict__ cand_i, int32_t *__restrict__ oidx,
                                    float *__restrict__ oval) {
    const int unit = blockIdx.x / kSTile, r = blockIdx.x % kSTile;
    const int64_t qrow = search_qrow(sp, g, unit, r);
    if (qrow < 0) return;
    float bv[kMaxFusedTopk];
    int32_t bi[kMaxFusedTopk];
    int cnt = 0;
    const int n = g.kc * K;
    for (int e = threadIdx.x; e < n; e += 32) {
        const int c = e / K, j = e % K;
        const size_t src = (((size_t)unit * g.kc + c) * kSTile + r) * K + j;
        const float v = cand_v[src];
        const int32_t ix = cand_i[src];
        if (ix == INT32_MAX) continue;
        if (cnt == K && !search_better(v, ix, bv[K - 1], bi[K - 1])) continue;
        int pos = cnt < K ? cnt : K - 1;
        while (pos > 0 && search_better(v, ix, bv[pos - 1], bi[pos - 1])) {
            bv[pos] = bv[pos - 1];
            bi[pos] = bi[pos - 1];
            --pos;
        }
        bv[pos] = v;
        bi[pos] = ix;
        if (cnt < K) ++cnt;
    }
    int head = 0;
    for (int round = 0; round < K; ++round) {
        float v = head < cnt ? bv[head] : -INFINITY;
        int32_t ix = head < cnt ? bi[head] : INT32_MAX;
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, v, o);
            const int32_t oi = __shfl_xor_sync(kFull, ix, o);
            if (search_better(ov, oi, v, ix)) {
                v = ov;
                ix = oi;
            }
        }
        if (threadIdx.x == 0) {
            oidx[qrow * K + round] = ix;
            oval[qrow * K + round] = v;
        }
        if (head < cnt && bi[head] == ix) ++head;
    }
}

template <int KB>
cudaError_t launch_search_kb(const Prepared &P, const ScoreProblem &sp, const SearchGeom &g, const uint8_t *qsw,
                             const int *uexp, float *scores, int K, float *cv, int32_t *ci, int32_t *dev_status,
                             cudaStream_t s) {
    const SearchSmem L = search_smem_layout(K);
    const size_t smem = L.total + 1024;
    auto kern = search_gemm_kernel<KB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<g.units * g.kc, kSThreads, smem, s>>>(P, sp, g, qsw, uexp, scores, K, cv, ci, dev_status);
    return cudaGetLastError();
}

struct SearchScratch {
    size_t qsw, uexp, cv, ci, total;
};

SearchScratch search_scratch_layout(const SearchGeom &g, int topk) {
    SearchScratch S;
    size_t o = 0;
    S.qsw = o;
    o = align_up(o + (size_t)g.units * g.nkb * 2 * kOpTile, 256);
    S.uexp = o;
    o = align_up(o + (size_t)g.units * 2 * sizeof(int), 256);
    const size_t lists = (size_t)g.units * g.kc * kSTile * (topk > 0 ? topk : 0) * 4;
    S.cv = o;
    o = align_up(o + lists, 256);
    S.ci = o;
    o = align_up(o + lists, 256);
    S.total = o;
    return S;
}

}  // namespace

bool search_tc_supported(const Prepared &P, const ScoreProblem &sp, int topk) {
    if (P.d % 64 || P.m % 64 || P.m < 64) return false;
    if (P.kbeta < 1 || P.kbeta > 3) return false;
    if (topk < 0 || topk > kMaxFusedTopk) return false;
    return (sp.Hq / sp.Hkv) * sp.Nq > 64;
}

size_t search_scratch_bytes(const Prepared &P, const ScoreProblem &sp, int topk) {
    return search_scratch_layout(search_geom(P, sp), topk).total;
}

cudaError_t launch_search(const Prepared &P, const ScoreProblem &sp, const float *qprep, void *scratch,
                          float *scores, int topk, int32_t *topk_idx, float *topk_val, int32_t *dev_status,
                          cudaStream_t s) {
    const SearchGeom g = search_geom(P, sp);
    const SearchScratch S = search_scratch_layout(g, topk);
    uint8_t *base = (uint8_t *)scratch;
    uint8_t *qsw = base + S.qsw;
    int *uexp = (int *)(base + S.uexp);
    float *cv = (float *)(base + S.cv);
    int32_t *ci = (int32_t *)(base + S.ci);
    search_prep_kernel<<<g.units, 256, 0, s>>>(sp, g, qprep, qsw, uexp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (P.kbeta) {
        case 1: e = launch_search_kb<1>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 2: e = launch_search_kb<2>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 3: e = launch_search_kb<3>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess || topk == 0) return e;
    search_merge_kernel<<<g.units * kSTile, 32, 0, s>>>(sp, g, topk, cv, ci, topk_idx, topk_val);
    return cudaGetLastError();
}

}  // namespace tq
