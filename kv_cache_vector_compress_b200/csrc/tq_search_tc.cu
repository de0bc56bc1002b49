// tq_search_tc.cu -- many queries against packed keys on the tensor cores, with a fused top-k.
//
// Nearest-neighbour search by estimated inner product (TurboQuantProd for vector databases:
// "TurboQuant er nå tilgjengelig som Python-bibliotek", jansverre.net, "Hva gjør
// Python-implementasjonen?"; the score is the asymmetric estimator of "turboquant-pytorch",
// nav.superapi.store, 核心 API):
//   s[r, t] = ||k_t|| ( <q_rot_r, c[idx_t]> + rho_t sqrt(pi/2)/m <sq_r, 2 sign_t - 1> )
// computed per tile of 128 keys x 128 query rows as one GEMM with K = d + m, streamed in
// 64-wide blocks into a single fp32 accumulator:
//   centroid blocks: C (fp16 hi + lo) x Qrot^T (fp16 hi + lo)          three products
//   sign blocks:     (+-rho_t, exact in fp16) x (gamma SQ)^T (hi + lo)   two products
// Decoder warps turn the packed codes of each key into its A rows and store them straight into
// tensor memory (the MMA reads A from TMEM, so shared-memory bandwidth is left to the B tiles);
// the queries' B tiles are split and swizzled once per call and arrive by bulk copy.  Two TMEM
// accumulator slots let the epilogue of one tile overlap the MMAs of the next; it transposes the
// scores through shared memory and keeps running per-row top-k lists, merged by a small kernel.
// Every operand product is exact in fp32 up to the dropped lo x lo terms (relative 2^-22).
// The single-product form (FP16 = true, tq_search) keeps only the hi x hi products: every operand
// is rounded to fp16 once (relative 2^-11), so a score moves by at most
// 2^-10 ||k|| (sum_i |q_rot,i c_i| + rho gamma sum_j |(S q)_j|) from the exact one.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {

namespace {

using namespace sm100;

constexpr int kSTile = 128;                  // keys per tile (MMA M) and query rows per tile (MMA N)
constexpr int kDecGroups = 2;                // key-decoder groups of four warps, one K-block each in turn
constexpr int kDecWarp0 = 2;                 // warps 2 .. 2 + 4 kDecGroups - 1: key decoders
constexpr int kEpiWarp0 = kDecWarp0 + 4 * kDecGroups;  // four epilogue warps
constexpr int kSThreads = 32 * (kEpiWarp0 + 4);
constexpr int kSStages = 4;                  // operand stages (B in shared memory, A in TMEM)
constexpr uint32_t kBTile = kSTile * 128;    // one 128 x 64 fp16 B tile (16 KB)
constexpr uint32_t kStageBytes = 2 * kBTile; // B hi, B lo
constexpr uint32_t kAccCols = 128;           // accumulator columns per slot
constexpr uint32_t kACol0 = 2 * kAccCols;    // first TMEM column of the A stages
constexpr uint32_t kAStageCols = 64;         // A hi (32 columns) | A lo (32 columns) per stage
constexpr int kScRows = 64;                  // query rows transposed at a time
constexpr int kScStride = kSTile + 4;        // transposed score row stride (floats, 16-byte rows)
constexpr int kSearchSms = 148;              // grid sizing (fixed so scratch sizes do not vary)
constexpr int kMaxFusedTopk = 16;            // longest per-row list kept in shared memory

constexpr int kQCap = 24;                    // per-row candidate queue entries per tile

struct SearchSmem {
    uint32_t stage, sc, lv, li, qv, qi, thr, qcnt, klut, rowoff, bars, misc, total;
};

__host__ __device__ inline SearchSmem search_smem_layout(int K, int KB) {
    SearchSmem L;
    uint32_t o = 0;
    L.stage = o;
    o += kSStages * kStageBytes;
    L.sc = o;  // transposed scores of 64 query rows (overflow path)
    o += kScRows * kScStride * 4;
    L.lv = o;  // per-row top-k lists, K entries each, padded with (-inf, INT32_MAX)
    o += kSTile * (K > 0 ? K : 1) * 4;
    L.li = o;
    o += kSTile * (K > 0 ? K : 1) * 4;
    L.qv = o;  // per-row candidate queues of the current tile
    o += kSTile * kQCap * 4;
    L.qi = o;
    o += kSTile * kQCap * 4;
    L.thr = o;  // per-row admission threshold (the k-th best so far, -inf until k are held)
    o += kSTile * 4;
    L.qcnt = o;
    o += kSTile * 4;
    o = (o + 15) & ~15u;
    L.klut = o;
    o += (1u << (2 * KB)) * 32 * 8;
    L.rowoff = o;
    o += kSTile * 8;
    L.bars = o;
    o += 32 * 8;
    L.misc = o;
    o += 64;
    L.total = o;
    return L;
}

enum SBar { kBFull = 0, kAFull = 4, kSEmpty = 8, kAccFull = 12, kAccEmpty = 14 };

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
// Exponent e with maxabs * 2^e in [512, 1024): fp16 operands far from overflow, and their lo
// halves far from the subnormal range.
__device__ __forceinline__ int pow2_exp(float maxabs) {
    if (!(maxabs > 0.f) || !isfinite(maxabs)) return 0;
    int e;
    frexpf(maxabs, &e);
    return 10 - e;
}
__device__ __forceinline__ float search_gamma(int m) { return sqrtf(1.5707963267948966f) / (float)m; }

// ------------------------------------------------------------------ query operands

// Per unit (slice, block of 128 query rows): max |q_rot| and max |gamma sq| over its rows, as
// float bits (non-negative floats order like their bit patterns); umax starts at zero.
__global__ void search_max_kernel(ScoreProblem sp, SearchGeom g, const float *__restrict__ qprep,
                                  unsigned *__restrict__ umax) {
    __shared__ float red[2][8];
    const int unit = blockIdx.x, rows_per = kSTile / gridDim.y;
    const int d = g.d, stride = g.d + g.m;
    const float gamma = search_gamma(g.m);
    float qm = 0.f, sm = 0.f;
    for (int e = threadIdx.x; e < rows_per * stride; e += blockDim.x) {
        const int r = blockIdx.y * rows_per + e / stride, col = e % stride;
        const int64_t qr = search_qrow(sp, g, unit, r);
        if (qr < 0) continue;
        const float v = qprep[qr * stride + col];
        if (col < d) qm = fmaxf(qm, fabsf(v));
        else sm = fmaxf(sm, fabsf(gamma * v));
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
        atomicMax(&umax[unit * 2 + threadIdx.x], __float_as_uint(mx));
    }
}

// Key-side centroid exponent: the codebook's largest |centroid| scaled into [512, 1024).
__device__ __forceinline__ int centroid_exp(const Prepared &P) {
    float kmax = 0.f;
    for (int k = 0; k < (1 << P.kbeta); ++k) kmax = fmaxf(kmax, fabsf(P.cb->kc[k]));
    return pow2_exp(kmax);
}

// One B tile (unit, K-block) per block: fp16 hi | lo of q_rot * 2^eq (centroid blocks) or of
// gamma sq * 2^eB (sign blocks), in the 128-byte-swizzled K-major layout.  The exponents make
// both parts of the accumulator carry the same scale 2^E: E = eq + ek for centroids (ek on the
// key side) and E = eB + eA for signs, where the key side holds +-rho * 2^eA (exact in fp16
// for eA in [-8, 14]).  E is lowered, if need be, so that eA <= 14 without pushing any B value
// above its [512, 1024) target.  uexp[unit] = {E, eA}.
__global__ void search_tiles_kernel(Prepared P, ScoreProblem sp, SearchGeom g, const float *__restrict__ qprep,
                                    const unsigned *__restrict__ umax, uint8_t *__restrict__ qsw,
                                    int *__restrict__ uexp) {
    const int unit = blockIdx.x, kb = blockIdx.y;
    const int d = g.d, stride = g.d + g.m, dkb = g.d / 64;
    const int eq = pow2_exp(__uint_as_float(umax[unit * 2]));
    const int ebn = pow2_exp(__uint_as_float(umax[unit * 2 + 1]));
    const int ek = centroid_exp(P);
    const int E = min(eq + ek, ebn + 14);
    const int eA = max(-8, E - ebn);
    if (kb == 0 && threadIdx.x == 0) {
        uexp[unit * 2] = E;
        uexp[unit * 2 + 1] = eA;
    }
    const bool sgn = kb >= dkb;
    const float scale = sgn ? search_gamma(g.m) * ldexpf(1.f, E - eA) : ldexpf(1.f, E - ek);
    const int col0 = sgn ? d + (kb - dkb) * 64 : kb * 64;
    uint8_t *hi = qsw + ((size_t)unit * g.nkb + kb) * kStageBytes;
    uint8_t *lo = hi + kBTile;
    for (int e = threadIdx.x; e < kSTile * 64; e += blockDim.x) {
        const int r = e >> 6, kk = e & 63;
        const int64_t qr = search_qrow(sp, g, unit, r);
        const float v = qr >= 0 ? qprep[qr * stride + col0 + kk] * scale : 0.f;
        const uint32_t off = (uint32_t)r * 128 + ((((uint32_t)kk >> 3) ^ (r & 7)) << 4) + (kk & 7) * 2;
        const __half h = __float2half_rn(v);
        *(__half *)(hi + off) = h;
        *(__half *)(lo + off) = __float2half_rn(v - __half2float(h));
    }
}

// ------------------------------------------------------------------------ GEMM

__device__ __forceinline__ bool search_better(float va, int32_t ia, float vb, int32_t ib) {
    return va > vb || (va == vb && ia < ib);
}


template <int KB, bool FP16>
__global__ void __launch_bounds__(kSThreads, 1)
    search_gemm_kernel(Prepared P, ScoreProblem sp, SearchGeom g, const uint8_t *__restrict__ qsw,
                       const int *__restrict__ uexp, float *__restrict__ scores, int K, float *__restrict__ cand_v,
                       int32_t *__restrict__ cand_i, int32_t *__restrict__ dev_status) {
    const int DKB = g.d / 64;          // centroid K-blocks
    const int KWPT = KB * (g.d / 32);  // code words per key
    const int SWPT = g.m / 32;         // sign words per key
    const int NKB = g.nkb;
    const SearchSmem L = search_smem_layout(K, KB);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    float *sc = (float *)(sm + L.sc);
    const uint2 *klut = (const uint2 *)(sm + L.klut);
    int64_t *rowoff = (int64_t *)(sm + L.rowoff);
    uint32_t *tmem_s = (uint32_t *)(sm + L.misc);
    volatile int *abort_s = (volatile int *)(sm + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x / g.kc, cidx = blockIdx.x % g.kc;
    const int sl = unit / g.nrb;
    const int my_tiles = (int)((g.nkt - cidx + g.kc - 1) / g.kc);
    const int total = my_tiles * NKB;
    const int64_t rec_base = (int64_t)sl * sp.Ts;
    const int E = uexp[unit * 2], eA = uexp[unit * 2 + 1];

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&bars[kBFull + s], 1);
            mbar_init(&bars[kAFull + s], 4);
            mbar_init(&bars[kSEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kAccFull + s], 1);
            mbar_init(&bars[kAccEmpty + s], 4);
        }
        *abort_s = 0;
        fence_mbar_init();
    }
    {
        // centroid pair table (hi pair, lo pair), one copy per lane so lookups never conflict:
        // entry idx holds coordinates whose plane bits interleave in idx (even bits: first)
        uint2 *lut = (uint2 *)(sm + L.klut);
        const float ksc = ldexpf(1.f, centroid_exp(P));
        for (int e = threadIdx.x; e < (32 << (2 * KB)); e += blockDim.x) {
            const int idx = e >> 5;
            int i0 = 0, i1 = 0;
            for (int p = 0; p < KB; ++p) {
                i0 |= ((idx >> (2 * p)) & 1) << p;
                i1 |= ((idx >> (2 * p + 1)) & 1) << p;
            }
            const float a0 = P.cb->kc[i0] * ksc, a1 = P.cb->kc[i1] * ksc;
            lut[e] = make_uint2(pack_h2s(a0, a1), pack_h2s(a0 - hi16(a0), a1 - hi16(a1)));
        }
        for (int r = threadIdx.x; r < kSTile; r += blockDim.x) {
            const int64_t qr = search_qrow(sp, g, unit, r);
            rowoff[r] = qr < 0 ? -1 : qr * sp.T;
        }
        for (int e = threadIdx.x; e < kSTile * K; e += blockDim.x) {
            ((float *)(sm + L.lv))[e] = -INFINITY;
            ((int32_t *)(sm + L.li))[e] = INT32_MAX;
        }
        for (int r = threadIdx.x; r < kSTile; r += blockDim.x) {
            ((float *)(sm + L.thr))[r] = search_qrow(sp, g, unit, r) >= 0 ? -INFINITY : INFINITY;
            ((int *)(sm + L.qcnt))[r] = 0;
        }
        if (threadIdx.x < 2) ((volatile int *)(sm + L.misc + 8))[threadIdx.x] = 0;  // queue overflow flags
    }
    if (warp == 0) {
        tmem_alloc(tmem_s, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_s;
    const uint8_t *qsw_u = qsw + (size_t)unit * NKB * kStageBytes;

    if (warp == 0) {
        // -------------------------------------------------------- query tiles (bulk copies)
        if (lane == 0) {
            int issued = 0;
            for (int gk = 0; gk < total; ++gk) {
                const int st = gk % kSStages;
                if (gk >= kSStages && !mbar_wait(&bars[kSEmpty + st], ((gk / kSStages) - 1) & 1, abort_s)) break;
                // the single-product form reads only the hi half of a B tile
                constexpr uint32_t kCopy = FP16 ? kBTile : kStageBytes;
                mbar_arrive_expect_tx(&bars[kBFull + st], kCopy);
                bulk_load(sm + L.stage + st * kStageBytes, qsw_u + (size_t)(gk % NKB) * kStageBytes, kCopy,
                          &bars[kBFull + st]);
                issued = gk + 1;
            }
            // every copy must land before the CTA can exit (bounded waits)
            int dummy = 0;
            for (int gk = issued > kSStages ? issued - kSStages : 0; gk < issued; ++gk)
                mbar_wait(&bars[kBFull + gk % kSStages], (gk / kSStages) & 1, (volatile int *)&dummy);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issue (A from TMEM)
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(kSTile, kSTile);
            const uint32_t sbase = smem_u32(sm + L.stage);
            bool ok = true;
            for (int i = 0; ok && i < my_tiles; ++i) {
                const int slot = i & 1;
                if (i >= 2 && !mbar_wait(&bars[kAccEmpty + slot], ((i >> 1) - 1) & 1, abort_s)) break;
                tc_fence_after();
                const uint32_t acc = tmem + slot * kAccCols;
                for (int kbi = 0; kbi < NKB; ++kbi) {
                    const int gk = i * NKB + kbi, st = gk % kSStages;
                    const uint32_t ph = (gk / kSStages) & 1;
                    if (!mbar_wait(&bars[kAFull + st], ph, abort_s) || !mbar_wait(&bars[kBFull + st], ph, abort_s)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = tmem + kACol0 + st * kAStageCols;
                    const uint32_t b_hi = sbase + st * kStageBytes, b_lo = b_hi + kBTile;
                    const bool cen = kbi < DKB;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t a_hi = a0 + 32 * (k >> 1) + 8 * (k & 1);
                        const uint64_t dh = sdesc_sw128(b_hi + 32 * k), dl = sdesc_sw128(b_lo + 32 * k);
                        mma_ts(acc, a_hi, dh, idesc, (kbi | k) ? 1u : 0u);
                        if constexpr (!FP16) {
                            mma_ts(acc, a_hi, dl, idesc, 1u);
                            if (cen) mma_ts(acc, a_hi + 16, dh, idesc, 1u);
                        }
                    }
                    mma_commit(&bars[kSEmpty + st]);
                }
                if (ok) mma_commit(&bars[kAccFull + slot]);
            }
        }
    } else if (warp < kEpiWarp0) {
        // -------------------------------------------------------- key decode into TMEM
        // group g fills the K-block steps g, g + kDecGroups, ...; within a group the four warps
        // cover the four TMEM lane quarters, one key per thread
        const int grp = (warp - kDecWarp0) >> 2;
        const int quarter = warp & 3;
        const int kr = 32 * quarter + lane;
        const uint32_t tq = tmem + ((uint32_t)(32 * quarter) << 16) + kACol0;
        auto fetch = [&](int gk, uint2 (&u)[KB], uint32_t &rb, bool &valid) {
            const int kbi = gk % NKB, i = gk / NKB;
            const int64_t t = (int64_t)(cidx + (int64_t)i * g.kc) * kSTile + kr;
            valid = t < sp.T;
#pragma unroll
            for (int p = 0; p < KB; ++p) u[p] = make_uint2(0u, 0u);
            rb = 0;
            if (!valid) return;
            const int64_t rec = rec_base + t;
            if (kbi < DKB) {
                const uint2 *src = (const uint2 *)(sp.kcodes + rec * KWPT + 2 * kbi * KB);
#pragma unroll
                for (int p = 0; p < KB; ++p) u[p] = __ldg(src + p);
            } else {
                u[0] = __ldg((const uint2 *)(sp.ksigns + rec * SWPT + 2 * (kbi - DKB)));
                rb = sp.krnorm[rec];
            }
        };
        // decode K-block step gk from its fetched words into its TMEM stage; false on abort
        auto decode = [&](int gk, const uint2 (&cu)[KB], uint32_t crb, bool cval) -> bool {
            const int st = gk % kSStages, kbi = gk % NKB;
            if (gk >= kSStages && !mbar_wait(&bars[kSEmpty + st], ((gk / kSStages) - 1) & 1, abort_s))
                return false;
            tc_fence_after();
            const uint32_t ta = tq + st * kAStageCols;
            if (kbi < DKB) {
                // coordinates 64 kbi + 32 h + (0..31): the KB plane words of group 2 kbi + h
                const char *lutl = (const char *)klut + 8 * lane;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t w[KB];
#pragma unroll
                    for (int p = 0; p < KB; ++p) {
                        const int wi = h * KB + p;
                        w[p] = (wi & 1) ? cu[wi >> 1].y : cu[wi >> 1].x;
                    }
                    uint32_t hp[16], lp[16];
                    if (cval) {
                        // byte k of ix[s] = table index of coordinate pair 4k + s: the pair's
                        // two bits of plane p moved to bits 2p, 2p + 1
                        uint32_t ix[4];
#pragma unroll
                        for (int s4 = 0; s4 < 4; ++s4) {
                            uint32_t e = 0;
#pragma unroll
                            for (int p = 0; p < KB; ++p) {
                                const int sh = 2 * s4 - 2 * p;
                                const uint32_t x = sh >= 0 ? (w[p] >> sh) : (w[p] << -sh);
                                e |= x & (0x03030303u << (2 * p));
                            }
                            ix[s4] = e;
                        }
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            // table offset idx * 256 (32 lane copies of 8 bytes per entry)
                            const uint32_t off = __byte_perm(ix[q & 3], 0u, 0x4404u | ((uint32_t)(q >> 2) << 4));
                            const uint2 e = *(const uint2 *)(lutl + off);
                            hp[q] = e.x;
                            lp[q] = e.y;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) hp[q] = lp[q] = 0u;
                    }
                    tmem_st16(ta + 32 * h, hp);
                    if constexpr (!FP16) tmem_st16(ta + 32 * h + 16, lp);
                }
            } else {
                // projections 64 (kbi - DKB) + 32 h + (0..31): +-rho 2^eA, sign bit set = +1
                const uint32_t hv =
                    cval ? (uint32_t)__half_as_ushort(__float2half_rn(ldexpf(f16_bits_to_f32((uint16_t)crb), eA)))
                         : 0u;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w = h ? cu[0].y : cu[0].x;
                    uint32_t v[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint32_t b = ~(w >> (2 * q));
                        v[q] = (hv | ((b & 1u) << 15)) | ((hv | ((b & 2u) << 14)) << 16);
                    }
                    tmem_st16(ta + 32 * h, v);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kAFull + st]);
            return true;
        };
        // three word buffers in turn: each step's words are fetched two of this group's steps
        // ahead, so their loads have two decodes to land in
        constexpr int D1 = kDecGroups, D2 = 2 * kDecGroups;
        uint2 b0[KB], b1[KB], b2[KB];
        uint32_t r0 = 0, r1 = 0, r2 = 0;
        bool v0 = false, v1 = false, v2 = false;
        if (grp < total) fetch(grp, b0, r0, v0);
        if (grp + D1 < total) fetch(grp + D1, b1, r1, v1);
        for (int gk = grp; gk < total; gk += 3 * D1) {
            if (gk + D2 < total) fetch(gk + D2, b2, r2, v2);
            if (!decode(gk, b0, r0, v0)) break;
            const int g1 = gk + D1;
            if (g1 >= total) break;
            if (g1 + D2 < total) fetch(g1 + D2, b0, r0, v0);
            if (!decode(g1, b1, r1, v1)) break;
            const int g2 = g1 + D1;
            if (g2 >= total) break;
            if (g2 + D2 < total) fetch(g2 + D2, b1, r1, v1);
            if (!decode(g2, b2, r2, v2)) break;
        }
    } else {
        // -------------------------------------------------------- scores and top-k
        // Each thread holds one key's scores for 32 query rows at a time (its TMEM lane) and
        // admits those above the row's threshold into the row's queue; after the tile, thread et
        // drains row et's queue into the row's sorted list.  A tile whose queues would overflow
        // (the first tile, while the lists fill up, or an adversarial key order) is instead
        // transposed through shared memory and scanned in full.
        const int q4 = warp & 3;                      // TMEM lane quarter this warp may read
        const int row = 32 * q4 + lane;               // key within the tile
        const int et = threadIdx.x - kEpiWarp0 * 32;  // 0..127: the query row this thread drains
        float *thr = (float *)(sm + L.thr);
        int *qcnt = (int *)(sm + L.qcnt);
        float *qv = (float *)(sm + L.qv);
        int32_t *qi = (int32_t *)(sm + L.qi);
        volatile int *ovf = (volatile int *)(sm + L.misc + 8);  // one flag per tile parity
        const float un = ldexpf(1.f, -E);
        float *lv = (float *)(sm + L.lv);
        int32_t *li = (int32_t *)(sm + L.li);
        const int ew = et >> 5;  // epilogue warp index 0..3
        for (int i = 0; i < my_tiles; ++i) {
            const int slot = i & 1;
            const int64_t t0 = (int64_t)(cidx + (int64_t)i * g.kc) * kSTile;
            const int64_t t = t0 + row;
            const bool valid = t < sp.T;
            float c = 0.f, bias = -INFINITY;
            if (valid) {
                c = f16_bits_to_f32(sp.knorm[rec_base + t]) * un;
                bias = 0.f;
            }
            if (!mbar_wait(&bars[kAccFull + slot], (i >> 1) & 1, abort_s)) break;
            tc_fence_after();
            const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16) + slot * kAccCols;
#pragma unroll 1
            for (int cc = 0; cc < kSTile / 16; ++cc) {
                uint32_t a[16];
                tmem_ld16(tl + 16 * cc, a);
                tmem_ld_wait();
                if (scores && valid) {
#pragma unroll
                    for (int l = 0; l < 16; ++l) {
                        const int64_t ro = rowoff[16 * cc + l];
                        if (ro >= 0) scores[ro + t] = fmaf(c, __uint_as_float(a[l]), bias);
                    }
                }
                if (K > 0) {
#pragma unroll
                    for (int l4 = 0; l4 < 4; ++l4) {
                        const float4 th = ((const float4 *)thr)[4 * cc + l4];
                        const float tv[4] = {th.x, th.y, th.z, th.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const float s = fmaf(c, __uint_as_float(a[4 * l4 + u]), bias);
                            if (s > tv[u]) {
                                const int r = 16 * cc + 4 * l4 + u;
                                const int qs = atomicAdd(&qcnt[r], 1);
                                if (qs < kQCap) {
                                    qv[r * kQCap + qs] = s;
                                    qi[r * kQCap + qs] = (int32_t)t;
                                } else {
                                    ovf[slot] = 1;
                                }
                            }
                        }
                    }
                }
            }
            if (K == 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kAccEmpty + slot]);
                continue;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ovf[slot] == 0) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kAccEmpty + slot]);
                const int n = min(qcnt[et], kQCap);
                if (n > 0) {
                    float *mv = lv + et * K;
                    int32_t *mi = li + et * K;
#pragma unroll 1
                    for (int j = 0; j < n; ++j) {
                        const float sv = qv[et * kQCap + j];
                        const int32_t ti = qi[et * kQCap + j];
                        if (!search_better(sv, ti, mv[K - 1], mi[K - 1])) continue;
                        int pos = K - 1;
                        while (pos > 0 && search_better(sv, ti, mv[pos - 1], mi[pos - 1])) {
                            mv[pos] = mv[pos - 1];
                            mi[pos] = mi[pos - 1];
                            --pos;
                        }
                        mv[pos] = sv;
                        mi[pos] = ti;
                    }
                    thr[et] = mv[K - 1];
                }
            } else {
                // transpose 64 query rows at a time and scan every key of the tile
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
#pragma unroll 1
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t a[32];
                        tmem_ld32(tl + 64 * h + 32 * cc, a);
                        tmem_ld_wait();
#pragma unroll
                        for (int l = 0; l < 32; ++l)
                            sc[(32 * cc + l) * kScStride + row] = fmaf(c, __uint_as_float(a[l]), bias);
                    }
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                    // warp ew selects, for 16 of these rows, the tile's best K by K rounds of
                    // warp arg-max, then merges them with the row's list by rank
#pragma unroll 1
                    for (int rr = 0; rr < 16; ++rr) {
                        const int rl = 16 * ew + rr, r = 64 * h + rl;
                        if (rowoff[r] < 0) continue;
                        const float4 v4 = ((const float4 *)(sc + rl * kScStride))[lane];
                        float vv[4] = {v4.x, v4.y, v4.z, v4.w};
                        float nv = -INFINITY;
                        int32_t ni = INT32_MAX;
                        for (int k = 0; k < K; ++k) {
                            float bvv = -INFINITY;
                            int32_t bii = INT32_MAX;
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const int32_t ix = vv[u] == -INFINITY ? INT32_MAX : (int32_t)(t0 + 4 * lane + u);
                                if (search_better(vv[u], ix, bvv, bii)) {
                                    bvv = vv[u];
                                    bii = ix;
                                }
                            }
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) {
                                const float ov = __shfl_xor_sync(kFull, bvv, o);
                                const int32_t oi = __shfl_xor_sync(kFull, bii, o);
                                if (search_better(ov, oi, bvv, bii)) {
                                    bvv = ov;
                                    bii = oi;
                                }
                            }
                            if (lane == k) {
                                nv = bvv;
                                ni = bii;
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                if (bii != INT32_MAX && (int32_t)(t0 + 4 * lane + u) == bii) vv[u] = -INFINITY;
                        }
                        // rank of each entry among both sorted lists (a permutation apart from
                        // the interchangeable padding), then scatter the first K
                        const float ev = lane < K ? lv[r * K + lane] : -INFINITY;
                        const int32_t ei = lane < K ? li[r * K + lane] : INT32_MAX;
                        int rn = lane, re = lane;
                        for (int k = 0; k < K; ++k) {
                            const float xe = __shfl_sync(kFull, ev, k), xn = __shfl_sync(kFull, nv, k);
                            const int32_t ie = __shfl_sync(kFull, ei, k), in = __shfl_sync(kFull, ni, k);
                            rn += search_better(xe, ie, nv, ni) ? 1 : 0;
                            re += search_better(xn, in, ev, ei) ? 1 : 0;
                        }
                        __syncwarp();
                        if (lane < K && rn < K) {
                            lv[r * K + rn] = nv;
                            li[r * K + rn] = ni;
                        }
                        if (lane < K && re < K) {
                            lv[r * K + re] = ev;
                            li[r * K + re] = ei;
                        }
                        __syncwarp();
                        if (lane == 0) thr[r] = lv[r * K + K - 1];
                    }
                    asm volatile("bar.sync 1, 128;" ::: "memory");
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kAccEmpty + slot]);
            }
            qcnt[et] = 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            // every thread read this parity's flag before the barrier; it is next set two tiles on
            if (et == 0) ovf[slot] = 0;
        }
        if (K > 0) {
            const size_t base = ((size_t)blockIdx.x * kSTile + et) * K;
            for (int j = 0; j < K; ++j) {
                cand_v[base + j] = lv[et * K + j];
                cand_i[base + j] = li[et * K + j];
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
    const int per = K;
    for (int e = threadIdx.x; e < g.kc * per; e += 32) {
        const int c = e / per, j = e % per;
        const size_t src = (((size_t)unit * g.kc + c) * kSTile + r) * per + j;
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

template <int KB, bool FP16>
cudaError_t launch_search_kb(const Prepared &P, const ScoreProblem &sp, const SearchGeom &g, const uint8_t *qsw,
                             const int *uexp, float *scores, int K, float *cv, int32_t *ci, int32_t *dev_status,
                             cudaStream_t s) {
    const SearchSmem L = search_smem_layout(K, KB);
    const size_t smem = L.total + 1024;
    auto kern = search_gemm_kernel<KB, FP16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<g.units * g.kc, kSThreads, smem, s>>>(P, sp, g, qsw, uexp, scores, K, cv, ci, dev_status);
    return cudaGetLastError();
}

struct SearchScratch {
    size_t qsw, umax, uexp, cv, ci, total;
};

SearchScratch search_scratch_layout(const SearchGeom &g, int topk) {
    SearchScratch S;
    size_t o = 0;
    S.qsw = o;
    o = align_up(o + (size_t)g.units * g.nkb * kStageBytes, 256);
    S.umax = o;
    o = align_up(o + (size_t)g.units * 2 * sizeof(unsigned), 256);
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
                          cudaStream_t s, bool fp16) {
    const SearchGeom g = search_geom(P, sp);
    const SearchScratch S = search_scratch_layout(g, topk);
    uint8_t *base = (uint8_t *)scratch;
    uint8_t *qsw = base + S.qsw;
    unsigned *umax = (unsigned *)(base + S.umax);
    int *uexp = (int *)(base + S.uexp);
    float *cv = (float *)(base + S.cv);
    int32_t *ci = (int32_t *)(base + S.ci);
    cudaError_t e = cudaMemsetAsync(umax, 0, (size_t)g.units * 2 * sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
    search_max_kernel<<<dim3((unsigned)g.units, 16), 256, 0, s>>>(sp, g, qprep, umax);
    search_tiles_kernel<<<dim3((unsigned)g.units, (unsigned)g.nkb), 256, 0, s>>>(P, sp, g, qprep, umax, qsw, uexp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    switch (P.kbeta * 2 + (fp16 ? 1 : 0)) {
        case 2: e = launch_search_kb<1, false>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 3: e = launch_search_kb<1, true>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 4: e = launch_search_kb<2, false>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 5: e = launch_search_kb<2, true>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 6: e = launch_search_kb<3, false>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        case 7: e = launch_search_kb<3, true>(P, sp, g, qsw, uexp, scores, topk, cv, ci, dev_status, s); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess || topk == 0) return e;
    search_merge_kernel<<<g.units * kSTile, 32, 0, s>>>(sp, g, topk, cv, ci, topk_idx, topk_val);
    return cudaGetLastError();
}

}  // namespace tq
