// tq_compress_big.cu -- key / value compression on the tensor cores for any head dimension
// d = 64 k <= 1024, fp16 or fp32 input, with both operands streamed.
//
// Per 128-vector tile (TurboQuantMSE.quantize / TurboQuantProd.compress; "turboquant-pytorch",
// nav.superapi.store, 核心 API and 算法细节; atskills.one, "What It Does" stage 1 + stage 2):
//   u = x / ||x||                          converter warps, one vector per thread: ||x|| in fp32,
//                                          then U = u 2^10 as fp16 hi + lo, 64 coordinates per
//                                          K-block, written into swizzled shared memory
//   y = R u                                N-chunks of 128 outputs: ACC = U (hi + lo) x
//                                          (R 2^8)(hi + lo), three products per k-step
//   codes, ||y - c[idx]||                  epilogue, one vector per thread (a TMEM lane)
//   p = S u - S' c[idx]  (S' = S R^T)      N-chunks of the projection: the S u products as above,
//                                          then, once the tile's codes are out, K-blocks of
//                                          -c[idx] 2^14 (hi + lo) x (S' 2^4)(hi + lo) into the
//                                          same accumulator, so only sign(ACC) is needed
// R is orthogonal, so ||u - R^T c|| = ||y - c||.  All products are exact in fp32 up to the
// dropped lo x lo terms (relative 2^-22); the bucket decisions are taken on fp32 y.
// Warp roles: 0 streams the B tiles and owns TMEM, 1 issues the MMAs, 2..9 convert the A
// tiles (two groups taking alternate K-blocks), 10..13 run the epilogue.  Two TMEM slots of
// 256 columns keep one chunk's epilogue under the next chunk's MMAs.
// fp16 input with d <= 256 (one rotation chunk; keys also m <= 256) takes the input itself as the
// A operand: fp16 is exact, so x (R 2^8)(hi + lo) needs two products per k-step, warp 0 loads the
// rows by TMA into the swizzled stage beside the B tiles (the converter warps have no work), and
// the epilogue takes ||x|| = ||ACC|| / 2^8 from the rotation accumulator (R orthogonal, to the
// 2^-22 of its split) before coding y = ACC / ||ACC||.  Keys then project the residual:
// p = S u - S' c[idx] = S' (y - c[idx]) (S u = S R^T y), so the epilogue writes
// 2^14 e = 2^14 (y - c[idx]) as fp16 hi | lo back into the rotation slot and the projection chunk
// multiplies that TMEM operand by (S' 2^4)(hi + lo), three products per k-step into one
// accumulator; there are no correction blocks.
#include <cudaTypedefs.h>

#include <cstring>

#include "tq_common.cuh"
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {

namespace {

using namespace sm100;

constexpr int kBRows = 128;                   // vectors per tile (MMA M)
constexpr int kBChunk = 256;                  // output columns per chunk (MMA N, at most)
constexpr int kBThreads = 448;                // 14 warps
constexpr int kCvtWarp0 = 2;                  // warps 2..9: A-tile converters, two groups of four
constexpr int kBEpiWarp0 = 10;                // warps 10..13: epilogue
constexpr int kBStages = 2;                   // A + B operand stages
constexpr uint32_t kATile = kBRows * 128;     // 128 x 64 fp16 (16 KB)
constexpr uint32_t kBTileMax = kBChunk * 128; // up to 256 x 64 fp16 (32 KB)
constexpr uint32_t kBStage = 2 * kATile + 2 * kBTileMax;  // A hi, A lo, B hi, B lo
constexpr int kUScaleLog2 = 10;               // U = u 2^10
constexpr int kCorrScaleLog2 = kUScaleLog2 + kRScaleLog2 - kSScaleLog2;  // correction A scale

enum BBar { kBFull = 0, kBEmpty = 2, kBAccFull = 4, kBAccEmpty = 6, kBCodes = 8, kBNorm = 10, kBEe = 12 };

struct BigSmem {
    uint32_t stage, ctab, bnd, cen, bars, misc, xchg, total;
};

__host__ __device__ inline BigSmem big_smem_layout() {
    BigSmem L;
    uint32_t o = 0;
    L.stage = o;
    o += kBStages * kBStage;
    L.ctab = o;  // 16 words: fp16 hi | lo << 16 of -c[k] 2^14 (correction operand)
    o += 16 * 4;
    L.bnd = o;  // 16 boundaries
    o += 16 * 4;
    L.cen = o;  // 16 centroids
    o += 16 * 4;
    L.bars = o;
    o += 32 * 8;
    L.misc = o;
    o += 64;
    L.xchg = o;  // exact path: partial squared norms [2][2][128], partial residual norms [2][128]
    o += 3 * 2 * 128 * 4;
    L.total = o;
    return L;
}

// The chunk sequence of one tile: R chunks (rotation outputs), then, for keys, S chunks
// (projection outputs), each with its K-blocks: d/64 over U, plus d/64 correction blocks for
// S chunks (the residual form of the exact path has only the d/64 blocks of S').
struct BigGeom {
    int d, m, nr, ns;  // dims; number of R chunks and S chunks
    __host__ __device__ int nchunks() const { return nr + ns; }
    __host__ __device__ int n0(int c) const { return c < nr ? c * kBChunk : (c - nr) * kBChunk; }
    __host__ __device__ int width(int c) const {
        const int tot = c < nr ? d : m;
        const int w = tot - n0(c);
        return w < kBChunk ? w : kBChunk;
    }
    __host__ __device__ int nkb(int c) const { return c < nr ? d / 64 : 2 * (d / 64); }
    __host__ __device__ int kb_per_tile() const { return nr * (d / 64) + ns * 2 * (d / 64); }
};

// The codebooks are symmetric (c[HL + k] = -c[HL - 1 - k], middle boundary 0, HL = 2^(BETA-1)),
// so the code of y follows from its sign and the digits of m = #{k : e[k] < |y|} over the HL - 1
// positive boundaries e[k] = b[HL + k]: the code is HL + m for y > 0 and HL - 1 - m otherwise, so
// its top bit is [y > 0] and its bit j < BETA - 1 is m_j when y > 0, not m_j otherwise.
// big_mag sets mb[j] = m_j by a binary search over thresholds held in registers.
template <int BETA>
__device__ __forceinline__ void big_mag(float u, const float *e, bool (&mb)[3]) {
    if constexpr (BETA == 2) {
        mb[0] = u > e[0];
    } else if constexpr (BETA == 3) {
        mb[1] = u > e[1];
        mb[0] = u > (mb[1] ? e[2] : e[0]);
    } else if constexpr (BETA == 4) {
        mb[2] = u > e[3];
        mb[1] = u > (mb[2] ? e[5] : e[1]);
        mb[0] = u > (mb[2] ? (mb[1] ? e[6] : e[4]) : (mb[1] ? e[2] : e[0]));
    }
}

// |c| = cm[m] from the digits of m (HL positive centroids in registers).
template <int BETA>
__device__ __forceinline__ float big_cmag(const bool (&mb)[3], const float *cm) {
    if constexpr (BETA == 1) {
        return cm[0];
    } else if constexpr (BETA == 2) {
        return mb[0] ? cm[1] : cm[0];
    } else if constexpr (BETA == 3) {
        return mb[1] ? (mb[0] ? cm[3] : cm[2]) : (mb[0] ? cm[1] : cm[0]);
    } else {
        const float hi = mb[1] ? (mb[0] ? cm[7] : cm[6]) : (mb[0] ? cm[5] : cm[4]);
        const float lo = mb[1] ? (mb[0] ? cm[3] : cm[2]) : (mb[0] ? cm[1] : cm[0]);
        return mb[2] ? hi : lo;
    }
}

__device__ __forceinline__ uint32_t hsplit2(float a, float b, bool lo) {
    const __half ha = __float2half_rn(a), hb = __float2half_rn(b);
    if (!lo) return (uint32_t)__half_as_ushort(ha) | ((uint32_t)__half_as_ushort(hb) << 16);
    const __half la = __float2half_rn(a - __half2float(ha)), lb = __float2half_rn(b - __half2float(hb));
    return (uint32_t)__half_as_ushort(la) | ((uint32_t)__half_as_ushort(lb) << 16);
}

constexpr float kSignRecheck = 1e-4f;  // |p| below which a sign is recomputed exactly
// The residual form has no cancelling O(1) terms: its error is the fp32 rounding of y carried
// through S' plus that of the d-term sum of S'_a e (a few 1e-6 at d <= 256 even with truncating
// accumulation), so it rechecks only below 2e-5.
constexpr float kSignRecheckResidual = 2e-5f;
constexpr float kPUnscaleInv = (float)(1 << (kUScaleLog2 + kRScaleLog2));  // ACC = p 2^18
constexpr float kEScale = (float)(1 << kCorrScaleLog2);  // residual operand 2^14 e

// p_a = S_a . u - S'_a . c[idx] of vector v in double, one warp: lane l takes coordinates
// 4 l + 128 i .. + 3 (row-major S and S', coalesced); the codes are the ones this CTA has just
// written for v.
template <int BETA, bool F16>
__device__ __noinline__ double exact_projection(const Prepared &P, const BigGeom &G, const void *xin,
                                                const uint32_t *codes, int64_t v, int a, int lane,
                                                const float *cen) {
    const int d = G.d, KWPT = BETA * (d / 32);
    const float *sr = P.S + (int64_t)a * d, *spr = P.Sp + (int64_t)a * d;
    double ss = 0.0, su = 0.0, sc = 0.0;
#pragma unroll 4
    for (int j = 4 * lane; j < d; j += 128) {
        float x4[4];
        if (F16) {
            const uint2 h = *(const uint2 *)((const __half *)xin + v * d + j);
            const float2 a2 = __half22float2(*(const __half2 *)&h.x), b2 = __half22float2(*(const __half2 *)&h.y);
            x4[0] = a2.x; x4[1] = a2.y; x4[2] = b2.x; x4[3] = b2.y;
        } else {
            const float4 f = *(const float4 *)((const float *)xin + v * d + j);
            x4[0] = f.x; x4[1] = f.y; x4[2] = f.z; x4[3] = f.w;
        }
        const float4 s4 = *(const float4 *)(sr + j), p4 = *(const float4 *)(spr + j);
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w}, pv[4] = {p4.x, p4.y, p4.z, p4.w};
        uint32_t w[BETA];
#pragma unroll
        for (int p = 0; p < BETA; ++p) w[p] = codes[v * KWPT + (j >> 5) * BETA + p] >> (j & 31);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            uint32_t idx = 0;
#pragma unroll
            for (int p = 0; p < BETA; ++p) idx |= ((w[p] >> e) & 1u) << p;
            const double xj = (double)x4[e];
            ss = fma(xj, xj, ss);
            su = fma((double)sv[e], xj, su);
            sc = fma((double)pv[e], (double)cen[idx], sc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ss += __shfl_xor_sync(kFull, ss, o);
        su += __shfl_xor_sync(kFull, su, o);
        sc += __shfl_xor_sync(kFull, sc, o);
    }
    const double nx = sqrt(ss);
    return (nx > 0.0 ? su / nx : 0.0) - sc;
}

template <bool IS_KEY, int BETA, bool F16, bool EX, bool SPLIT>
__global__ void __launch_bounds__(kBThreads, 1)
    compress_big_kernel(const __grid_constant__ CUtensorMap xmap, Prepared P, BigGeom G, const void *__restrict__ xin,
                        int64_t n, uint32_t *__restrict__ codes,
                        uint32_t *__restrict__ signs, uint16_t *__restrict__ norm, uint16_t *__restrict__ rnorm,
                        int32_t *__restrict__ dev_status) {
    const BigSmem L = big_smem_layout();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    uint32_t *ctab = (uint32_t *)(sm + L.ctab);
    float *bnd_s = (float *)(sm + L.bnd);
    float *cen_s = (float *)(sm + L.cen);
    uint32_t *tmem_s = (uint32_t *)(sm + L.misc);
    volatile int *abort_s = (volatile int *)(sm + L.misc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = G.d, dkb = G.d / 64;
    const int KWPT = BETA * (d / 32);
    const int SWPT = G.m / 32;
    const int NC = G.nchunks();
    // EX: A = the fp16 input itself, loaded by TMA (see the header); warps 2 .. kEpi0 - 1 idle.
    // SPLIT (exact path with a heavier code step): eight epilogue warps (6..13, two column halves)
    // code each tile.
    constexpr bool exact = EX;
    // RP (exact keys): the projection is p = S' e of the residual e = y - c[idx], which the
    // epilogue writes back into the rotation slot (fp16 hi | lo of 2^14 e) as the A operand of the
    // projection chunk, whose B is S' 2^4 (d/64 K-blocks, three products): no converter work
    constexpr bool RP = EX && IS_KEY;
    auto nkb_of = [&](int c) { return (RP && c >= G.nr) ? G.d / 64 : G.nkb(c); };
    constexpr int kEpi0 = SPLIT ? 6 : kBEpiWarp0;
    constexpr int kNEpi = SPLIT ? 8 : 4;
    float *xn_s = (float *)(sm + L.xchg);         // [tile parity][half][row] partial ||ACC||^2
    float *xe_s = xn_s + 2 * 2 * kBRows;          // [tile parity][row] half 1's part of ||y - c||^2
    const int64_t ntiles = (n + kBRows - 1) / kBRows;
    const int my_tiles = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBStages; ++s) {
            // the four converter warps of a group + the B copy; exact path: the copies of A and B
            mbar_init(&bars[kBFull + s], EX ? 1 : 5);
            mbar_init(&bars[kBEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBAccFull + s], 1);
            mbar_init(&bars[kBAccEmpty + s], kNEpi);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBCodes + s], kNEpi);
            mbar_init(&bars[kBNorm + s], kNEpi);
            mbar_init(&bars[kBEe + s], 4);
        }
        *abort_s = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 16) {
        const int k = threadIdx.x;
        const int K = 1 << BETA;
        bnd_s[k] = k < K - 1 ? (IS_KEY ? P.cb->kb[k] : P.cb->vb[k]) : INFINITY;
        const float c = k < K ? (IS_KEY ? P.cb->kc[k] : P.cb->vc[k]) : 0.f;
        cen_s[k] = c;
        const float cs = -c * (float)(1 << kCorrScaleLog2);
        const __half h = __float2half_rn(cs);
        const __half lo = __float2half_rn(cs - __half2float(h));
        ctab[k] = (uint32_t)__half_as_ushort(h) | ((uint32_t)__half_as_ushort(lo) << 16);
    }
    if (warp == 0) {
        tmem_alloc(tmem_s, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_s;

    if (warp == 0) {
        // -------------------------------------------------------- B tiles (bulk copies)
        if (lane == 0) {
            const int wrows = IS_KEY ? d + G.m : d;
            const uint8_t *W = (const uint8_t *)(IS_KEY ? P.RSsw : P.Rsw);
            const size_t wlo = (size_t)wrows * d * 2;
            const uint8_t *Sp = (const uint8_t *)P.Ssw;
            const size_t slo = (size_t)G.m * d * 2;
            int gk = 0, issued = 0;
            bool ok = true;
            if (EX) prefetch_tmap(&xmap);
            for (int i = 0; ok && i < my_tiles; ++i)
                for (int c = 0; ok && c < NC; ++c) {
                    const int w = G.width(c), n0 = G.n0(c), nkb = nkb_of(c);
                    const uint32_t bytes = (uint32_t)w * 128;
                    for (int kb = 0; kb < nkb; ++kb, ++gk) {
                        const int st = gk % kBStages;
                        const bool sp_blk = RP ? c >= G.nr : kb >= dkb;  // a K-block of S'
                        const int kbs = RP ? kb : kb - dkb;
                        if (gk >= kBStages && !mbar_wait(&bars[kBEmpty + st], ((gk / kBStages) - 1) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
                        const uint8_t *src;
                        size_t lo;
                        if (!sp_blk) {
                            const int row0 = c < G.nr ? n0 : d + n0;
                            src = W + ((size_t)kb * wrows + row0) * 128;
                            lo = wlo;
                        } else {
                            src = Sp + ((size_t)kbs * G.m + n0) * 128;
                            lo = slo;
                        }
                        uint8_t *dst = sm + L.stage + st * kBStage + 2 * kATile;
                        // exact path: A is the fp16 input tile itself, 128 rows x 64 coordinates in
                        // the 128-byte swizzle (rows past n read as zeros)
                        const bool xa = EX && c < G.nr;
                        mbar_arrive_expect_tx(&bars[kBFull + st], 2 * bytes + (xa ? kATile : 0u));
                        if (xa)
                            tma_load_2d(sm + L.stage + st * kBStage, &xmap, &bars[kBFull + st], 64 * kb,
                                        (int)((blockIdx.x + (int64_t)i * gridDim.x) * kBRows));
                        bulk_load(dst, src, bytes, &bars[kBFull + st]);
                        bulk_load(dst + kBTileMax, src + lo, bytes, &bars[kBFull + st]);
                        issued = gk + 1;
                    }
                }
            // every copy must land before the CTA can exit (bounded waits)
            int dummy = 0;
            for (int g = issued > kBStages ? issued - kBStages : 0; g < issued; ++g)
                mbar_wait(&bars[kBFull + g % kBStages], (g / kBStages) & 1, (volatile int *)&dummy);
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t sbase = smem_u32(sm + L.stage);
            int gk = 0, gc = 0;
            bool ok = true;
            for (int i = 0; ok && i < my_tiles; ++i)
                for (int c = 0; ok && c < NC; ++c, ++gc) {
                    const int slot = gc & 1;
                    if constexpr (RP) {
                        // slot 0: rotation of tile i, then its residual; slot 1: its projection
                        bool w = true;
                        if (c < G.nr) {
                            // the projection of tile i - 1 has read the residual in slot 0
                            if (i >= 1) w = mbar_wait(&bars[kBAccFull + 1], (i - 1) & 1, abort_s);
                        } else {
                            // tile i's residual is written; tile i - 1's projection has been read
                            w = mbar_wait(&bars[kBAccEmpty + 0], i & 1, abort_s);
                            if (w && i >= 1) w = mbar_wait(&bars[kBAccEmpty + 1], (i - 1) & 1, abort_s);
                        }
                        if (!w) {
                            ok = false;
                            break;
                        }
                    } else if (gc >= 2 && !mbar_wait(&bars[kBAccEmpty + slot], ((gc >> 1) - 1) & 1, abort_s)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t acc0 = tmem + slot * kBChunk;
                    const uint32_t idesc = idesc_f16_f32(kBRows, G.width(c));
                    const int nkb = nkb_of(c);
                    if (RP && c >= G.nr) {
                        // projection: A = 2^14 e (hi | lo per 32 coordinates) in slot 0
                        for (int kb = 0; kb < nkb; ++kb, ++gk) {
                            const int st = gk % kBStages;
                            if (!mbar_wait(&bars[kBFull + st], (gk / kBStages) & 1, abort_s)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const uint32_t b_hi = sbase + st * kBStage + 2 * kATile, b_lo = b_hi + kBTileMax;
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int K = 4 * kb + k;
                                const uint32_t a_hi = tmem + 32 * (K >> 1) + 8 * (K & 1), a_lo = a_hi + 16;
                                const uint64_t dh = sdesc_sw128(b_hi + 32 * k), dl = sdesc_sw128(b_lo + 32 * k);
                                mma_ts(acc0, a_hi, dh, idesc, (kb | k) ? 1u : 0u);
                                mma_ts(acc0, a_hi, dl, idesc, 1u);
                                mma_ts(acc0, a_lo, dh, idesc, 1u);
                            }
                            mma_commit(&bars[kBEmpty + st]);
                        }
                        if (ok) mma_commit(&bars[kBAccFull + slot]);
                        continue;
                    }
                    for (int kb = 0; kb < nkb; ++kb, ++gk) {
                        const int st = gk % kBStages;
                        if (!mbar_wait(&bars[kBFull + st], (gk / kBStages) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_hi = sbase + st * kBStage, a_lo = a_hi + kATile;
                        const uint32_t b_hi = a_hi + 2 * kATile, b_lo = b_hi + kBTileMax;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint32_t o = 32 * k;
                            mma_ss(acc0, sdesc_sw128(a_hi + o), sdesc_sw128(b_hi + o), idesc, (kb | k) ? 1u : 0u);
                            mma_ss(acc0, sdesc_sw128(a_hi + o), sdesc_sw128(b_lo + o), idesc, 1u);
                            if (!exact) mma_ss(acc0, sdesc_sw128(a_lo + o), sdesc_sw128(b_hi + o), idesc, 1u);
                        }
                        mma_commit(&bars[kBEmpty + st]);
                    }
                    if (ok) mma_commit(&bars[kBAccFull + slot]);
                }
        }
    } else if (warp < kEpi0) {
        // -------------------------------------------------------- A tiles, one vector per thread
        // (the exact path's producer loads A by TMA: no converter work)
        if constexpr (!EX) {
        const int cg = SPLIT ? 0 : (warp - kCvtWarp0) >> 2;  // group: K-block steps gk with gk % 2 == cg
        const int r = (threadIdx.x - kCvtWarp0 * 32) & 127;  // the vector this thread converts
        const uint32_t rowb = (uint32_t)r * 128;
        int gk = 0;
        bool ok = true;
        for (int i = 0; ok && i < my_tiles; ++i) {
            const int64_t v = (blockIdx.x + (int64_t)i * gridDim.x) * kBRows + r;
            const bool valid = v < n;
            // ||x|| in fp32 from the input row (the exact path takes it from the accumulator)
            float ss = 0.f;
            if (valid && !exact) {
                if (F16) {
                    const uint4 *xr = (const uint4 *)((const __half *)xin + v * d);
                    for (int j = 0; j < d / 8; ++j) {
                        const uint4 q = __ldg(xr + j);
                        const uint32_t u4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __half22float2(*(const __half2 *)&u4[e]);
                            ss = fmaf(f.x, f.x, ss);
                            ss = fmaf(f.y, f.y, ss);
                        }
                    }
                } else {
                    const float4 *xr = (const float4 *)((const float *)xin + v * d);
                    for (int j = 0; j < d / 4; ++j) {
                        const float4 f = __ldg(xr + j);
                        ss = fmaf(f.x, f.x, ss);
                        ss = fmaf(f.y, f.y, ss);
                        ss = fmaf(f.z, f.z, ss);
                        ss = fmaf(f.w, f.w, ss);
                    }
                }
            }
            const float nrm = sqrtf(ss);
            const float us = nrm > 0.f ? (float)(1 << kUScaleLog2) / nrm : 0.f;
            if (valid && cg == 0 && !exact) norm[v] = f32_to_f16_bits(nrm);
            bool have_codes = false;
            for (int c = 0; ok && c < NC; ++c) {
                const int nkb = nkb_of(c);
                for (int kb = 0; kb < nkb; ++kb, ++gk) {
                    if (!SPLIT && (gk & 1) != cg) continue;
                    const int st = gk % kBStages;
                    uint8_t *ah = sm + L.stage + st * kBStage;
                    uint8_t *al = ah + kATile;
                    if (RP && c >= G.nr) {
                        // the projection's A operand is in TMEM: only keep the stage's arrivals
                        if (gk >= kBStages && !mbar_wait(&bars[kBEmpty + st], ((gk / kBStages) - 1) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
                    } else if (kb < dkb) {
                        // U = u 2^10 for coordinates 64 kb .. 64 kb + 63, fp16 hi | lo; the inputs
                        // are fetched before waiting for the stage to free up
                        constexpr int NQ = F16 ? 8 : 16;
                        uint4 q[NQ];
#pragma unroll
                        for (int e = 0; e < NQ; ++e) {
                            q[e] = make_uint4(0u, 0u, 0u, 0u);
                            if (valid)
                                q[e] = __ldg((const uint4 *)((const char *)xin + (v * d + 64 * kb) * (F16 ? 2 : 4)) + e);
                        }
                        if (gk >= kBStages && !mbar_wait(&bars[kBEmpty + st], ((gk / kBStages) - 1) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
                        if (F16 && exact) {
                            // the fp16 row itself, one 16-byte chunk of 8 coordinates at a time
#pragma unroll
                            for (int cc = 0; cc < 8; ++cc)
                                *(uint4 *)(ah + rowb + (((uint32_t)cc ^ (r & 7)) << 4)) = q[cc];
                        } else {
#pragma unroll
                        for (int cc = 0; cc < 8; ++cc) {
                            float f[8];
                            if (F16) {
                                const uint32_t u4[4] = {q[cc].x, q[cc].y, q[cc].z, q[cc].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 h2 = __half22float2(*(const __half2 *)&u4[e]);
                                    f[2 * e] = h2.x;
                                    f[2 * e + 1] = h2.y;
                                }
                            } else {
                                const uint4 a0 = q[2 * cc], a1 = q[2 * cc + 1];
                                f[0] = __uint_as_float(a0.x); f[1] = __uint_as_float(a0.y);
                                f[2] = __uint_as_float(a0.z); f[3] = __uint_as_float(a0.w);
                                f[4] = __uint_as_float(a1.x); f[5] = __uint_as_float(a1.y);
                                f[6] = __uint_as_float(a1.z); f[7] = __uint_as_float(a1.w);
                            }
                            uint32_t hv[4], lv4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                hv[e] = hsplit2(f[2 * e] * us, f[2 * e + 1] * us, false);
                                lv4[e] = hsplit2(f[2 * e] * us, f[2 * e + 1] * us, true);
                            }
                            const uint32_t off = rowb + (((uint32_t)cc ^ (r & 7)) << 4);
                            *(uint4 *)(ah + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                            *(uint4 *)(al + off) = make_uint4(lv4[0], lv4[1], lv4[2], lv4[3]);
                        }
                        }
                    } else {
                        // correction: -c[idx] 2^14 for coordinates 64 kbc .. 64 kbc + 63 from the
                        // tile's codes, which the epilogue has just written
                        if (!have_codes) {
                            if (!mbar_wait(&bars[kBCodes + (i & 1)], (i >> 1) & 1, abort_s)) {
                                ok = false;
                                break;
                            }
                            have_codes = true;
                        }
                        const int kbc = kb - dkb;
                        uint32_t w[2][BETA];
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int p = 0; p < BETA; ++p)
                                w[h][p] = valid ? codes[v * KWPT + (2 * kbc + h) * BETA + p] : 0u;
                        if (gk >= kBStages && !mbar_wait(&bars[kBEmpty + st], ((gk / kBStages) - 1) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
#pragma unroll
                            for (int cc = 0; cc < 4; ++cc) {
                                uint32_t hv[4], lv4[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int l = 8 * cc + 2 * e;
                                    uint32_t i0 = 0, i1 = 0;
#pragma unroll
                                    for (int p = 0; p < BETA; ++p) {
                                        i0 |= ((w[h][p] >> l) & 1u) << p;
                                        i1 |= ((w[h][p] >> (l + 1)) & 1u) << p;
                                    }
                                    const uint32_t t0 = ctab[i0], t1 = ctab[i1];
                                    hv[e] = valid ? __byte_perm(t0, t1, 0x5410) : 0u;
                                    lv4[e] = valid ? __byte_perm(t0, t1, 0x7632) : 0u;
                                }
                                const uint32_t off = rowb + (((uint32_t)(4 * h + cc) ^ (r & 7)) << 4);
                                *(uint4 *)(ah + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                                *(uint4 *)(al + off) = make_uint4(lv4[0], lv4[1], lv4[2], lv4[3]);
                            }
                        }
                    }
                    // generic-proxy stores must be visible to the tensor core (async proxy)
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kBFull + st]);
                }
            }
        }
        }
    } else {
        // -------------------------------------------------------- epilogue, one vector per thread
        const int q4 = warp & 3;  // TMEM lane quarter this warp may read
        const int r = 32 * q4 + lane;
        const int hf = SPLIT ? (warp - kEpi0) >> 2 : 0;  // column half of this warp
        constexpr int NHF = SPLIT ? 2 : 1;
        constexpr int HL = 1 << (BETA - 1);
        float edge[HL > 1 ? HL - 1 : 1], cmag[HL];  // positive boundaries; 2^14 |c| (keys)
#pragma unroll
        for (int k = 0; k < HL - 1; ++k) edge[k] = bnd_s[HL + k];
#pragma unroll
        for (int k = 0; k < HL; ++k) cmag[k] = cen_s[HL + k] * kEScale;
        constexpr float kYUnscale = 1.0f / (float)(1 << (kUScaleLog2 + kRScaleLog2));
        int gc = 0;
        bool ok = true;
        for (int i = 0; ok && i < my_tiles; ++i) {
            const int64_t v = (blockIdx.x + (int64_t)i * gridDim.x) * kBRows + r;
            const bool valid = v < n;
            float2 ee2 = make_float2(0.f, 0.f);  // (2^14 ||y - c||)^2 over even | odd coordinates
            float na = 0.f;  // exact path: ||ACC|| of the rotation chunk (2^8 ||x||)
            for (int c = 0; c < NC; ++c, ++gc) {
                const int slot = gc & 1;
                if (!mbar_wait(&bars[kBAccFull + slot], (gc >> 1) & 1, abort_s)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tl = tmem + ((uint32_t)(32 * q4) << 16) + slot * kBChunk;
                const int ng = G.width(c) / 32, g0 = G.n0(c) / 32;
                const int gA = hf * ng / NHF, gB = (hf + 1) * ng / NHF;  // this warp's column groups
                // exact path: ACC = 2^8 R x; ||x|| = ||ACC|| / 2^8 and y = ACC / ||ACC||
                float yscale = kYUnscale;
                if (exact && c < G.nr) {
                    float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll 1
                    for (int g = gA; g < gB; ++g) {
                        uint32_t a[32];
                        tmem_ld32(tl + 32 * g, a);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float2 a2 = make_float2(__uint_as_float(a[2 * k]), __uint_as_float(a[2 * k + 1]));
                            ss2 = __ffma2_rn(a2, a2, ss2);
                        }
                    }
                    if constexpr (SPLIT) {
                        // the halves meet in shared memory (slots of tile parity; a slot is next
                        // written two tiles on, after both halves have released this tile's chunks)
                        float *xn = xn_s + (i & 1) * 2 * kBRows;
                        xn[hf * kBRows + r] = ss2.x + ss2.y;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars[kBNorm + (i & 1)]);
                        if (!mbar_wait(&bars[kBNorm + (i & 1)], (i >> 1) & 1, abort_s)) {
                            ok = false;
                            break;
                        }
                        na = sqrtf(xn[r] + xn[kBRows + r]);
                    } else {
                        na = sqrtf(ss2.x + ss2.y);
                    }
                    yscale = na > 0.f ? 1.0f / na : 0.f;
                    if (valid && hf == 0) norm[v] = f32_to_f16_bits(na * (1.0f / (float)(1 << kRScaleLog2)));
                }
                if (c < G.nr) {
                    // codes of rotated coordinates 32 (g0 + g) .. + 31, planar words.  y = ACC yscale
                    // is compared as ACC against the boundaries scaled by 1 / yscale; a zero vector
                    // compares its zero accumulator against the unscaled ones (y = 0).
                    const float sc = yscale > 0.f ? (exact ? na : 1.0f / kYUnscale) : 1.f;
                    float ep[HL > 1 ? HL - 1 : 1];
#pragma unroll
                    for (int k = 0; k < HL - 1; ++k) ep[k] = edge[k] * sc;
                    const float ys14 = yscale * kEScale;  // ACC -> 2^14 y
#pragma unroll 1
                    for (int g = gA; g < gB; ++g) {
                        uint32_t a[32];
                        tmem_ld32(tl + 32 * g, a);
                        tmem_ld_wait();
                        // words of [y > 0] and of the magnitude digits; the code planes follow per word
                        uint32_t sgn = 0u, mbw[BETA > 1 ? BETA - 1 : 1];
#pragma unroll
                        for (int j = 0; j < BETA - 1; ++j) mbw[j] = 0u;
                        uint32_t hp[RP ? 16 : 1], lp[RP ? 16 : 1];  // RP: fp16 hi | lo of 2^14 e, pairs
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            float es[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int l = 2 * k + u;
                                const float av = __uint_as_float(a[l]), ua = fabsf(av);
                                const bool pos = av > 0.f;
                                bool mb[3] = {false, false, false};
                                big_mag<BETA>(ua, ep, mb);
                                if (pos) sgn |= 1u << l;
#pragma unroll
                                for (int j = 0; j < BETA - 1; ++j)
                                    if (mb[j]) mbw[j] |= 1u << l;
                                if (IS_KEY) {
                                    // y - c = sign(y) (|y| - |c|), 2^14 scaled
                                    const float em = fmaf(ua, ys14, -big_cmag<BETA>(mb, cmag));
                                    es[u] = pos ? em : -em;
                                }
                            }
                            if (IS_KEY) {
                                const float2 e2 = make_float2(es[0], es[1]);
                                ee2 = __ffma2_rn(e2, e2, ee2);
                                if constexpr (RP) {
                                    const __half2 hh = __floats2half2_rn(e2.x, e2.y);
                                    const float2 h2 = __half22float2(hh);
                                    const __half2 ll = __floats2half2_rn(e2.x - h2.x, e2.y - h2.y);
                                    hp[k] = *(const uint32_t *)&hh;
                                    lp[k] = *(const uint32_t *)&ll;
                                }
                            }
                        }
                        uint32_t wp[BETA];
                        wp[BETA - 1] = sgn;
#pragma unroll
                        for (int j = 0; j < BETA - 1; ++j) wp[j] = ~(mbw[j] ^ sgn);
                        if constexpr (RP) {
                            // in place: group g's 32 fp32 columns become its hi (16) and lo (16)
                            tmem_st16(tl + 32 * g, hp);
                            tmem_st16(tl + 32 * g + 16, lp);
                        }
                        if (valid) {
#pragma unroll
                            for (int p = 0; p < BETA; ++p) codes[v * KWPT + (g0 + g) * BETA + p] = wp[p];
                        }
                    }
                    if (IS_KEY && c == G.nr - 1) {
                        // every code word of this tile is out: release the correction operands.
                        // Exact path: half 1 hands its part of ||y - c||^2 to half 0 first.
                        float ee = (ee2.x + ee2.y) * (1.0f / (kEScale * kEScale));
                        if (SPLIT && hf == 1) {
                            xe_s[(i & 1) * kBRows + r] = ee;
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&bars[kBEe + (i & 1)]);
                        } else {
                            if (SPLIT) {
                                if (!mbar_wait(&bars[kBEe + (i & 1)], (i >> 1) & 1, abort_s)) {
                                    ok = false;
                                    break;
                                }
                                ee += xe_s[(i & 1) * kBRows + r];
                            }
                            if (valid) rnorm[v] = f32_to_f16_bits(sqrtf(ee));
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bars[kBCodes + (i & 1)]);
                    }
                } else {
                    // signs of the projections 32 (g0 + g) .. + 31: sign(S u - S' c) = sign(ACC).
                    // In the two-term form the terms are O(1) and cancel to p; the accumulator's
                    // rounding grows with d (a few 1e-5 of p at d = 1024), so projections with
                    // |p| < kSignRecheck (kSignRecheckResidual in the residual form) are recomputed
                    // in double by the warp, from x, the codes, S and S'.
                    const int64_t vbase = v - lane;
                    // a recheck reads the vector's codes from both column halves
                    if (RP && !mbar_wait(&bars[kBCodes + (i & 1)], (i >> 1) & 1, abort_s)) {
                        ok = false;
                        break;
                    }
#pragma unroll 1
                    for (int g = gA; g < gB; ++g) {
                        uint32_t a[32];
                        tmem_ld32(tl + 32 * g, a);
                        tmem_ld_wait();
                        uint32_t sw = 0, unc = 0;
#pragma unroll
                        for (int l = 0; l < 32; ++l) {
                            const float pv = __uint_as_float(a[l]);
                            sw |= (uint32_t)(pv >= 0.f) << l;
                            unc |= (uint32_t)(fabsf(pv) < (RP ? kSignRecheckResidual : kSignRecheck) * kPUnscaleInv) << l;
                        }
                        if (!valid) unc = 0;
                        uint32_t pend = __ballot_sync(kFull, unc != 0);
                        while (pend) {
                            const int src = __ffs(pend) - 1;
                            pend &= pend - 1;
                            uint32_t um = __shfl_sync(kFull, unc, src);
                            while (um) {
                                const int l = __ffs(um) - 1;
                                um &= um - 1;
                                const double pe = exact_projection<BETA, F16>(P, G, xin, codes, vbase + src,
                                                                              32 * (g0 + g) + l, lane, cen_s);
                                if (lane == src) sw = (sw & ~(1u << l)) | ((uint32_t)(pe >= 0.0) << l);
                            }
                        }
                        if (valid) signs[v * SWPT + g0 + g] = sw;
                    }
                }
                if (RP && c < G.nr) tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kBAccEmpty + slot]);
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

PFN_cuTensorMapEncodeTiled_v12000 big_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

template <bool IS_KEY, int BETA, bool F16>
cudaError_t launch_big(const Prepared &P, const BigGeom &G, const void *x, int64_t n, uint32_t *codes, uint32_t *signs,
                       uint16_t *norm, uint16_t *rnorm, int32_t *dev_status, cudaStream_t s) {
    const BigSmem L = big_smem_layout();
    const size_t smem = L.total + 1024;
    // the exact path for fp16 input with one rotation chunk; its code step split over eight warps
    // where it is heavy (keys; values of 3 or 4 bits)
    const bool ex = F16 && G.nr == 1 && (!IS_KEY || G.ns == 1) && n <= (int64_t)INT32_MAX;
    const bool split = ex && (IS_KEY || BETA >= 3);
    auto kern = compress_big_kernel<IS_KEY, BETA, F16, false, false>;
    if (split) kern = compress_big_kernel<IS_KEY, BETA, F16, F16, F16>;
    if constexpr (!IS_KEY) {
        if (ex && !split) kern = compress_big_kernel<IS_KEY, BETA, F16, F16, false>;
    }
    // exact path: a tensor map over the fp16 rows (n x d), 64 x 128 boxes in the 128-byte swizzle
    CUtensorMap xmap;
    memset(&xmap, 0, sizeof(xmap));
    if (ex) {
        auto encode = big_encode_fn();
        if (!encode) return cudaErrorNotSupported;
        cuuint64_t dims[2] = {(cuuint64_t)G.d, (cuuint64_t)n};
        cuuint64_t strides[1] = {(cuuint64_t)G.d * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)kBRows};
        cuuint32_t estr[2] = {1, 1};
        if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ntiles = (n + kBRows - 1) / kBRows;
    const int grid = (int)(ntiles < sms ? ntiles : sms);
    kern<<<grid, kBThreads, smem, s>>>(xmap, P, G, x, n, codes, signs, norm, rnorm, dev_status);
    return cudaGetLastError();
}

template <bool IS_KEY, bool F16>
cudaError_t launch_big_beta(const Prepared &P, const BigGeom &G, int beta, const void *x, int64_t n, uint32_t *codes,
                            uint32_t *signs, uint16_t *norm, uint16_t *rnorm, int32_t *dev_status, cudaStream_t s) {
    switch (beta) {
        case 1: return launch_big<IS_KEY, 1, F16>(P, G, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 2: return launch_big<IS_KEY, 2, F16>(P, G, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 3: return launch_big<IS_KEY, 3, F16>(P, G, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 4:
            if constexpr (!IS_KEY) return launch_big<IS_KEY, 4, F16>(P, G, x, n, codes, signs, norm, rnorm, dev_status, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool compress_big_supported(const Prepared &P, bool is_key) {
    if (P.d < 64 || P.d > 1024 || P.d % 64) return false;
    if (is_key && (P.m < 32 || P.m % 32)) return false;
    return true;
}

cudaError_t launch_compress_big(const Prepared &P, bool is_key, const void *x, bool x_f16, int64_t n,
                                uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                                int32_t *dev_status, cudaStream_t s) {
    BigGeom G;
    G.d = P.d;
    G.m = is_key ? P.m : 0;
    G.nr = (P.d + kBChunk - 1) / kBChunk;
    G.ns = is_key ? (P.m + kBChunk - 1) / kBChunk : 0;
    const int beta = is_key ? P.kbeta : P.vbeta;
    if (is_key)
        return x_f16 ? launch_big_beta<true, true>(P, G, beta, x, n, codes, signs, norm, rnorm, dev_status, s)
                     : launch_big_beta<true, false>(P, G, beta, x, n, codes, signs, norm, rnorm, dev_status, s);
    return x_f16 ? launch_big_beta<false, true>(P, G, beta, x, n, codes, signs, norm, rnorm, dev_status, s)
                 : launch_big_beta<false, false>(P, G, beta, x, n, codes, signs, norm, rnorm, dev_status, s);
}

}  // namespace tq
