// tq_compress_tc.cu -- key / value compression on the fifth-generation tensor cores.
//
// Per 128-vector tile (TurboQuantMSE.quantize / TurboQuantProd.compress; "turboquant-pytorch",
// nav.superapi.store, 核心 API; atskills.one, "What It Does" stage 1 + stage 2):
//   rotation    ACC[v, j] = sum_i X[v, i] (R_hi + R_lo)[j, i]          tcgen05, smem x smem
//               (X is the fp16 input tile, exact in fp16; R * 2^8 = R_hi + R_lo in fp16, so
//               the product carries ~22 bits of R and the accumulator is fp32)
//   code step   n = ||R x|| = ||ACC|| / 2^8 (the two halves of a row summed by its two threads),
//               y = ACC / (2^8 n), idx = code of y, planar pack;
//               keys: e = 2^14 (y - c[idx]) split into fp16 hi + lo, written back into TMEM
//   projection  P[v, a] = sum_j (E_hi (S'_hi + S'_lo) + E_lo S'_hi)[v, j]   tcgen05, tmem x smem
//               with S' = S R^T, so P is a positive multiple of S r for the residual r = R^T e;
//   sign step   QJL sign bits of P.
// One thread owns one vector (one TMEM lane) and half of its coordinates.  Warp roles (10 warps):
// warp 0 loads (TMA) and owns TMEM, warp 1 issues the MMAs, warps 2..9 run the norm, code and
// sign steps of every tile.  TMEM holds up to four rotation accumulators
// (keys: three beside two projection accumulators), so the rotation of later tiles and the
// projection of earlier ones keep the tensor cores busy while a tile is being coded.
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {

namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kEpiWarp0 = 2;   // warps 2..9: epilogue (two groups of four)
constexpr int kEpiWarps = 8;   // warps 2..9
constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);

constexpr int kEScaleLog2 = 14;  // residual scale before the fp16 hi/lo split

struct TcSmem {
    // offsets from the 1024-aligned dynamic shared memory base
    uint32_t R, S, X, bars, misc;
    uint32_t total;
    int nst;  // input stages
    int nrs;  // rotation accumulators in TMEM
};

// Rotation accumulators (D columns each) that fit in the 512 TMEM columns beside the keys' two
// projection accumulators (m columns each); at most four.
__host__ __device__ inline int tc_rotation_slots(int D, int m, bool is_key) {
    const int r = is_key ? (512 - 2 * m) / D : 512 / D;
    return r > 4 ? 4 : r;
}

// misc block: codebook and flags (256 B), squared row norms [4][128], half residual norms [4][128]
constexpr uint32_t kMiscNorm = 256, kMiscEe = 256 + 4096;
constexpr uint32_t kMiscBytes = kMiscEe + 2048;

__host__ __device__ inline TcSmem tc_smem_layout(int D, int m, bool is_key) {
    TcSmem L;
    uint32_t o = 0;
    L.R = o;
    o += 2u * D * D * 2;  // R hi | lo
    L.S = o;
    if (is_key) o += 2u * m * D * 2;  // S' = S R^T, hi | lo
    L.X = o;
    const uint32_t xs = kTileRows * D * 2;
    const uint32_t budget = 225u * 1024 - o - 256 - kMiscBytes;
    int nst = (int)(budget / xs);
    if (nst > 4) nst = 4;
    L.nst = nst;
    L.nrs = tc_rotation_slots(D, m, is_key);
    o += nst * xs;
    L.bars = o;
    o += 256;
    L.misc = o;
    o += kMiscBytes;
    L.total = o;
    return L;
}

enum BarIdx {
    kOpnd = 0,
    kFull = 1,       // [4] input stage landed
    kEmpty = 5,      // [4] input stage consumed (its rotation MMAs completed)
    kRotFull = 9,    // [4] rotation accumulator ready
    kEReady = 13,    // [4] codes written; keys: residual in TMEM; values: accumulator free
    kNormReady = 17, // [4] both halves' squared row norms of the slot's tile
    kPartReady = 21, // [4] half-1 residual norms handed to half 0
    kProjFull = 25,  // [2] projection accumulator ready (and its residual operand consumed)
    kAccFree = 27    // [2] projection accumulator read
};

// Magnitude digits of u = |y| against the HL - 1 = 2^(BETA-1) - 1 positive boundaries e[] of a
// symmetric codebook (binary search, thresholds selected from registers): mb[j] receives bit j
// of m = #{k : e[k] < u}.  The code of y is then HL + m for y > 0 and HL - 1 - m otherwise, so its
// low bits are m's bits, complemented on the negative side, and its top bit is the sign.
template <int BETA>
__device__ __forceinline__ void magnitude_bits(float u, const float *e, bool (&mb)[3]) {
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

template <int D, bool IS_KEY, int BETA>
__global__ void __launch_bounds__(kThreads, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap tmap, Prepared P, int64_t n,
                       uint32_t *__restrict__ codes, uint32_t *__restrict__ signs, uint16_t *__restrict__ norm,
                       uint16_t *__restrict__ rnorm, int32_t *__restrict__ dev_status) {
    constexpr int KSTEPS = D / 16;
    constexpr int CHUNKS = D / 32;
    constexpr uint32_t XSTAGE = kTileRows * D * 2;
    const int m = IS_KEY ? P.m : 0;
    const TcSmem L = tc_smem_layout(D, m, IS_KEY);
    const int NST = L.nst, NRS = L.nrs;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    float *bnd_s = (float *)(sm + L.misc);
    float *cen_s = bnd_s + kMaxLevels;
    uint32_t *tmem_s = (uint32_t *)(cen_s + kMaxLevels);
    volatile int *abort_s = (volatile int *)(tmem_s + 1);
    float *norm_s = (float *)(sm + L.misc + kMiscNorm);    // [half][slot][row] partial squared norms
    float *ee_s = (float *)(sm + L.misc + kMiscEe);        // [slot][row] half residual norms

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntiles = (n + kTileRows - 1) / kTileRows;
    const int my_tiles = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

    if (threadIdx.x == 0) {
        mbar_init(&bars[kOpnd], 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars[kFull + s], 1);
            mbar_init(&bars[kEmpty + s], 1);  // MMA commit
            mbar_init(&bars[kRotFull + s], 1);
            mbar_init(&bars[kEReady + s], 8);
            mbar_init(&bars[kNormReady + s], kEpiWarps);
            mbar_init(&bars[kPartReady + s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kProjFull + s], 1);
            mbar_init(&bars[kAccFree + s], 8);
        }
        *abort_s = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kMaxLevels) {
        bnd_s[threadIdx.x] = IS_KEY ? P.cb->kb[threadIdx.x] : P.cb->vb[threadIdx.x];
        cen_s[threadIdx.x] = IS_KEY ? P.cb->kc[threadIdx.x] : P.cb->vc[threadIdx.x];
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap);
            const uint32_t rbytes = 2u * D * D * 2;
            const uint32_t sbytes = IS_KEY ? 2u * m * D * 2 : 0u;
            mbar_arrive_expect_tx(&bars[kOpnd], rbytes + sbytes);
            bulk_load(sm + L.R, P.Rsw, rbytes, &bars[kOpnd]);
            if (IS_KEY) bulk_load(sm + L.S, P.Ssw, sbytes, &bars[kOpnd]);
            int issued = 0;
            for (int i = 0; i < my_tiles; ++i) {
                const int stage = i % NST;
                if (i >= NST && !mbar_wait(&bars[kEmpty + stage], ((i / NST) - 1) & 1, abort_s)) break;
                const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
                uint8_t *dst = sm + L.X + stage * XSTAGE;
                mbar_arrive_expect_tx(&bars[kFull + stage], XSTAGE);
#pragma unroll
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_2d(dst + kb * (kTileRows * 128), &tmap, &bars[kFull + stage], kb * 64,
                                (int)(tile * kTileRows));
                ++issued;
            }
            // never leave with copies in flight: wait (bounded) for the last stages to land
            for (int i = (issued > NST ? issued - NST : 0); i < issued; ++i) {
                int dummy = 0;
                mbar_wait(&bars[kFull + (i % NST)], (i / NST) & 1, (volatile int *)&dummy);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_rot = idesc_f16_f32(128, D);
            const uint32_t idesc_prj = idesc_f16_f32(128, m > 0 ? m : 16);
            const uint32_t sR = smem_u32(sm + L.R), sS = smem_u32(sm + L.S), sX = smem_u32(sm + L.X);
            bool ok = mbar_wait(&bars[kOpnd], 0, abort_s);
            // rotation of tile i into accumulator slot i % NRS, once the slot's previous tile has
            // released it (keys: its residual was consumed by the projection; values: its codes
            // are out)
            auto rotation = [&](int i) -> bool {
                const int rs = i % NRS, stage = i % NST;
                if (i >= NRS) {
                    const bool w = IS_KEY ? mbar_wait(&bars[kProjFull + ((i - NRS) & 1)], ((i - NRS) >> 1) & 1, abort_s)
                                          : mbar_wait(&bars[kEReady + rs], ((i / NRS) - 1) & 1, abort_s);
                    if (!w) return false;
                }
                if (!mbar_wait(&bars[kFull + stage], (i / NST) & 1, abort_s)) return false;
                tc_fence_after();
                const uint32_t acc = tmem + rs * D;
                const uint32_t xbase = sX + stage * XSTAGE;
                uint32_t first = 0;
#pragma unroll
                for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                    for (int k = 0; k < KSTEPS; ++k) {
                        const uint32_t aoff = (uint32_t)(k >> 2) * (kTileRows * 128) + (k & 3) * 32;
                        const uint32_t boff = (uint32_t)pass * (D * D * 2) + (uint32_t)(k >> 2) * (D * 128) + (k & 3) * 32;
                        mma_ss(acc, sdesc_sw128(xbase + aoff), sdesc_sw128(sR + boff), idesc_rot, first);
                        first = 1;
                    }
                mma_commit(&bars[kEmpty + stage]);
                mma_commit(&bars[kRotFull + rs]);
                return true;
            };
            // projection of tile j's residual (hi | lo in its rotation slot) into accumulator j & 1
            auto projection = [&](int j) -> bool {
                const int rs = j % NRS, pa = j & 1;
                if (!mbar_wait(&bars[kEReady + rs], (j / NRS) & 1, abort_s)) return false;
                if (j >= 2 && !mbar_wait(&bars[kAccFree + pa], ((j >> 1) - 1) & 1, abort_s)) return false;
                tc_fence_after();
                const uint32_t acc = tmem + NRS * D + pa * m;
                const uint32_t sbytes = (uint32_t)m * D * 2;
                uint32_t first = 0;
                // unrolled: a single thread issues the MMAs, and loop overhead between issues
                // would starve the tensor cores (N = 64 MMAs take about 45 cycles each)
#pragma unroll
                for (int k = 0; k < KSTEPS; ++k) {
                    const uint32_t a_hi = tmem + rs * D + 32 * (k >> 1) + 8 * (k & 1);
                    const uint32_t a_lo = a_hi + 16;
                    const uint32_t boff = (uint32_t)(k >> 2) * m * 128 + (k & 3) * 32;
                    const uint64_t b_hi = sdesc_sw128(sS + boff);
                    const uint64_t b_lo = sdesc_sw128(sS + sbytes + boff);
                    mma_ts(acc, a_hi, b_hi, idesc_prj, first);
                    first = 1;
                    mma_ts(acc, a_hi, b_lo, idesc_prj, 1);
                    mma_ts(acc, a_lo, b_hi, idesc_prj, 1);
                }
                mma_commit(&bars[kProjFull + pa]);
                return true;
            };
            if (IS_KEY) {
                // rotations run NRS - 1 tiles ahead of the projections
                for (int i = 0; ok && i < NRS - 1 && i < my_tiles; ++i) ok = rotation(i);
                for (int j = 0; ok && j < my_tiles; ++j) {
                    if (!projection(j)) break;
                    if (j + NRS - 1 < my_tiles && !rotation(j + NRS - 1)) break;
                }
            } else {
                for (int i = 0; ok && i < my_tiles; ++i) ok = rotation(i);
            }
        }
    } else if (warp < kEpiWarp0 + kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        // Every tile goes to all eight warps: warp (q, h) takes rows 32q..32q+31 (its TMEM lane
        // quarter) and half h of the coordinates and of the projections.  Keys run the code step
        // of tile i, then the sign step of tile i - 1, so the projection of tile i - 1 executes
        // on the tensor cores while tile i is being coded.
        const int ew = warp - kEpiWarp0;   // 0..7
        const int h = ew >> 2;             // which half of the columns
        const int q = warp & 3;            // TMEM subpartition this warp may access
        const int row = 32 * q + lane;     // vector within the tile
        const uint32_t lanes = (uint32_t)(32 * q) << 16;
        constexpr int CH = CHUNKS / 2;     // 32-coordinate chunks per warp
        constexpr int wpv = BETA * CHUNKS;
        const int spk = m >> 5;
        // Both codebooks are symmetric (c[HL + k] = -c[HL - 1 - k] exactly, middle boundary 0), so a
        // coordinate is coded from its sign and the magnitude digits of |y| against the HL - 1
        // positive boundaries; a key's centroid is sign(y) cmag[m] and (y - c)^2 = (|y| - cmag[m])^2.
        constexpr int HL = 1 << (BETA - 1);
        float edge[HL > 1 ? HL - 1 : 1];
#pragma unroll
        for (int k = 0; k < HL - 1; ++k) edge[k] = bnd_s[HL + k];
        float cmag[HL];  // 2^14 |c| (keys)
#pragma unroll
        for (int k = 0; k < HL; ++k) cmag[k] = cen_s[HL + k] * (float)(1 << kEScaleLog2);

        // codes of tile i; keys also leave 2^14 (y - c) as fp16 hi | lo in the slot's columns
        auto code_step = [&](int i) -> bool {
            const int rs = i % NRS;
            const uint32_t ph = (uint32_t)(i / NRS) & 1;
            const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
            const int64_t v = tile * kTileRows + row;
            const bool valid = v < n;
            if (!mbar_wait(&bars[kRotFull + rs], ph, abort_s)) return false;
            tc_fence_after();
            const uint32_t tl = tmem + lanes + rs * D;
            // ||x|| = ||R x|| (R orthogonal, to the 2^-22 of its split) from the accumulator: each
            // half of the row sums its squares, the halves meet in shared memory.  norm_s[.][rs] is
            // next written NRS tiles on, after every warp has released this slot.
            {
                uint32_t r[32];
                float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll 1
                for (int c = h * CH; c < h * CH + CH; ++c) {
                    tmem_ld32(tl + 32 * c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float2 a2 = make_float2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
                        ss2 = __ffma2_rn(a2, a2, ss2);
                    }
                }
                norm_s[(h * 4 + rs) * kTileRows + row] = ss2.x + ss2.y;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kNormReady + rs]);
                if (!mbar_wait(&bars[kNormReady + rs], ph, abort_s)) return false;
            }
            const float nx = sqrtf(norm_s[rs * kTileRows + row] + norm_s[(4 + rs) * kTileRows + row]) *
                             (1.0f / (float)(1 << kRScaleLog2));
            // the accumulator holds 2^8 R x; y = R x / ||x||
            const float inv = nx > 0.f ? (1.0f / (float)(1 << kRScaleLog2)) / nx : 0.f;
            const float inve = inv * (float)(1 << kEScaleLog2);
            // the accumulator itself is compared against boundaries scaled by 2^8 ||x||; a zero
            // vector compares its zero accumulator against the unscaled ones (y = 0)
            const float sc = nx > 0.f ? nx * (float)(1 << kRScaleLog2) : 1.f;
            float ep[HL > 1 ? HL - 1 : 1];
#pragma unroll
            for (int k = 0; k < HL - 1; ++k) ep[k] = edge[k] * sc;
            float2 ee2 = make_float2(0.f, 0.f);  // sums of (2^14 (y - c))^2 over even / odd coordinates
            uint32_t *dst = codes + v * wpv;
            uint32_t r[32];
            // the loop stays rolled so the unrolled body fits the instruction cache
#pragma unroll 1
            for (int c = h * CH; c < h * CH + CH; ++c) {
                tmem_ld32(tl + 32 * c, r);
                tmem_ld_wait();
                uint32_t wp[4] = {0u, 0u, 0u, 0u};
                if constexpr (IS_KEY) {
                    // coordinate pairs: codes, then 2^14 (y - c) and its fp16 hi | lo split with
                    // packed two-wide fp32 arithmetic (one column holds the pair)
                    uint32_t hp[16], lp[16];
                    const float2 inve2 = make_float2(inve, inve);
                    const float2 mone2 = make_float2(-1.f, -1.f);
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float ncs[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int l = 2 * k + u;
                            const float a = __uint_as_float(r[l]);
                            const bool pos = a > 0.f;
                            bool mb[3];
                            magnitude_bits<BETA>(fabsf(a), ep, mb);
                            if (pos) wp[BETA - 1] |= 1u << l;
#pragma unroll
                            for (int j = 0; j < BETA - 1; ++j)
                                if (mb[j] == pos) wp[j] |= 1u << l;
                            float cm;
                            if constexpr (HL == 1) cm = cmag[0];
                            else if constexpr (HL == 2) cm = mb[0] ? cmag[1] : cmag[0];
                            else cm = mb[1] ? (mb[0] ? cmag[3] : cmag[2]) : (mb[0] ? cmag[1] : cmag[0]);
                            ncs[u] = __uint_as_float(__float_as_uint(cm) ^ (pos ? 0x80000000u : 0u));  // -2^14 c
                        }
                        const float2 a2 = make_float2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
                        const float2 e2 = __ffma2_rn(a2, inve2, make_float2(ncs[0], ncs[1]));  // 2^14 (y - c)
                        ee2 = __ffma2_rn(e2, e2, ee2);
                        const __half2 hh = __floats2half2_rn(e2.x, e2.y);
                        const float2 d2 = __ffma2_rn(__half22float2(hh), mone2, e2);
                        const __half2 ll = __floats2half2_rn(d2.x, d2.y);
                        hp[k] = *(const uint32_t *)&hh;
                        lp[k] = *(const uint32_t *)&ll;
                    }
                    tmem_st16(tl + 32 * c, hp);
                    tmem_st16(tl + 32 * c + 16, lp);
                } else {
#pragma unroll
                    for (int l = 0; l < 32; ++l) {
                        const float a = __uint_as_float(r[l]);
                        const bool pos = a > 0.f;
                        bool mb[3];
                        magnitude_bits<BETA>(fabsf(a), ep, mb);
                        if (pos) wp[BETA - 1] |= 1u << l;
#pragma unroll
                        for (int j = 0; j < BETA - 1; ++j)
                            if (mb[j] == pos) wp[j] |= 1u << l;
                    }
                }
                if (valid) {
#pragma unroll
                    for (int p = 0; p < BETA; ++p) dst[c * BETA + p] = wp[p];
                }
            }
            if constexpr (IS_KEY) {
                tmem_st_wait();
                // half 1 hands its part of ||y - c||^2 to half 0; ee_s[rs] is next written NRS
                // tiles on, after half 0 has released this slot
                const float ee = ee2.x + ee2.y;
                if (h == 1) {
                    ee_s[rs * kTileRows + row] = ee;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kPartReady + rs]);
                } else {
                    if (!mbar_wait(&bars[kPartReady + rs], ph, abort_s)) return false;
                    const float ss = (ee + ee_s[rs * kTileRows + row]) * (1.0f / (float)(1 << (2 * kEScaleLog2)));
                    if (valid) rnorm[v] = f32_to_f16_bits(sqrtf(ss));
                }
            }
            if (valid && h == 0) norm[v] = f32_to_f16_bits(nx);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kEReady + rs]);
            return true;
        };

        // QJL signs of tile j from its projection accumulator (2^18 S' (y - c))
        auto sign_step = [&](int j) -> bool {
            const int pa = j & 1;
            const int64_t tile = blockIdx.x + (int64_t)j * gridDim.x;
            const int64_t v = tile * kTileRows + row;
            const bool valid = v < n;
            if (!mbar_wait(&bars[kProjFull + pa], (j >> 1) & 1, abort_s)) return false;
            tc_fence_after();
            const uint32_t ta = tmem + lanes + NRS * D + pa * m;
            uint32_t r[32];
#pragma unroll 1
            for (int g = h; g < spk; g += 2) {
                tmem_ld32(ta + 32 * g, r);
                tmem_ld_wait();
                uint32_t sw = 0;
#pragma unroll
                for (int l = 0; l < 32; ++l) sw |= (uint32_t)(__uint_as_float(r[l]) >= 0.f) << l;
                if (valid) signs[v * spk + g] = sw;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kAccFree + pa]);
            return true;
        };

        if (IS_KEY) {
            bool ok = true;
            for (int i = 0; ok && i < my_tiles; ++i) {
                ok = code_step(i);
                if (ok && i >= 1) ok = sign_step(i - 1);
            }
            if (ok && my_tiles > 0) sign_step(my_tiles - 1);
        } else {
            for (int i = 0; i < my_tiles; ++i)
                if (!code_step(i)) break;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

template <int D, bool IS_KEY, int BETA>
cudaError_t launch_tc(const Prepared &P, const void *x, int64_t n, uint32_t *codes, uint32_t *signs,
                      uint16_t *norm, uint16_t *rnorm, int32_t *dev_status, cudaStream_t s) {
    auto encode = get_encode();
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap map;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)n};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kTileRows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(x), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    const TcSmem L = tc_smem_layout(D, IS_KEY ? P.m : 0, IS_KEY);
    const size_t smem = L.total + 1024;
    cudaError_t e = cudaFuncSetAttribute(compress_tc_kernel<D, IS_KEY, BETA>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ntiles = (n + kTileRows - 1) / kTileRows;
    const int grid = (int)(ntiles < sms ? ntiles : sms);
    compress_tc_kernel<D, IS_KEY, BETA><<<grid, kThreads, smem, s>>>(map, P, n, codes, signs, norm, rnorm,
                                                                   dev_status);
    return cudaGetLastError();
}

}  // namespace

bool compress_tc_supported(const Prepared &P, bool is_key, bool x_f16) {
    if (!x_f16) return false;
    if (P.d != 128 && P.d != 64) return false;
    // keys need two rotation accumulators beside the two projection accumulators
    if (is_key && (P.m < 32 || P.m % 32 || P.m > 256 || tc_rotation_slots(P.d, P.m, true) < 2)) return false;
    return true;
}

template <int D, bool IS_KEY>
cudaError_t launch_tc_beta(const Prepared &P, int beta, const void *x, int64_t n, uint32_t *codes,
                           uint32_t *signs, uint16_t *norm, uint16_t *rnorm, int32_t *dev_status, cudaStream_t s) {
    switch (beta) {
        case 1: return launch_tc<D, IS_KEY, 1>(P, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 2: return launch_tc<D, IS_KEY, 2>(P, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 3: return launch_tc<D, IS_KEY, 3>(P, x, n, codes, signs, norm, rnorm, dev_status, s);
        case 4:
            if constexpr (!IS_KEY) return launch_tc<D, IS_KEY, 4>(P, x, n, codes, signs, norm, rnorm, dev_status, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_compress_tc(const Prepared &P, bool is_key, const void *x, int64_t n, uint32_t *codes,
                               uint32_t *signs, uint16_t *norm, uint16_t *rnorm, int32_t *dev_status,
                               cudaStream_t s) {
    const int beta = is_key ? P.kbeta : P.vbeta;
    if (P.d == 128)
        return is_key ? launch_tc_beta<128, true>(P, beta, x, n, codes, signs, norm, rnorm, dev_status, s)
                      : launch_tc_beta<128, false>(P, beta, x, n, codes, signs, norm, rnorm, dev_status, s);
    return is_key ? launch_tc_beta<64, true>(P, beta, x, n, codes, signs, norm, rnorm, dev_status, s)
                  : launch_tc_beta<64, false>(P, beta, x, n, codes, signs, norm, rnorm, dev_status, s);
}

}  // namespace tq
