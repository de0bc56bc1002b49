// tq_compress_tc.cu -- key / value compression on the fifth-generation tensor cores.
//
// Per 128-vector tile (TurboQuantMSE.quantize / TurboQuantProd.compress; "turboquant-pytorch",
// nav.superapi.store, 核心 API; atskills.one, "What It Does" stage 1 + stage 2):
//   rotation    ACC[v, j] = sum_i X[v, i] (R_hi + R_lo)[j, i]          tcgen05, smem x smem
//               (X is the fp16 input tile, exact in fp16; R * 2^8 = R_hi + R_lo in fp16, so
//               the product carries ~22 bits of R and the accumulator is fp32)
//   epilogue    n = ||ACC row|| (R orthogonal), y = ACC / n, idx = code of y, planar pack,
//               keys: e = y - c[idx] split into fp16 hi + lo, written back into TMEM
//   projection  P[v, a] = sum_j (E_hi (S'_hi + S'_lo) + E_lo S'_hi)[v, j]   tcgen05, tmem x smem
//               with S' = S R^T (so P = S r for the residual r = R^T e); sign bits of P.
// One thread of the epilogue owns one vector (one TMEM lane), so norms and residual norms are
// thread-local.  Warp roles: warp 0 loads (TMA) and owns TMEM, warp 1 issues the MMAs, two
// groups of four epilogue warps take alternate tiles, each with its own half of TMEM.
#include <cudaTypedefs.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"
#include "tq_sm100.cuh"

namespace tq {

namespace {

using namespace sm100;

constexpr int kTileRows = 128;
constexpr int kThreads = 384;  // 12 warps
constexpr int kEpiWarp0 = 2;   // warps 2..9: epilogue (two groups of four)
constexpr int kNormWarp0 = 10; // warps 10..11: row norms of the input tiles
constexpr int kCScaleLog2 = 10;  // centroid scale before the fp16 hi/lo split

struct TcSmem {
    // offsets from the 1024-aligned dynamic shared memory base
    uint32_t R, S, X, bars, misc;
    uint32_t total;
    int nst;
};

__host__ __device__ inline TcSmem tc_smem_layout(int D, int m, bool is_key) {
    TcSmem L;
    uint32_t o = 0;
    L.R = o;
    o += 2u * (is_key ? D + m : D) * D * 2;  // [R; S] (keys) or R (values), hi | lo
    L.S = o;
    if (is_key) o += 2u * m * D * 2;
    L.X = o;
    const uint32_t xs = kTileRows * D * 2;
    uint32_t budget = 225u * 1024 - o - 2048;
    int nst = (int)(budget / xs);
    if (nst > 4) nst = 4;
    L.nst = nst;
    o += nst * xs;
    L.bars = o;
    o += 256;
    L.misc = o;
    o += 2048;
    L.total = o;
    return L;
}

enum BarIdx {
    kOpnd = 0,
    kFull = 1,
    kEmpty = 5,
    kRotFull = 9,
    kEReady = 11,
    kProjFull = 13,
    kTmemEmpty = 15,
    kNormReady = 17
};

// Code of y against ascending boundaries b[0..2^BETA-2] (#{k : b[k] < y}) by a binary
// search whose thresholds are selected from registers; t[p] receives bit p of the code.
template <int BETA>
__device__ __forceinline__ void bucket_bits(float y, const float (&b)[16], bool (&t)[4]) {
    if constexpr (BETA == 1) {
        t[0] = y > b[0];
    } else if constexpr (BETA == 2) {
        t[1] = y > b[1];
        t[0] = y > (t[1] ? b[2] : b[0]);
    } else if constexpr (BETA == 3) {
        t[2] = y > b[3];
        t[1] = y > (t[2] ? b[5] : b[1]);
        t[0] = y > (t[2] ? (t[1] ? b[6] : b[4]) : (t[1] ? b[2] : b[0]));
    } else {
        t[3] = y > b[7];
        t[2] = y > (t[3] ? b[11] : b[3]);
        t[1] = y > (t[3] ? (t[2] ? b[13] : b[9]) : (t[2] ? b[5] : b[1]));
        t[0] = y > (t[3] ? (t[2] ? (t[1] ? b[14] : b[12]) : (t[1] ? b[10] : b[8]))
                         : (t[2] ? (t[1] ? b[6] : b[4]) : (t[1] ? b[2] : b[0])));
    }
}

template <int N>
__device__ __forceinline__ uint32_t umux(const uint32_t *v, uint32_t idx) {
    if constexpr (N == 1) {
        return v[0];
    } else {
        const uint32_t lo = umux<N / 2>(v, idx);
        const uint32_t hi = umux<N / 2>(v + N / 2, idx);
        return (idx & (N / 2)) ? hi : lo;
    }
}

// v[idx] for a register array, as a tree of selects.
template <int N>
__device__ __forceinline__ float mux(const float *v, uint32_t idx) {
    if constexpr (N == 1) {
        return v[0];
    } else {
        const float lo = mux<N / 2>(v, idx);
        const float hi = mux<N / 2>(v + N / 2, idx);
        return (idx & (N / 2)) ? hi : lo;
    }
}

template <int D, bool IS_KEY, int BETA>
__global__ void __launch_bounds__(kThreads, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap tmap, Prepared P, int64_t n,
                       uint32_t *__restrict__ codes, uint32_t *__restrict__ signs, uint16_t *__restrict__ norm,
                       uint16_t *__restrict__ rnorm, int32_t *__restrict__ dev_status) {
    constexpr int KB = D / 64;
    constexpr int KSTEPS = D / 16;
    constexpr int CHUNKS = D / 32;
    constexpr uint32_t XSTAGE = kTileRows * D * 2;
    const int m = IS_KEY ? P.m : 0;
    const TcSmem L = tc_smem_layout(D, m, IS_KEY);
    const int NST = L.nst;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = (uint64_t *)(sm + L.bars);
    float *bnd_s = (float *)(sm + L.misc);
    float *cen_s = bnd_s + kMaxLevels;
    uint32_t *tmem_s = (uint32_t *)(cen_s + kMaxLevels);
    volatile int *abort_s = (volatile int *)(tmem_s + 1);
    float *norm_s = (float *)(sm + L.misc + 256);  // [2 slots][128 rows] squared norms
    uint32_t *cbit_s = (uint32_t *)(sm + L.misc + 256 + 1024);  // centroid fp16 hi/lo bits

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t ntiles = (n + kTileRows - 1) / kTileRows;
    const int my_tiles = (int)((ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

    if (threadIdx.x == 0) {
        mbar_init(&bars[kOpnd], 1);
        for (int s = 0; s < 4; ++s) {
            mbar_init(&bars[kFull + s], 1);
            mbar_init(&bars[kEmpty + s], 3);  // MMA commit + the two norm warps
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kRotFull + s], 1);
            mbar_init(&bars[kEReady + s], 4);
            mbar_init(&bars[kProjFull + s], 1);
            mbar_init(&bars[kTmemEmpty + s], 4);
            mbar_init(&bars[kNormReady + s], 2);
        }
        *abort_s = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kMaxLevels) {
        bnd_s[threadIdx.x] = IS_KEY ? P.cb->kb[threadIdx.x] : P.cb->vb[threadIdx.x];
        const float c = IS_KEY ? P.cb->kc[threadIdx.x] : P.cb->vc[threadIdx.x];
        cen_s[threadIdx.x] = c;
        const float cs = c * (float)(1 << kCScaleLog2);
        const __half h = __float2half_rn(cs);
        const __half lo = __float2half_rn(cs - __half2float(h));
        cbit_s[threadIdx.x] = ((uint32_t)__half_as_ushort(h) << 16) | (uint32_t)__half_as_ushort(lo);
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
            const uint32_t rbytes = 2u * (IS_KEY ? D + m : D) * D * 2;
            const uint32_t sbytes = IS_KEY ? 2u * m * D * 2 : 0u;
            mbar_arrive_expect_tx(&bars[kOpnd], rbytes + sbytes);
            bulk_load(sm + L.R, IS_KEY ? P.RSsw : P.Rsw, rbytes, &bars[kOpnd]);
            if (IS_KEY) bulk_load(sm + L.S, P.Ssw, sbytes, &bars[kOpnd]);
            int issued = 0;
            for (int i = 0; i < my_tiles; ++i) {
                const int stage = i % NST;
                if (i >= NST && !mbar_wait(&bars[kEmpty + stage], ((i / NST) - 1) & 1, abort_s)) break;
                const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
                uint8_t *dst = sm + L.X + stage * XSTAGE;
                mbar_arrive_expect_tx(&bars[kFull + stage], XSTAGE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
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
            const int rowsB = IS_KEY ? D + m : D;
            const uint32_t idesc_rot = idesc_f16_f32(128, rowsB);
            const uint32_t idesc_prj = idesc_f16_f32(128, m > 0 ? m : 16);
            const uint32_t sR = smem_u32(sm + L.R), sS = smem_u32(sm + L.S), sX = smem_u32(sm + L.X);
            bool ok = mbar_wait(&bars[kOpnd], 0, abort_s);
            auto projection = [&](int j) -> bool {
                const int slot = j & 1;
                if (!mbar_wait(&bars[kEReady + slot], (j >> 1) & 1, abort_s)) return false;
                tc_fence_after();
                const uint32_t acc = tmem + slot * 256 + D + m;
                const uint32_t sbytes = (uint32_t)m * D * 2;
                uint32_t first = 0;
#pragma unroll 1
                for (int k = 0; k < KSTEPS; ++k) {
                    const uint32_t a_hi = tmem + slot * 256 + 32 * (k >> 1) + 8 * (k & 1);
                    const uint32_t a_lo = a_hi + 16;
                    const uint32_t boff = (uint32_t)(k >> 2) * m * 128 + (k & 3) * 32;
                    const uint64_t b_hi = sdesc_sw128(sS + boff);
                    const uint64_t b_lo = sdesc_sw128(sS + sbytes + boff);
                    mma_ts(acc, a_hi, b_hi, idesc_prj, first);
                    first = 1;
                    mma_ts(acc, a_hi, b_lo, idesc_prj, 1);
                    mma_ts(acc, a_lo, b_hi, idesc_prj, 1);
                }
                mma_commit(&bars[kProjFull + slot]);
                return true;
            };
            auto rotation = [&](int i) -> bool {
                const int slot = i & 1, stage = i % NST;
                if (i >= 2 && !mbar_wait(&bars[kTmemEmpty + slot], ((i >> 1) - 1) & 1, abort_s)) return false;
                if (!mbar_wait(&bars[kFull + stage], (i / NST) & 1, abort_s)) return false;
                tc_fence_after();
                const uint32_t acc = tmem + slot * 256;
                const uint32_t xbase = sX + stage * XSTAGE;
                uint32_t first = 0;
#pragma unroll
                for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                    for (int k = 0; k < KSTEPS; ++k) {
                        const uint32_t aoff = (uint32_t)(k >> 2) * (kTileRows * 128) + (k & 3) * 32;
                        const uint32_t boff = (uint32_t)pass * (rowsB * D * 2) + (uint32_t)(k >> 2) * (rowsB * 128) +
                                              (k & 3) * 32;
                        mma_ss(acc, sdesc_sw128(xbase + aoff), sdesc_sw128(sR + boff), idesc_rot, first);
                        first = 1;
                    }
                mma_commit(&bars[kEmpty + stage]);
                mma_commit(&bars[kRotFull + slot]);
                return true;
            };
            // Two tiles in flight (one per TMEM slot); the projection of tile j goes out as soon
            // as its residual is ready, before the rotation that reuses tile j's slot.
            if (ok && my_tiles > 0) ok = rotation(0);
            if (ok && my_tiles > 1) ok = rotation(1);
            for (int j = 0; ok && j < my_tiles; ++j) {
                if (IS_KEY && !projection(j)) break;
                if (j + 2 < my_tiles && !rotation(j + 2)) break;
            }
        }
    } else if (warp < kNormWarp0) {
        // ------------------------------------------------------------ epilogue
        const int ew = warp - kEpiWarp0;   // 0..7
        const int wg = ew >> 2;            // which half of the tiles / TMEM
        const int q = warp & 3;            // TMEM subpartition this warp may access
        const int row = 32 * q + lane;     // vector within the tile
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)wg * 256;
        constexpr int wpv = BETA * CHUNKS;
        float bnd_r[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) bnd_r[k] = bnd_s[k];
        for (int i = wg; i < my_tiles; i += 2) {
            const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
            const int64_t v = tile * kTileRows + row;
            const bool valid = v < n;
            if (!mbar_wait(&bars[kNormReady + wg], (i >> 1) & 1, abort_s)) break;
            if (!mbar_wait(&bars[kRotFull + wg], (i >> 1) & 1, abort_s)) break;
            tc_fence_after();
            const float nx = sqrtf(norm_s[wg * kTileRows + row]);
            // the accumulator holds 2^8 R x; y = R x / ||x||
            const float inv = nx > 0.f ? (1.0f / (float)(1 << kRScaleLog2)) / nx : 0.f;
            float ee = 0.f;
            uint32_t r[32];
            uint32_t *dst = codes + v * wpv;
            // chunks of 32 coordinates; the loop stays rolled so the unrolled body fits the
            // instruction cache, and each chunk's code words go straight to global memory
#pragma unroll 1
            for (int c = 0; c < CHUNKS; ++c) {
                tmem_ld32(tl + 32 * c, r);
                tmem_ld_wait();
                uint32_t wp[4] = {0u, 0u, 0u, 0u};
                uint32_t hp[16], lp[16];
#pragma unroll
                for (int l = 0; l < 32; ++l) {
                    const float y = __uint_as_float(r[l]) * inv;
                    bool t[4];
                    bucket_bits<BETA>(y, bnd_r, t);
                    uint32_t idx = 0;
#pragma unroll
                    for (int p = 0; p < BETA; ++p) {
                        if (t[p]) wp[p] |= 1u << l;
                        idx |= (t[p] ? 1u : 0u) << p;
                    }
                    if (IS_KEY) {
                        // centroid and its fp16 hi/lo bit pattern from shared-memory tables
                        const float e = y - cen_s[idx];
                        ee = fmaf(e, e, ee);
                        const uint32_t cb = cbit_s[idx];
                        if (l & 1) {
                            hp[l >> 1] = __byte_perm(hp[l >> 1], cb, 0x7632);
                            lp[l >> 1] = __byte_perm(lp[l >> 1], cb, 0x5410);
                        } else {
                            hp[l >> 1] = cb;
                            lp[l >> 1] = cb;
                        }
                    }
                }
                if (IS_KEY) {
                    tmem_st16(tl + 32 * c, hp);
                    tmem_st16(tl + 32 * c + 16, lp);
                }
                if (valid) {
#pragma unroll
                    for (int p = 0; p < BETA; ++p) dst[c * BETA + p] = wp[p];
                }
            }
            if (IS_KEY) tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(IS_KEY ? &bars[kEReady + wg] : &bars[kTmemEmpty + wg]);
            if (valid) norm[v] = f32_to_f16_bits(nx);
            if (IS_KEY) {
                if (valid) rnorm[v] = f32_to_f16_bits(sqrtf(ee));
                if (!mbar_wait(&bars[kProjFull + wg], (i >> 1) & 1, abort_s)) break;
                tc_fence_after();
                // p = S u - S' c[idx]: S u from the rotation accumulator (2^8 S x), S' c from the
                // projection accumulator (2^(kCScaleLog2 + kSScaleLog2) S' c)
                const int spk = m >> 5;
                const float pun = 1.0f / (float)(1 << (kCScaleLog2 + kSScaleLog2));
#pragma unroll 1
                for (int g = 0; g < spk; ++g) {
                    uint32_t r2[32];
                    tmem_ld32(tl + D + 32 * g, r);
                    tmem_ld32(tl + D + m + 32 * g, r2);
                    tmem_ld_wait();
                    uint32_t sw = 0;
#pragma unroll
                    for (int l = 0; l < 32; ++l) {
                        const float pv = fmaf(__uint_as_float(r[l]), inv, -__uint_as_float(r2[l]) * pun);
                        sw |= (uint32_t)(pv >= 0.f) << l;
                    }
                    if (valid) signs[v * spk + g] = sw;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kTmemEmpty + wg]);
            }
        }
    } else {
        // ------------------------------------------------------------ row norms
        // ||x||^2 of every row of the fp16 input tile, read from the swizzled stage in
        // shared memory (exact fp16 inputs, fp32 sums); two warps, 64 rows each.
        const int nw = warp - kNormWarp0;
        for (int i = 0; i < my_tiles; ++i) {
            const int slot = i & 1, stage = i % NST;
            if (i >= 2 && !mbar_wait(&bars[kTmemEmpty + slot], ((i >> 1) - 1) & 1, abort_s)) break;
            if (!mbar_wait(&bars[kFull + stage], (i / NST) & 1, abort_s)) break;
            const uint8_t *xs = sm + L.X + stage * XSTAGE;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = nw * 64 + h * 32 + lane;
                float ss = 0.f;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    const int kb = c >> 3, cc = c & 7;
                    const uint4 w = *(const uint4 *)(xs + kb * (kTileRows * 128) + r * 128 + ((cc ^ (r & 7)) << 4));
                    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(*(const __half2 *)&u[e]);
                        ss = fmaf(f.x, f.x, ss);
                        ss = fmaf(f.y, f.y, ss);
                    }
                }
                norm_s[slot * kTileRows + r] = ss;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[kNormReady + slot]);
                mbar_arrive(&bars[kEmpty + stage]);
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
    // keys keep [R x | S x] and the projection in one 256-column TMEM slot
    if (is_key && (P.m < 32 || P.m % 32 || P.d + 2 * P.m > 256)) return false;
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
