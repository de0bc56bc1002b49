// tq_attend_planes.cu -- decode attention and scores straight from the packed keys and values,
// with the code bits themselves as 8-bit integer tensor-core operands.
//
// Math (asymmetric scores from the compressed keys, softmax, weighted sum over the MSE-
// dequantized values; "turboquant-pytorch", nav.superapi.store, 常见使用模式 and 核心 API):
//   s_tr = ||k_t|| ( <q_rot_r, c[kidx_t]> + rho_t sqrt(pi/2)/m <sq_r, 2 sign_t - 1> )
//   o_rot_r = sum_t softmax_t(scale s_tr) ||v_t|| c[vidx_t],   out_r = R^T o_rot_r
//
// Walsh form of the codebook.  The Lloyd-Max codebooks are exactly antisymmetric
// (c[K-1-k] = -c[k]), so as a function of the code bits b_0..b_{beta-1} (s_i = 2 b_i - 1)
//   c[idx] = sum over odd-sized subsets S of {0..beta-1} of alpha_S prod_{i in S} s_i,
// with 1, 2, 4 or 8 terms for beta = 1..4.  A product of an odd number of s_i equals
// 2 (xor of those bits) - 1, so every term is one bit plane (a stored plane, or the xor of three)
// times a real coefficient alpha_S = (1/K) sum_idx c[idx] prod_{i in S} s_i(idx).  Hence
//   <q, c[kidx]> = sum_S alpha_S sum_j q_j (2 b_Sj - 1)
//   sum_t y_t c[vidx_tj] = sum_S alpha_S (2 sum_t y_t b_S(t, j) - sum_t y_t)
// and both products take the bits as exact integer operands.  The real factors are rounded to
// integers and split into 8-bit digits, one product column per digit, so the tensor core
// accumulates exact int32 sums:
//   - keys (m16n8k32, A = key bits, B = query digits): per query row the 2 alpha_S q_j and the
//     2 (S q)_i are rounded to 31-bit integers with one power-free scale per row (relative error
//     2^-30 of the row's largest coefficient), as four balanced base-256 digits;
//   - values (m16n8k32, A = value bits of one coordinate for four tokens, B = weight digits):
//     the softmax weights times the value norms are rounded to 16-bit fixed point relative to the
//     largest value norm of the CTA's token range (absolute error 2^-17 of it per token).
// Two passes per CTA over a range of at most kPRange tokens: (1) scores of the whole range into
// shared memory (and the row maxima); (2) the fixed-point weights, then the value products.  Each
// CTA writes its range's (max, sum, o_rot) partial; the last CTA of a (batch, KV head) slice to
// finish (an atomic count per slice) merges them by log-sum-exp and applies R^T, or writes the
// merged partial for tq_attend_partial.  A separate kernel (planes_qfrag_kernel) prepares each
// slice's query operands first.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.cuh"

namespace tq {

namespace {

constexpr int kPRows = 4;      // query rows per KV head (G * Nq) this kernel takes
constexpr int kPRange = 1024;  // most tokens per CTA
constexpr int kPStage = 32;    // tokens per copy stage
constexpr int kCounterWord = 48;  // in a slice's constants block: CTAs of the slice finished
constexpr double kLog2e = 1.4426950408889634;

__host__ __device__ constexpr int walsh_terms(int beta) { return beta <= 1 ? 1 : beta == 2 ? 2 : beta == 3 ? 4 : 8; }

// bit subset of Walsh term s of a beta-bit code: the single bits first, then the triples
__host__ __device__ constexpr int walsh_subset(int beta, int s) {
    return s < beta ? (1 << s) : (beta == 3 ? 0x7 : s == 4 ? 0x7 : s == 5 ? 0xB : s == 6 ? 0xD : 0xE);
}

template <int D, int KB, int VB>
struct PlanesCfg {
    static constexpr int G32 = D / 32;
    static constexpr int M = D / 2;  // proj_dim = head_dim / 2
    static constexpr int SW = M / 32;
    static constexpr int KWPT = KB * G32;
    static constexpr int VWPT = VB * G32;
    static constexpr int KPL = walsh_terms(KB);
    static constexpr int VPL = walsh_terms(VB);
    static constexpr int NC = G32 * KPL;  // key products (32 positions each) on code planes
    static constexpr int NK = NC + SW;    // ... and on sign words
    static constexpr bool KREG = NK <= 12;
    static constexpr int CPW = VB <= 3 ? 64 : 32;  // coordinates per warp in the value products
    static constexpr int GPW = CPW / 32;
    static constexpr int TPW = CPW / 16;
    static constexpr int VW = D / CPW;
    static constexpr int NW = VW > 4 ? VW : 4;
    static constexpr int TS = NW / VW;  // token subsets of the value pass
    static constexpr int SLW = 32 * NK * 4 + 64;  // words per slice of prepared query operands
};

// Prepared query operands of one slice: [lane][NK][4] fragment words, then per row r:
// Ec[4], Es[4] (int32 digit sums), lam_c, lam_s (floats).

__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D = A B + C with C in other registers (the start of a product chain)
__device__ __forceinline__ void mma_u8s8_c(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                           const uint32_t (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]), "r"(c[2]),
          "r"(c[3]));
}
__device__ __forceinline__ void mma_u8u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
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

// Copy `words` 32-bit words with the widest cp.async the per-record word count allows.
template <int RECW>
__device__ __forceinline__ void stage_copy(uint32_t *dst, const uint32_t *src, int words, int lane) {
    constexpr int G = (RECW % 4 == 0) ? 4 : (RECW % 2 == 0) ? 2 : 1;
    for (int i = lane * G; i < words; i += 32 * G) cp_async<4 * G>(dst + i, src + i);
}

// Plane word of Walsh term s from the beta stored plane words of one 32-coordinate group.
template <int BETA>
__device__ __forceinline__ uint32_t plane_word(const uint32_t *w, int s) {
    const int sub = walsh_subset(BETA, s);
    uint32_t r = 0;
#pragma unroll
    for (int i = 0; i < BETA; ++i)
        if (sub & (1 << i)) r ^= w[i];
    return r;
}

// Byte b of each of four words, in word order.
__device__ __forceinline__ uint32_t gather_byte(uint4 q, uint32_t sel2) {
    const uint32_t lo = __byte_perm(q.x, q.y, sel2);
    const uint32_t hi = __byte_perm(q.z, q.w, sel2);
    return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ int32_t digit(int64_t &q) {
    const int32_t d = (int32_t)(((q + 128) & 255) - 128);
    q = (q - d) >> 8;
    return d;
}

// ------------------------------------------------------------------ query operands
//
// One warp per slice (batch, KV head).  Key position k (0..31) of product kappa holds bit
// beta(k) of that product's 32-bit plane word with the element value 2 e(k):
//   k = 4 t + i        -> bit 2 t + 8 i,      e = 1
//   k = 16 + 4 t + i   -> bit 2 t + 1 + 8 i,  e = 2
// (t = lane % 4, i = byte within the register), which is how the kernel below builds its A
// registers with one funnel shift and two masks.  The B value is Q / e with
// Q = round(gamma / Lambda), gamma = 2 alpha_S q_rot[32 g + beta] (code planes) or 2 sq[...]
// (signs), and Lambda = max |gamma| / 2^30 per row and kind.
// Rows of R^T and S^T staged in shared memory per chunk of input coordinates (at most ~96 KB).
template <int D>
struct QfragChunk {
    static constexpr int NQ = D + D / 2;
    static constexpr int KC = (NQ * D * 4 <= 96 * 1024) ? D : (96 * 1024) / (NQ * 4) / 32 * 32;
    static constexpr uint32_t BYTES = (uint32_t)KC * NQ * 4;
};

template <int D, int KB>
__global__ void __launch_bounds__(256) planes_qfrag_kernel(Prepared P, ScoreProblem sp, float scale,
                                                         uint32_t *__restrict__ frag) {
    using C = PlanesCfg<D, KB, 1>;
    constexpr int NQ = D + C::M;
    constexpr int NTH = 256;
    static_assert(QfragChunk<D>::NQ == NQ && D % QfragChunk<D>::KC == 0, "chunking");
    extern __shared__ __align__(16) float wsm[];  // [KC][NQ] rows of R^T | S^T
    __shared__ __align__(16) float4 qT[D];        // qT[j] = (q_0[j], q_1[j], q_2[j], q_3[j])
    __shared__ float qs[kPRows][NQ];
    __shared__ uint32_t Qd[kPRows][C::NK][32];  // the four balanced base-256 digits, as bytes
    __shared__ double alpha[8];
    __shared__ double inv[kPRows][2];
    __shared__ float lamf[kPRows][2];
    __shared__ int esum[kPRows][2][4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t sl = blockIdx.x;
    const int b = (int)(sl / sp.Hkv), kv = (int)(sl % sp.Hkv);
    const int G = sp.Hq / sp.Hkv, nrows = G * sp.Nq;
    uint32_t *out = frag + sl * (int64_t)C::SLW;
    // the slice's query rows (zero beyond nrows), coordinate-major
    for (int e = tid; e < kPRows * D; e += NTH) {
        const int r = e / D, c = e % D;
        float v = 0.f;
        if (r < nrows) {
            const int g = r / sp.Nq, i = r % sp.Nq;
            v = sp.q[(((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i) * D + c];
        }
        (&qT[c].x)[r] = v;
    }
    if (tid < C::KPL) {
        const int sub = walsh_subset(KB, tid), K = 1 << KB;
        double a = 0.0;
        for (int idx = 0; idx < K; ++idx) {
            double sgn = 1.0;
            for (int i = 0; i < KB; ++i)
                if (sub & (1 << i)) sgn *= ((idx >> i) & 1) ? 1.0 : -1.0;
            a += (double)P.cb->kc[idx] * sgn;
        }
        alpha[tid] = a / K;
    }
    if (tid < kPRows * 2 * 4) (&esum[0][0][0])[tid] = 0;
    __syncthreads();
    // q_rot = R q and S q: thread t takes outputs t, t + 256, ...; the rows of R^T and S^T (input
    // coordinate j: the weights of all outputs) come through shared memory in chunks of KC
    // coordinates, copied with every load of a chunk in flight at once
    constexpr int KC = QfragChunk<D>::KC;
    constexpr int OPT = (NQ + NTH - 1) / NTH;
    float acc[OPT][kPRows];
#pragma unroll
    for (int o = 0; o < OPT; ++o)
#pragma unroll
        for (int r = 0; r < kPRows; ++r) acc[o][r] = 0.f;
    for (int k0 = 0; k0 < D; k0 += KC) {
        if (k0 > 0) __syncthreads();  // the previous chunk is consumed
        for (int e = tid; e < KC * (NQ / 4); e += NTH) {
            const int j = e / (NQ / 4), c4 = 4 * (e % (NQ / 4));
            const float *src = c4 < D ? P.RT + (int64_t)(k0 + j) * D + c4 : P.ST + (int64_t)(k0 + j) * C::M + (c4 - D);
            cp_async<16>(wsm + j * NQ + c4, src);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
#pragma unroll 4
        for (int j = 0; j < KC; ++j) {
            const float4 q4 = qT[k0 + j];
#pragma unroll
            for (int o = 0; o < OPT; ++o) {
                const int c = tid + o * NTH;
                if (c < NQ) {
                    const float w = wsm[j * NQ + c];
                    acc[o][0] = fmaf(w, q4.x, acc[o][0]);
                    acc[o][1] = fmaf(w, q4.y, acc[o][1]);
                    acc[o][2] = fmaf(w, q4.z, acc[o][2]);
                    acc[o][3] = fmaf(w, q4.w, acc[o][3]);
                }
            }
        }
    }
#pragma unroll
    for (int o = 0; o < OPT; ++o) {
        const int c = tid + o * NTH;
        if (c < NQ)
#pragma unroll
            for (int r = 0; r < kPRows; ++r) qs[r][c] = acc[o][r];
    }
    __syncthreads();
    // gamma of (row, product, position k): 2 alpha_S q_rot[32 g + bit] or 2 (S q)[32 g' + bit]
    auto gamma_at = [&](int r, int kappa, int k) -> double {
        const int tq = (k & 15) >> 2, i = k & 3;
        const int bit = (k < 16) ? 2 * tq + 8 * i : 2 * tq + 1 + 8 * i;
        if (kappa < C::NC) {
            const int g = kappa / C::KPL, s = kappa % C::KPL;
            return 2.0 * alpha[s] * (double)qs[r][32 * g + bit];
        }
        return 2.0 * (double)qs[r][D + 32 * (kappa - C::NC) + bit];
    };
    // per-row scales: Lambda = max |gamma| / 2^30 over the code positions and over the sign positions
    if (warp < kPRows) {
        const int r = warp;
        double mc = 0.0, ms = 0.0;
        for (int kappa = 0; kappa < C::NK; ++kappa) {
            const double g = fabs(gamma_at(r, kappa, lane));
            if (kappa < C::NC) mc = fmax(mc, g);
            else ms = fmax(ms, g);
        }
        for (int o = 16; o > 0; o >>= 1) {
            mc = fmax(mc, __shfl_xor_sync(kFull, mc, o));
            ms = fmax(ms, __shfl_xor_sync(kFull, ms, o));
        }
        if (lane == 0) {
            inv[r][0] = mc > 0.0 ? 1073741824.0 / mc : 0.0;
            inv[r][1] = ms > 0.0 ? 1073741824.0 / ms : 0.0;
            lamf[r][0] = (float)((double)scale * kLog2e * (mc / 1073741824.0) * 0.5);
            lamf[r][1] = (float)((double)scale * kLog2e * sqrt(1.5707963267948966) / C::M * (ms / 1073741824.0) * 0.5);
        }
    }
    __syncthreads();
    // Q = round(gamma / (Lambda e)), e = 1 for k < 16 and 2 above, as four balanced digits;
    // digit sums E = sum of e * digit (exact integers, so the order of the additions is immaterial)
    // (a warp takes the 32 positions of one (row, product); its lanes' digit sums meet by shuffles)
    for (int e = tid; e < kPRows * C::NK * 32; e += NTH) {
        const int r = e / (C::NK * 32), kappa = (e / 32) % C::NK, k = e % 32;
        const int kind = kappa < C::NC ? 0 : 1;
        const int ek = (k < 16) ? 1 : 2;
        int64_t q = (int64_t)llrint(gamma_at(r, kappa, k) * inv[r][kind] * (k < 16 ? 1.0 : 0.5));
        uint32_t packed = 0;
#pragma unroll
        for (int dg = 0; dg < 4; ++dg) {
            const int32_t dd = digit(q);
            packed |= ((uint32_t)dd & 0xFFu) << (8 * dg);
            int v = ek * dd;
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
            if (lane == 0) atomicAdd(&esum[r][kind][dg], v);
        }
        Qd[r][kappa][k] = packed;
    }
    __syncthreads();
    // fragment words of lane (gid, t4): column gid = (row gid / 2, digit 2 nu + gid % 2)
    for (int e = tid; e < 32 * C::NK; e += NTH) {
        const int ln = e / C::NK, kappa = e % C::NK;
        const int gid = ln >> 2, t4 = ln & 3, row = gid >> 1;
        uint32_t w[4];
#pragma unroll
        for (int nu = 0; nu < 2; ++nu) {
            const int sh = 8 * (2 * nu + (gid & 1));
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint32_t *q4 = &Qd[row][kappa][16 * j + 4 * t4];
                w[2 * nu + j] = ((q4[0] >> sh) & 0xFFu) | (((q4[1] >> sh) & 0xFFu) << 8) |
                                (((q4[2] >> sh) & 0xFFu) << 16) | (((q4[3] >> sh) & 0xFFu) << 24);
            }
        }
        *(uint4 *)(out + ((int64_t)ln * C::NK + kappa) * 4) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (tid == 0) out[32 * C::NK * 4 + kCounterWord] = 0u;  // CTAs of this slice done (attention)
    if (tid < kPRows) {
        const int r = tid;
        uint32_t *cr = out + 32 * C::NK * 4 + r * 10;
        for (int dg = 0; dg < 4; ++dg) {
            cr[dg] = (uint32_t)esum[r][0][dg];
            cr[4 + dg] = (uint32_t)esum[r][1][dg];
        }
        // z = scale * log2(e) * n * (Lambda_c / 2 * F_c + rho * sqrt(pi/2)/m * Lambda_s / 2 * F_s)
        cr[8] = __float_as_uint(lamf[r][0]);
        cr[9] = __float_as_uint(lamf[r][1]);
    }
}

// ------------------------------------------------------------------ shared memory layout

// Per-warp copy ring: key stages (codes, signs, key norms and residual norms, the norms copied
// from an even record index) and, in the value pass, value stages, in the same slots.
template <int D, int KB, int VB, bool ATTEND>
struct PlanesRing {
    using C = PlanesCfg<D, KB, VB>;
    static constexpr uint32_t NB = ((kPStage + 2) * 2 + 15) & ~15u;
    static constexpr uint32_t KC = 0;
    static constexpr uint32_t KS = kPStage * C::KWPT * 4;
    static constexpr uint32_t KN = KS + kPStage * C::SW * 4;
    static constexpr uint32_t KR = KN + NB;
    static constexpr uint32_t KEYB = KR + NB;
    static constexpr uint32_t VALB = (uint32_t)(C::GPW * VB * kPStage * 4);
    static constexpr uint32_t STAGE = (((ATTEND && VALB > KEYB) ? VALB : KEYB) + 15) & ~15u;
    static constexpr int NST = (C::NW * 4 * STAGE <= 24u * 1024) ? 4 : 2;
};

struct PlanesSmem {
    uint32_t sbuf, vnb, wfrag, kf, red, ring, total;
};

template <int D, int KB, int VB, bool ATTEND>
__host__ __device__ inline PlanesSmem planes_smem(int range, int splits_cap) {
    using C = PlanesCfg<D, KB, VB>;
    PlanesSmem L;
    uint32_t o = 0;
    const uint32_t r32 = (uint32_t)((range + 31) & ~31);
    L.sbuf = o;
    if (ATTEND) {
        // scores of the range; reused at the end for the token subsets' value sums
        const uint32_t xch = (uint32_t)((C::TS - 1) * C::VW * C::VPL * C::TPW * 4 * 32 * 4);
        uint32_t sb = r32 * kPRows * 4;
        if (xch > sb) sb = xch;
        const uint32_t mrg = (uint32_t)(kPRows * (D + splits_cap) * 4);  // merge: o_rot rows, split weights
        if (mrg > sb) sb = mrg;
        o += (sb + 15) & ~15u;
    }
    L.vnb = o;
    if (ATTEND) o += ((r32 + 8) * 2 + 15) & ~15u;
    L.wfrag = o;
    if (ATTEND) o += r32 * 8;  // [r32/32][32 lanes][2 words]
    L.kf = o;
    if (!C::KREG) o += 32 * C::NK * 16;
    L.red = o;
    o += 1024;
    L.ring = o;
    using RG = PlanesRing<D, KB, VB, ATTEND>;
    o += C::NW * RG::NST * RG::STAGE;
    L.total = o;
    return L;
}

// ------------------------------------------------------------------ the kernel

template <int D, int KB, int VB, bool ATTEND>
__global__ void __launch_bounds__(PlanesCfg<D, KB, VB>::NW * 32)
    planes_attend_kernel(Prepared P, ScoreProblem sp, uint32_t *__restrict__ frag, int range, int splits,
                         float *__restrict__ out, float *__restrict__ partials, int merged_partial) {
    using C = PlanesCfg<D, KB, VB>;
    using RG = PlanesRing<D, KB, VB, ATTEND>;
    constexpr int NT = C::NW * 32;
    constexpr int NST = RG::NST;
    const PlanesSmem L = planes_smem<D, KB, VB, ATTEND>(range, splits);
    extern __shared__ __align__(16) uint8_t smem[];
    float *sbuf = (float *)(smem + L.sbuf);
    uint16_t *vnb = (uint16_t *)(smem + L.vnb);
    uint32_t *wfrag = (uint32_t *)(smem + L.wfrag);
    float *red = (float *)(smem + L.red);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, t4 = lane & 3;
    const int split = blockIdx.x;
    const int64_t sl = blockIdx.y;
    const int b = (int)(sl / sp.Hkv), kv = (int)(sl % sp.Hkv);
    const int G = sp.Hq / sp.Hkv, nrows = G * sp.Nq;
    const int64_t t0 = (int64_t)split * range;
    const int len = (int)min((int64_t)range, sp.T - t0);  // >= 1 (host)
    const int64_t rec_base = sl * sp.Ts + t0;
    const int64_t nrec = (int64_t)sp.B * sp.Hkv * sp.Ts;
    auto qrow_of = [&](int r) {
        const int g = r / sp.Nq, i = r % sp.Nq;
        return ((int64_t)b * sp.Hq + (int64_t)kv * G + g) * sp.Nq + i;
    };

    // ---- query operands (registers, or shared memory when there are many products)
    const uint32_t *fs = frag + sl * (int64_t)C::SLW;
    uint4 kf[C::KREG ? C::NK : 1];
    if constexpr (C::KREG) {
#pragma unroll
        for (int k = 0; k < C::NK; ++k) kf[k] = *(const uint4 *)(fs + ((int64_t)lane * C::NK + k) * 4);
    } else {
        uint4 *d = (uint4 *)(smem + L.kf);
        for (int i = tid; i < 32 * C::NK; i += NT) d[i] = ((const uint4 *)fs)[i];
    }
    const uint32_t *crow = fs + 32 * C::NK * 4 + t4 * 10;
    int Ec[4], Es[4];
#pragma unroll
    for (int dg = 0; dg < 4; ++dg) {
        Ec[dg] = (int)crow[dg];
        Es[dg] = (int)crow[4 + dg];
    }
    const float lam_c = __uint_as_float(crow[8]), lam_s = __uint_as_float(crow[9]);

    // ---- value norms of the range (and their maximum), every load of a thread in flight at once;
    // the Walsh coefficients of the value codebook (read at the end of the CTA)
    __shared__ double va_s[8];
    float nmax = 0.f;
    if constexpr (ATTEND) {
        constexpr int NPT = (kPRange + NT - 1) / NT;
        uint16_t hv[NPT];
#pragma unroll
        for (int k = 0; k < NPT; ++k) {
            const int i = tid + k * NT;
            hv[k] = i < len ? sp.vnorm[rec_base + i] : (uint16_t)0;
        }
#pragma unroll
        for (int k = 0; k < NPT; ++k) {
            const int i = tid + k * NT;
            if (i < len) {
                vnb[i] = hv[k];
                nmax = fmaxf(nmax, f16_bits_to_f32(hv[k]));
            }
        }
        nmax = warp_max(nmax);
        if (lane == 0) red[64 + warp] = nmax;
        if (tid < C::VPL) {
            constexpr int K = 1 << VB;
            const int sub = walsh_subset(VB, tid);
            double a = 0.0;
            for (int idx = 0; idx < K; ++idx) {
                const int par = __popc(idx & sub) ^ __popc(sub);  // number of zero bits in S, mod 2
                a += (par & 1) ? -(double)P.cb->vc[idx] : (double)P.cb->vc[idx];
            }
            va_s[tid] = a / K;
        }
    }
    if constexpr (!C::KREG) __syncthreads();

    // ================= pass 1: scores of the range
    // Each warp takes a contiguous run of 32-token stages.  Per stage, tile A holds tokens
    // (2 gid, 2 gid + 1) in its rows (gid, gid + 8) and tile B tokens (16 + 2 gid, 17 + 2 gid).
    const int rot = (2 * t4 + 31) & 31;  // funnel rotation: bit 2 t4 + 8 i -> position 8 i + 1
    float rmax = -INFINITY;
    {
        const int wlen = ((len + C::NW * kPStage - 1) / (C::NW * kPStage)) * kPStage;
        const int wt0 = min(len, warp * wlen);
        const int wt1 = min(len, wt0 + wlen);
        uint8_t *wring = smem + L.ring + (size_t)warp * NST * RG::STAGE;
        float *orow = nullptr;
        if constexpr (!ATTEND) {
            if (t4 < nrows) orow = out + qrow_of(t4) * sp.T + t0;
        }
        // accumulator start values: minus the digit sums, so the products end as 2X - E digits
        const uint32_t ic0[4] = {(uint32_t)-Ec[0], (uint32_t)-Ec[1], (uint32_t)-Ec[0], (uint32_t)-Ec[1]};
        const uint32_t ic1[4] = {(uint32_t)-Ec[2], (uint32_t)-Ec[3], (uint32_t)-Ec[2], (uint32_t)-Ec[3]};
        const uint32_t is0[4] = {(uint32_t)-Es[0], (uint32_t)-Es[1], (uint32_t)-Es[0], (uint32_t)-Es[1]};
        const uint32_t is1[4] = {(uint32_t)-Es[2], (uint32_t)-Es[3], (uint32_t)-Es[2], (uint32_t)-Es[3]};
        // copy sources of this lane: 16-byte code chunks, 8- or 4-byte sign chunks, and 4-byte
        // words of the fp16 norm arrays taken from the even record index at or below the stage's
        // first record (the norms' parity offset is the same for every stage of the warp)
        // chunk sizes in words: the widest copy that every record offset keeps aligned
        constexpr int CG = (C::KWPT % 4 == 0) ? 4 : (C::KWPT % 2 == 0) ? 2 : 1;
        constexpr int SG = (C::SW % 4 == 0) ? 4 : (C::SW % 2 == 0) ? 2 : 1;
        constexpr int CCH = C::KWPT * kPStage / CG;  // code chunks per stage
        constexpr int SCH = C::SW * kPStage / SG;    // sign chunks per stage
        const int64_t wrec0 = rec_base + wt0;
        const int noff = (int)(wrec0 & 1);
        const uint32_t *gcode = sp.kcodes + wrec0 * C::KWPT;
        const uint32_t *gsign = sp.ksigns + wrec0 * C::SW;
        const uint32_t *gkn = (const uint32_t *)(sp.knorm + (wrec0 - noff));
        const uint32_t *gkr = (const uint32_t *)(sp.krnorm + (wrec0 - noff));
        auto issue = [&](int s) {
            const int tb = s * kPStage;  // relative to wt0
            if (wt0 + tb < wt1) {
                const int ntok = min(kPStage, wt1 - wt0 - tb);
                uint8_t *st = wring + (s % NST) * RG::STAGE;
                const int cch = ntok * C::KWPT / CG, sch = ntok * C::SW / SG;
#pragma unroll
                for (int c = lane; c < CCH; c += 32)
                    if (c < cch) cp_async<4 * CG>((uint32_t *)(st + RG::KC) + CG * c, gcode + (int64_t)tb * C::KWPT + CG * c);
#pragma unroll
                for (int c = lane; c < SCH; c += 32)
                    if (c < sch) cp_async<4 * SG>((uint32_t *)(st + RG::KS) + SG * c, gsign + (int64_t)tb * C::SW + SG * c);
                // norm words: (noff + ntok + 1) / 2 of them; a last word that would pass the end of
                // the arrays is copied as its one valid half
                const int nw = (noff + ntok + 1) >> 1;
                if (lane < nw) {
                    const int64_t hw = wrec0 - noff + tb + 2 * lane;  // first halfword of this word
                    if (hw + 2 <= nrec) {
                        cp_async<4>((uint32_t *)(st + RG::KN) + lane, gkn + tb / 2 + lane);
                        cp_async<4>((uint32_t *)(st + RG::KR) + lane, gkr + tb / 2 + lane);
                    } else {
                        ((uint16_t *)(st + RG::KN))[2 * lane] = sp.knorm[hw];
                        ((uint16_t *)(st + RG::KR))[2 * lane] = sp.krnorm[hw];
                    }
                }
            }
            cp_async_commit();
        };
        const int nstages = (wt1 - wt0 + kPStage - 1) / kPStage;
        for (int k = 0; k < NST - 1; ++k) issue(k);
        const int tA = 2 * gid, tB = 16 + 2 * gid;
        for (int s = 0; s < nstages; ++s) {
            issue(s + NST - 1);
            if (NST == 4) cp_async_wait<3>();
            else cp_async_wait<1>();
            __syncwarp();
            const uint8_t *st = wring + (s % NST) * RG::STAGE;
            const int tb = wt0 + s * kPStage;  // first token of the stage, in the range
            const int nv = wt1 - tb;           // valid tokens from tb on
            const uint16_t *skn = (const uint16_t *)(st + RG::KN) + noff;
            const uint16_t *skr = (const uint16_t *)(st + RG::KR) + noff;
            const uint32_t *skc = (const uint32_t *)(st + RG::KC);
            const uint32_t *sks = (const uint32_t *)(st + RG::KS);
            int cA[2][4], cB[2][4], sA[2][4], sB[2][4];
            {
                uint32_t w0[C::KWPT], w1[C::KWPT], w2[C::KWPT], w3[C::KWPT];
                load_words<C::KWPT>(skc + tA * C::KWPT, w0);
                load_words<C::KWPT>(skc + (tA + 1) * C::KWPT, w1);
                load_words<C::KWPT>(skc + tB * C::KWPT, w2);
                load_words<C::KWPT>(skc + (tB + 1) * C::KWPT, w3);
#pragma unroll
                for (int g = 0; g < C::G32; ++g) {
#pragma unroll
                    for (int sidx = 0; sidx < C::KPL; ++sidx) {
                        const int kap = g * C::KPL + sidx;
                        const uint32_t W0 = plane_word<KB>(w0 + g * KB, sidx), W1 = plane_word<KB>(w1 + g * KB, sidx);
                        const uint32_t W2 = plane_word<KB>(w2 + g * KB, sidx), W3 = plane_word<KB>(w3 + g * KB, sidx);
                        const uint32_t r0 = __funnelshift_r(W0, W0, rot), r1 = __funnelshift_r(W1, W1, rot);
                        const uint32_t r2 = __funnelshift_r(W2, W2, rot), r3 = __funnelshift_r(W3, W3, rot);
                        const uint32_t aA[4] = {r0 & 0x02020202u, r1 & 0x02020202u, r0 & 0x04040404u, r1 & 0x04040404u};
                        const uint32_t aB[4] = {r2 & 0x02020202u, r3 & 0x02020202u, r2 & 0x04040404u, r3 & 0x04040404u};
                        uint4 f;
                        if constexpr (C::KREG) f = kf[kap];
                        else f = ((const uint4 *)(smem + L.kf))[lane * C::NK + kap];
                        if (kap == 0) {
                            mma_u8s8_c(cA[0], aA, f.x, f.y, ic0);
                            mma_u8s8_c(cA[1], aA, f.z, f.w, ic1);
                            mma_u8s8_c(cB[0], aB, f.x, f.y, ic0);
                            mma_u8s8_c(cB[1], aB, f.z, f.w, ic1);
                        } else {
                            mma_u8s8(cA[0], aA, f.x, f.y);
                            mma_u8s8(cA[1], aA, f.z, f.w);
                            mma_u8s8(cB[0], aB, f.x, f.y);
                            mma_u8s8(cB[1], aB, f.z, f.w);
                        }
                    }
                }
            }
            {
                uint32_t s0[C::SW], s1[C::SW], s2[C::SW], s3[C::SW];
                load_words<C::SW>(sks + tA * C::SW, s0);
                load_words<C::SW>(sks + (tA + 1) * C::SW, s1);
                load_words<C::SW>(sks + tB * C::SW, s2);
                load_words<C::SW>(sks + (tB + 1) * C::SW, s3);
#pragma unroll
                for (int g = 0; g < C::SW; ++g) {
                    const int kap = C::NC + g;
                    const uint32_t r0 = __funnelshift_r(s0[g], s0[g], rot), r1 = __funnelshift_r(s1[g], s1[g], rot);
                    const uint32_t r2 = __funnelshift_r(s2[g], s2[g], rot), r3 = __funnelshift_r(s3[g], s3[g], rot);
                    const uint32_t aA[4] = {r0 & 0x02020202u, r1 & 0x02020202u, r0 & 0x04040404u, r1 & 0x04040404u};
                    const uint32_t aB[4] = {r2 & 0x02020202u, r3 & 0x02020202u, r2 & 0x04040404u, r3 & 0x04040404u};
                    uint4 f;
                    if constexpr (C::KREG) f = kf[kap];
                    else f = ((const uint4 *)(smem + L.kf))[lane * C::NK + kap];
                    if (g == 0) {
                        mma_u8s8_c(sA[0], aA, f.x, f.y, is0);
                        mma_u8s8_c(sA[1], aA, f.z, f.w, is1);
                        mma_u8s8_c(sB[0], aB, f.x, f.y, is0);
                        mma_u8s8_c(sB[1], aB, f.z, f.w, is1);
                    } else {
                        mma_u8s8(sA[0], aA, f.x, f.y);
                        mma_u8s8(sA[1], aA, f.z, f.w);
                        mma_u8s8(sB[0], aB, f.x, f.y);
                        mma_u8s8(sB[1], aB, f.z, f.w);
                    }
                }
            }
            // exact digit sums -> float: F = (D3 * 256 + D2) * 65536 + (D1 * 256 + D0); e = 0 for the
            // tile's first token (accumulator row gid), 2 for its second (row gid + 8)
            auto digits_f = [](const int (&c)[2][4], int e) {
                return (float)(c[1][e + 1] * 256 + c[1][e]) * 65536.f + (float)(c[0][e + 1] * 256 + c[0][e]);
            };
            const int toks[4] = {tA, tA + 1, tB, tB + 1};
            const float fc[4] = {digits_f(cA, 0), digits_f(cA, 2), digits_f(cB, 0), digits_f(cB, 2)};
            const float fsg[4] = {digits_f(sA, 0), digits_f(sA, 2), digits_f(sB, 0), digits_f(sB, 2)};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int tk = toks[u];
                const float kn = f16_bits_to_f32(skn[tk]), kr = f16_bits_to_f32(skr[tk]);
                const float z = tk < nv ? kn * fmaf(kr * lam_s, fsg[u], lam_c * fc[u]) : -INFINITY;
                if constexpr (ATTEND) {
                    sbuf[(tb + tk) * kPRows + t4] = z;
                    rmax = fmaxf(rmax, z);
                } else {
                    // scores only: lam_c, lam_s carry log2(e) (scale 1); undo it here
                    if (orow != nullptr && tk < nv) orow[tb + tk] = z * 0.6931471805599453f;
                }
            }
            __syncwarp();
        }
        cp_async_wait<0>();
    }
    if constexpr (!ATTEND) return;

    // ---- row maxima, largest value norm
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, 4));
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, 8));
    rmax = fmaxf(rmax, __shfl_xor_sync(kFull, rmax, 16));
    if (lane < 4) red[warp * 4 + lane] = rmax;
    __syncthreads();
    float Mr[kPRows];
#pragma unroll
    for (int r = 0; r < kPRows; ++r) {
        float m = -INFINITY;
        for (int w = 0; w < C::NW; ++w) m = fmaxf(m, red[w * 4 + r]);
        Mr[r] = m;
    }
    float Nmax = 0.f;
    for (int w = 0; w < C::NW; ++w) Nmax = fmaxf(Nmax, red[64 + w]);
    const float ysc = Nmax > 0.f ? 65535.f / Nmax : 0.f;

    // ================= pass 2a: fixed-point weights y = w * n * 65535 / Nmax as B fragments
    // unit (kappa, quad): tokens 32 kappa + 16 j + 4 quad + i -> lanes (2 r + digit, quad), word j
    const int nk = (len + 31) >> 5;
    float lsum[kPRows] = {0.f, 0.f, 0.f, 0.f};
    uint32_t usum[kPRows] = {0u, 0u, 0u, 0u};
    for (int u = tid; u < nk * 4; u += NT) {
        const int kap = u >> 2, quad = u & 3;
        uint32_t wlo[kPRows][2], whi[kPRows][2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            uint32_t y[4][kPRows];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tk = 32 * kap + 16 * j + 4 * quad + i;
                const bool valid = tk < len;
                const float4 z = valid ? *(const float4 *)(sbuf + tk * kPRows) : make_float4(0.f, 0.f, 0.f, 0.f);
                const float nf = valid ? f16_bits_to_f32(vnb[tk]) * ysc : 0.f;
                const float zz[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
                for (int r = 0; r < kPRows; ++r) {
                    const float w = valid ? exp2f(zz[r] - Mr[r]) : 0.f;
                    lsum[r] += w;
                    const uint32_t q = __float2uint_rn(w * nf);
                    usum[r] += q;
                    y[i][r] = q;
                }
            }
#pragma unroll
            for (int r = 0; r < kPRows; ++r) {
                const uint32_t p01 = __byte_perm(y[0][r], y[1][r], 0x5140);  // [y0.b0, y1.b0, y0.b1, y1.b1]
                const uint32_t p23 = __byte_perm(y[2][r], y[3][r], 0x5140);
                wlo[r][j] = __byte_perm(p01, p23, 0x5410);
                whi[r][j] = __byte_perm(p01, p23, 0x7632);
            }
        }
#pragma unroll
        for (int r = 0; r < kPRows; ++r) {
            *(uint2 *)(wfrag + ((kap * 32 + (2 * r) * 4 + quad) * 2)) = make_uint2(wlo[r][0], wlo[r][1]);
            *(uint2 *)(wfrag + ((kap * 32 + (2 * r + 1) * 4 + quad) * 2)) = make_uint2(whi[r][0], whi[r][1]);
        }
    }
#pragma unroll
    for (int r = 0; r < kPRows; ++r) {
        lsum[r] = warp_sum(lsum[r]);
        uint32_t v = usum[r];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        usum[r] = v;
    }
    if (lane == 0) {
#pragma unroll
        for (int r = 0; r < kPRows; ++r) {
            red[128 + warp * 4 + r] = lsum[r];
            ((uint32_t *)red)[192 + warp * 4 + r] = usum[r];
        }
    }
    __syncthreads();

    // ================= pass 2b: value products
    const int cw = warp % C::VW, ts = warp / C::VW;
    int cv[C::VPL][C::TPW][4];
#pragma unroll
    for (int s = 0; s < C::VPL; ++s)
#pragma unroll
        for (int t = 0; t < C::TPW; ++t) cv[s][t][0] = cv[s][t][1] = cv[s][t][2] = cv[s][t][3] = 0;
    const int gg = (C::GPW == 2) ? (gid >> 2) : 0;
    const uint32_t bsel = (C::CPW == 64) ? (uint32_t)(gid & 3) : (uint32_t)(gid >> 1);
    const int IB = (C::CPW == 32) ? 4 * (gid & 1) : 0;
    const uint32_t sel2 = bsel | ((bsel + 4) << 4);
    {
        const int kper = (nk + C::TS - 1) / C::TS;
        const int k0 = min(nk, ts * kper), k1 = min(nk, k0 + kper);
        uint8_t *wring = smem + L.ring + (size_t)warp * NST * RG::STAGE;
        constexpr int PW = C::GPW * VB;  // plane words of this warp's groups per token
        const int woff = cw * C::GPW * VB;
        // this lane copies its token's plane words of the warp's groups, one stage per product
        const uint32_t *gv = sp.vcodes + (rec_base + 32 * k0 + lane) * C::VWPT + woff;
        auto issue = [&](int s) {
            const int kap = k0 + s;
            if (kap < k1 && 32 * kap + lane < len) {
                uint32_t *st = (uint32_t *)(wring + (s % NST) * RG::STAGE);
                const uint32_t *src = gv + (int64_t)s * 32 * C::VWPT;
#pragma unroll
                for (int p = 0; p < PW; ++p) cp_async<4>(st + p * 32 + lane, src + p);
            }
            cp_async_commit();
        };
        for (int k = 0; k < NST - 1; ++k) issue(k);
        for (int s = 0; s < k1 - k0; ++s) {
            issue(s + NST - 1);
            if (NST == 4) cp_async_wait<3>();
            else cp_async_wait<1>();
            __syncwarp();
            const uint32_t *st = (const uint32_t *)(wring + (s % NST) * RG::STAGE);
            const int kap = k0 + s;
            const uint2 bw = *(const uint2 *)(wfrag + (kap * 32 + lane) * 2);
            uint32_t X[VB][2];
#pragma unroll
            for (int p = 0; p < VB; ++p) {
                const uint32_t *row = st + (gg * VB + p) * 32;
                X[p][0] = gather_byte(*(const uint4 *)(row + 4 * t4), sel2);
                X[p][1] = gather_byte(*(const uint4 *)(row + 16 + 4 * t4), sel2);
            }
#pragma unroll
            for (int sidx = 0; sidx < C::VPL; ++sidx) {
                const int sub = walsh_subset(VB, sidx);
                uint32_t x0 = 0, x1 = 0;
#pragma unroll
                for (int p = 0; p < VB; ++p)
                    if (sub & (1 << p)) {
                        x0 ^= X[p][0];
                        x1 ^= X[p][1];
                    }
#pragma unroll
                for (int t = 0; t < C::TPW; ++t) {
                    const uint32_t m0 = 0x01010101u << (IB + 2 * t), m1 = m0 << 1;
                    const uint32_t a[4] = {x0 & m0, x0 & m1, x1 & m0, x1 & m1};
                    mma_u8u8(cv[sidx][t], a, bw.x, bw.y);
                }
            }
            __syncwarp();
        }
        cp_async_wait<0>();
    }

    // ---- sum the token subsets, then o_rot = (Nmax / 65535) sum_S alpha_S (2 U_S / 2^iota - U)
    constexpr int NCV = C::VPL * C::TPW * 4;
    if constexpr (C::TS > 1) {
        __syncthreads();  // sbuf is free
        int *xch = (int *)sbuf;
        if (ts > 0) {
            int *dst = xch + ((size_t)((ts - 1) * C::VW + cw) * NCV) * 32 + lane;
#pragma unroll
            for (int s = 0; s < C::VPL; ++s)
#pragma unroll
                for (int t = 0; t < C::TPW; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[((s * C::TPW + t) * 4 + e) * 32] = cv[s][t][e];
        }
        __syncthreads();
#pragma unroll
        for (int o = 1; o < C::TS; ++o) {
            if (ts != 0) break;
            const int *src = xch + ((size_t)((o - 1) * C::VW + cw) * NCV) * 32 + lane;
#pragma unroll
            for (int s = 0; s < C::VPL; ++s)
#pragma unroll
                for (int t = 0; t < C::TPW; ++t)
#pragma unroll
                    for (int e = 0; e < 4; ++e) cv[s][t][e] += src[((s * C::TPW + t) * 4 + e) * 32];
        }
    }
    // Walsh coefficients of the value codebook (computed in the prologue; barriers since)
    double va[C::VPL];
#pragma unroll
    for (int s = 0; s < C::VPL; ++s) va[s] = va_s[s];
    // row t4: sum of weights and of fixed-point weights over the range
    float lrow = 0.f;
    int64_t utot = 0;
    for (int w = 0; w < C::NW; ++w) {
        lrow += red[128 + w * 4 + t4];
        utot += ((const uint32_t *)red)[192 + w * 4 + t4];
    }
    const double unit = (double)Nmax / 65535.0;
    // the warps of token subset 0 hold the range's sums and write the partial
    if (ts == 0 && t4 < nrows) {
        float *op = partials + (qrow_of(t4) * splits + split) * (int64_t)(D + 2);
        if (gid == 0 && cw == 0) {
            const float mrow = t4 == 0 ? Mr[0] : t4 == 1 ? Mr[1] : t4 == 2 ? Mr[2] : Mr[3];
            op[0] = mrow * 0.6931471805599453f;  // natural-log units
            op[1] = lrow;
        }
#pragma unroll
        for (int t = 0; t < C::TPW; ++t)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int iota = IB + 2 * t + u;
                const int c = 32 * (cw * C::GPW + gg) + 8 * (int)bsel + iota;
                double acc = 0.0;
#pragma unroll
                for (int s = 0; s < C::VPL; ++s) {
                    const int64_t U = (int64_t)cv[s][t][2 * u + 1] * 256 + (int64_t)cv[s][t][2 * u];
                    acc += va[s] * (double)(2 * U - (utot << iota));
                }
                op[2 + c] = (float)(acc * unit / (double)(1 << iota));
            }
    }

    // ---- the slice's last CTA to finish merges the partials of all its ranges and rotates back:
    // out = R^T (sum_s e^{M_s - M} o_s) / (sum_s e^{M_s - M} l_s)
    __shared__ uint32_t last;
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(frag + sl * (int64_t)C::SLW + 32 * C::NK * 4 + kCounterWord, 1u) == (uint32_t)(splits - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();
    float *orow = sbuf;                 // [kPRows][D] merged o_rot
    float *wsp = sbuf + kPRows * D;     // [kPRows][splits] split weights e^{M_s - M}
    __shared__ float msh[kPRows], lsh[kPRows];
    for (int r = warp; r < nrows; r += C::NW) {
        const float *pp = partials + qrow_of(r) * splits * (int64_t)(D + 2);
        float M = -INFINITY;
        for (int s2 = lane; s2 < splits; s2 += 32) M = fmaxf(M, pp[(int64_t)s2 * (D + 2)]);
        M = warp_max(M);
        float Ls = 0.f;
        for (int s2 = lane; s2 < splits; s2 += 32) {
            const float *ps = pp + (int64_t)s2 * (D + 2);
            const float w = (ps[0] == -INFINITY) ? 0.f : expf(ps[0] - M);
            wsp[r * splits + s2] = w;
            Ls = fmaf(w, ps[1], Ls);
        }
        Ls = warp_sum(Ls);
        if (lane == 0) {
            msh[r] = M;
            lsh[r] = Ls;
        }
    }
    __syncthreads();
    for (int e = tid; e < nrows * D; e += NT) {
        const int r = e / D, j = e % D;
        const float *pj = partials + qrow_of(r) * splits * (int64_t)(D + 2) + 2 + j;
        const float *ww = wsp + r * splits;
        float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        int s2 = 0;
        for (; s2 + 8 <= splits; s2 += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = pj[(int64_t)(s2 + u) * (D + 2)];
#pragma unroll
            for (int u = 0; u < 8; ++u) a8[u] = fmaf(ww[s2 + u], v[u], a8[u]);
        }
        for (; s2 < splits; ++s2) a8[0] = fmaf(ww[s2], pj[(int64_t)s2 * (D + 2)], a8[0]);
        const float sum = ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
        if (merged_partial) {
            // the slice's partial over its whole context: (M, l, o_rot), unnormalised
            float *po = out + qrow_of(r) * (int64_t)(D + 2);
            if (j == 0) {
                po[0] = msh[r];
                po[1] = lsh[r];
            }
            po[2 + j] = sum;
        } else {
            orow[r * D + j] = sum / lsh[r];
        }
    }
    if (merged_partial) return;
    __syncthreads();
    for (int j = tid; j < D; j += NT) {
        float a4[kPRows] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
        for (int i = 0; i < D; ++i) {
            const float rv = P.R[(int64_t)i * D + j];
#pragma unroll
            for (int r = 0; r < kPRows; ++r) a4[r] = fmaf(rv, orow[r * D + i], a4[r]);
        }
#pragma unroll
        for (int r = 0; r < kPRows; ++r)
            if (r < nrows) out[qrow_of(r) * D + j] = a4[r];
    }
}

template <int D, int KB, int VB, bool ATTEND>
cudaError_t launch_planes_t(const Prepared &P, const ScoreProblem &sp, float scale, uint32_t *frag,
                            int range, int splits, float *out, float *partials, cudaStream_t s, int mp) {
    using C = PlanesCfg<D, KB, VB>;
    const int64_t slices = (int64_t)sp.B * sp.Hkv;
    auto qk = planes_qfrag_kernel<D, KB>;
    cudaError_t e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QfragChunk<D>::BYTES);
    if (e != cudaSuccess) return e;
    qk<<<(unsigned)slices, 256, QfragChunk<D>::BYTES, s>>>(P, sp, ATTEND ? scale : 1.0f, frag);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const PlanesSmem L = planes_smem<D, KB, VB, ATTEND>(range, splits);
    auto kern = planes_attend_kernel<D, KB, VB, ATTEND>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)splits, (unsigned)slices);
    kern<<<grid, C::NW * 32, L.total, s>>>(P, sp, frag, range, splits, out, partials, mp);
    return cudaGetLastError();
}

template <int D, bool ATTEND>
cudaError_t launch_planes_d(const Prepared &P, const ScoreProblem &sp, float scale, uint32_t *frag, int range,
                            int splits, float *out, float *partials, cudaStream_t s, int mp) {
    const int kb = P.kbeta, vb = P.vbeta;
    if constexpr (ATTEND) {
        if (kb == 1 && vb == 2) return launch_planes_t<D, 1, 2, true>(P, sp, scale, frag, range, splits, out, partials, s, mp);
        if (kb == 2 && vb == 3) return launch_planes_t<D, 2, 3, true>(P, sp, scale, frag, range, splits, out, partials, s, mp);
        if (kb == 3 && vb == 4) return launch_planes_t<D, 3, 4, true>(P, sp, scale, frag, range, splits, out, partials, s, mp);
    } else {
        if (kb == 1) return launch_planes_t<D, 1, 2, false>(P, sp, scale, frag, range, splits, out, partials, s, mp);
        if (kb == 2) return launch_planes_t<D, 2, 2, false>(P, sp, scale, frag, range, splits, out, partials, s, mp);
        if (kb == 3) return launch_planes_t<D, 3, 2, false>(P, sp, scale, frag, range, splits, out, partials, s, mp);
    }
    return cudaErrorInvalidValue;
}

int planes_nk(int d, int kbeta) {
    const int kpl = walsh_terms(kbeta);
    return (d / 32) * kpl + d / 64;
}

}  // namespace

bool planes_supported(const Prepared &P, const ScoreProblem &sp, bool attend) {
    if (P.d != 64 && P.d != 128 && P.d != 256) return false;
    if (P.m * 2 != P.d) return false;  // proj_dim = head_dim / 2
    if ((sp.Hq / sp.Hkv) * sp.Nq > kPRows) return false;
    const int kb = P.kbeta, vb = P.vbeta;
    if (kb < 1 || kb > 3) return false;
    return !attend || vb == kb + 1;
}

PlanesPlan plan_planes(const ScoreProblem &sp) {
    PlanesPlan pl;
    const int64_t slices = (int64_t)sp.B * sp.Hkv;
    // at least one CTA per kPRange tokens; enough CTAs for about three per SM
    int64_t splits = (sp.T + kPRange - 1) / kPRange;
    const int64_t want = (148 * 3 + slices - 1) / slices;
    const int64_t cap = (sp.T + 255) / 256;  // keep ranges of at least ~256 tokens
    if (splits < want) splits = want < cap ? want : cap;
    if (splits < 1) splits = 1;
    int64_t range = (sp.T + splits - 1) / splits;
    range = (range + 31) & ~(int64_t)31;
    if (range > kPRange) range = kPRange;
    splits = (sp.T + range - 1) / range;
    pl.range = (int)range;
    pl.splits = (int)splits;
    return pl;
}

size_t planes_frag_bytes(const Prepared &P, const ScoreProblem &sp) {
    const int nk = planes_nk(P.d, P.kbeta);
    return align_up(sizeof(uint32_t) * (size_t)sp.B * sp.Hkv * (size_t)(32 * nk * 4 + 64), 256);
}

cudaError_t launch_planes(const Prepared &P, const ScoreProblem &sp, float scale, uint32_t *frag,
                          const PlanesPlan &pl, bool attend, float *out, float *partials, cudaStream_t s,
                          bool merged_partial) {
    const int mp = merged_partial ? 1 : 0;
    switch (P.d) {
        case 64:
            return attend ? launch_planes_d<64, true>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp)
                          : launch_planes_d<64, false>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp);
        case 128:
            return attend ? launch_planes_d<128, true>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp)
                          : launch_planes_d<128, false>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp);
        case 256:
            return attend ? launch_planes_d<256, true>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp)
                          : launch_planes_d<256, false>(P, sp, scale, frag, pl.range, pl.splits, out, partials, s, mp);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tq
