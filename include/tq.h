/*
 * tq.h -- C ABI of libtq, a B200 (sm_100a) implementation of the TurboQuant
 * KV-cache vector compression hot path.
 *
 * What the method computes (web pages on the turboquant-pytorch / turboquant-py
 * implementations of Google's TurboQuant):
 *   - stage 1 ("TurboQuantMSE"): normalise a vector, rotate it by a fixed random
 *     orthogonal matrix R so every coordinate follows N(0, 1/d), and Lloyd-Max
 *     quantize each coordinate with b bits
 *       ["turboquant-pytorch" (atskills.one), "What It Does" and
 *        "Algorithm Details: Why Random Rotation?";
 *        "turboquant-pytorch" (nav.superapi.store), 主要能力, 核心 API, 算法细节];
 *   - stage 2 ("TurboQuantProd", keys only): a 1-bit QJL sign sketch of the residual
 *     through a Gaussian matrix S with proj_dim = head_dim/2 rows, which makes inner
 *     product estimates unbiased [same pages, "Why QJL for Keys but Not Values?",
 *     算法细节 "proj_dim 选择"];
 *   - attention straight from the compressed keys ("asymmetric_attention_scores"),
 *     softmax, weighted sum over the MSE-dequantized values
 *       [nav.superapi.store page, 常见使用模式 "压缩整个模型的 KV 缓存"].
 *
 * Conventions (all functions):
 *   - Every call returns a tq_status.  Argument errors are detected on the host and
 *     returned before anything is launched; nothing is written in that case.
 *   - The caller allocates and owns every buffer.  The library never allocates or
 *     frees device memory; the one device memory it keeps is the fixed scratch array
 *     of tq_attend_static (declared last), which exists only for that call.
 *   - Device work is enqueued asynchronously on the caller's stream; results are
 *     ready when that stream is synchronised.  Outputs are bit-identical run to run.
 *   - Device pointers must be 16-byte aligned (TQ_ERR_INVALID_ARG otherwise).
 *   - dev_status (optional, may be NULL) is a device int32 that kernels set to a
 *     nonzero tq_status if they detect an error on the device; it is never cleared
 *     by the library.
 *
 * Packed layout (a contract of this library; the pages do not fix one):
 *   codes  : per vector, dim/32 groups of beta little-endian uint32 words; word
 *            g*beta + p holds bit p of the code of coordinate 32g+l at bit l
 *            (beta = bits-1 for keys, bits for values);
 *   signs  : per key, proj_dim/32 words; word g bit l = [p_{32g+l} >= 0];
 *   norms  : IEEE binary16 (round to nearest even) of the fp32 value.
 *   Keys take (bits-1)*dim/8 + proj_dim/8 + 4 bytes, values bits*dim/8 + 2 bytes.
 *   Records of a cache are ordered [B, Hkv, T] (row-major).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *tq_stream_t; /* binary-compatible with cudaStream_t */

typedef enum tq_status {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size or value      */
    TQ_ERR_UNSUPPORTED = 2, /* valid arguments outside what the kernels implement */
    TQ_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed               */
    TQ_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (dev_status)    */
} tq_status;

typedef enum tq_dtype { TQ_F16 = 0, TQ_F32 = 1 } tq_dtype;

/* Human-readable name of a status code.  Never returns NULL. */
const char *tq_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
int tq_version(void);

/*
 * Lloyd-Max codebook for one coordinate of a randomly rotated unit vector, whose law
 * is taken as N(0, 1/dim) (nav.superapi.store page, 核心 API
 * "build_lloyd_max_codebook(dim=128, bits=3) returns (boundaries, centroids)";
 * atskills.one page, "Why Random Rotation?").  HOST function, no device work.
 *   dim        : vector dimension (>= 1)
 *   bits       : 1..4
 *   boundaries : host array of 2^bits - 1 floats, ascending; the middle one is 0
 *   centroids  : host array of 2^bits floats, ascending, antisymmetric
 * A coordinate y gets code #{k : boundaries[k] < y} (ties go to the lower cell).
 */
tq_status tq_codebook(int dim, int bits, float *boundaries, float *centroids);

/*
 * The same Lloyd-Max conditions under the exact law of one coordinate of a uniformly random
 * unit vector in R^dim, density proportional to (1 - y^2)^((dim-3)/2) on (-1, 1): the
 * "concentrated Beta" law of "TurboQuant er nå tilgjengelig som Python-bibliotek"
 * (jansverre.net), section "Hva er TurboQuant, kort fortalt?".  N(0, 1/dim) is its large-dim
 * limit.  HOST function, no device work.  Arguments as tq_codebook; dim >= 3.
 */
tq_status tq_codebook_beta(int dim, int bits, float *boundaries, float *centroids);

/* Coordinate laws a parameter set's codebooks can be built for (tq_prepare_law). */
enum { TQ_LAW_GAUSSIAN = 0, TQ_LAW_BETA = 1 };

/*
 * Quantizer parameters.  R and S are caller-generated (the pages use a fixed random
 * orthogonal R and an i.i.d. N(0,1) matrix S; the library takes them as inputs).
 *   dim      : head dimension d; a multiple of 32, 32..1024
 *   bits     : nominal bits per coordinate b, 1..4.  Values use b MSE bits; keys use
 *              b-1 MSE bits plus one QJL sign per projection (so keys need b >= 2)
 *   proj_dim : QJL projection count m; a multiple of 32, 32..1024 (0 = values only)
 *   R        : device fp32 [dim, dim], row-major, orthogonal; rotation y = R u
 *   S        : device fp32 [proj_dim, dim], row-major (NULL when proj_dim == 0)
 *   workspace: device buffer of at least tq_workspace_bytes(dim, bits, proj_dim)
 *              bytes, filled by tq_prepare; read by every other call
 */
typedef struct tq_params {
    int dim;
    int bits;
    int proj_dim;
    const float *R;
    const float *S;
    void *workspace;
    size_t workspace_bytes;
} tq_params;

/* Bytes of workspace tq_prepare needs for these sizes (0 if the sizes are invalid). */
size_t tq_workspace_bytes(int dim, int bits, int proj_dim);

/*
 * Derive everything the kernels need from (R, S, codebooks) into p->workspace:
 * the fp32 codebooks for bits-1 and bits, S' = S R^T (the QJL projection expressed on
 * rotated coordinates) and the split-precision operand copies of R and S'.  Call it
 * once per (R, S), and again whenever they change.  Enqueued on `stream`.
 */
tq_status tq_prepare(const tq_params *p, int32_t *dev_status, tq_stream_t stream);

/*
 * tq_prepare with the codebooks of a chosen coordinate law: TQ_LAW_GAUSSIAN (what tq_prepare
 * uses, tq_codebook) or TQ_LAW_BETA (tq_codebook_beta).  Every other call then quantizes,
 * scores and dequantizes with those codebooks.  TQ_ERR_INVALID_ARG for any other law.
 */
tq_status tq_prepare_law(const tq_params *p, int law, int32_t *dev_status, tq_stream_t stream);

/*
 * Compress n key vectors (TurboQuantProd.compress / TurboQuantCompressorV2;
 * nav.superapi.store page, 核心 API; atskills.one page, "What It Does" stages 1+2):
 *   n_k = ||x||, u = x / n_k, y = R u, idx_j = code of y_j with the (dim, bits-1)
 *   codebook, e = y - c[idx] (so the residual r = R^T e), rho = ||e||,
 *   sign_i = [ (S r)_i >= 0 ].
 *   x      : device [n, dim], fp16 or fp32 (dtype), row-major
 *   codes  : device uint32 [n, (bits-1)*dim/32]
 *   signs  : device uint32 [n, proj_dim/32]
 *   norm   : device fp16 bits [n]  (||x||)
 *   rnorm  : device fp16 bits [n]  (||r|| of the unit vector's residual)
 * n may be 0 (no work).  A zero vector gets norm 0 and the codes of y = 0.
 */
tq_status tq_compress_keys(const tq_params *p, const void *x, tq_dtype dtype, int64_t n,
                           uint32_t *codes, uint32_t *signs, uint16_t *norm, uint16_t *rnorm,
                           int32_t *dev_status, tq_stream_t stream);

/*
 * Compress n value vectors (TurboQuantMSE.quantize / TurboQuantCompressorMSE: stage 1
 * only; atskills.one page, "Why QJL for Keys but Not Values?").
 *   codes : device uint32 [n, bits*dim/32];  norm : device fp16 bits [n]
 */
tq_status tq_compress_values(const tq_params *p, const void *x, tq_dtype dtype, int64_t n,
                             uint32_t *codes, uint16_t *norm, int32_t *dev_status,
                             tq_stream_t stream);

/*
 * Asymmetric inner-product estimates straight from packed keys
 * (TurboQuantProd.inner_product / asymmetric_attention_scores; nav.superapi.store page,
 * 核心 API and 常见使用模式):
 *   s = ||k|| * ( <R q, c[idx]> + rho * sqrt(pi/2)/proj_dim * <S q, 2*sign - 1> )
 * (the raw estimate of <q, k>; no 1/sqrt(d) scaling).
 *   q      : device fp32 [B, Hq, Nq, dim];  query head h reads KV head h / (Hq/Hkv)
 *   keys   : the four arrays of tq_compress_keys for [B, Hkv, T] records
 *   scores : device fp32 [B, Hq, Nq, T], or NULL when only top-k is wanted
 *   topk   : 0, or 1..64: also return the topk largest scores of every (b, h, query)
 *            row, descending, ties to the smaller token index
 *   topk_idx / topk_val : device int32 / fp32 [B, Hq, Nq, topk] (when topk > 0)
 *   scratch: device buffer of tq_scores_scratch_bytes(...) bytes (may be NULL if 0)
 */
size_t tq_scores_scratch_bytes(const tq_params *p, int B, int Hq, int Hkv, int Nq, int64_t T,
                               int topk);
tq_status tq_scores(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, float *scores, int topk, int32_t *topk_idx,
                    float *topk_val, void *scratch, size_t scratch_bytes, int32_t *dev_status,
                    tq_stream_t stream);

/*
 * tq_search -- tq_scores for vector-database search ("TurboQuant er nå tilgjengelig som
 * Python-bibliotek", jansverre.net, "Hvem er dette nyttig for?": nearest-neighbour search over
 * compressed vectors), with the tensor-core products taken on single fp16 operands.
 * Arguments, layouts, scratch size (tq_scores_scratch_bytes), ownership and errors are those of
 * tq_scores.  Where the tensor-core search path runs (more than 64 query rows per KV head,
 * dim and proj_dim multiples of 64, 2-4 bit keys) each operand of a product is the fp16
 * rounding of its exact value (relative 2^-11), so a score differs from the exact estimator by at
 * most 2^-10 ||k|| (sum_i |q_rot,i c_i| + rho sqrt(pi/2)/m sum_j |(S q)_j|) beyond fp32
 * accumulation; with unit queries and keys at dim 1024 the typical difference is about 1e-5.
 * Other shapes run exactly as tq_scores.  The top-k is the k best of these scores.
 */
tq_status tq_search(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, float *scores, int topk, int32_t *topk_idx,
                    float *topk_val, void *scratch, size_t scratch_bytes, int32_t *dev_status,
                    tq_stream_t stream);

/*
 * Attention over a compressed cache, fused: scores from the packed keys, softmax of
 * scale*scores over all T tokens (no mask), weighted sum of the dequantized values
 * (nav.superapi.store page, 常见使用模式: "softmax 后对解压的值做加权求和"):
 *   out = sum_t softmax_t(scale * s_t) * ||v_t|| * R^T c[vidx_t]
 *   q      : device fp32 [B, Hq, Nq, dim]
 *   keys   : as tq_scores;  vcodes / vnorm: the arrays of tq_compress_values
 *   scale  : softmax temperature; <= 0 selects 1/sqrt(dim)
 *   out    : device fp32 [B, Hq, Nq, dim]
 *   scratch: device buffer of tq_attend_scratch_bytes(...) bytes (query operands, split-context
 *            partials, and room to stage the new records of tq_append_attend)
 * T must be >= 1.
 */
size_t tq_attend_scratch_bytes(const tq_params *p, int B, int Hq, int Hkv, int Nq, int64_t T);
tq_status tq_attend(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                    const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                    const uint16_t *krnorm, const uint32_t *vcodes, const uint16_t *vnorm,
                    float scale, float *out, void *scratch, size_t scratch_bytes,
                    int32_t *dev_status, tq_stream_t stream);

/*
 * tq_append_attend -- one decode step on caches with spare capacity: append the new token of
 * every (batch, KV head), then attend over the cache including it.
 * The append is TurboQuantProd.compress / TurboQuantMSE.quantize of the new key / value and the
 * attention is that of tq_attend, as the cache wrapper does them token by token
 * ("turboquant-pytorch", nav.superapi.store, 核心 API: TurboQuantKVCache with append_key,
 * append_value, attention_scores; "TurboQuant: онлайн-квантование векторов без калибровки",
 * ai-manual.ru, "Где TurboQuant выстреливает, а где нет?": keys and values compressed during
 * generation).  With at most 4 query rows per KV head (the bit-plane attention shapes) the new
 * rows go through the tensor-core compress kernels into a staging part of the scratch and are
 * scattered to slot t; with 5 to 64 rows (register-MMA attention shapes) the compression runs
 * inside the attention kernel, in the CTA whose context range holds slot t.
 *   q            : device fp32 [B, Hq, Nq, dim]
 *   k_new, v_new : device [B, Hkv, dim] of dtype (TQ_F16 or TQ_F32), 16-byte aligned
 *   t            : the slot the new token takes, 0 <= t < t_cap; slots 0 .. t-1 hold the cache
 *   t_cap        : cache capacity: every array below holds B * Hkv * t_cap records, record
 *                  (b * Hkv + h) * t_cap + s for slot s of (b, h), in the layouts of
 *                  tq_compress_keys / tq_compress_values; slot t is overwritten
 *   scale, out   : as tq_attend; the attention covers slots 0 .. t (t + 1 tokens)
 *   scratch      : tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, t + 1) bytes
 * For other shapes (outside dim 64, 128 or 256 with proj_dim = dim / 2 and 2-4 bit keys) the
 * append is a small kernel of its own, launched before the attention.
 * Returns the errors of tq_attend.
 */
tq_status tq_append_attend(const tq_params *p, const float *q, const void *k_new, const void *v_new,
                           tq_dtype dtype, int B, int Hq, int Hkv, int Nq, int64_t t, int64_t t_cap,
                           uint32_t *kcodes, uint32_t *ksigns, uint16_t *knorm, uint16_t *krnorm,
                           uint32_t *vcodes, uint16_t *vnorm, float scale, float *out, void *scratch,
                           size_t scratch_bytes, int32_t *dev_status, tq_stream_t stream);

/*
 * tq_selftest_wait_timeout -- exercises the device-side failure path of every kernel.
 * (The pages have no counterpart: this is a diagnostic of the library.)
 * Every wait of the kernels on another warp or on a copy is bounded; when one runs out, the
 * kernel records TQ_ERR_TIMEOUT in dev_status, drains its copies, frees its tensor memory and
 * returns, so the context stays usable.  This call launches one small kernel whose wait can only
 * end by its time limit (a barrier nothing ever arrives at) and so must leave TQ_ERR_TIMEOUT in
 * *dev_status after about timeout_ms milliseconds.
 *   dev_status : device int32 (required); set, never cleared
 *   timeout_ms : 1 .. 10000, else TQ_ERR_INVALID_ARG
 * Returns TQ_OK once the kernel is enqueued on stream.
 */
tq_status tq_selftest_wait_timeout(int32_t *dev_status, uint32_t timeout_ms, tq_stream_t stream);

/*
 * Attention over one piece of a longer context, for splitting a long context across GPUs
 * (nav.superapi.store page, 适用场景: long-context inference; the method's softmax is exact
 * over any partition of the tokens).  Arguments as tq_attend, with T the tokens of this piece
 * (records [B, Hkv, T] of this piece only); instead of the output it writes, per query row
 * [B, Hq, Nq], a partial of dim + 2 floats:
 *   partial[0]     = M, the largest logit scale * s_t of the piece,
 *   partial[1]     = l = sum_t e^{scale s_t - M},
 *   partial[2 + j] = sum_t e^{scale s_t - M} ||v_t|| c[vidx_tj]   (rotated coordinates, unnormalised)
 *   partial    : device fp32 [B * Hq * Nq, dim + 2]
 *   scratch    : device, tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T) bytes
 */
tq_status tq_attend_partial(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                            const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                            const uint16_t *krnorm, const uint32_t *vcodes, const uint16_t *vnorm, float scale,
                            float *partial, void *scratch, size_t scratch_bytes, int32_t *dev_status,
                            tq_stream_t stream);

/*
 * Merge the partials of `parts` pieces of a context (for example gathered from the GPUs that
 * each attended one piece with tq_attend_partial) into the attention output:
 *   M = max_k M_k,  out = R^T (sum_k e^{M_k - M} o_k) / (sum_k e^{M_k - M} l_k)
 *   partials : device fp32 [parts, rows, dim + 2] (piece-major, as an all-gather leaves them)
 *   out      : device fp32 [rows, dim]   (rows = B * Hq * Nq)
 * The result equals tq_attend over the whole context up to floating-point rounding.
 */
tq_status tq_attend_merge(const tq_params *p, const float *partials, int parts, int64_t rows, float *out,
                          int32_t *dev_status, tq_stream_t stream);

/*
 * tq_compress_attend_host -- one whole prefill-and-decode step from host memory: copy fp16/fp32
 * keys, values and queries from the host, compress the keys and values into the caller's device
 * cache arrays, attend, and copy the attention output back to the host, all enqueued on `stream`
 * (the cache wrapper's prefill then attention_scores / weighted value sum: "turboquant-pytorch",
 * nav.superapi.store, 核心 API and 常见使用模式).
 *   k_host, v_host : host [B, Hkv, T, dim] of dtype (TQ_F16 or TQ_F32)
 *   q_host         : host fp32 [B, Hq, Nq, dim]
 *   kcodes .. vnorm: device cache arrays for B * Hkv * T records (tq_compress_keys /
 *                    tq_compress_values layouts), overwritten
 *   scale          : as tq_attend
 *   out_host       : host fp32 [B, Hq, Nq, dim]; valid once `stream` has been synchronised
 *   scratch        : device buffer of tq_compress_attend_host_scratch_bytes(...) bytes (staging
 *                    of the inputs and the output, and the attention's scratch)
 * Host buffers should be page-locked (cudaHostAlloc) for the copies to run asynchronously; with
 * pageable memory the CUDA runtime stages them and the call returns later.  The host buffers
 * must stay valid and unmodified until the stream has been synchronised.  Errors: those of
 * tq_compress_keys, tq_compress_values and tq_attend (host pointers may not be NULL).
 */
size_t tq_compress_attend_host_scratch_bytes(const tq_params *p, tq_dtype dtype, int B, int Hq, int Hkv,
                                             int Nq, int64_t T);
tq_status tq_compress_attend_host(const tq_params *p, const void *k_host, const void *v_host, tq_dtype dtype,
                                  const float *q_host, int B, int Hq, int Hkv, int Nq, int64_t T,
                                  uint32_t *kcodes, uint32_t *ksigns, uint16_t *knorm, uint16_t *krnorm,
                                  uint32_t *vcodes, uint16_t *vnorm, float scale, float *out_host,
                                  void *scratch, size_t scratch_bytes, int32_t *dev_status,
                                  tq_stream_t stream);

/*
 * tq_attend_static -- tq_attend for callers that cannot allocate device memory when they call.
 * (The pages have no counterpart: this is an addition of the library.)
 * A serving loop whose device memory is all handed to its own pool up front, or code that must
 * not pay the device synchronisation cudaMalloc / cudaFree can cause inside a decode step, has
 * no scratch buffer to pass.  This call takes its scratch from a library-owned device array of
 * TQ_STATIC_SCRATCH_BYTES instead; every GPU that loads the library holds that array until the
 * process exits.  Arguments and results are those of tq_attend, without scratch/scratch_bytes.
 *   - Problems whose tq_attend_scratch_bytes(...) exceeds TQ_STATIC_SCRATCH_BYTES are rejected
 *     with TQ_ERR_UNSUPPORTED before any work; use tq_attend with your own scratch for them.
 *   - The call never allocates: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's address on that device (with that device
 *     current); make that first call before any stream capture.  The address is kept for the
 *     life of the process and belongs to the device's primary context (the one the CUDA runtime
 *     uses): do not call this after cudaDeviceReset, or with a different driver context current
 *     on that device.
 *   - All calls share the one array, which keeps the last call's contents (nothing in it needs
 *     to start at zero).  Calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on it: serialise them.
 */
#define TQ_STATIC_SCRATCH_BYTES (16u << 20)
tq_status tq_attend_static(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq, int64_t T,
                           const uint32_t *kcodes, const uint32_t *ksigns, const uint16_t *knorm,
                           const uint16_t *krnorm, const uint32_t *vcodes, const uint16_t *vnorm,
                           float scale, float *out, int32_t *dev_status, tq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
