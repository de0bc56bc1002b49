// tq_prepare.cu -- derive the kernels' operand copies of R and S into the workspace.
#include "tq_internal.cuh"

namespace tq {

namespace {

__global__ void prepare_kernel(const float *__restrict__ R, const float *__restrict__ S, int d, int m,
                               Codebooks cb, WsHeader hdr, char *__restrict__ ws, WsLayout L) {
    float *Rc = (float *)(ws + L.R);
    float *RT = (float *)(ws + L.RT);
    float *ST = (float *)(ws + L.ST);
    float *SpT = (float *)(ws + L.SpT);
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nth = (int64_t)gridDim.x * blockDim.x;
    if (tid == 0) {
        *(WsHeader *)(ws + L.header) = hdr;
        *(Codebooks *)(ws + L.codebooks) = cb;
    }
    uint16_t *Rhi = (uint16_t *)(ws + L.Rsw);
    uint16_t *Rlo = Rhi + (size_t)d * d;
    for (int64_t e = tid; e < (int64_t)d * d; e += nth) {
        int i = (int)(e / d), j = (int)(e % d);
        float v = R[e];
        Rc[e] = v;
        RT[(int64_t)j * d + i] = v;
        // split operand: R * 2^s = hi + lo, both fp16, row i = output coordinate, k = j
        const float sv = v * (float)(1 << kRScaleLog2);
        const __half hi = __float2half_rn(sv);
        const __half lo = __float2half_rn(sv - __half2float(hi));
        const size_t off = sw128_offset(d, i, j) / 2;
        Rhi[off] = __half_as_ushort(hi);
        Rlo[off] = __half_as_ushort(lo);
    }
    // keys' rotation operand [R; S] * 2^s split into fp16 hi + lo, d + m rows
    {
        const int rows = d + (m > 0 ? m : 0);
        uint16_t *Xhi = (uint16_t *)(ws + L.RSsw);
        uint16_t *Xlo = Xhi + (size_t)d * rows;
        for (int64_t e = tid; e < (int64_t)rows * d; e += nth) {
            const int i = (int)(e / d), j = (int)(e % d);
            const float v = (i < d) ? R[(int64_t)i * d + j] : S[(int64_t)(i - d) * d + j];
            const float sv = v * (float)(1 << kRScaleLog2);
            const __half hi = __float2half_rn(sv);
            const __half lo = __float2half_rn(sv - __half2float(hi));
            const size_t off = sw128_offset(rows, i, j) / 2;
            Xhi[off] = __half_as_ushort(hi);
            Xlo[off] = __half_as_ushort(lo);
        }
    }
    if (m <= 0) return;
    float *Srow = (float *)(ws + L.S);
    float *Sprow = (float *)(ws + L.Sp);
    for (int64_t e = tid; e < (int64_t)m * d; e += nth) {
        int a = (int)(e / d), j = (int)(e % d);
        ST[(int64_t)j * m + a] = S[e];
        Srow[e] = S[e];
    }
    // S' = S R^T expressed on rotated coordinates: S'[a][i] = sum_k S[a][k] R[i][k],
    // accumulated in double and rounded once.
    for (int64_t e = tid; e < (int64_t)m * d; e += nth) {
        int a = (int)(e / d), i = (int)(e % d);
        const float *sr = S + (int64_t)a * d;
        const float *rr = R + (int64_t)i * d;
        double acc = 0.0;
        for (int k = 0; k < d; ++k) acc += (double)sr[k] * (double)rr[k];
        SpT[(int64_t)i * m + a] = (float)acc;
        Sprow[e] = (float)acc;
        // split operand of S' * 2^s: row a = projection index, k = i (rotated coordinate)
        const double sv = acc * (double)(1 << kSScaleLog2);
        const __half hi = __double2half(sv);
        const __half lo = __float2half_rn((float)(sv - (double)__half2float(hi)));
        uint16_t *Shi = (uint16_t *)(ws + L.Ssw);
        uint16_t *Slo = Shi + (size_t)m * d;
        const size_t off = sw128_offset(m, a, i) / 2;
        Shi[off] = __half_as_ushort(hi);
        Slo[off] = __half_as_ushort(lo);
    }
}

}  // namespace

cudaError_t launch_prepare(const tq_params *p, const Codebooks &cb, cudaStream_t s) {
    WsLayout L = ws_layout(p->dim, p->proj_dim);
    WsHeader h{kWsMagic, p->dim, p->bits, p->proj_dim};
    int64_t work = (int64_t)p->dim * (p->dim > p->proj_dim ? p->dim : p->proj_dim);
    int blocks = (int)((work + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    prepare_kernel<<<blocks, 256, 0, s>>>(p->R, p->S, p->dim, p->proj_dim, cb, h,
                                         (char *)p->workspace, L);
    return cudaGetLastError();
}

}  // namespace tq
