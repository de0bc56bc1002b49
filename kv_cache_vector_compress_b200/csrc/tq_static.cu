// tq_static.cu -- tq_attend_static: fused attention without a caller-provided scratch buffer.
//
// Some callers cannot allocate device memory when they call the library: a serving loop whose
// device memory is fully handed to its own pool up front, or code that must not pay the device
// synchronisation that cudaMalloc / cudaFree can cause in the middle of a decode step.  For them
// this entry point takes its scratch (rotated queries and split-context partial results) from a
// fixed array that belongs to the library instead of from the caller.
#include <mutex>

#include "tq_internal.cuh"

namespace {

// The library-owned scratch array.  Every GPU that loads the library holds it until exit.
static __device__ __align__(256) unsigned char tq_static_scratch[TQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per device.  In host code
// the array's name only stands for it; the address has to come from cudaGetSymbolAddress.
tq_status static_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, tq_static_scratch) != cudaSuccess || !p) return TQ_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_attend_static(const tq_params *p, const float *q, int B, int Hq, int Hkv, int Nq,
                                      int64_t T, const uint32_t *kcodes, const uint32_t *ksigns,
                                      const uint16_t *knorm, const uint16_t *krnorm, const uint32_t *vcodes,
                                      const uint16_t *vnorm, float scale, float *out, int32_t *dev_status,
                                      tq_stream_t stream) {
    const size_t need = tq_attend_scratch_bytes(p, B, Hq, Hkv, Nq, T);
    if (need == 0) return TQ_ERR_INVALID_ARG;
    if (need > (size_t)TQ_STATIC_SCRATCH_BYTES) return TQ_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    const tq_status st = static_scratch(&scratch);
    if (st != TQ_OK) return st;
    // every byte the call reads from the array is written earlier in the same call, so the
    // previous call's contents never need clearing
    return tq_attend(p, q, B, Hq, Hkv, Nq, T, kcodes, ksigns, knorm, krnorm, vcodes, vnorm, scale, out, scratch,
                     (size_t)TQ_STATIC_SCRATCH_BYTES, dev_status, stream);
}
