// rda_prefill_chunked_noalloc: the fixed-length prefill for callers that
// cannot hand the library a workspace.  Some host programs own every byte of
// device memory themselves -- an inference server that plans its memory pool
// once at start-up, or a plug-in whose host framework gives it tensors but no
// way to request scratch -- and must not call cudaMalloc after that point.
// This entry point needs no workspace from them: its scratch is a file-scope
// device array of fixed size, which every GPU that loads this library holds
// until the process exits.
//
// The array is shared by every call on a device and keeps the last call's
// contents; calls whose work overlaps on the GPU (for example on two streams
// without ordering between them) race on it.  The device error word at its
// start is cleared at the beginning of each call.
#include <mutex>

#include "rda_internal.h"

namespace {

// Largest scratch this entry point can use, bytes: enough for the chunked
// path's per-chunk images of about 1,600 (chunk, head) pairs at Dv = 128,
// e.g. B = 1, T = 4096, H = 16.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code may not use the array's name as a device address: it resolves the
// address once per device, with that device current.
std::mutex g_mu;
void *g_scratch_addr[64] = {};

cudaError_t scratch_for_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" rda_status_t rda_prefill_chunked_noalloc(const void *q, const void *k, const void *v,
                                                   const float *log_alpha, const float *beta,
                                                   const float *write_gate,
                                                   const float *initial_state, float *final_state,
                                                   void *out, rda_dtype_t dtype,
                                                   int B, int T, int H, int Dk, int Dv, float scale,
                                                   void *stream) {
    if (B < 0 || T < 0 || H <= 0) return RDA_ERR_INVALID_ARG;
    const size_t need = rda_prefill_workspace_bytes(B, T, H, Dk, Dv, 0);
    if (need == 0) return (Dk == 64 || Dk == 128) && (Dv == 64 || Dv == 128) ? RDA_ERR_INVALID_ARG
                                                                              : RDA_ERR_UNSUPPORTED;
    if (need > kNoAllocScratchBytes) return RDA_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return RDA_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return RDA_ERR_CUDA;
    return rda_prefill_chunked(q, k, v, log_alpha, beta, write_gate, initial_state, final_state, out, dtype,
                               B, T, H, Dk, Dv, scale, scratch, kNoAllocScratchBytes, stream);
}
