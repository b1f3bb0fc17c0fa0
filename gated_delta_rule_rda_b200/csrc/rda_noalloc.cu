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
// start is cleared at the beginning of each call that passes the argument
// checks; a call that fails them enqueues nothing.
#include "rda_internal.h"

namespace {

// Largest scratch this entry point can use, bytes: the chunked path's
// per-chunk images of about 1,600 (chunk, head) pairs at Dv = 128 (H = 16:
// T up to about 6,400).
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" rda_status_t rda_prefill_chunked_noalloc(const void *q, const void *k, const void *v,
                                                   const float *log_alpha, const float *beta,
                                                   const float *write_gate,
                                                   const float *initial_state, float *final_state,
                                                   void *out, rda_dtype_t dtype,
                                                   int B, int T, int H, int Dk, int Dv, float scale,
                                                   void *stream) {
    size_t need = 0;
    rda_status_t st = rda::validate_prefill_chunked(q, k, v, log_alpha, beta, write_gate, initial_state,
                                                    final_state, out, dtype, B, T, H, Dk, Dv, &need);
    if (st != RDA_OK) return st;
    if (need > kNoAllocScratchBytes) return RDA_ERR_WORKSPACE;
    // The array's name is not a device address in host code.  Its address is
    // looked up in the current context on every call, so a context created
    // after a device reset (or another context on the same device) gets its
    // own array's address, never a stale one.
    void *scratch = nullptr;
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch) return RDA_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess) return RDA_ERR_CUDA;
    return rda_prefill_chunked(q, k, v, log_alpha, beta, write_gate, initial_state, final_state, out, dtype,
                               B, T, H, Dk, Dv, scale, scratch, kNoAllocScratchBytes, stream);
}
