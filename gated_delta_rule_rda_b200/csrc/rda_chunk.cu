// Chunked tensor-core prefill (placeholder until the sm_100a kernel lands).
#include "rda_internal.h"

namespace rda {

bool chunked_supported(rda_dtype_t, int, int) { return false; }

cudaError_t launch_chunked(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace rda
