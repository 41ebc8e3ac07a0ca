// Chunked-prefill attention (query rows of sequences with q_len > 1).
#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

cudaError_t launch_prefill(const PrefillArgs&, const CUtensorMap&, const CUtensorMap&,
                           const CUtensorMap&, const pa_cache_desc&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pa
