// prefill_chunk.cu -- chunked tensor-core Gated DeltaNet prefill (sm_100a).
#include "common.cuh"

bool prefill_chunked_supported(const GdnPrefillArgs &) { return false; }

cudaError_t launch_prefill_chunked(const GdnPrefillArgs &, cudaStream_t)
{
    return cudaErrorNotSupported;
}
