// prefill_noalloc.cu -- gdn_prefill_noalloc: the sequence-parallel prefill without any
// allocation, its workspace taken from a fixed array inside the library.
//
// Some callers cannot call cudaMalloc: code that runs where allocation is forbidden or
// unavailable (a host runtime that owns all device memory through its own pool and gives
// kernels no allocator, a C caller with no memory manager of its own, code on a hot serving
// path that must never allocate), or that cannot know how much scratch a call needs.  For them
// this entry point uses a file-scope device array instead of a caller-provided workspace.
//
// The array is a static __device__ object: every GPU that loads the library holds its own
// kNoAllocScratchBytes of it until the process exits.  Host code never uses the array's name
// as a pointer (on the host it is only a stand-in symbol); its device address is looked up
// with cudaGetSymbolAddress once per device, with that device current, on the first call made
// on that device, and cached.
#include <mutex>

#include "common.cuh"

namespace {

// 8 MiB: the split workspace of 32 (request, value head) units of 128 x 128 heads, e.g. one
// request with 32 value heads (the long-context workload)
constexpr uint64_t kNoAllocScratchBytes = 8ull << 20;

static __device__ __align__(256) unsigned char g_prefill_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mu;
void *g_addr[kMaxDevices] = {};

// device address of g_prefill_scratch on the current device (looked up on first use)
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_prefill_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

gdn_status gdn_prefill_noalloc(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *a_log, const float *dt_bias,
                               const int32_t *cu_seqlens, const float *initial_state,
                               float *final_state, void *out, int32_t B, int64_t N, int32_t Hq,
                               int32_t Hv, int32_t Dk, int32_t Dv, gdn_dtype dtype, float scale,
                               int32_t qk_l2norm, uint32_t flags, int32_t *dev_status,
                               void *stream)
{
    const uint64_t need = gdn_prefill_workspace_size(B, N, Hq, Hv, Dk, Dv, dtype, flags);
    if (need > kNoAllocScratchBytes) return GDN_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (need > 0) {
        const cudaError_t e = scratch_address(&ws);
        if (e != cudaSuccess) return gdn_report_cuda_failure(e, "gdn_prefill_noalloc scratch address");
    }
    // every workspace byte the split reads is written earlier in the same call (segment 1's
    // start state, A and B by pass 1, segment 2's start state by the composition), so the
    // array's contents left by an earlier call need no clearing
    return gdn_prefill_ws(q, k, v, g, beta, a_log, dt_bias, cu_seqlens, initial_state,
                          final_state, out, B, N, Hq, Hv, Dk, Dv, dtype, scale, qk_l2norm, flags,
                          ws, need, dev_status, stream);
}

}  // extern "C"
