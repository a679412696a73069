// common.cuh -- small device helpers shared by the libgdn kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "gdn.h"

namespace gdn {

__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

// 4 consecutive bf16 (8 bytes) -> float4
__device__ __forceinline__ float4 ld_bf16x4(const __nv_bfloat16 *p)
{
    uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&raw.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&raw.y);
    float2 a = __bfloat1622float2(lo);
    float2 b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}

// the same from shared memory (a plain load; the read-only global path does not apply)
__device__ __forceinline__ float4 lds_bf16x4(const __nv_bfloat16 *p)
{
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// streaming (evict-first) 16-byte global load / store
__device__ __forceinline__ float4 ld_stream(const float *p)
{
    return __ldcs(reinterpret_cast<const float4 *>(p));
}
__device__ __forceinline__ void st_stream(float *p, float4 v)
{
    __stcs(reinterpret_cast<float4 *>(p), v);
}

__device__ __forceinline__ float dot4(float4 a, float4 b)
{
    return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

template <int WIDTH>
__device__ __forceinline__ float group_sum(float x)
{
#pragma unroll
    for (int m = 1; m < WIDTH; m <<= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

__device__ __forceinline__ float warp_sum(float x) { return group_sum<32>(x); }

__device__ __forceinline__ int64_t clamp_i64(int64_t x, int64_t lo, int64_t hi)
{
    return x < lo ? lo : (x > hi ? hi : x);
}

// softplus with the threshold-20 rule of the decode gate
__device__ __forceinline__ float softplus20(float x)
{
    return x > 20.f ? x : log1pf(expf(x));
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// ---------------------------------------------------------------- checked builds
// Compiled with GDN_CHECKS, every global access and every data-dependent shared-memory access
// is first tested against its buffer; one outside it is skipped (a load yields zero) and
// GDN_DEV_BOUNDS is OR-ed into the status word.  Without GDN_CHECKS the tests are constant
// true and vanish.
#ifdef GDN_CHECKS
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif

// elements [i, i + len) inside [0, n)
__device__ __forceinline__ bool in_range(int64_t i, int64_t len, int64_t n, int32_t *status)
{
    if constexpr (!kChecked) return true;
    if (i >= 0 && len >= 0 && i + len <= n) return true;
    if (status) atomicOr(status, GDN_DEV_BOUNDS);
    return false;
}

// bytes [p, p + len) inside the block's dynamic shared memory
__device__ __forceinline__ bool in_smem(const void *p, uint32_t len, int32_t *status)
{
    if constexpr (!kChecked) return true;
    extern __shared__ unsigned char gdn_dynamic_smem[];
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    const int64_t off = (int64_t)__cvta_generic_to_shared(p) -
                        (int64_t)__cvta_generic_to_shared(gdn_dynamic_smem);
    if (off >= 0 && off + len <= dyn) return true;
    if (status) atomicOr(status, GDN_DEV_BOUNDS);
    return false;
}

// checked builds: the caller asked for the timeout path to be exercised (GDN_DEV_TEST_STALL)
__device__ __forceinline__ bool test_stall_requested(const int32_t *status)
{
    if constexpr (!kChecked) return false;
    return status && (*reinterpret_cast<const volatile int32_t *>(status) & GDN_DEV_TEST_STALL);
}

}  // namespace gdn

// Launchers implemented by the kernel translation units.
struct GdnPrefillArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    const int32_t *cu_seqlens;
    const float *initial_state;
    float *final_state;
    void *out;
    int32_t B;
    int64_t N;
    int32_t Hq, Hv, Dk, Dv;
    gdn_dtype dtype;
    float scale;
    int32_t qk_l2norm;
    int32_t *dev_status;
    // update_rule of the op: which of the decay and the delta retrieval survive; a rule
    // without decay has g == NULL (g = 0), one without retrieval has beta == NULL (beta = 1)
    int32_t has_decay, has_retrieval;
    const float *a_log, *dt_bias;   // non-NULL: qwen gate on g
    int32_t beta_sigmoid;
    int32_t g_per_key;              // g is [N, Hv, Dk]: one decay per key dimension
    // caller-owned device workspace for the sequence-parallel split (NULL: no split)
    void *workspace;
    uint64_t workspace_bytes;
};

struct GdnDecodeArgs {
    const void *q, *k, *v;
    float *pool;
    int32_t pool_size;
    int64_t slot_stride, head_stride;
    const void *read_idx, *write_idx;   // int32, or int64 when idx64
    const int32_t *scatter_idx;
    int32_t idx64;
    const float *A_log;
    const void *a;
    const float *dt_bias;
    const void *b;
    float scale;
    void *out;
    int32_t B, T, nh, H, HV, Dk, Dv;
    int32_t disable_state_update;
    int32_t use_qk_l2norm;
    int32_t *dev_status;
};

struct GdnConv1dArgs {
    const void *x;            // [N, conv_dim] dtype
    const void *weight;       // [conv_dim, K] dtype
    void *conv_state;         // [max_slots, conv_dim, K-1] dtype, in place (NULL when K == 1)
    const uint32_t *slot_idx; // [B]
    const uint32_t *offsets;  // [B+1]
    void *out;                // [N, conv_dim] dtype
    int32_t B, conv_dim, K, max_slots;
    int64_t N;
    int32_t dtype, write_state;
    int32_t *dev_status;
};

// Host-side setup done once per device (kernel attribute opt-ins): run() calls f() unless it
// already succeeded on the current device.  Threads that race may both call f, which must
// therefore be idempotent; devices numbered 32 and up call it every time.
struct DeviceOnce {
    std::atomic<uint32_t> done{0};
    template <class F>
    cudaError_t run(F &&f)
    {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const uint32_t bit = dev < 32 ? (1u << dev) : 0u;
        if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
        e = f();
        if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
        return e;
    }
};

cudaError_t launch_decode(const GdnDecodeArgs &a, cudaStream_t stream);
cudaError_t launch_conv1d(const GdnConv1dArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_sequential(const GdnPrefillArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_chunked(const GdnPrefillArgs &a, cudaStream_t stream);
bool prefill_chunked_supported(const GdnPrefillArgs &a);
// bytes of workspace with which gdn_prefill may split long requests (0: never splits)
uint64_t prefill_split_workspace_bytes(const GdnPrefillArgs &a);
cudaError_t launch_seq_compose(const GdnPrefillArgs &a, void *workspace, int G, cudaStream_t stream);
// the chunked tensor-core kernel for the per-key-dimension decay (prefill_kd.cu)
bool prefill_kd_supported(const GdnPrefillArgs &a);
cudaError_t launch_prefill_kd(const GdnPrefillArgs &a, cudaStream_t stream);
// records a CUDA failure for gdn_last_error() and returns GDN_ERR_CUDA
gdn_status gdn_report_cuda_failure(cudaError_t e, const char *where);
