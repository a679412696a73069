// gdn_api.cu -- the C ABI of libgdn: host-side validation and kernel dispatch.
//
// Nothing here reads tensor contents or synchronises: every check uses only
// the scalars and pointer values the caller passes, then one kernel is
// launched on the caller's stream.
#include <stdio.h>
#include <string.h>

#include "common.cuh"

namespace {

thread_local char g_last_error[256] = "";

gdn_status cuda_fail(cudaError_t e, const char *where)
{
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
             (int)e);
    return GDN_ERR_CUDA;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

// [p, p + bytes) and [q, q + qbytes) intersect (both non-empty)
bool overlaps(const void *p, size_t bytes, const void *q, size_t qbytes)
{
    if (!p || !q || bytes == 0 || qbytes == 0) return false;
    uintptr_t a0 = (uintptr_t)p, a1 = a0 + bytes;
    uintptr_t b0 = (uintptr_t)q, b1 = b0 + qbytes;
    return a0 < b1 && b0 < a1;
}

}  // namespace

gdn_status gdn_report_cuda_failure(cudaError_t e, const char *where) { return cuda_fail(e, where); }

extern "C" {

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

const char *gdn_last_error(void) { return g_last_error; }

const char *gdn_status_string(int32_t s)
{
    switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_NULL: return "GDN_ERR_NULL";
    case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE";
    case GDN_ERR_DTYPE: return "GDN_ERR_DTYPE";
    case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN";
    case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    default: return "GDN_ERR_UNKNOWN";
    }
}

}  // extern "C"

namespace {

// the chunked tensor-core kernel takes the call: its own size/dtype rule, and a scalar decay
// (the per-key-dimension spelling has a tensor-core kernel of its own, prefill_kd.cu)
bool chunked_path(const GdnPrefillArgs &a)
{
    return !a.g_per_key && prefill_chunked_supported(a);
}

}  // namespace

extern "C" {

int32_t gdn_prefill_uses_chunked(gdn_dtype dtype, int32_t Hv, int32_t Dk, int32_t Dv,
                                 uint32_t flags)
{
    if (flags & GDN_PREFILL_SEQUENTIAL) return 0;
    GdnPrefillArgs a;
    memset(&a, 0, sizeof(a));
    a.dtype = dtype; a.Dk = Dk; a.Dv = Dv; a.Hq = 1; a.Hv = Hv;
    a.g_per_key = (flags & GDN_DECAY_PER_KEY) ? 1 : 0;
    a.has_decay = 1;   // the per-key spelling always comes with a decay input
    return (chunked_path(a) || prefill_kd_supported(a)) ? 1 : 0;
}

}  // extern "C"

namespace {

// scalar part of the prefill arguments (enough for host-only queries)
GdnPrefillArgs prefill_shape(int32_t B, int64_t N, int32_t Hq, int32_t Hv, int32_t Dk, int32_t Dv,
                             gdn_dtype dtype, uint32_t flags)
{
    GdnPrefillArgs a;
    memset(&a, 0, sizeof(a));
    const uint32_t rule = flags & GDN_RULE_MASK;
    a.B = B; a.N = N; a.Hq = Hq; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.dtype = dtype;
    a.has_decay = rule == 0 || rule == GDN_RULE_GATED;
    a.has_retrieval = rule == 0 || rule == GDN_RULE_DELTA;
    a.beta_sigmoid = (flags & GDN_BETA_SIGMOID) ? 1 : 0;
    a.g_per_key = (flags & GDN_DECAY_PER_KEY) ? 1 : 0;
    return a;
}

gdn_status prefill_impl(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, const float *a_log, const float *dt_bias,
                        const int32_t *cu_seqlens, const float *initial_state,
                        float *final_state, void *out, int32_t B, int64_t N, int32_t Hq,
                        int32_t Hv, int32_t Dk, int32_t Dv, gdn_dtype dtype, float scale,
                        int32_t qk_l2norm, uint32_t flags, void *workspace,
                        uint64_t workspace_bytes, int32_t *dev_status, void *stream)
{
    if (dtype != GDN_F32 && dtype != GDN_BF16 && dtype != GDN_F16) return GDN_ERR_DTYPE;
    if (B < 0 || N < 0 || Hq < 1 || Hv < 1 || Dk < 1 || Dv < 1) return GDN_ERR_SHAPE;
    if (Hv % Hq != 0) return GDN_ERR_SHAPE;
    if (Dk > 256 || Dv > 256) return GDN_ERR_UNSUPPORTED;
    const uint32_t known = GDN_PREFILL_SEQUENTIAL | GDN_RULE_MASK | GDN_GATE_QWEN |
                           GDN_BETA_SIGMOID | GDN_DECAY_PER_KEY;
    if (flags & ~known) return GDN_ERR_UNSUPPORTED;
    // update_rule: decay input exactly for gated / gated_delta, beta exactly for delta /
    // gated_delta, qwen parameters exactly with the qwen gate (which needs a decay)
    const uint32_t rule = flags & GDN_RULE_MASK;
    const bool has_decay = rule == 0 || rule == GDN_RULE_GATED;
    const bool has_retrieval = rule == 0 || rule == GDN_RULE_DELTA;
    const bool qwen = (flags & GDN_GATE_QWEN) != 0;
    const bool per_key = (flags & GDN_DECAY_PER_KEY) != 0;
    if ((qwen || per_key) && !has_decay) return GDN_ERR_SHAPE;
    if ((flags & GDN_BETA_SIGMOID) && !has_retrieval) return GDN_ERR_SHAPE;
    if (B == 0) return N == 0 ? GDN_OK : GDN_ERR_SHAPE;
    if (!cu_seqlens && N % B != 0) return GDN_ERR_SHAPE;
    if (N > ((int64_t)1 << 31) - 1) return GDN_ERR_UNSUPPORTED;
    if (!final_state) return GDN_ERR_NULL;
    if (N > 0 && (!q || !k || !v || !out)) return GDN_ERR_NULL;
    if (N > 0 && (has_decay != (g != nullptr) || has_retrieval != (beta != nullptr)))
        return GDN_ERR_NULL;
    if (qwen != (a_log != nullptr) || qwen != (dt_bias != nullptr)) return GDN_ERR_NULL;

    const size_t esz = dtype == GDN_F32 ? 4 : 2;
    const size_t qk_bytes = (size_t)N * Hq * Dk * esz;
    const size_t v_bytes = (size_t)N * Hv * Dv * esz;
    const size_t gb_bytes = (size_t)N * Hv * 4;
    const size_t g_bytes = per_key ? gb_bytes * Dk : gb_bytes;
    const size_t st_bytes = (size_t)B * Hv * Dv * Dk * 4;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(initial_state, 16) || !aligned(final_state, 16) || !aligned(g, 16) ||
        !aligned(beta, 16) || !aligned(cu_seqlens, 4) || !aligned(a_log, 4) || !aligned(dt_bias, 4))
        return GDN_ERR_ALIGN;
    if (overlaps(initial_state, st_bytes, final_state, st_bytes)) return GDN_ERR_ALIAS;
    if (overlaps(out, v_bytes, q, qk_bytes) || overlaps(out, v_bytes, k, qk_bytes) ||
        overlaps(out, v_bytes, v, v_bytes) || overlaps(out, v_bytes, g, g_bytes) ||
        overlaps(out, v_bytes, beta, gb_bytes) || overlaps(out, v_bytes, final_state, st_bytes) ||
        overlaps(out, v_bytes, initial_state, st_bytes) ||
        overlaps(final_state, st_bytes, q, qk_bytes) ||
        overlaps(final_state, st_bytes, k, qk_bytes) ||
        overlaps(final_state, st_bytes, v, v_bytes) ||
        overlaps(final_state, st_bytes, g, g_bytes) ||
        overlaps(final_state, st_bytes, beta, gb_bytes) ||
        overlaps(final_state, st_bytes, cu_seqlens, (size_t)(B + 1) * 4) ||
        overlaps(out, v_bytes, a_log, (size_t)Hv * 4) || overlaps(out, v_bytes, dt_bias, (size_t)Hv * 4) ||
        overlaps(final_state, st_bytes, a_log, (size_t)Hv * 4) ||
        overlaps(final_state, st_bytes, dt_bias, (size_t)Hv * 4))
        return GDN_ERR_ALIAS;

    GdnPrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.cu_seqlens = cu_seqlens;
    a.initial_state = initial_state; a.final_state = final_state; a.out = out;
    a.B = B; a.N = N; a.Hq = Hq; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.dtype = dtype;
    a.scale = scale; a.qk_l2norm = qk_l2norm ? 1 : 0; a.dev_status = dev_status;
    a.has_decay = has_decay; a.has_retrieval = has_retrieval;
    a.a_log = a_log; a.dt_bias = dt_bias; a.beta_sigmoid = (flags & GDN_BETA_SIGMOID) ? 1 : 0;
    a.g_per_key = per_key ? 1 : 0;
    a.workspace = nullptr;
    a.workspace_bytes = 0;

    // workspace of the sequence-parallel split: used only when the call can split and the
    // chunked kernel runs; then it must be large enough, aligned, and overlap nothing
    if (workspace && !(flags & GDN_PREFILL_SEQUENTIAL) && chunked_path(a)) {
        const uint64_t need = prefill_split_workspace_bytes(a);
        if (need > 0) {
            if (workspace_bytes < need) return GDN_ERR_SHAPE;
            if (!aligned(workspace, 16)) return GDN_ERR_ALIGN;
            const size_t wb = (size_t)need;
            if (overlaps(workspace, wb, q, qk_bytes) || overlaps(workspace, wb, k, qk_bytes) ||
                overlaps(workspace, wb, v, v_bytes) || overlaps(workspace, wb, g, g_bytes) ||
                overlaps(workspace, wb, beta, gb_bytes) || overlaps(workspace, wb, out, v_bytes) ||
                overlaps(workspace, wb, initial_state, st_bytes) ||
                overlaps(workspace, wb, final_state, st_bytes) ||
                overlaps(workspace, wb, cu_seqlens, (size_t)(B + 1) * 4))
                return GDN_ERR_ALIAS;
            a.workspace = workspace;
            a.workspace_bytes = workspace_bytes;
        }
    }

    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (!(flags & GDN_PREFILL_SEQUENTIAL) && chunked_path(a))
        e = launch_prefill_chunked(a, s);
    else if (!(flags & GDN_PREFILL_SEQUENTIAL) && prefill_kd_supported(a))
        e = launch_prefill_kd(a, s);
    else
        e = launch_prefill_sequential(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_prefill launch");
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_prefill(const void *q, const void *k, const void *v, const float *g,
                       const float *beta, const float *a_log, const float *dt_bias,
                       const int32_t *cu_seqlens, const float *initial_state,
                       float *final_state, void *out, int32_t B, int64_t N, int32_t Hq,
                       int32_t Hv, int32_t Dk, int32_t Dv, gdn_dtype dtype, float scale,
                       int32_t qk_l2norm, uint32_t flags, int32_t *dev_status, void *stream)
{
    return prefill_impl(q, k, v, g, beta, a_log, dt_bias, cu_seqlens, initial_state, final_state,
                        out, B, N, Hq, Hv, Dk, Dv, dtype, scale, qk_l2norm, flags, nullptr, 0,
                        dev_status, stream);
}

gdn_status gdn_prefill_ws(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, const float *a_log, const float *dt_bias,
                          const int32_t *cu_seqlens, const float *initial_state,
                          float *final_state, void *out, int32_t B, int64_t N, int32_t Hq,
                          int32_t Hv, int32_t Dk, int32_t Dv, gdn_dtype dtype, float scale,
                          int32_t qk_l2norm, uint32_t flags, void *workspace,
                          uint64_t workspace_bytes, int32_t *dev_status, void *stream)
{
    return prefill_impl(q, k, v, g, beta, a_log, dt_bias, cu_seqlens, initial_state, final_state,
                        out, B, N, Hq, Hv, Dk, Dv, dtype, scale, qk_l2norm, flags, workspace,
                        workspace_bytes, dev_status, stream);
}

uint64_t gdn_prefill_workspace_size(int32_t B, int64_t N, int32_t Hq, int32_t Hv, int32_t Dk,
                                    int32_t Dv, gdn_dtype dtype, uint32_t flags)
{
    if ((flags & GDN_PREFILL_SEQUENTIAL) || B < 1 || Hq < 1 || Hv < 1 || Hv % Hq != 0 || N < 0)
        return 0;
    const GdnPrefillArgs a = prefill_shape(B, N, Hq, Hv, Dk, Dv, dtype, flags);
    if ((flags & GDN_GATE_QWEN) || !chunked_path(a)) return 0;
    return prefill_split_workspace_bytes(a);
}

gdn_status gdn_decode(const void *q, const void *k, const void *v, float *state_pool,
                      int32_t pool_size, int64_t slot_stride, int64_t head_stride,
                      const void *read_idx, const void *write_idx,
                      const int32_t *scatter_idx, const float *A_log, const void *a,
                      const float *dt_bias, const void *b, float scale, void *out, int32_t B,
                      int32_t T, int32_t nh, int32_t H, int32_t HV, int32_t Dk, int32_t Dv,
                      uint32_t flags, int32_t *dev_status, void *stream)
{
    const uint32_t known = GDN_DISABLE_STATE_UPDATE | GDN_DECODE_QK_L2NORM | GDN_DECODE_IDX64;
    if (flags & ~known) return GDN_ERR_UNSUPPORTED;
    if (B < 0 || T < 1 || nh < 1 || H < 1 || HV < 1 || Dk < 1 || Dv < 1 || pool_size < 1)
        return GDN_ERR_SHAPE;
    if (H != HV) return GDN_ERR_SHAPE;
    if (T > 16 || nh > 4 || Dk != 128 || (Dv != 64 && Dv != 128)) return GDN_ERR_UNSUPPORTED;
    if (scatter_idx && (flags & GDN_DISABLE_STATE_UPDATE)) return GDN_ERR_SHAPE;
    if (head_stride < (int64_t)Dv * Dk || slot_stride < (int64_t)HV * head_stride)
        return GDN_ERR_SHAPE;
    if (B == 0) return GDN_OK;
    if (!q || !k || !v || !state_pool || !read_idx || !A_log || !a || !dt_bias || !b || !out)
        return GDN_ERR_NULL;
    if (!aligned(state_pool, 16) || (slot_stride & 3) || (head_stride & 3))
        return GDN_ERR_ALIGN;
    const uintptr_t idx_align = (flags & GDN_DECODE_IDX64) ? 8 : 4;
    if (!aligned(q, 8) || !aligned(k, 8) || !aligned(v, 8) || !aligned(out, 8) ||
        !aligned(a, 2) || !aligned(b, 2) || !aligned(A_log, 4) || !aligned(dt_bias, 4) ||
        !aligned(read_idx, idx_align) || !aligned(write_idx, idx_align) || !aligned(scatter_idx, 4))
        return GDN_ERR_ALIGN;
    const size_t pool_bytes =
        ((size_t)(pool_size - 1) * slot_stride + (size_t)(HV - 1) * head_stride +
         (size_t)Dv * Dk) * 4;
    const size_t out_bytes = (size_t)B * T * HV * Dv * 2;
    if (overlaps(out, out_bytes, state_pool, pool_bytes) ||
        overlaps(out, out_bytes, q, (size_t)B * T * H * Dk * 2) ||
        overlaps(out, out_bytes, k, (size_t)B * T * nh * H * Dk * 2) ||
        overlaps(out, out_bytes, v, (size_t)B * T * nh * HV * Dv * 2) ||
        overlaps(state_pool, pool_bytes, q, (size_t)B * T * H * Dk * 2) ||
        overlaps(state_pool, pool_bytes, k, (size_t)B * T * nh * H * Dk * 2) ||
        overlaps(state_pool, pool_bytes, v, (size_t)B * T * nh * HV * Dv * 2))
        return GDN_ERR_ALIAS;

    GdnDecodeArgs d;
    d.q = q; d.k = k; d.v = v; d.pool = state_pool; d.pool_size = pool_size;
    d.slot_stride = slot_stride; d.head_stride = head_stride;
    d.read_idx = read_idx; d.write_idx = write_idx; d.scatter_idx = scatter_idx;
    d.A_log = A_log; d.a = a; d.dt_bias = dt_bias; d.b = b; d.scale = scale; d.out = out;
    d.B = B; d.T = T; d.nh = nh; d.H = H; d.HV = HV; d.Dk = Dk; d.Dv = Dv;
    d.disable_state_update = (flags & GDN_DISABLE_STATE_UPDATE) ? 1 : 0;
    d.use_qk_l2norm = (flags & GDN_DECODE_QK_L2NORM) ? 1 : 0;
    d.idx64 = (flags & GDN_DECODE_IDX64) ? 1 : 0;
    d.dev_status = dev_status;
    cudaError_t e = launch_decode(d, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_decode launch");
    return GDN_OK;
}

gdn_status gdn_conv1d(const void *x, const void *weight, void *conv_state,
                      const uint32_t *slot_idx, const uint32_t *row_offsets, void *out,
                      int32_t B, int64_t N, int32_t conv_dim, int32_t kernel_size,
                      int32_t max_slots, gdn_dtype dtype, int32_t write_state,
                      int32_t *dev_status, void *stream)
{
    if (dtype != GDN_F32 && dtype != GDN_BF16 && dtype != GDN_F16) return GDN_ERR_DTYPE;
    if (B < 0 || N < 0 || conv_dim < 1 || kernel_size < 1 || max_slots < 1) return GDN_ERR_SHAPE;
    if (kernel_size > 8) return GDN_ERR_UNSUPPORTED;
    if (N > ((int64_t)1 << 31) - 1) return GDN_ERR_UNSUPPORTED;
    if (B == 0) return GDN_OK;
    if (!x || !weight || !out || !slot_idx || !row_offsets) return GDN_ERR_NULL;
    if (kernel_size > 1 && !conv_state) return GDN_ERR_NULL;
    const size_t esz = dtype == GDN_F32 ? 4 : 2;
    if (!aligned(x, esz) || !aligned(weight, esz) || !aligned(out, esz) ||
        !aligned(conv_state, esz) || !aligned(slot_idx, 4) || !aligned(row_offsets, 4))
        return GDN_ERR_ALIGN;
    const size_t x_bytes = (size_t)N * conv_dim * esz;
    const size_t w_bytes = (size_t)conv_dim * kernel_size * esz;
    const size_t st_bytes = (size_t)max_slots * conv_dim * (kernel_size - 1) * esz;
    const size_t si_bytes = (size_t)B * 4, ro_bytes = (size_t)(B + 1) * 4;
    if (overlaps(out, x_bytes, x, x_bytes) || overlaps(out, x_bytes, weight, w_bytes) ||
        overlaps(out, x_bytes, conv_state, st_bytes) || overlaps(out, x_bytes, slot_idx, si_bytes) ||
        overlaps(out, x_bytes, row_offsets, ro_bytes) ||
        overlaps(conv_state, st_bytes, x, x_bytes) || overlaps(conv_state, st_bytes, weight, w_bytes) ||
        overlaps(conv_state, st_bytes, slot_idx, si_bytes) ||
        overlaps(conv_state, st_bytes, row_offsets, ro_bytes))
        return GDN_ERR_ALIAS;

    GdnConv1dArgs c;
    c.x = x; c.weight = weight; c.conv_state = conv_state; c.slot_idx = slot_idx;
    c.offsets = row_offsets; c.out = out; c.B = B; c.conv_dim = conv_dim; c.K = kernel_size;
    c.max_slots = max_slots; c.N = N; c.dtype = dtype; c.write_state = write_state ? 1 : 0;
    c.dev_status = dev_status;
    cudaError_t e = launch_conv1d(c, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "gdn_conv1d launch");
    return GDN_OK;
}

}  // extern "C"
