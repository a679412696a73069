/*
 * gdn.h -- C ABI of libgdn: the Gated DeltaNet recurrence on NVIDIA B200
 * (sm_100a).
 *
 * Three entry points:
 *   gdn_prefill  chunked / sequential scan over ragged requests;
 *   gdn_decode   decode / MTP update of an fp32 slot-indexed state pool;
 *   gdn_conv1d   the causal depthwise conv1d that feeds q, k, v, with a
 *                slot-indexed pool of conv windows.
 *
 * Conventions shared by every call
 *   - Every tensor argument is a DEVICE pointer owned by the caller.  The
 *     library allocates no device memory and keeps no pointer after the call
 *     returns (device-side it only holds read-only constant tables).  Scratch
 *     memory, where a call can use some (gdn_prefill_ws), is passed in by the
 *     caller.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL means the
 *     legacy default stream).  The library never reads tensor contents on the
 *     host and never synchronises, so a call may be captured in a CUDA graph.
 *   - Inputs are never modified.  The only buffers written are `out`,
 *     `final_state` (prefill), `state_pool`, `out` (decode) and `out`,
 *     `conv_state` (conv1d), plus the optional `dev_status` word.
 *   - Errors the host can see (null pointers, shapes, alignment, aliasing,
 *     unsupported sizes) are returned as a gdn_status before anything is
 *     launched.  Errors only the device can see (a slot index >= pool_size)
 *     skip the affected unit and OR a GDN_DEV_* bit into *dev_status when
 *     `dev_status` is non-NULL.  No kernel traps or asserts.
 *   - Layouts are dense, row-major, with the strides implied by the shapes
 *     below (decode's pool alone takes explicit strides).
 */
#ifndef GDN_H
#define GDN_H

#include <stdint.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_NULL = 1,        /* a required pointer is NULL */
    GDN_ERR_SHAPE = 2,       /* inconsistent sizes (e.g. Hv % Hq != 0, H != HV) */
    GDN_ERR_DTYPE = 3,       /* unknown dtype code */
    GDN_ERR_ALIGN = 4,       /* a pointer or stride breaks the alignment rule */
    GDN_ERR_ALIAS = 5,       /* an output overlaps an input it must not overlap */
    GDN_ERR_UNSUPPORTED = 6, /* valid, but outside what the kernels implement */
    GDN_ERR_CUDA = 7         /* a CUDA runtime call failed; see gdn_last_error() */
} gdn_status;

typedef enum {
    GDN_F32 = 0,   /* float32 activations */
    GDN_BF16 = 1,  /* bfloat16 activations */
    GDN_F16 = 2    /* float16 activations (prefill, conv1d) */
} gdn_dtype;

/* flags */
enum {
    GDN_PREFILL_SEQUENTIAL = 1u << 0,   /* prefill: force the per-token kernel */
    GDN_DISABLE_STATE_UPDATE = 1u << 1, /* decode: leave the pool unchanged */
    GDN_DECODE_QK_L2NORM = 1u << 2,     /* decode: L2-normalise q and k in the kernel */
    GDN_DECODE_IDX64 = 1u << 7,         /* decode: read_idx and write_idx are int64 */
    /* prefill update_rule (two bits; 0 = gated_delta, both terms) */
    GDN_RULE_GATED = 1u << 3,           /* decay only: S_t = exp(g_t) S_{t-1} + k_t v_t^T */
    GDN_RULE_DELTA = 2u << 3,           /* retrieval only: g = 0 */
    GDN_RULE_LINEAR = 3u << 3,          /* neither: S_t = S_{t-1} + k_t v_t^T */
    GDN_RULE_MASK = 3u << 3,
    GDN_GATE_QWEN = 1u << 5,            /* prefill: g <- -exp(a_log[h]) softplus(g + dt_bias[h]) */
    GDN_BETA_SIGMOID = 1u << 6,         /* prefill: beta <- sigmoid(beta) */
    GDN_DECAY_PER_KEY = 1u << 8         /* prefill: g is [N, Hv, Dk], one decay per key dimension */
};

/* bits OR-ed into *dev_status by the kernels */
enum {
    GDN_DEV_BAD_SLOT = 1,  /* a slot index >= the pool size was skipped (decode, conv1d) */
    GDN_DEV_TIMEOUT = 2,   /* a kernel-internal wait exceeded its bound; outputs invalid */
    GDN_DEV_INTERNAL = 4,  /* a kernel's layout self-check failed; nothing was computed */
    /* Checked builds only (libgdn_checked.so, compiled with GDN_CHECKS): every global and
     * data-dependent shared-memory access is tested against its buffer first; one outside it
     * is skipped (a load reads zero) and this bit is set.  Ordinary builds never set it. */
    GDN_DEV_BOUNDS = 8,
    /* Checked builds only, set by the CALLER in *dev_status before a gdn_decode or a
     * chunked gdn_prefill call: the persistent decode kernel, or the chunked prefill
     * kernel's first q/k stage, posts 16 bytes more than its copies deliver (the per-key
     * decay kernel's first CTA waits for its first W/U~ MMA group on a barrier that nothing
     * arrives on), so the waits run out after their bound (about a second), GDN_DEV_TIMEOUT
     * is set and the kernel returns.  Exercises the timeout path without a fault; ignored by
     * ordinary builds. */
    GDN_DEV_TEST_STALL = 1 << 30
};

/*
 * gdn_prefill -- the log-space Gated DeltaNet recurrence over ragged requests.
 *
 * Defined by "com.microsoft.GatedDeltaNet" (ONNX Runtime contrib operator),
 * Description and Inputs/Outputs/Attributes tables: per value head h,
 *     S_t = exp(g_t) S_{t-1} + k_t (beta_t (v_t - exp(g_t) S_{t-1}^T k_t))^T
 *     o_t = scale * S_t^T q_t
 * with value head h reading query/key head floor(h * Hq / Hv).  This is the
 * gamma form of "Gated DeltaNet State Update" (statement) with gamma = exp(g).
 *
 * Arguments (N = total tokens, B = requests):
 *   q, k           [N, Hq, Dk]  `dtype`
 *   v              [N, Hv, Dv]  `dtype`
 *   g              [N, Hv] float32, log-space decay (g <= 0; -inf allowed);
 *                  required exactly for the rules with decay (gated_delta,
 *                  gated), NULL otherwise.  With GDN_GATE_QWEN it is the raw
 *                  `decay` input and the kernels use
 *                  -exp(a_log[h]) * softplus(g + dt_bias[h]) (softplus(x) = x
 *                  for x > 20), in float32.
 *                  With GDN_DECAY_PER_KEY, g is [N, Hv, Dk] float32, the op's
 *                  per-key-dimension spelling of `decay` (Inputs table): exp(g_t)
 *                  becomes diag(exp(g_t[0..Dk))) on the key axis of the state,
 *                  in both places of the recurrence,
 *                    S_t = D_t S_{t-1} + k_t (beta_t (v_t - (D_t S_{t-1})^T k_t))^T
 *                  (V-major: column i of S scales by exp(g_t[i])); the qwen gate
 *                  maps every element with its head's a_log and dt_bias.  The
 *                  page lists this spelling as not implemented by its own kernels.
 *                  bf16 heads of 8 to 128 run a chunked tensor-core kernel of
 *                  their own, which floors each per-dimension log-decay at -9
 *                  (a decay factor below e^-9 ~ 1.2e-4 counts as 1.2e-4) so that
 *                  its decay-scaled operands stay in range; fp16, fp32 and other
 *                  head sizes run the per-token kernel (no floor).
 *   beta           [N, Hv] float32, update rate; required exactly for the rules
 *                  with the delta retrieval (gated_delta, delta), NULL
 *                  otherwise (the write is then k_t v_t^T).  With
 *                  GDN_BETA_SIGMOID the kernels use sigmoid(beta).
 *   a_log, dt_bias [Hv] float32, required exactly with GDN_GATE_QWEN.
 *   cu_seqlens     [B+1] int32 exclusive prefix sums, or NULL for uniform
 *                  packing (then N % B == 0 and request b is tokens
 *                  [b*N/B, (b+1)*N/B)).  Entries are clamped on the device to
 *                  [0, N]; a request whose end <= start is empty.
 *   initial_state  [B, Hv, Dv, Dk] float32 (V-major), or NULL for zero
 *   final_state    [B, Hv, Dv, Dk] float32, written; must not overlap
 *                  initial_state.  An empty request copies its initial state.
 *   out            [N, Hv, Dv] `dtype`, written for every token that a
 *                  request covers (others keep the caller's values).
 *   scale          applied as given (the Python binding maps 0/None to
 *                  1/sqrt(Dk), the op's default).
 *   qk_l2norm      non-zero: q and k vectors are scaled by
 *                  (sum x^2 + 1e-12)^(-1/2) before use.
 *   flags          GDN_PREFILL_SEQUENTIAL, one GDN_RULE_* (update_rule of the
 *                  op's Attributes table: which of the decay and the delta
 *                  retrieval survive), GDN_GATE_QWEN, GDN_BETA_SIGMOID,
 *                  GDN_DECAY_PER_KEY (needs a rule with decay, else GDN_ERR_SHAPE).
 *   dev_status     optional device int32; GDN_DEV_TIMEOUT is OR-ed in if an
 *                  internal pipeline wait of the chunked kernel exceeds its
 *                  bound (the call's outputs are then invalid).
 * Requirements: 1 <= Dk, Dv <= 256; Hv % Hq == 0; q, k, v, g, beta, out,
 * initial_state and final_state 16-byte aligned (the chunked kernel reads g
 * and beta through tensor maps, whose base must be 16-byte aligned; the rule
 * holds for every call, so a view such as g[1:] of a 4-byte aligned buffer is
 * GDN_ERR_ALIGN, not a launch failure); out must not overlap any input.
 * bf16 or fp16 with Dk, Dv <= 128 runs the chunked tensor-core kernel (unless
 * GDN_PREFILL_SEQUENTIAL; its operand tiles take the activations' type, fp32
 * accumulation and state; rows that a tensor map cannot describe -- Dk or Dv
 * not a multiple of 8, or Hv % 4 != 0 -- are copied into its zero-padded tiles
 * with plain loads); everything else (fp32, heads wider than 128) runs the
 * per-token kernel, which computes in fp32.  The chunked kernel floors each g at -30
 * (exp(-30) ~ 9e-14) so that in-chunk decay differences stay finite.
 * Overlapping request ranges are not supported (their outputs are undefined).
 */
GDN_API gdn_status gdn_prefill(const void *q, const void *k, const void *v,
                       const float *g, const float *beta,
                       const float *a_log, const float *dt_bias,
                       const int32_t *cu_seqlens,
                       const float *initial_state, float *final_state,
                       void *out,
                       int32_t B, int64_t N, int32_t Hq, int32_t Hv,
                       int32_t Dk, int32_t Dv, gdn_dtype dtype,
                       float scale, int32_t qk_l2norm, uint32_t flags,
                       int32_t *dev_status, void *stream);

/*
 * gdn_prefill_ws -- gdn_prefill with a caller-owned device workspace, which lets
 * the call cut long requests into segments that run in parallel.
 *
 * Defined by the same operation as gdn_prefill ("com.microsoft.GatedDeltaNet",
 * Description); the op's Attributes table states that how the sequence is cut
 * into chunks does not change the result.  The recurrence is affine in the
 * state: over a run of tokens S_end = A S_start + B.  When a call holds too few
 * (request, value head) units to fill the GPU, a long request is cut into three
 * segments of whole 64-token chunks: segment 0 runs from the true initial state;
 * segment 1 runs twice in parallel with it, from the identity with v = 0 (giving
 * A_1) and from zero (giving B_1); a small kernel composes the start state of
 * segment 2; then segments 1 and 2 run from their true start states.  Results
 * equal gdn_prefill's within the same tolerance (every product still goes
 * through bf16 operands with fp32 state).
 *
 * Arguments: those of gdn_prefill, plus
 *   workspace        device buffer of at least gdn_prefill_workspace_size(...)
 *                    bytes, 16-byte aligned, overlapping no other argument; it
 *                    holds per (request, value head) the start states of
 *                    segments 1 and 2 and segment 1's A and B (fp32).  Owned
 *                    by the caller, written and read by the call on `stream`
 *                    (calls sharing one workspace must be ordered).  NULL: no
 *                    split (exactly gdn_prefill).
 *   workspace_bytes  its size.
 * Whether a request is split is decided on the device from cu_seqlens (the host
 * reads no tensor): a request of fewer than 24 chunks never is, nor any request
 * of a call whose split would not shorten its longest chain.  The split applies
 * to the default rule (gated_delta, no gate or beta activation), bf16,
 * Dk = Dv = 128, at most 8 requests and at most one (request, head) unit per SM;
 * any other call ignores the workspace.  Errors: GDN_ERR_SHAPE if a non-NULL
 * workspace is smaller than the size the call needs, GDN_ERR_ALIGN, GDN_ERR_ALIAS;
 * otherwise as gdn_prefill.
 */
GDN_API gdn_status gdn_prefill_ws(const void *q, const void *k, const void *v,
                          const float *g, const float *beta,
                          const float *a_log, const float *dt_bias,
                          const int32_t *cu_seqlens,
                          const float *initial_state, float *final_state,
                          void *out,
                          int32_t B, int64_t N, int32_t Hq, int32_t Hv,
                          int32_t Dk, int32_t Dv, gdn_dtype dtype,
                          float scale, int32_t qk_l2norm, uint32_t flags,
                          void *workspace, uint64_t workspace_bytes,
                          int32_t *dev_status, void *stream);

/* Workspace bytes gdn_prefill_ws needs for these sizes (0: the call never splits,
 * pass NULL).  Host-only: reads the current device's SM count, launches nothing. */
GDN_API uint64_t gdn_prefill_workspace_size(int32_t B, int64_t N, int32_t Hq, int32_t Hv,
                                            int32_t Dk, int32_t Dv, gdn_dtype dtype,
                                            uint32_t flags);

/*
 * gdn_prefill_noalloc -- gdn_prefill_ws whose workspace is a fixed array inside the
 * library, so the call allocates nothing and needs no workspace from the caller.
 *
 * No passage of the pages corresponds to this entry point: it serves callers that cannot
 * allocate device memory for a call -- a host runtime that owns all device memory
 * through its own pool, a C caller without a memory manager, a serving path that must
 * never allocate -- and still want the sequence-parallel split of gdn_prefill_ws.
 *
 * Arguments and results: exactly those of gdn_prefill (inputs and outputs are the
 * caller's).  The workspace is a static device array of 8 MiB (8388608 bytes) that every
 * GPU loading the library holds until the process exits; 8 MiB covers 32 (request, value
 * head) units of 128 x 128 heads, e.g. one request with 32 value heads.  A call whose split
 * would need more (gdn_prefill_workspace_size > 8 MiB) returns GDN_ERR_UNSUPPORTED before
 * launching anything; a call that cannot split runs as gdn_prefill.
 * The array's device address is looked up (cudaGetSymbolAddress) on the first call made on
 * each device, with that device current; make that first call before any stream capture.
 * All calls on a device share the one array: calls that overlap on the GPU (on different
 * streams, without ordering) race on it and must not be issued.  Nothing in the array needs
 * to start at zero: every byte a call reads was written earlier by the same call.
 */
GDN_API gdn_status gdn_prefill_noalloc(const void *q, const void *k, const void *v,
                               const float *g, const float *beta,
                               const float *a_log, const float *dt_bias,
                               const int32_t *cu_seqlens,
                               const float *initial_state, float *final_state,
                               void *out,
                               int32_t B, int64_t N, int32_t Hq, int32_t Hv,
                               int32_t Dk, int32_t Dv, gdn_dtype dtype,
                               float scale, int32_t qk_l2norm, uint32_t flags,
                               int32_t *dev_status, void *stream);

/*
 * gdn_decode -- Gated DeltaProduct decode / MTP over an fp32 state pool.
 *
 * Defined by "flashinfer.cake_gdp.cake_gated_delta_product_mtp" (description,
 * Parameters): for every batch row b and head h with r = read_idx[b] >= 0,
 * S = pool[r, h]; for each token t:
 *     S <- alpha_t S,  alpha_t = exp(-exp(A_log[h]) softplus(a[b,t,h] + dt_bias[h]))
 *                      (softplus(x) = x for x > 20)
 *     for j < nh:  S <- S + k_tj (beta_tj (v_tj - S^T k_tj))^T,  beta_tj = sigmoid(b[b,t,j,h])
 *     out[b,t,h] = scale * S^T q_t
 *     if scatter_idx: pool[scatter_idx[b,t], h] <- S   (negative entry: skipped)
 * and after the last token, unless scatter_idx or GDN_DISABLE_STATE_UPDATE:
 *     pool[w, h] <- S with w = write_idx ? write_idx[b] : r (negative: skipped).
 * With GDN_DECODE_QK_L2NORM, q_t and every k_tj are first scaled by
 * (sum x^2 + 1e-6)^(-1/2).  A row with read_idx < 0 is padding: nothing is
 * read, computed or stored and its `out` rows keep the caller's values.
 *
 * Arguments:
 *   q      [B, T, H, Dk] bf16            k  [B, T, nh, H, Dk] bf16
 *   v      [B, T, nh, HV, Dv] bf16       out [B, T, HV, Dv] bf16 (written)
 *   state_pool  fp32, slot s head h row j at
 *               state_pool + s*slot_stride + h*head_stride + j*Dk (rows dense);
 *               read and written in place.  pool_size slots.
 *   read_idx [B], write_idx [B] or NULL (= read_idx): int32, or int64 with
 *          GDN_DECODE_IDX64 (the page allows either); scatter_idx [B, T] or NULL: int32
 *   A_log, dt_bias [HV] float32;  a [B, T, HV] bf16;  b [B, T, nh, HV] bf16
 *   scale  applied as given (the Python binding maps None to 1/sqrt(Dk))
 *   flags  GDN_DISABLE_STATE_UPDATE | GDN_DECODE_QK_L2NORM | GDN_DECODE_IDX64, or 0
 *   dev_status  optional device int32; GDN_DEV_BAD_SLOT is OR-ed in when a
 *               slot index >= pool_size is met (that read/write is skipped);
 *               GDN_DEV_TIMEOUT if a copy into shared memory did not complete
 *               within its bound (the CTA stops; outputs invalid).
 * Requirements: H == HV; Dk == 128; Dv in {64, 128}; 1 <= T <= 16;
 * 1 <= nh <= 4; scatter_idx requires the update enabled; state_pool 16-byte
 * aligned with slot_stride and head_stride multiples of 4 elements,
 * head_stride >= Dv*Dk, slot_stride >= HV*head_stride; q, k, v, out 8-byte
 * aligned; index arrays aligned to their element size.  A slot index beyond
 * int32 range is >= pool_size (skipped and flagged).  Rows must not write a
 * slot that another row reads (a row's own
 * write slot may equal its read slot).
 */
GDN_API gdn_status gdn_decode(const void *q, const void *k, const void *v,
                      float *state_pool, int32_t pool_size,
                      int64_t slot_stride, int64_t head_stride,
                      const void *read_idx, const void *write_idx,
                      const int32_t *scatter_idx,
                      const float *A_log, const void *a, const float *dt_bias,
                      const void *b, float scale, void *out,
                      int32_t B, int32_t T, int32_t nh, int32_t H, int32_t HV,
                      int32_t Dk, int32_t Dv, uint32_t flags,
                      int32_t *dev_status, void *stream);

/*
 * gdn_conv1d -- causal depthwise conv1d over ragged requests with a
 * slot-indexed pool of conv windows, updated in place.
 *
 * Defined by "max.nn.legacy.state_space.gated_delta_conv1d_fwd" (description,
 * Parameters, example).  For request b with tokens [s, e) =
 * [row_offsets[b], row_offsets[b+1]) (clamped to [0, N]; e <= s is empty) and
 * slot r = slot_idx[b], channel c sees the sequence
 *     xe = (conv_state[r, c, 0 .. K-2], x[s, c], ..., x[e-1, c])
 * (the window is stored oldest first) and
 *     out[s + i, c] = sum_{j=0}^{K-1} weight[c, j] * xe[i + j]
 * accumulated in float32 and rounded to `dtype`; no activation follows.
 * With write_state != 0, conv_state[r] receives the last K-1 entries of xe
 * (a request shorter than K-1 keeps the newest old entries ahead of its
 * inputs); with write_state == 0 the pool is only read.  Slots no request
 * names keep their values; so does an empty request's slot.
 *
 * Arguments (N = total tokens, B = requests, K = kernel_size):
 *   x            [N, conv_dim] `dtype` (the projected q/k/v rows)
 *   weight       [conv_dim, K] `dtype`
 *   conv_state   [max_slots, conv_dim, K-1] `dtype`, read and written in
 *                place; may be NULL only when K == 1
 *   slot_idx     [B] uint32;  row_offsets [B+1] uint32
 *   out          [N, conv_dim] `dtype`, written for every token a request
 *                with a valid slot covers (others keep the caller's values)
 *   dev_status   optional device int32; GDN_DEV_BAD_SLOT is OR-ed in when a
 *                slot >= max_slots is met (that request is skipped: no
 *                output rows, no pool access).
 * Requirements: 1 <= K <= 8; conv_dim >= 1; dtype F32, BF16 or F16; all
 * tensors naturally aligned for `dtype` (16-byte alignment of every tensor
 * and conv_dim * element size a multiple of 16 select the vector path);
 * out and conv_state overlap no input and not each other.  Requests must
 * name distinct slots when write_state != 0 (a shared slot is a race).
 */
GDN_API gdn_status gdn_conv1d(const void *x, const void *weight, void *conv_state,
                              const uint32_t *slot_idx, const uint32_t *row_offsets,
                              void *out, int32_t B, int64_t N, int32_t conv_dim,
                              int32_t kernel_size, int32_t max_slots, gdn_dtype dtype,
                              int32_t write_state, int32_t *dev_status, void *stream);

/* 1 when gdn_prefill with these arguments runs a chunked tensor-core kernel,
 * 0 when it runs the per-token kernel (host-only query, no launch).  The chunked
 * kernel takes bf16 or fp16 with Dk, Dv up to 128 (smaller heads run as
 * zero-padded 128-wide tiles) and any Hv; with GDN_DECAY_PER_KEY, bf16 with Dk,
 * Dv from 8 to 128. */
GDN_API int32_t gdn_prefill_uses_chunked(gdn_dtype dtype, int32_t Hv, int32_t Dk, int32_t Dv,
                                         uint32_t flags);

/* Name of a gdn_status code (static string). */
GDN_API const char *gdn_status_string(int32_t status);

/* Text of the last GDN_ERR_CUDA on the calling thread (static per thread). */
GDN_API const char *gdn_last_error(void);

/* ABI version of this header: increments on any incompatible change. */
GDN_API int32_t gdn_abi_version(void);

#define GDN_ABI_VERSION 2

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
