// prefill_seq.cu -- per-token Gated DeltaNet prefill for any head size <= 256.
//
// Operation ("com.microsoft.GatedDeltaNet", Description; "Gated DeltaNet
// State Update", statement): per request and value head, for every token
//   p   = S_{t-1}^T k_t
//   S_t = exp(g_t) S_{t-1} + k_t (beta_t (v_t - exp(g_t) p))^T
//   o_t = scale * S_t^T q_t
// The state stays in fp32 registers for the whole request.
//
// The op's update_rule keeps or drops the decay (g = 0) and the delta
// retrieval (the -exp(g_t) p term, with beta = 1 when the rule has no beta);
// its qwen gate maps g to -exp(a_log[h]) softplus(g + dt_bias[h]) and its
// sigmoid activation maps beta to sigmoid(beta), both in fp32.
//
// With the per-key-dimension decay (the op's Inputs table, `decay` of shape
// (..., num_heads_v, head_size_qk)) exp(g_t) becomes diag(exp(g_t)) on the key
// axis: each lane scales its own key columns of S by their decay before the
// retrieval and the write, S_t = D_t S_{t-1} + k_t (beta_t (v_t - (D_t S_{t-1})^T k_t))^T.
//
// This is the general path: fp32, bf16 or fp16 activations, any Dk, Dv in
// [1, 256], any Hq | Hv.  It is also the sequential counterpart the chunked
// tensor-core kernel is checked against.  Layout: a 1-D grid of (request, value
// head, tile of 32 V-rows) blocks, the tile index fastest and the requests
// longest first (for up to 256 requests), so that the longest chains start in
// the first wave of blocks; a warp owns 4 V-rows of S (V-major, one row = Dk
// floats), lane l owns elements l + 32 j of each row; row dot products are warp
// reductions.
#include <cuda_fp16.h>

#include "common.cuh"

namespace gdn {

constexpr int kSeqWarps = 8;
constexpr int kSeqRows = 4;  // V-rows per warp

template <typename Tin>
__device__ __forceinline__ float load_act(const Tin *p);
template <>
__device__ __forceinline__ float load_act<float>(const float *p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_act<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(p[0]);
}

template <>
__device__ __forceinline__ float load_act<__half>(const __half *p)
{
    return __half2float(p[0]);
}

template <typename Tout>
__device__ __forceinline__ void store_act(Tout *p, float x);
template <>
__device__ __forceinline__ void store_act<float>(float *p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_act<__nv_bfloat16>(__nv_bfloat16 *p, float x)
{
    *p = __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ void store_act<__half>(__half *p, float x)
{
    *p = __float2half_rn(x);
}

template <typename Tin, int EPL, bool PER_KEY>
__global__ void __launch_bounds__(kSeqWarps * 32)
prefill_seq_kernel(const GdnPrefillArgs p)
{
    constexpr int R = kSeqRows;
    constexpr int NT = kSeqWarps * 32;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int Hv = p.Hv, Hq = p.Hq, Dk = p.Dk, Dv = p.Dv;
    const int tiles = (Dv + kSeqWarps * R - 1) / (kSeqWarps * R);
    const int unit = (int)(blockIdx.x / (unsigned)tiles);
    const int tile = (int)blockIdx.x - unit * tiles;
    int b = unit / Hv;
    const int h = unit - b * Hv;
    // request of rank b in decreasing length (ties by index)
    if (p.cu_seqlens && p.B > 1 && p.B <= NT) {
        __shared__ int lens[NT];
        __shared__ int pick;
        const int t = threadIdx.x;
        if (t < p.B) {
            const int64_t st = clamp_i64(p.cu_seqlens[t], 0, p.N);
            const int64_t en = clamp_i64(p.cu_seqlens[t + 1], 0, p.N);
            lens[t] = en > st ? (int)(en - st) : 0;
        }
        __syncthreads();
        if (t < p.B) {
            const int li = lens[t];
            int rank = 0;
            for (int j2 = 0; j2 < p.B; ++j2) rank += (lens[j2] > li) || (lens[j2] == li && j2 < t);
            if (rank == b) pick = t;
        }
        __syncthreads();
        b = pick;
    }
    const int qh = (int)(((int64_t)h * Hq) / Hv);
    const int row_base = tile * (kSeqWarps * R) + warp * R;
    if (row_base >= Dv) return;  // whole warp idle (uniform)

    int64_t start, end;
    if (p.cu_seqlens) {
        start = clamp_i64(p.cu_seqlens[b], 0, p.N);
        end = clamp_i64(p.cu_seqlens[b + 1], 0, p.N);
    } else {
        const int64_t S = p.N / p.B;
        start = (int64_t)b * S;
        end = start + S;
    }

    const Tin *qg = static_cast<const Tin *>(p.q);
    const Tin *kg = static_cast<const Tin *>(p.k);
    const Tin *vg = static_cast<const Tin *>(p.v);
    Tin *og = static_cast<Tin *>(p.out);

    float S[R][EPL];
    const int64_t state_off = ((int64_t)b * Hv + h) * Dv * (int64_t)Dk;
    // (checked builds) every access below lies in the tokens [start, end), query head qh and
    // this head's state slice: test those ranges once
    if constexpr (kChecked) {
        if (!in_range(start, end > start ? end - start : 0, p.N, p.dev_status) ||
            !in_range(qh, 1, Hq, p.dev_status) ||
            !in_range(state_off, (int64_t)Dv * Dk, (int64_t)p.B * Hv * Dv * Dk, p.dev_status))
            return;
    }
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            const int row = row_base + i;
            S[i][j] = (p.initial_state && e < Dk && row < Dv)
                          ? p.initial_state[state_off + (int64_t)row * Dk + e]
                          : 0.f;
        }

    // The raw inputs of token t + 1 (k, q, the decay, beta and this warp's R values) are
    // loaded while token t is computed, so the loop waits on no global load; the R rows'
    // warp reductions run interleaved (same butterfly order as warp_sum, so every value is
    // the one a row-by-row loop computes).
    constexpr int NG = PER_KEY ? EPL : 1;
    float nk[EPL], nq[EPL], nlg[NG], nbt = 1.f, nv[R];
    auto load_token = [&](int64_t t) {
        const int64_t qk_off = (t * Hq + qh) * (int64_t)Dk;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            nk[j] = e < Dk ? load_act<Tin>(kg + qk_off + e) : 0.f;
            nq[j] = e < Dk ? load_act<Tin>(qg + qk_off + e) : 0.f;
        }
        if constexpr (PER_KEY) {
            const float *gt = p.g + (t * Hv + h) * (int64_t)Dk;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = lane + 32 * j;
                nlg[j] = e < Dk ? __ldg(gt + e) : 0.f;
            }
        } else {
            nlg[0] = p.has_decay ? __ldg(p.g + t * Hv + h) : 0.f;
        }
        nbt = p.has_retrieval ? __ldg(p.beta + t * Hv + h) : 1.f;
        const int64_t vo = (t * Hv + h) * (int64_t)Dv;
#pragma unroll
        for (int i = 0; i < R; ++i)
            nv[i] = row_base + i < Dv ? load_act<Tin>(vg + vo + row_base + i) : 0.f;
    };
    if (start < end) load_token(start);

    for (int64_t t = start; t < end; ++t) {
        float kx[EPL], qx[EPL], lgv[NG], vv[R];
        float bt = nbt;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            kx[j] = nk[j];
            qx[j] = nq[j];
        }
#pragma unroll
        for (int j = 0; j < NG; ++j) lgv[j] = nlg[j];
#pragma unroll
        for (int i = 0; i < R; ++i) vv[i] = nv[i];
        if (t + 1 < end) load_token(t + 1);

        if (p.qk_l2norm) {
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                sk += kx[j] * kx[j];
                sq += qx[j] * qx[j];
            }
            sk = warp_sum(sk);
            sq = warp_sum(sq);
            const float rk = 1.0f / sqrtf(sk + 1e-12f);
            const float rq = 1.0f / sqrtf(sq + 1e-12f);
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                kx[j] *= rk;
                qx[j] *= rq;
            }
        }
        if (p.has_retrieval && p.beta_sigmoid) bt = sigmoidf_(bt);
        // gam: the decay of each of this lane's key columns (one value without PER_KEY);
        // kr: the key as the retrieval sees it -- D_t k_t per key, k_t (scaled by gamma
        // after the sum) for the scalar decay
        float gam[NG], kr[EPL];
#pragma unroll
        for (int j = 0; j < NG; ++j) {
            float lg = lgv[j];
            if (p.has_decay && p.a_log)
                lg = -expf(__ldg(p.a_log + h)) * softplus20(lg + __ldg(p.dt_bias + h));
            gam[j] = expf(lg);
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j)
            kr[j] = PER_KEY ? (p.has_retrieval ? gam[j] * kx[j] : 0.f) : kx[j];
        // weight of the retrieval term (per key it sits in kr)
        const float rg = PER_KEY ? 1.f : (p.has_retrieval ? gam[0] : 0.f);

        float pd[R], o[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            pd[i] = 0.f;
#pragma unroll
            for (int j = 0; j < EPL; ++j) pd[i] += S[i][j] * kr[j];
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1)
#pragma unroll
            for (int i = 0; i < R; ++i) pd[i] += __shfl_xor_sync(0xffffffffu, pd[i], m);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const float u = PER_KEY ? bt * (vv[i] - pd[i]) : bt * (vv[i] - rg * pd[i]);
            o[i] = 0.f;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                S[i][j] = fmaf(kx[j], u, gam[PER_KEY ? j : 0] * S[i][j]);
                o[i] += S[i][j] * qx[j];
            }
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1)
#pragma unroll
            for (int i = 0; i < R; ++i) o[i] += __shfl_xor_sync(0xffffffffu, o[i], m);
        // lane i stores row row_base + i
        float oi = o[0];
#pragma unroll
        for (int i = 1; i < R; ++i) oi = lane == i ? o[i] : oi;
        if (lane < R && row_base + lane < Dv)
            store_act<Tin>(og + (t * Hv + h) * (int64_t)Dv + row_base + lane, p.scale * oi);
    }

#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            const int row = row_base + i;
            if (e < Dk && row < Dv) p.final_state[state_off + (int64_t)row * Dk + e] = S[i][j];
        }
}

template <typename Tin, bool PER_KEY>
static cudaError_t launch_seq_t(const GdnPrefillArgs &a, cudaStream_t stream)
{
    const unsigned tiles = (unsigned)((a.Dv + kSeqWarps * kSeqRows - 1) / (kSeqWarps * kSeqRows));
    if ((uint64_t)a.B * a.Hv * tiles > 0x7fffffffull) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)a.B * (unsigned)a.Hv * tiles);
    dim3 block(kSeqWarps * 32);
    if (a.Dk <= 32)
        prefill_seq_kernel<Tin, 1, PER_KEY><<<grid, block, 0, stream>>>(a);
    else if (a.Dk <= 64)
        prefill_seq_kernel<Tin, 2, PER_KEY><<<grid, block, 0, stream>>>(a);
    else if (a.Dk <= 128)
        prefill_seq_kernel<Tin, 4, PER_KEY><<<grid, block, 0, stream>>>(a);
    else
        prefill_seq_kernel<Tin, 8, PER_KEY><<<grid, block, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_seq_t(const GdnPrefillArgs &a, cudaStream_t stream)
{
    return a.g_per_key ? launch_seq_t<Tin, true>(a, stream) : launch_seq_t<Tin, false>(a, stream);
}

}  // namespace gdn

cudaError_t launch_prefill_sequential(const GdnPrefillArgs &a, cudaStream_t stream)
{
    if (a.B == 0 || a.Hv == 0) return cudaSuccess;
    if (a.dtype == GDN_F32) return gdn::launch_seq_t<float>(a, stream);
    if (a.dtype == GDN_F16) return gdn::launch_seq_t<__half>(a, stream);
    return gdn::launch_seq_t<__nv_bfloat16>(a, stream);
}
