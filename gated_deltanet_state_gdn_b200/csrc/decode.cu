// decode.cu -- Gated DeltaProduct decode / MTP over an fp32 slot pool.
//
// Operation ("flashinfer.cake_gdp.cake_gated_delta_product_mtp", description
// and Parameters): per (batch row, head) read the slot, per token decay once
// with alpha = exp(-exp(A_log) softplus(a + dt_bias)), apply nh delta
// sub-steps with beta = sigmoid(b), read out, and write the state back (to the
// write slot after the last token, or to the per-token scatter slots).
//
// Design (HBM-bound): one CTA per (row, head).  The Dv x 128 fp32 state is
// streamed HBM -> registers once with 16-byte evict-first loads, updated in
// registers for all T x nh sub-steps, and streamed back once per store.
// A state row (128 floats, 512 B) is split over an 8-lane group: lane `sub`
// holds elements {32 j + 4 sub + c : j < 4, c < 4}, so one load instruction
// moves four contiguous 128-byte segments.  A lane keeps R rows, a warp 4R
// rows, a CTA Dv rows.  Row dot products reduce over the 8-lane group with
// three xor-shuffles.
#include "common.cuh"

namespace gdn {

constexpr int kDecodeDk = 128;

// slot index i of an int32 or int64 index array
__device__ __forceinline__ int64_t slot_at(const void *idx, int i, bool wide)
{
    return wide ? (int64_t)__ldg(static_cast<const long long *>(idx) + i)
                : (int64_t)__ldg(static_cast<const int *>(idx) + i);
}

template <int DV, int R>
__global__ void __launch_bounds__(DV / (4 * R) * 32)
decode_kernel(const GdnDecodeArgs p)
{
    constexpr int DK = kDecodeDk;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane & 7;
    const int grp = lane >> 3;
    const int HV = p.HV;
    const int b = blockIdx.x / HV;
    const int h = blockIdx.x - b * HV;

    const int64_t r = slot_at(p.read_idx, b, p.idx64 != 0);
    if (r < 0) return;  // padding row: nothing is read, computed or stored
    if (r >= p.pool_size) {
        if (p.dev_status && threadIdx.x == 0) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
        return;
    }
    const int row0 = warp * (4 * R) + grp * R;
    const int64_t head_off = (int64_t)h * p.head_stride + (int64_t)row0 * DK + 4 * sub;

    // 1. stream the state in (all loads in flight before any use)
    float4 s[R][4];
    {
        const float *src = p.pool + (int64_t)r * p.slot_stride + head_off;
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) s[i][j] = ld_stream(src + i * DK + 32 * j);
    }

    const float neg_A = -expf(__ldg(p.A_log + h));
    const float dtb = __ldg(p.dt_bias + h);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);
    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *ag = static_cast<const __nv_bfloat16 *>(p.a);
    const __nv_bfloat16 *bg = static_cast<const __nv_bfloat16 *>(p.b);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.out);
    const int T = p.T, nh = p.nh, H = p.H;

    // 2. every token's k, q, v rows and gates for this (row, head) staged in shared memory by
    //    the whole CTA while the state streams in, so that the token loop below waits on no
    //    global load; alpha and beta are evaluated here once
    extern __shared__ __align__(16) unsigned char stage_raw[];
    __nv_bfloat16 *sk = reinterpret_cast<__nv_bfloat16 *>(stage_raw);   // [T][nh][DK]
    __nv_bfloat16 *sq = sk + T * nh * DK;                                 // [T][DK]
    __nv_bfloat16 *sv = sq + T * DK;                                      // [T][nh][DV]
    float *salpha = reinterpret_cast<float *>(sv + T * nh * DV);          // [T]
    float *sbeta = salpha + T;                                            // [T][nh]
    {
        constexpr int RW = DK / 4;   // 8-byte pieces of a k or q row
        constexpr int VW = DV / 4;
        const int nk = T * nh * RW, nq = T * RW, nv = T * nh * VW;
        for (int i = threadIdx.x; i < nk + nq + nv; i += blockDim.x) {
            if (i < nk) {
                const int row = i / RW, c = i - row * RW;   // row = t * nh + j
                const int64_t src = (((int64_t)b * T * nh + row) * H + h) * DK + 4 * c;
                reinterpret_cast<uint2 *>(sk)[i] = __ldg(reinterpret_cast<const uint2 *>(kg + src));
            } else if (i < nk + nq) {
                const int e = i - nk, t = e / RW, c = e - t * RW;
                const int64_t src = (((int64_t)b * T + t) * H + h) * DK + 4 * c;
                reinterpret_cast<uint2 *>(sq)[e] = __ldg(reinterpret_cast<const uint2 *>(qg + src));
            } else {
                const int e = i - nk - nq, row = e / VW, c = e - row * VW;
                const int64_t src = (((int64_t)b * T * nh + row) * HV + h) * DV + 4 * c;
                reinterpret_cast<uint2 *>(sv)[e] = __ldg(reinterpret_cast<const uint2 *>(vg + src));
            }
        }
        for (int i = threadIdx.x; i < T * (1 + nh); i += blockDim.x) {
            if (i < T) {
                // alpha = exp(-exp(A_log) * softplus20(a + dt_bias))
                const int64_t bt = (int64_t)b * T + i;
                salpha[i] = expf(neg_A * softplus20(bf16_to_f32(ag[bt * HV + h]) + dtb));
            } else {
                const int sj = i - T;   // t * nh + j
                sbeta[sj] = 1.0f / (1.0f + expf(-bf16_to_f32(bg[((int64_t)b * T * nh + sj) * HV + h])));
            }
        }
        __syncthreads();
    }

    for (int t = 0; t < T; ++t) {
        const int64_t bt = (int64_t)b * T + t;
        // 3. decay by alpha_t
        const float alpha = salpha[t];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s[i][j].x *= alpha; s[i][j].y *= alpha; s[i][j].z *= alpha; s[i][j].w *= alpha;
            }

        // 4. nh delta sub-steps
        for (int jh = 0; jh < nh; ++jh) {
            const int tj = t * nh + jh;
            const __nv_bfloat16 *kp = sk + tj * DK + 4 * sub;
            float4 kx[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) kx[j] = lds_bf16x4(kp + 32 * j);
            if (p.use_qk_l2norm) {
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) ss += dot4(kx[j], kx[j]);
                ss = group_sum<8>(ss);
                const float rn = 1.0f / sqrtf(ss + 1e-6f);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    kx[j].x *= rn; kx[j].y *= rn; kx[j].z *= rn; kx[j].w *= rn;
                }
            }
            const float beta = sbeta[tj];
            float vr[R];
            const __nv_bfloat16 *vp = sv + tj * DV + row0;
            if constexpr (R == 4) {
                float4 v4 = lds_bf16x4(vp);
                vr[0] = v4.x; vr[1] = v4.y; vr[2] = v4.z; vr[3] = v4.w;
            } else {
#pragma unroll
                for (int i = 0; i < R; ++i) vr[i] = bf16_to_f32(vp[i]);
            }
            float pd[R];
#pragma unroll
            for (int i = 0; i < R; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) acc += dot4(s[i][j], kx[j]);
                pd[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < R; ++i) pd[i] = group_sum<8>(pd[i]);
#pragma unroll
            for (int i = 0; i < R; ++i) {
                const float u = beta * (vr[i] - pd[i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    s[i][j].x = fmaf(kx[j].x, u, s[i][j].x);
                    s[i][j].y = fmaf(kx[j].y, u, s[i][j].y);
                    s[i][j].z = fmaf(kx[j].z, u, s[i][j].z);
                    s[i][j].w = fmaf(kx[j].w, u, s[i][j].w);
                }
            }
        }

        // 5. readout o = scale * S q
        {
            const __nv_bfloat16 *qp = sq + t * DK + 4 * sub;
            float4 qx[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) qx[j] = lds_bf16x4(qp + 32 * j);
            float qs = p.scale;
            if (p.use_qk_l2norm) {
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) ss += dot4(qx[j], qx[j]);
                ss = group_sum<8>(ss);
                qs *= 1.0f / sqrtf(ss + 1e-6f);
            }
            float o[R];
#pragma unroll
            for (int i = 0; i < R; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < 4; ++j) acc += dot4(s[i][j], qx[j]);
                o[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < R; ++i) o[i] = group_sum<8>(o[i]) * qs;
            if (sub == 0) {
                __nv_bfloat16 *op = og + (bt * HV + h) * DV + row0;
                if constexpr (R == 4) {
                    uint2 w;
                    w.x = pack_bf16x2(o[0], o[1]);
                    w.y = pack_bf16x2(o[2], o[3]);
                    *reinterpret_cast<uint2 *>(op) = w;
                } else if constexpr (R == 2) {
                    *reinterpret_cast<uint32_t *>(op) = pack_bf16x2(o[0], o[1]);
                } else {
#pragma unroll
                    for (int i = 0; i < R; ++i) op[i] = __float2bfloat16_rn(o[i]);
                }
            }
        }

        // 6. per-token scatter
        if (p.scatter_idx) {
            const int sidx = __ldg(p.scatter_idx + bt);
            if (sidx >= p.pool_size) {
                if (p.dev_status && threadIdx.x == 0) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
            } else if (sidx >= 0) {
                float *dst = p.pool + (int64_t)sidx * p.slot_stride + head_off;
#pragma unroll
                for (int i = 0; i < R; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_stream(dst + i * DK + 32 * j, s[i][j]);
            }
        }
    }

    // 7. end-of-sequence write-back
    if (!p.scatter_idx && !p.disable_state_update) {
        const int64_t w = p.write_idx ? slot_at(p.write_idx, b, p.idx64 != 0) : r;
        if (w >= p.pool_size) {
            if (p.dev_status && threadIdx.x == 0) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
        } else if (w >= 0) {
            float *dst = p.pool + (int64_t)w * p.slot_stride + head_off;
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) st_stream(dst + i * DK + 32 * j, s[i][j]);
        }
    }
}

}  // namespace gdn

cudaError_t launch_decode(const GdnDecodeArgs &a, cudaStream_t stream)
{
    const unsigned grid = (unsigned)a.B * (unsigned)a.HV;
    if (grid == 0) return cudaSuccess;
    // staged k, q, v rows (bf16) and gates (fp32): at most 37 KB (T = 16, nh = 4, Dv = 128)
    const size_t smem = (size_t)a.T * a.nh * gdn::kDecodeDk * 2 + (size_t)a.T * gdn::kDecodeDk * 2 +
                        (size_t)a.T * a.nh * a.Dv * 2 + (size_t)a.T * (1 + a.nh) * 4;
    if (a.Dv == 128) {
        constexpr int R = 4;
        gdn::decode_kernel<128, R><<<grid, 128 / (4 * R) * 32, smem, stream>>>(a);
    } else {
        constexpr int R = 4;
        gdn::decode_kernel<64, R><<<grid, 64 / (4 * R) * 32, smem, stream>>>(a);
    }
    return cudaGetLastError();
}
