// decode.cu -- Gated DeltaProduct decode / MTP over an fp32 slot pool.
//
// Operation ("flashinfer.cake_gdp.cake_gated_delta_product_mtp", description
// and Parameters): per (batch row, head) read the slot, per token decay once
// with alpha = exp(-exp(A_log) softplus(a + dt_bias)), apply nh delta
// sub-steps with beta = sigmoid(b), read out, and write the state back (to the
// write slot after the last token, or to the per-token scatter slots).
//
// Design (HBM-bound).  The unit of work is one (row, head): its Dv x 128 fp32
// state is held in registers for all T x nh sub-steps and streamed back with
// 16-byte evict-first stores.  A state row (128 floats, 512 B) is split over an
// 8-lane group: lane `sub` holds elements {32 j + 4 sub + c : j < 4, c < 4}, so
// one access instruction moves four contiguous 128-byte segments.  A lane keeps
// R rows, a warp 4R rows, a CTA Dv rows.  Row dot products reduce over the
// 8-lane group with three xor-shuffles.  Every token's k, q, v rows, gates and
// scatter slot are staged in shared memory before the token loop, so the loop
// waits on no global load.
//
// Two launch forms share that per-unit code:
//   decode_kernel         one CTA per unit; the state is loaded straight into
//                         registers (8 rows per lane at Dv = 128: 128 threads,
//                         three CTAs per SM).  Used for single-token units that
//                         fill several waves of resident CTAs.
//   decode_stream_kernel  persistent: one CTA per resident slot walks the units
//                         blockIdx.x + i * gridDim.x.  While it updates and
//                         stores unit i, one bulk copy brings unit i+1's state
//                         into shared memory and cp.async its k, q, v rows,
//                         all completing on one mbarrier, so loads, arithmetic
//                         and stores of consecutive units overlap.
#include "common.cuh"
#include "sm100.cuh"

#include <atomic>

namespace gdn {

constexpr int kDecodeDk = 128;

// slot index i of an int32 or int64 index array
__device__ __forceinline__ int64_t slot_at(const void *idx, int i, bool wide)
{
    return wide ? (int64_t)__ldg(static_cast<const long long *>(idx) + i)
                : (int64_t)__ldg(static_cast<const int *>(idx) + i);
}

// Per-unit staging area in shared memory: k [T][nh][128], q [T][128], v [T][nh][Dv] (bf16),
// alpha [T], beta [T][nh] (fp32), scatter slot [T] (int32).
struct Stage {
    __nv_bfloat16 *k, *q, *v;
    float *alpha, *beta;
    int32_t *scat;
};

__host__ __device__ inline size_t stage_bytes(int T, int nh, int Dv)
{
    const size_t n = (size_t)T * nh * kDecodeDk * 2 + (size_t)T * kDecodeDk * 2 +
                     (size_t)T * nh * Dv * 2 + (size_t)T * (1 + nh) * 4 + (size_t)T * 4;
    return (n + 15) & ~(size_t)15;
}

template <int DV>
__device__ __forceinline__ Stage stage_at(unsigned char *base, int T, int nh)
{
    Stage s;
    s.k = reinterpret_cast<__nv_bfloat16 *>(base);
    s.q = s.k + T * nh * kDecodeDk;
    s.v = s.q + T * kDecodeDk;
    s.alpha = reinterpret_cast<float *>(s.v + T * nh * DV);
    s.beta = s.alpha + T;
    s.scat = reinterpret_cast<int32_t *>(s.beta + T * nh);
    return s;
}

// Input piece i of unit (b, h): an 8-byte global source and its shared-memory destination.
// Pieces run over the k rows, then the q rows, then the v rows of every token.  Returns false
// (checked builds only) when either side lies outside its buffer.
template <int DV>
__device__ __forceinline__ bool input_piece(const GdnDecodeArgs &p, const Stage &st, int b, int h,
                                            int i, const void *&src, void *&dst)
{
    constexpr int RW = kDecodeDk / 4;   // 8-byte pieces of a k or q row
    constexpr int VW = DV / 4;
    const int T = p.T, nh = p.nh, H = p.H;
    const int nk = T * nh * RW, nq = T * RW;
    int64_t e_src, n_src;
    if (i < nk) {
        const int row = i / RW, c = i - row * RW;   // row = t * nh + j
        e_src = (((int64_t)b * T * nh + row) * H + h) * kDecodeDk + 4 * c;
        n_src = (int64_t)p.B * T * nh * H * kDecodeDk;
        src = static_cast<const __nv_bfloat16 *>(p.k) + e_src;
        dst = st.k + 4 * i;
    } else if (i < nk + nq) {
        const int e = i - nk, t = e / RW, c = e - t * RW;
        e_src = (((int64_t)b * T + t) * H + h) * kDecodeDk + 4 * c;
        n_src = (int64_t)p.B * T * H * kDecodeDk;
        src = static_cast<const __nv_bfloat16 *>(p.q) + e_src;
        dst = st.q + 4 * e;
    } else {
        const int e = i - nk - nq, row = e / VW, c = e - row * VW;
        e_src = (((int64_t)b * T * nh + row) * p.HV + h) * DV + 4 * c;
        n_src = (int64_t)p.B * T * nh * p.HV * DV;
        src = static_cast<const __nv_bfloat16 *>(p.v) + e_src;
        dst = st.v + 4 * e;
    }
    return in_range(e_src, 4, n_src, p.dev_status) && in_smem(dst, 8, p.dev_status);
}

// elements of the pool the strides can reach
template <int DV>
__device__ __forceinline__ int64_t pool_elems(const GdnDecodeArgs &p)
{
    return (int64_t)(p.pool_size - 1) * p.slot_stride + (int64_t)(p.HV - 1) * p.head_stride +
           (int64_t)DV * kDecodeDk;
}

// a lane's R x 4 float4 of state rows at pool element `base` (row stride 128), evict-first
template <int DV, int R>
__device__ __forceinline__ void store_state(const GdnDecodeArgs &p, int64_t base, const float4 (&s)[R][4])
{
    const int64_t n = pool_elems<DV>(p);
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t e = base + i * kDecodeDk + 32 * j;
            if (in_range(e, 4, n, p.dev_status)) st_stream(p.pool + e, s[i][j]);
        }
}

template <int DV>
__device__ __forceinline__ int input_pieces(const GdnDecodeArgs &p)
{
    return p.T * p.nh * (kDecodeDk / 4) + p.T * (kDecodeDk / 4) + p.T * p.nh * (DV / 4);
}

// Raw gate i of unit (b, h): i < T is a[b, t], otherwise b[b, t, j] with i - T = t nh + j.
__device__ __forceinline__ unsigned short gate_raw(const GdnDecodeArgs &p, int b, int h, int i)
{
    const int T = p.T;
    const unsigned short *ag = static_cast<const unsigned short *>(p.a);
    const unsigned short *bg = static_cast<const unsigned short *>(p.b);
    if (i < T) {
        const int64_t e = ((int64_t)b * T + i) * p.HV + h;
        return in_range(e, 1, (int64_t)p.B * T * p.HV, p.dev_status) ? __ldg(ag + e) : (unsigned short)0;
    }
    const int64_t e = ((int64_t)b * T * p.nh + (i - T)) * p.HV + h;
    return in_range(e, 1, (int64_t)p.B * T * p.nh * p.HV, p.dev_status) ? __ldg(bg + e) : (unsigned short)0;
}

// alpha = exp(-exp(A_log) softplus20(a + dt_bias)), beta = sigmoid(b)
__device__ __forceinline__ void gate_store(const GdnDecodeArgs &p, const Stage &st, int h, int i,
                                           unsigned short raw)
{
    const float x = __uint_as_float((uint32_t)raw << 16);
    if (i < p.T) {
        const float neg_A = -expf(__ldg(p.A_log + h));
        st.alpha[i] = expf(neg_A * softplus20(x + __ldg(p.dt_bias + h)));
    } else {
        st.beta[i - p.T] = 1.0f / (1.0f + expf(-x));
    }
}

// The T tokens of one unit on a state held in registers: decay, nh delta sub-steps, readout,
// per-token scatter, then the end-of-sequence write-back.  `r` is the unit's read slot and `w`
// its write slot (already resolved; unused with scatter or disable_state_update).
template <int DV, int R>
__device__ __forceinline__ void update_unit(float4 (&s)[R][4], const GdnDecodeArgs &p,
                                            const Stage &st, int b, int h, int row0, int sub,
                                            int64_t head_off, int64_t w)
{
    constexpr int DK = kDecodeDk;
    const int T = p.T, nh = p.nh, HV = p.HV;
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.out);

    for (int t = 0; t < T; ++t) {
        const int64_t bt = (int64_t)b * T + t;
        // decay by alpha_t
        const float alpha = st.alpha[t];
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                s[i][j].x *= alpha; s[i][j].y *= alpha; s[i][j].z *= alpha; s[i][j].w *= alpha;
            }

        // nh delta sub-steps
        for (int jh = 0; jh < nh; ++jh) {
            const int tj = t * nh + jh;
            const __nv_bfloat16 *kp = st.k + tj * DK + 4 * sub;
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
            const float beta = st.beta[tj];
            float vr[R];
            const __nv_bfloat16 *vp = st.v + tj * DV + row0;
            if constexpr (R == 4 || R == 8) {
#pragma unroll
                for (int h = 0; h < R / 4; ++h) {
                    const float4 v4 = lds_bf16x4(vp + 4 * h);
                    vr[4 * h] = v4.x; vr[4 * h + 1] = v4.y; vr[4 * h + 2] = v4.z; vr[4 * h + 3] = v4.w;
                }
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

        // readout o = scale * S q
        {
            const __nv_bfloat16 *qp = st.q + t * DK + 4 * sub;
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
            if (sub == 0 && in_range((bt * HV + h) * DV + row0, R, (int64_t)p.B * T * HV * DV, p.dev_status)) {
                __nv_bfloat16 *op = og + (bt * HV + h) * DV + row0;
                if constexpr (R == 8) {
                    // two 8-byte stores: `out` is only required to be 8-byte aligned
                    uint2 w0, w1;
                    w0.x = pack_bf16x2(o[0], o[1]);
                    w0.y = pack_bf16x2(o[2], o[3]);
                    w1.x = pack_bf16x2(o[4], o[5]);
                    w1.y = pack_bf16x2(o[6], o[7]);
                    reinterpret_cast<uint2 *>(op)[0] = w0;
                    reinterpret_cast<uint2 *>(op)[1] = w1;
                } else if constexpr (R == 4) {
                    uint2 wv;
                    wv.x = pack_bf16x2(o[0], o[1]);
                    wv.y = pack_bf16x2(o[2], o[3]);
                    *reinterpret_cast<uint2 *>(op) = wv;
                } else if constexpr (R == 2) {
                    *reinterpret_cast<uint32_t *>(op) = pack_bf16x2(o[0], o[1]);
                } else {
#pragma unroll
                    for (int i = 0; i < R; ++i) op[i] = __float2bfloat16_rn(o[i]);
                }
            }
        }

        // per-token scatter
        if (p.scatter_idx) {
            const int sidx = st.scat[t];
            if (sidx >= p.pool_size) {
                if (p.dev_status && threadIdx.x == 0) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
            } else if (sidx >= 0) {
                store_state<DV, R>(p, (int64_t)sidx * p.slot_stride + head_off, s);
            }
        }
    }

    // end-of-sequence write-back
    if (!p.scatter_idx && !p.disable_state_update) {
        if (w >= p.pool_size) {
            if (p.dev_status && threadIdx.x == 0) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
        } else if (w >= 0) {
            store_state<DV, R>(p, w * p.slot_stride + head_off, s);
        }
    }
}

// write slot of row b (read slot r when there is no write array)
__device__ __forceinline__ int64_t write_slot(const GdnDecodeArgs &p, int b, int64_t r)
{
    if (p.scatter_idx || p.disable_state_update) return -1;
    return p.write_idx ? slot_at(p.write_idx, b, p.idx64 != 0) : r;
}

// Side value i of unit (b, h), fetched into a register and stored to the stage later: the gates
// (i < T (1 + nh), raw bf16) and then the T scatter slots.
__device__ __forceinline__ uint32_t side_raw(const GdnDecodeArgs &p, int b, int h, int i)
{
    const int ng = p.T * (1 + p.nh);
    if (i < ng) return gate_raw(p, b, h, i);
    const int64_t e = (int64_t)b * p.T + (i - ng);
    return in_range(e, 1, (int64_t)p.B * p.T, p.dev_status) ? (uint32_t)__ldg(p.scatter_idx + e) : 0xffffffffu;
}

__device__ __forceinline__ void side_store(const GdnDecodeArgs &p, const Stage &st, int h, int i,
                                           uint32_t raw)
{
    const int ng = p.T * (1 + p.nh);
    if (i < ng) gate_store(p, st, h, i, (unsigned short)raw);
    else st.scat[i - ng] = (int32_t)raw;
}

__device__ __forceinline__ int side_count(const GdnDecodeArgs &p)
{
    return p.T * (1 + p.nh) + (p.scatter_idx ? p.T : 0);
}

// ---------------------------------------------------------------- one CTA per (row, head)
template <int DV, int R>
__global__ void __launch_bounds__(DV / (4 * R) * 32, R == 8 ? 3 : 1)
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

    // the state streams in (all loads in flight before any use)
    float4 s[R][4];
    {
        const int64_t n = pool_elems<DV>(p);
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t e = r * p.slot_stride + head_off + i * DK + 32 * j;
                s[i][j] = in_range(e, 4, n, p.dev_status) ? ld_stream(p.pool + e) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
    }
    const int64_t w = write_slot(p, b, r);

    // meanwhile the whole CTA stages the unit's inputs and evaluates its gates
    extern __shared__ __align__(16) unsigned char stage_raw[];
    const Stage st = stage_at<DV>(stage_raw, p.T, p.nh);
    {
        const int n = input_pieces<DV>(p);
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const void *src;
            void *dst;
            if (input_piece<DV>(p, st, b, h, i, src, dst))
                *static_cast<uint2 *>(dst) = __ldg(static_cast<const uint2 *>(src));
        }
        const int ns = side_count(p);
        for (int i = threadIdx.x; i < ns; i += blockDim.x) side_store(p, st, h, i, side_raw(p, b, h, i));
        __syncthreads();
    }
    update_unit<DV, R>(s, p, st, b, h, row0, sub, head_off, w);
}

// ---------------------------------------------------------------- persistent, prefetching
// bounded wait on an mbarrier phase: false when it does not complete within `limit` cycles
// (2^31, about a second, for a wait on the pipeline)
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, long long limit = 1ll << 31)
{
    if (sm100::mbar_try_wait(bar, parity)) return true;
    const long long start = clock64();
    while (!sm100::mbar_try_wait(bar, parity))
        if (clock64() - start > limit) return false;
    return true;
}

template <int DV, int R, int MINB>
__global__ void __launch_bounds__(DV / (4 * R) * 32, MINB)
decode_stream_kernel(const GdnDecodeArgs p)
{
    using namespace sm100;
    constexpr int DK = kDecodeDk;
    constexpr int NT = DV / (4 * R) * 32;
    constexpr uint32_t kStateBytes = DV * DK * 4;
    static_assert(NT >= 16 * (1 + 4) + 16, "one side value per thread at T = 16, nh = 4");
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane & 7;
    const int grp = lane >> 3;
    const int HV = p.HV, T = p.T, nh = p.nh;
    const int units = p.B * HV;
    const bool wide = p.idx64 != 0;
    const int row0 = warp * (4 * R) + grp * R;
    const int npieces = input_pieces<DV>(p);
    const int nside = side_count(p);

    // state buffer [DV][128] fp32, then two stages (units i and i+1)
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar_mem;
    const float *sstate = reinterpret_cast<const float *>(smem);
    const size_t sbytes = stage_bytes(T, nh, DV);
    unsigned char *stage0 = smem + kStateBytes;
    const uint32_t bar = smem_u32(&bar_mem);

    int u = blockIdx.x;
    if (u >= units) return;
    if (threadIdx.x == 0) {
        mbar_init(bar, NT + 1);   // one cp.async arrival per thread + thread 0's expect_tx
        fence_mbar_init();
    }
    __syncthreads();

    // copies of unit uu (read slot rr) into the state buffer and stage `buf`; every thread
    // arrives once, thread 0 also posts the state's byte count (0 for a skipped unit)
    // (checked builds: a caller-requested stall makes the first wait run out)
    bool stall = threadIdx.x == 0 && test_stall_requested(p.dev_status);
    auto issue = [&](int uu, int64_t rr, int buf) {
        const int bb = uu / HV, hh = uu - bb * HV;
        const bool live = rr >= 0 && rr < p.pool_size;
        if (threadIdx.x == 0) {
            if (rr >= p.pool_size && p.dev_status) atomicOr(p.dev_status, GDN_DEV_BAD_SLOT);
            const int64_t e = rr * p.slot_stride + (int64_t)hh * p.head_stride;
            const bool copy = live && in_range(e, DV * DK, pool_elems<DV>(p), p.dev_status) &&
                              in_smem(sstate, kStateBytes, p.dev_status);
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(bar, (copy ? kStateBytes : 0u) + (stall ? 16u : 0u));
            stall = false;
            if (copy) bulk_load_1d(smem_u32(sstate), p.pool + e, kStateBytes, bar);
        }
        if (live && in_smem(stage0 + buf * sbytes, (uint32_t)sbytes, p.dev_status)) {
            const Stage st = stage_at<DV>(stage0 + buf * sbytes, T, nh);
            for (int i = threadIdx.x; i < npieces; i += NT) {
                const void *src;
                void *dst;
                if (input_piece<DV>(p, st, bb, hh, i, src, dst)) cp_async8(smem_u32(dst), src);
            }
        }
        cp_async_arrive(bar);
    };

    int un = u + gridDim.x;
    int64_t r = slot_at(p.read_idx, u / HV, wide);
    int64_t r_next = un < units ? slot_at(p.read_idx, un / HV, wide) : -1;
    issue(u, r, 0);
    {
        const int b0 = u / HV, h0 = u - b0 * HV;
        if (threadIdx.x < nside)
            side_store(p, stage_at<DV>(stage0, T, nh), h0, threadIdx.x, side_raw(p, b0, h0, threadIdx.x));
    }

    for (int it = 0; u < units; ++it) {
        const int buf = it & 1;
        const int b = u / HV, h = u - b * HV;
        const bool live = r >= 0 && r < p.pool_size;
        // global loads first consumed later (after this unit's arithmetic or in the next
        // iteration): the read slot after next, the next unit's side values, the write slot
        const int unn = un + gridDim.x;
        const int64_t r_nn = unn < units ? slot_at(p.read_idx, unn / HV, wide) : -1;
        const bool has_next = un < units;
        const int bn = un / HV, hn = un - bn * HV;
        const uint32_t side_n = (has_next && threadIdx.x < nside) ? side_raw(p, bn, hn, threadIdx.x) : 0u;
        const int64_t w = live ? write_slot(p, b, r) : -1;

        // this unit's state and inputs
        const bool timed_out = !wait_phase(bar, (uint32_t)(it & 1));
        float4 s[R][4];
        if (live) {
            const float *src = sstate + row0 * DK + 4 * sub;
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) s[i][j] = *reinterpret_cast<const float4 *>(src + i * DK + 32 * j);
        }
        // the state buffer and the other stage are free from here on
        if (__syncthreads_or(timed_out)) {
            if (threadIdx.x == 0) {
                if (p.dev_status) atomicOr(p.dev_status, GDN_DEV_TIMEOUT);
                // let copies still in flight land before the CTA's shared memory goes away;
                // one that is on its way lands within microseconds, so this wait is short
                // (2^24 cycles, ~8 ms) rather than a second bound on bytes that never come
                wait_phase(bar, (uint32_t)(it & 1), 1ll << 24);
            }
            return;
        }
        if (has_next) issue(un, r_next, buf ^ 1);
        if (live) {
            const int64_t head_off = (int64_t)h * p.head_stride + (int64_t)row0 * DK + 4 * sub;
            update_unit<DV, R>(s, p, stage_at<DV>(stage0 + buf * sbytes, T, nh), b, h, row0, sub,
                               head_off, w);
        }
        if (has_next && threadIdx.x < nside)
            side_store(p, stage_at<DV>(stage0 + (buf ^ 1) * sbytes, T, nh), hn, threadIdx.x, side_n);
        u = un;
        un = unn;
        r = r_next;
        r_next = r_nn;
    }
}

}  // namespace gdn

namespace {

constexpr int kMaxDevices = 16;
constexpr long long kPerUnitWaves = 4;   // waves of resident one-CTA-per-unit CTAs

int sm_count()
{
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < kMaxDevices) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev < kMaxDevices) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// persistent launch: one CTA per resident slot (occupancy cached per device and T x nh)
template <int DV, int R, int MINB>
cudaError_t launch_stream(const GdnDecodeArgs &a, cudaStream_t stream)
{
    constexpr int NT = DV / (4 * R) * 32;
    auto kern = gdn::decode_stream_kernel<DV, R, MINB>;
    const size_t smem = (size_t)DV * gdn::kDecodeDk * 4 + 2 * gdn::stage_bytes(a.T, a.nh, DV);
    static std::atomic<int> occ[kMaxDevices][17][5];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int nb = dev < kMaxDevices ? occ[dev][a.T][a.nh].load(std::memory_order_relaxed) : 0;
    if (nb <= 0) {
        const size_t max_smem = (size_t)DV * gdn::kDecodeDk * 4 + 2 * gdn::stage_bytes(16, 4, DV);
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, NT, smem);
        if (e != cudaSuccess) return e;
        if (nb <= 0) return cudaErrorInvalidConfiguration;
        if (dev < kMaxDevices) occ[dev][a.T][a.nh].store(nb, std::memory_order_relaxed);
    }
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const long long units = (long long)a.B * a.HV;
    const unsigned grid = (unsigned)std::min<long long>(units, (long long)nb * sms);
    kern<<<grid, NT, smem, stream>>>(a);
    return cudaGetLastError();
}

template <int DV, int R>
cudaError_t launch_per_unit(const GdnDecodeArgs &a, cudaStream_t stream)
{
    const unsigned grid = (unsigned)a.B * (unsigned)a.HV;
    // staged inputs: at most 37 KB (T = 16, nh = 4, Dv = 128)
    const size_t smem = gdn::stage_bytes(a.T, a.nh, DV);
    gdn::decode_kernel<DV, R><<<grid, DV / (4 * R) * 32, smem, stream>>>(a);
    return cudaGetLastError();
}

// resident one-CTA-per-unit CTAs per SM (cached per device)
template <int DV, int R>
int per_unit_occupancy()
{
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < kMaxDevices) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, gdn::decode_kernel<DV, R>, DV / (4 * R) * 32,
                                                      gdn::stage_bytes(1, 1, DV)) != cudaSuccess)
        return 0;
    if (dev < kMaxDevices) cache[dev].store(nb, std::memory_order_relaxed);
    return nb;
}

template <int DV, int R, int MINB, int RU>
cudaError_t launch_form(const GdnDecodeArgs &a, cudaStream_t stream)
{
    // One CTA per unit keeps every state load of its resident CTAs in flight at once and wins
    // once the units fill several waves of them; with fewer waves, or several tokens per unit
    // (scatter stores, longer arithmetic), the persistent form's overlap of the next unit's
    // loads with this unit's arithmetic and stores wins.  RU rows per lane for the one-CTA
    // form (8 at Dv = 128: 128 threads, three CTAs and 192 KB of state loads per SM).
    const long long units = (long long)a.B * a.HV;
    const long long resident = (long long)sm_count() * per_unit_occupancy<DV, RU>();
    if (a.T == 1 && resident > 0 && units >= kPerUnitWaves * resident)
        return launch_per_unit<DV, RU>(a, stream);
    return launch_stream<DV, R, MINB>(a, stream);
}

}  // namespace

cudaError_t launch_decode(const GdnDecodeArgs &a, cudaStream_t stream)
{
    if ((long long)a.B * a.HV == 0) return cudaSuccess;
    constexpr int R = 4;
    if (a.Dv == 128) return launch_form<128, R, 2, 8>(a, stream);
    return launch_form<64, R, 4, 4>(a, stream);
}
