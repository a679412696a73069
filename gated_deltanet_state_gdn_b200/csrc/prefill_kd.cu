// prefill_kd.cu -- chunked prefill with a per-key-dimension decay on sm_100a tensor cores.
//
// Operation: the recurrence of "com.microsoft.GatedDeltaNet" (Description) with `decay`
// in its per-key-dimension spelling (Inputs table, shape (..., num_heads_v, head_size_qk)),
// read as D_t = diag(exp(g_t)) on the key axis of the state:
//   S_t = D_t S_{t-1} + k_t (beta_t (v_t - (D_t S_{t-1})^T k_t))^T,   o_t = scale S_t^T q_t.
// bf16 q/k/v with 8 <= Dk, Dv <= 128 (zero-padded to 128-wide tiles), 64 tokens a chunk.
// The scaled operands below reach 2^104, beyond fp16's exponent range (2^15), so fp16
// activations take the per-token kernel; bf16 has fp32's exponent range.  Every operand
// here carries one bf16 rounding of a decayed product (the scalar-decay kernel feeds the raw
// bytes and decays in fp32 after the MMA); heads narrower than 8 have no rows to average that
// over and no tensor-core work worth the rounding, so they take the per-token fp32 kernel.
//
// Chunk form (derived from the recurrence as for the scalar decay, with every decay factor
// now a vector over the key dimensions).  For a chunk with incoming state S0 (Dk x Dv),
// per-dimension cumulative log-decay G_i = sum_{l<=i} g_l, normalised rows k^_i, q^_i:
//   A_ij = beta_i sum_d k^_i[d] k^_j[d] e^{G_i[d] - G_j[d]}  (j < i),   T = (I + A)^-1
//   P_ij = sum_d q^_i[d] k^_j[d] e^{G_i[d] - G_j[d]}          (j <= i)
//   W = T diag(beta) (K^ * e^G),   U~ = T diag(beta) V,   U = U~ - W S0
//   O = scale ((Q^ * e^G) S0 + P U)
//   S_C = diag(e^{G_C}) S0 + (K^ * e^{G_C - G})^T U
// The decay sits inside the contractions of A and P, so it is split between the two
// operands relative to a reference.  Each 16-token block I of the chunk takes as reference
// M_I = G at its eighth token: the row operand is x_i * e^{G_i - M_I} (one tile for all
// rows), the key operand of block I is k^_j * e^{M_I - G_j} for every j up to the block's
// end, and the four key operands are stacked into one 160-row tile, so a single MMA
// (N = 160) gives every block's products at once.  Every factor stays within 2^104 once
// each per-dimension log-decay is floored at -9 (at most 8 tokens lie between a token and
// its reference, 8 * 9 * log2(e) < 104): the products that are used are <= 1, the others
// (j > i) are masked out by selection.  The floor changes a per-token decay factor below
// e^-9 ~ 1.2e-4 into 1.2e-4, far below the bf16 operand rounding.
// All state-dependent products are evaluated transposed (rows = value index dv, M = 128):
//   (G)  [K^;Q^]*e^{G-M} x Bcat^T  -> TMEM (128 x 160)
//   (W)  W^T = (K^ e^G)^T Tb^T      (U~) U~^T = V^T Tb^T,   Tb = T diag(beta)
//   (1a) U^T += S^T (-W)^T          (1b) Y = S^T (Q^ e^G)^T
//   (2)  S^T = S^T diag(e^{G_C}) + U^T (K^ e^{G_C - G})
//   (3)  Z = U^T P^T                O^T = scale (Y + Z)
//
// One CTA of 512 threads per (request, value head), longest requests first: four
// warpgroups, whose thread t owns TMEM lane t (the state row dv = t) and which split each
// row's columns between them.  The phases of a chunk run one after another: plain loads stage
// and scale the operand tiles, thread 0 issues the MMAs and a bounded wait on an mbarrier ends
// each group.  (1b) alone is issued by another thread, with its own mbarrier, while the tensor
// pipe is idle, and the output phase waits for it.
// The triangular solve works on 16 x 16 blocks: fp32 forward substitution inside the four
// diagonal blocks, then tf32 warp MMAs merge the blocks below the diagonal.
#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "tile16.cuh"

using namespace sm100;

namespace gdn_kd {

using gdn_tile::a_slot;
using gdn_tile::blk_mma;
using gdn_tile::blk_store;
using gdn_tile::elem16;
using gdn_tile::pack2;
using gdn_tile::pack8;
using gdn_tile::SOLVE_BLK;
using gdn_tile::SOLVE_LD;
using gdn_tile::sw128;

constexpr int C = 64;            // chunk length (tokens)
constexpr int NT = 512;          // threads per CTA: four warpgroups over the 128 TMEM lanes
constexpr int NWG = NT / 128;    // warpgroups
constexpr int BPW = 4 / NWG;     // 32-column state blocks per warpgroup
constexpr int CPW = 64 / NWG;    // chunk columns (tokens) per warpgroup
static_assert(NWG == 4 && CPW == 16, "the decay scan gives warpgroup I the tokens of block I");
constexpr float G_FLOOR = -9.f;  // per-dimension log-decay floor
constexpr float LOG2E = 1.4426950408889634f;

// ---- shared memory (bytes from a 1024-aligned base) ----
// region Y: the Gram operands, then (after the Gram) P, -W and the bf16 U
constexpr uint32_t OFF_ASIDE = 0;        // [kb 2][128 rows: K^ 0-63, Q^ 64-127][128 B], kb 16384
constexpr uint32_t ASIDE_KB = 16384;
constexpr uint32_t OFF_BCAT = 32768;     // [kb 2][160 rows][128 B], kb 20480
constexpr uint32_t BCAT_KB = 20480;
constexpr uint32_t OFF_P = 0;            // [64 rows i][64 j], K-major
constexpr uint32_t OFF_WNEG = 8192;      // [128 rows dk][64 i], MN-major B of (1a)
constexpr uint32_t OFF_UB = 24576;       // [128 rows dv][64 j], K-major A of (2), (3)
constexpr uint32_t OFF_GN = 40960;       // raw log-decays of the next chunk, fp32 [64][128]:
                                         // staged once the Gram has read the key operands
// region Z: decayed operands and v
constexpr uint32_t OFF_KG = 73728;       // K^ e^G        [kb 2][64 rows j][128 B], kb 8192
constexpr uint32_t OFF_QG = 90112;       // Q^ e^G
constexpr uint32_t OFF_KD = 106496;      // K^ e^{G_C-G}
constexpr uint32_t OFF_VT = 122880;      // v             [dv half 2][64 rows j][128 B]
constexpr uint32_t TILE_KB = 8192;
constexpr uint32_t OFF_SB = 139264;      // bf16 S^T      [kb 2][128 rows dv][128 B], kb 16384
// region X: log-decays, then (after the operands are built) A and Tb
constexpr uint32_t OFF_G2 = 172032;      // fp32 [64][128]: G * log2(e)
constexpr uint32_t OFF_A = 172032;       // solve area: 16 fp32 blocks of 16 x SOLVE_LD
constexpr uint32_t OFF_TB = 192512;      // [64 rows i][64 j], K-major B of (W), (U~)
constexpr uint32_t OFF_VEC = 204800;     // per-dimension vectors, fp32
constexpr int VEC_EM = 0;        // e^{M_I}                 [4][128]
constexpr int VEC_CM = 512;      // e^{M_I' - M_I}, I' > I  [6][128]
constexpr int VEC_EC3 = 1280;    // e^{G_C - M_3}           [128]
constexpr int VEC_GC = 1408;     // e^{G_C}                 [128]
constexpr int VEC_M2 = 1536;     // M_I * log2(e)           [4][128]
constexpr int VEC_TOT = VEC_CM;  // segment totals of the scan [3][128], before e^{M_I' - M_I}
constexpr uint32_t OFF_ROW = OFF_VEC + 2048 * 4;   // per-token values, fp32
constexpr int ROW_BETA = 0, ROW_QK = 64;   // beta_j; rq_j rk_j (q_j . k_j)
constexpr uint32_t OFF_BAR = OFF_ROW + 1024;       // mbarrier, TMEM base, flag
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_BCAT + 2 * BCAT_KB <= OFF_KG && OFF_UB + 16384 <= OFF_GN &&
              OFF_GN + 64 * 128 * 4 <= OFF_KG, "region Y");
static_assert(OFF_A + 16 * SOLVE_BLK * 4 <= OFF_TB && OFF_TB + 8192 <= OFF_VEC &&
              OFF_G2 + 64 * 128 * 4 <= OFF_VEC, "region X");
static_assert(OFF_TB % 1024 == 0 && OFF_SB % 1024 == 0 && OFF_VT % 1024 == 0 &&
              OFF_BCAT % 1024 == 0 && OFF_KD % 1024 == 0, "swizzled tiles need 1024 alignment");

// TMEM columns: the Gram's 160 columns are reused by W and U once A and P are read
constexpr uint32_t TM_S = 0, TM_G = 128, TM_W = 128, TM_U = 192, TM_Y = 288, TM_Z = 352;

// the thread that issues (1b): lane 0 of warp 12, whose lane quarter (key rows of blocks 0-1)
// needs only three A/P loads, dealt to warpgroups 0-2
constexpr int Y_ISSUER = 384;

template <bool F16>
__device__ __forceinline__ float to_f(uint16_t b)
{
    if constexpr (F16) return __half2float(*reinterpret_cast<const __half *>(&b));
    else return __uint_as_float((uint32_t)b << 16);
}

// 16-byte global -> shared asynchronous copy (both addresses 16-byte aligned)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// 8 consecutive floats from 32-byte aligned shared memory
__device__ __forceinline__ void lds8(const float *src, float (&x)[8])
{
    const float4 a = *reinterpret_cast<const float4 *>(src);
    const float4 b = *reinterpret_cast<const float4 *>(src + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// the bits of elements [8c, 8c + 8) of a row of `n` 16-bit values (zero past n)
__device__ __forceinline__ uint4 load_raw8(const uint16_t *row, int c, int n, bool vec)
{
    if (vec) return 8 * c < n ? __ldg(reinterpret_cast<const uint4 *>(row) + c) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int d = 8 * c + 2 * e;
        const uint32_t lo = d < n ? row[d] : 0u, hi = d + 1 < n ? row[d + 1] : 0u;
        w[e] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <bool F16>
__device__ __forceinline__ void unpack8(uint4 r, float (&x)[8])
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        x[2 * e] = to_f<F16>((uint16_t)(w[e] & 0xffffu));
        x[2 * e + 1] = to_f<F16>((uint16_t)(w[e] >> 16));
    }
}

// one state row (32 fp32 columns of block `blk`) into the bf16 S^T tile (K-major, dk across)
template <bool F16>
__device__ __forceinline__ void store_sb(uint8_t *sb, int dv, int blk, const float (&x)[32])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int ch = 4 * (blk & 1) + q;   // 16-byte chunk within the 64-dk k-block
        *reinterpret_cast<uint4 *>(sb + (blk >> 1) * 16384 + sw128(dv, ch)) = pack8<F16>(x + 8 * q);
    }
}

// block (I, J) of T (times sgn) into Tb = T diag(beta) (bf16, K-major, 128B-swizzled)
template <bool F16>
__device__ __forceinline__ void blk_store_tb(const float (&acc)[2][4], float sgn, int I, int J,
                                             const float *beta, uint8_t *tb)
{
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int j = 16 * J + 8 * nh + 2 * t;
        const float b0 = beta[j], b1 = beta[j + 1];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const uint32_t off = sw128(16 * I + g + 8 * hh, j >> 3) + (uint32_t)(j & 7) * 2u;
            *reinterpret_cast<uint32_t *>(tb + off) =
                pack2<F16>(sgn * acc[nh][2 * hh] * b0, sgn * acc[nh][2 * hh + 1] * b1);
        }
    }
}

// a chunk's raw log-decays (rows of Dk floats, zero past the request's ln tokens and past Dk)
// into dst fp32 [64][128]: asynchronous 16-byte copies when rows are 16-byte multiples
__device__ __forceinline__ void stage_g(float *dst, const GdnPrefillArgs &p, int64_t t0, int ln, int h)
{
    const int Dk = p.Dk, Hv = p.Hv;
    if ((Dk & 3) == 0) {
        const int pieces = Dk >> 2;
        for (int u = threadIdx.x; u < C * 32; u += NT) {
            const int i = u >> 5, c4 = u & 31;
            float *d = dst + i * 128 + 4 * c4;
            if (i < ln && c4 < pieces)
                cp_async16(smem_u32(d), p.g + ((t0 + i) * Hv + h) * (int64_t)Dk + 4 * c4);
            else
                *reinterpret_cast<float4 *>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    } else {
        for (int u = threadIdx.x; u < C * 128; u += NT) {
            const int i = u >> 7, d = u & 127;
            dst[u] = (i < ln && d < Dk) ? __ldg(p.g + ((t0 + i) * Hv + h) * (int64_t)Dk + d) : 0.f;
        }
    }
}

// bounded wait for the phase of `wbar` with parity `parity`
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t wbar, uint32_t parity)
{
    bool good = mbar_try_wait(wbar, parity);
    if (!good) {
        const long long t0 = clock64();
        while (!(good = mbar_try_wait(wbar, parity)))
            if (clock64() - t0 > (1ll << 31)) break;
    }
    return good;
}

// thread 0 waits (bounded) on `wbar` for the MMA group committed to it, and also on `wbar2`
// when given; every thread gets the outcome.  (Checked builds with GDN_DEV_TEST_STALL pass,
// once, a barrier that nothing arrives on instead of the commit barrier, with `fresh` set: a
// barrier that has completed no phase is waited on with parity 0, since parity 1 would name
// the phase before its first, which counts as complete.)
__device__ __forceinline__ bool cta_wait_mma(uint32_t wbar, uint32_t &phase, volatile int *flag,
                                             int32_t *status, uint32_t wbar2 = 0,
                                             uint32_t *phase2 = nullptr, bool fresh = false)
{
    if (threadIdx.x == 0) {
        bool good = mbar_wait_bounded(wbar, fresh ? 0u : (phase & 1));
        if (good && wbar2) good = mbar_wait_bounded(wbar2, *phase2 & 1);
        if (!good && status) atomicOr(status, GDN_DEV_TIMEOUT);
        *flag = good ? 1 : 0;
    }
    ++phase;
    if (wbar2) ++*phase2;
    __syncthreads();
    const bool good = *flag != 0;
    tc_fence_after();
    return good;
}

template <bool F16>
__global__ void __launch_bounds__(NT, 1) gdn_prefill_kd_kernel(const __grid_constant__ GdnPrefillArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int wg = tid >> 7, lt = tid & 127;   // warpgroup; TMEM lane = state row
    const int Hv = p.Hv, Hq = p.Hq, Dk = p.Dk, Dv = p.Dv;
    // CTAs take the (request, head) units longest request first (ties by request index), so
    // that the chains of the longest requests start in the first wave of CTAs
    int b = blockIdx.x / Hv;
    const int h = blockIdx.x - b * Hv;
    if (p.cu_seqlens && p.B > 1 && p.B <= NT) {
        int *lens = reinterpret_cast<int *>(smem + OFF_KG);     // scratch before the first chunk
        int *pick = reinterpret_cast<int *>(smem + OFF_BAR + 32);
        if (tid < p.B) {
            const int64_t st = gdn::clamp_i64(p.cu_seqlens[tid], 0, p.N);
            const int64_t en = gdn::clamp_i64(p.cu_seqlens[tid + 1], 0, p.N);
            lens[tid] = en > st ? (int)(en - st) : 0;
        }
        __syncthreads();
        if (tid < p.B) {
            const int li = lens[tid];
            int rank = 0;
            for (int j2 = 0; j2 < p.B; ++j2) {
                const int lj = lens[j2];
                rank += (lj > li) || (lj == li && j2 < tid);
            }
            if (rank == b) *pick = tid;
        }
        __syncthreads();
        b = *pick;
    }
    const int qh = (int)(((int64_t)h * Hq) / Hv);
    const bool retrieval = p.has_retrieval != 0;

    int64_t start, end;
    if (p.cu_seqlens) {
        start = gdn::clamp_i64(p.cu_seqlens[b], 0, p.N);
        end = gdn::clamp_i64(p.cu_seqlens[b + 1], 0, p.N);
    } else {
        const int64_t S = p.N / p.B;
        start = (int64_t)b * S;
        end = start + S;
    }
    const int len = end > start ? (int)(end - start) : 0;
    const int nc = (len + C - 1) / C;
    const int64_t soff = ((int64_t)b * Hv + h) * Dv * (int64_t)Dk;
    if constexpr (gdn::kChecked) {
        if (!gdn::in_range(start, len, p.N, p.dev_status) || !gdn::in_range(qh, 1, Hq, p.dev_status) ||
            !gdn::in_range(soff, (int64_t)Dv * Dk, (int64_t)p.B * Hv * Dv * Dk, p.dev_status))
            return;
    }

    const uint16_t *kg = static_cast<const uint16_t *>(p.k);
    const uint16_t *qg = static_cast<const uint16_t *>(p.q);
    const uint16_t *vg = static_cast<const uint16_t *>(p.v);
    uint16_t *og = static_cast<uint16_t *>(p.out);
    const bool kvec = (Dk & 7) == 0, vvec = (Dv & 7) == 0;

    const uint32_t bar = sbase + OFF_BAR;
    const uint32_t bar_y = sbase + OFF_BAR + 40;   // commits of (1b), issued by Y_ISSUER
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8);
    volatile int *flag = reinterpret_cast<volatile int *>(smem + OFF_BAR + 12);
    // checked builds, GDN_DEV_TEST_STALL: CTA 0's wait for its first (W, U~) group runs on a
    // barrier that nothing arrives on, so it runs out and the CTA leaves through the timeout
    // path while (1b) and, in a request of more than one chunk, the next decay tile's copies
    // are in flight
    uint32_t stall_bar = (blockIdx.x == 0 && gdn::test_stall_requested(p.dev_status)) ? sbase + OFF_BAR + 16 : 0u;
    float *G2 = reinterpret_cast<float *>(smem + OFF_G2);
    float *solve = reinterpret_cast<float *>(smem + OFF_A);
    float *vec = reinterpret_cast<float *>(smem + OFF_VEC);
    float *rowv = reinterpret_cast<float *>(smem + OFF_ROW);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(sbase + OFF_BAR + 16, 1);
        mbar_init(bar_y, 1);
        fence_mbar_init();
        *flag = 1;
    }
    if (warp == 0) {
        tmem_alloc(sbase + OFF_BAR + 8, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);   // this warp's TMEM lanes
    uint32_t phase = 0, phase_y = 0;
    // a (1b) group was committed to bar_y (completing the phase of parity y_parity) and its
    // completion has not been seen yet
    bool y_pending = false;
    uint32_t y_parity = 0;

    // state S^T (row dv = lt, column blocks BPW wg .. BPW wg + BPW - 1) into TMEM, and its bf16
    // copy
    {
        float x[32];
#pragma unroll 1
        for (int blk = BPW * wg; blk < BPW * (wg + 1); ++blk) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int dk = 32 * blk + e;
                x[e] = (p.initial_state && lt < Dv && dk < Dk) ? p.initial_state[soff + (int64_t)lt * Dk + dk] : 0.f;
            }
            tmem_st32(tl + TM_S + 32 * blk, x);
            store_sb<F16>(smem + OFF_SB, lt, blk, x);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    constexpr uint32_t ID_G = idesc_f16kind(128, 160, 0, 0, !F16);
    constexpr uint32_t ID_WU = idesc_f16kind(128, 64, 1, 0, !F16);
    constexpr uint32_t ID_1A = idesc_f16kind(128, 64, 0, 1, !F16);
    constexpr uint32_t ID_1B = idesc_f16kind(128, 64, 0, 0, !F16);
    constexpr uint32_t ID_2 = idesc_f16kind(128, 128, 0, 1, !F16);
    constexpr uint32_t ID_3 = idesc_f16kind(128, 64, 0, 0, !F16);

    // the raw rows of chunk n (unit (token j, 8 dimensions 8c..8c+7), UNITS units per thread),
    // requested one chunk ahead, while the Gram runs: they travel while the rest of the chunk
    // runs.  A row's 16 units sit on 16 consecutive lanes; the first unit of a thread lies in
    // blocks 0-1 and the second, counted from the end, in blocks 3-2, so that every warp stores
    // the same number of stacked key rows (block I writes 4 - I of them).
    constexpr int UNITS = C * 16 / NT;
    static_assert(UNITS == 2, "unit map");
    uint4 rk8[UNITS], rq8[UNITS], rv8[UNITS];
    float rbeta = 0.f;   // beta of token tid (threads < 64), raw
    auto unit_of = [&](int it) { return it == 0 ? tid : 2 * NT - 1 - tid; };
    auto load_unit = [&](int n, int it) {
        const int64_t t0 = start + (int64_t)n * C;
        const int ln = min(C, len - n * C);
        const int u = unit_of(it), j = u >> 4, c = u & 15;
        if (j < ln) {
            const int64_t qk = ((t0 + j) * Hq + qh) * (int64_t)Dk;
            rk8[it] = load_raw8(kg + qk, c, Dk, kvec);
            rq8[it] = load_raw8(qg + qk, c, Dk, kvec);
            rv8[it] = load_raw8(vg + ((t0 + j) * Hv + h) * (int64_t)Dv, c, Dv, vvec);
        } else {
            rk8[it] = rq8[it] = rv8[it] = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto load_beta = [&](int n) {
        const int64_t t0 = start + (int64_t)n * C;
        const int ln = min(C, len - n * C);
        if (tid < C) rbeta = (tid < ln && retrieval) ? __ldg(p.beta + (t0 + tid) * Hv + h) : 0.f;
    };
    float *gn = reinterpret_cast<float *>(smem + OFF_GN);
    if (nc > 0) {
        load_beta(0);
#pragma unroll
        for (int it = 0; it < UNITS; ++it) load_unit(0, it);
        stage_g(gn, p, start, min(C, len), h);
    }

    bool ok = true;
    for (int n = 0; n < nc && ok; ++n) {
        const int64_t t0 = start + (int64_t)n * C;
        const int ln = min(C, len - n * C);

        // ---- this chunk's raw log-decays (staged during the previous chunk or before the loop)
        //      are in gn
        cp_async_wait_all();
        __syncthreads();
        // ---- per-dimension cumulative log-decay (log2 units) into G2: thread = key dimension,
        //      warpgroup wg holds tokens [16 wg, 16 wg + 16) in registers, publishes their
        //      total, and scans from the totals of the segments before it.  Segment wg is block
        //      I = wg, so the same thread has the block's reference M_I (its eighth token) and,
        //      in the last block, G_C.
        {
            const int d = lt;
            float gv[CPW];
#pragma unroll
            for (int e = 0; e < CPW; ++e) gv[e] = gn[(CPW * wg + e) * 128 + d];
            if (p.a_log) {
                const float ea = expf(__ldg(p.a_log + h)), dtb = __ldg(p.dt_bias + h);
#pragma unroll
                for (int e = 0; e < CPW; ++e)
                    if (CPW * wg + e < ln && d < Dk) gv[e] = -ea * gdn::softplus20(gv[e] + dtb);
            }
            float tot = 0.f;
#pragma unroll
            for (int e = 0; e < CPW; ++e) {
                // positions past the request or past Dk hold the zeros staged for them
                if (CPW * wg + e < ln && d < Dk) gv[e] = fmaxf(gv[e], G_FLOOR);
                gv[e] *= LOG2E;
                tot += gv[e];
            }
            if (wg < NWG - 1) vec[VEC_TOT + wg * 128 + d] = tot;
            __syncthreads();
            float acc = 0.f;
            for (int m = 0; m < wg; ++m) acc += vec[VEC_TOT + m * 128 + d];
            float mref = 0.f;
#pragma unroll
            for (int e = 0; e < CPW; ++e) {
                acc += gv[e];
                G2[(CPW * wg + e) * 128 + d] = acc;
                if (e == 7) mref = acc;
            }
            vec[VEC_M2 + wg * 128 + d] = mref;
            vec[VEC_EM + wg * 128 + d] = ex2_approx(mref);
            if (wg == NWG - 1) {
                vec[VEC_EC3 + d] = ex2_approx(acc - mref);
                vec[VEC_GC + d] = ex2_approx(acc);
            }
        }
        if (tid < C) {
            float bt = 0.f;
            if (tid < ln) {
                bt = retrieval ? rbeta : 1.f;
                if (retrieval && p.beta_sigmoid) bt = gdn::sigmoidf_(bt);
            }
            rowv[ROW_BETA + tid] = bt;
        }
        __syncthreads();
        // e^{M_I2 - M_I} for I < I2 (pair index I2 (I2 - 1) / 2 + I), per key dimension; the
        // segment totals above are read by now
        for (int u = tid; u < 6 * 128; u += NT) {
            const int pr = u >> 7, d = u & 127;
            const int I2 = pr < 1 ? 1 : (pr < 3 ? 2 : 3);
            const int I = pr - I2 * (I2 - 1) / 2;
            vec[VEC_CM + pr * 128 + d] = ex2_approx(vec[VEC_M2 + I2 * 128 + d] - vec[VEC_M2 + I * 128 + d]);
        }
        __syncthreads();

        // ---- operand tiles from the raw rows; a row's 16 units sit on 16 consecutive lanes,
        //      so its norms come from a 16-lane reduction.  q_j . k_j (from the raw bytes) is
        //      kept for the diagonal of P: its decay factor is 1, and taken from the
        //      bf16-rounded decayed operands its value would carry their rounding relative to
        //      |q^||k^| rather than to the product, which near-orthogonal q and k make small.
#pragma unroll
        for (int it = 0; it < UNITS; ++it) {
            const int u = unit_of(it), j = u >> 4, c = u & 15;
            const int I = j >> 4;
            float kx[8], qx[8];
            unpack8<F16>(rk8[it], kx);
            unpack8<F16>(rq8[it], qx);
            const uint4 v8 = rv8[it];   // v enters its tile as it is (the tile has v's type)
            float ssk = 0.f, ssq = 0.f, sqk = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                ssk = fmaf(kx[e], kx[e], ssk);
                ssq = fmaf(qx[e], qx[e], ssq);
                sqk = fmaf(qx[e], kx[e], sqk);
            }
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) {
                ssk += __shfl_xor_sync(0xffffffffu, ssk, m);
                ssq += __shfl_xor_sync(0xffffffffu, ssq, m);
                sqk += __shfl_xor_sync(0xffffffffu, sqk, m);
            }
            const float rk = p.qk_l2norm ? 1.0f / sqrtf(ssk + 1e-12f) : 1.f;
            const float rq = p.qk_l2norm ? 1.0f / sqrtf(ssq + 1e-12f) : 1.f;
            if (c == 0) rowv[ROW_QK + j] = rq * rk * sqk;

            float g2[8], mI[8], em[8];
            lds8(G2 + j * 128 + 8 * c, g2);
            lds8(vec + VEC_M2 + I * 128 + 8 * c, mI);
            lds8(vec + VEC_EM + I * 128 + 8 * c, em);
            float ak[8], aq[8], kgm[8], qgm[8], bk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float f = ex2_approx(g2[e] - mI[e]);    // e^{G_j - M_I}
                const float kh = kx[e] * rk;
                ak[e] = kh * f;
                aq[e] = qx[e] * rq * f;
                kgm[e] = ak[e] * em[e];                        // k^ e^{G_j}
                qgm[e] = aq[e] * em[e];
                bk[e] = kh * ex2_approx(mI[e] - g2[e]);        // k^ e^{M_I - G_j}
            }
            const uint32_t kb = (uint32_t)(c >> 3) , ch = (uint32_t)(c & 7);
            *reinterpret_cast<uint4 *>(smem + OFF_ASIDE + kb * ASIDE_KB + sw128(j, ch)) = pack8<F16>(ak);
            *reinterpret_cast<uint4 *>(smem + OFF_ASIDE + kb * ASIDE_KB + sw128(64 + j, ch)) = pack8<F16>(aq);
            *reinterpret_cast<uint4 *>(smem + OFF_KG + kb * TILE_KB + sw128(j, ch)) = pack8<F16>(kgm);
            *reinterpret_cast<uint4 *>(smem + OFF_QG + kb * TILE_KB + sw128(j, ch)) = pack8<F16>(qgm);
            *reinterpret_cast<uint4 *>(smem + OFF_VT + kb * TILE_KB + sw128(j, ch)) = v8;
            // key operand of every block I2 >= I: k^ e^{M_I2 - G_j} = bk e^{M_I2 - M_I}; the
            // last one also gives k^ e^{G_C - G_j} = k^ e^{M_3 - G_j} e^{G_C - M_3}
#pragma unroll
            for (int I2 = I; I2 < 4; ++I2) {
                float bb[8];
                if (I2 == I) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) bb[e] = bk[e];
                } else {
                    float cm[8];
                    lds8(vec + VEC_CM + (I2 * (I2 - 1) / 2 + I) * 128 + 8 * c, cm);
#pragma unroll
                    for (int e = 0; e < 8; ++e) bb[e] = bk[e] * cm[e];
                }
                const int row = 8 * I2 * (I2 + 1) + j;   // 16 * I2 (I2 + 1) / 2 + j
                *reinterpret_cast<uint4 *>(smem + OFF_BCAT + kb * BCAT_KB + sw128(row, ch)) = pack8<F16>(bb);
                if (I2 == 3) {
                    float kd[8], ec[8];
                    lds8(vec + VEC_EC3 + 8 * c, ec);
#pragma unroll
                    for (int e = 0; e < 8; ++e) kd[e] = bb[e] * ec[e];
                    *reinterpret_cast<uint4 *>(smem + OFF_KD + kb * TILE_KB + sw128(j, ch)) = pack8<F16>(kd);
                }
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- (G): all blocks' products in one MMA
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dA = sdesc_sw128(sbase + OFF_ASIDE, 16, 1024);
            const uint64_t dB = sdesc_sw128(sbase + OFF_BCAT, 16, 1024);
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16(tmem + TM_G, dA + (((kk >> 2) * ASIDE_KB + (kk & 3) * 32) >> 4),
                          dB + (((kk >> 2) * BCAT_KB + (kk & 3) * 32) >> 4), ID_G, kk > 0);
            umma_commit(bar);
        }
        // the next chunk's rows are requested while the Gram runs; the issuing thread's warp
        // requests its own after the wait, when the others' requests have left the queue
        auto load_next = [&] {
            if (n + 1 < nc) {
                load_beta(n + 1);
#pragma unroll
                for (int it = 0; it < UNITS; ++it) load_unit(n + 1, it);
            }
        };
        if (warp != 0) load_next();
        ok = cta_wait_mma(bar, phase, flag, p.dev_status);
        if (!ok) break;
        if (warp == 0) load_next();
        if (n + 1 < nc) stage_g(gn, p, t0 + C, min(C, len - (n + 1) * C), h);

        // ---- (1b) Y = S^T (Q^ e^G)^T needs only the state's bf16 copy and this chunk's tile:
        //      a thread of a warp that has no A/P load issues it while the tensor pipe is idle,
        //      with a commit to its own barrier, which the output phase waits for
        if (tid == Y_ISSUER) {
            const uint64_t dSB = sdesc_sw128(sbase + OFF_SB, 16, 1024);
            const uint64_t dQG = sdesc_sw128(sbase + OFF_QG, 16, 1024);
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk)
                umma_bf16(tmem + TM_Y, dSB + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                          dQG + (((kk >> 2) * TILE_KB + (kk & 3) * 32) >> 4), ID_1B, kk > 0);
            umma_commit(bar_y);
        }
        y_pending = true;
        y_parity = phase_y & 1;

        // ---- A (key rows, fp32) and P (query rows, bf16 tile) from the Gram; TMEM lane = row.
        //      The lanes of warp quarter g4 hold the key (g4 < 2) or query rows of blocks 2h and
        //      2h + 1 (h = g4 & 1), whose key columns are contiguous in the Gram: 3 loads of 16
        //      columns from column 0 (h = 0) or 7 from column 48 (h = 1), dealt to the four
        //      warpgroups; each load belongs to one block and serves that block's 16 lanes
        {
            const int g4 = warp & 3, hb = g4 & 1;
            const bool isq = g4 >= 2;
            const int i = lt & 63;
            const int myI = i >> 4;
            const float bi = rowv[ROW_BETA + i];
            uint8_t *P = smem + OFF_P;
            const int nld = hb ? 7 : 3;
#pragma unroll 1
            for (int ld = wg; ld < nld; ld += NWG) {
                const int col = (hb ? 48 : 0) + 16 * ld;
                float x[16];
                tmem_ld16(tl + TM_G + col, x);
                tmem_wait_ld();
                const int I = hb ? (ld < 3 ? 2 : 3) : (ld < 1 ? 0 : 1);
                if (myI != I) continue;
                const int blk = (col - 8 * I * (I + 1)) >> 4;   // key block of these columns
                const int j0 = 16 * blk;
                if (!isq) {
                    float *row = solve + (blk == I ? I : a_slot(I, blk)) * SOLVE_BLK + (i & 15) * SOLVE_LD;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int j = j0 + 4 * q4 + e;
                            y[e] = (retrieval && j < i) ? bi * x[4 * q4 + e] : 0.f;
                        }
                        *reinterpret_cast<float4 *>(row + 4 * q4) = make_float4(y[0], y[1], y[2], y[3]);
                    }
                } else {
                    // the diagonal from the raw bytes in fp32: rq_i rk_i (q_i . k_i)
                    const float pii = rowv[ROW_QK + i];
                    float y[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) y[e] = (j0 + e < i) ? x[e] : (j0 + e == i ? pii : 0.f);
                    *reinterpret_cast<uint4 *>(P + sw128(i, 2 * blk)) = pack8<F16>(y);
                    *reinterpret_cast<uint4 *>(P + sw128(i, 2 * blk + 1)) = pack8<F16>(y + 8);
                }
            }
            // P blocks right of the row's own block are zero (the solve reads no A block there);
            // the last warpgroup writes them for the query rows
            if (isq && wg == NWG - 1)
                for (int blk = myI + 1; blk < 4; ++blk) {
                    *reinterpret_cast<uint4 *>(P + sw128(i, 2 * blk)) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(P + sw128(i, 2 * blk + 1)) = make_uint4(0u, 0u, 0u, 0u);
                }
        }
        tc_fence_before();
        __syncthreads();

        // ---- T = (I + A)^-1 by blocks, written as Tb = T diag(beta) (bf16 B operand of (W),
        //      (U~)); the blocks above the diagonal of Tb are zero
        {
            const float *beta = rowv + ROW_BETA;
            uint8_t *tb = smem + OFF_TB;
            {
                // diagonal inverses D_I = (I + A_II)^-1 by a column sweep: warps 4I .. 4I + 3
                // take block I, and lane (row r, half) holds row r of columns c0 and c0 + 1
                // (c0 = 4 (warp & 3) + 2 half).  At step m the lanes of row m, final by then,
                // broadcast their entries and every later row subtracts A_rm times them.
                const int lane = tid & 31;
                const int I = warp >> 2, r = lane & 15;
                const int c0 = 4 * (warp & 3) + 2 * (lane >> 4);
                const float *Ar = solve + I * SOLVE_BLK + r * SOLVE_LD;
                float a[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 v = *reinterpret_cast<const float4 *>(Ar + 4 * q4);
                    a[4 * q4] = v.x;
                    a[4 * q4 + 1] = v.y;
                    a[4 * q4 + 2] = v.z;
                    a[4 * q4 + 3] = v.w;
                }
                float x0 = (r == c0) ? 1.f : 0.f, x1 = (r == c0 + 1) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < 15; ++m) {
                    const float y0 = __shfl_sync(0xffffffffu, x0, (lane & 16) | m);
                    const float y1 = __shfl_sync(0xffffffffu, x1, (lane & 16) | m);
                    if (m < r) {
                        x0 = fmaf(-a[m], y0, x0);
                        x1 = fmaf(-a[m], y1, x1);
                    }
                }
                float *Db = solve + (10 + I) * SOLVE_BLK;
                *reinterpret_cast<float2 *>(Db + r * SOLVE_LD + c0) = make_float2(x0, x1);
                const int j = 16 * I + c0;
                *reinterpret_cast<uint32_t *>(tb + sw128(16 * I + r, j >> 3) + (j & 7) * 2) =
                    pack2<F16>(x0 * beta[j], x1 * beta[j + 1]);
                // zero blocks above the diagonal: (I, J) with J > I, 16 rows x 32 bytes each
                for (int u = tid; u < 6 * 16 * 2; u += NT) {
                    const int pr = u >> 5, rr = (u >> 1) & 15, hf = u & 1;
                    const int Iz = pr < 3 ? 0 : (pr < 5 ? 1 : 2);
                    const int Jz = pr < 3 ? 1 + pr : (pr < 5 ? pr - 1 : 3);
                    *reinterpret_cast<uint4 *>(tb + sw128(16 * Iz + rr, 2 * Jz + hf)) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            __syncthreads();
            // T_10 = -D_1 (A_10 D_0) (warp 0), T_32 = -D_3 (A_32 D_2) (warp 1)
            if (warp < 2) {
                float *tmp = solve + (warp ? 15 : 14) * SOLVE_BLK;
                float acc[2][4] = {};
                blk_mma(acc, solve + (warp ? 5 : 4) * SOLVE_BLK, solve + (warp ? 12 : 10) * SOLVE_BLK);
                blk_store(tmp, acc, 1.f);
                __syncwarp();
                float acc2[2][4] = {};
                blk_mma(acc2, solve + (warp ? 13 : 11) * SOLVE_BLK, tmp);
                __syncwarp();
                blk_store(tmp, acc2, -1.f);
                blk_store_tb<F16>(acc2, -1.f, warp ? 3 : 1, warp ? 2 : 0, beta, tb);
            }
            __syncthreads();
            // lower-left 2 x 2 of blocks: X = A_BA T_AA (slots 2p+q), then T_BA = -T_BB X
#pragma unroll 1
            for (int ph = 0; ph < 2; ++ph) {
                const int pp = (warp >> 1) & 1, q = warp & 1;
                const float *X0, *Y0, *X1 = nullptr, *Y1 = nullptr;
                if (ph == 0) {
                    if (q == 0) {
                        X0 = solve + a_slot(2 + pp, 0) * SOLVE_BLK; Y0 = solve + 10 * SOLVE_BLK;
                        X1 = solve + a_slot(2 + pp, 1) * SOLVE_BLK; Y1 = solve + 14 * SOLVE_BLK;
                    } else {
                        X0 = solve + a_slot(2 + pp, 1) * SOLVE_BLK; Y0 = solve + 11 * SOLVE_BLK;
                    }
                } else {
                    if (pp == 0) {
                        X0 = solve + 12 * SOLVE_BLK; Y0 = solve + q * SOLVE_BLK;
                    } else {
                        X0 = solve + 15 * SOLVE_BLK; Y0 = solve + q * SOLVE_BLK;
                        X1 = solve + 13 * SOLVE_BLK; Y1 = solve + (2 + q) * SOLVE_BLK;
                    }
                }
                if (warp < 4) {
                    float acc[2][4] = {};
                    const int np = X1 ? 2 : 1;
#pragma unroll 1
                    for (int t = 0; t < np; ++t) blk_mma(acc, t ? X1 : X0, t ? Y1 : Y0);
                    if (ph == 0) blk_store(solve + (2 * pp + q) * SOLVE_BLK, acc, 1.f);
                    else blk_store_tb<F16>(acc, -1.f, 2 + pp, q, beta, tb);
                }
                __syncthreads();
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        // ---- (W), (U~)
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dKG = sdesc_sw128(sbase + OFF_KG, TILE_KB, 1024);
            const uint64_t dVT = sdesc_sw128(sbase + OFF_VT, TILE_KB, 1024);
            const uint64_t dTB = sdesc_sw128(sbase + OFF_TB, 16, 1024);
            if (retrieval) {
#pragma unroll 1
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + TM_W, dKG + ((kk * 2048) >> 4), dTB + ((kk * 32) >> 4), ID_WU, kk > 0);
            }
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_U, dVT + ((kk * 2048) >> 4), dTB + ((kk * 32) >> 4), ID_WU, kk > 0);
            umma_commit(bar);
        }
        ok = cta_wait_mma(stall_bar ? stall_bar : bar, phase, flag, p.dev_status, 0, nullptr,
                          stall_bar != 0);
        stall_bar = 0;
        if (!ok) break;

        // ---- -W as the MN-major B operand of (1a): lane = dk row, tokens CPW wg .. + CPW - 1
        if (retrieval) {
            uint8_t *wn = smem + OFF_WNEG;
#pragma unroll
            for (int c16 = 0; c16 < CPW / 16; ++c16) {
                const int col = CPW * wg + 16 * c16;
                float x[16];
                tmem_ld16(tl + TM_W + col, x);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = -x[e];
                *reinterpret_cast<uint4 *>(wn + sw128(lt, col / 8)) = pack8<F16>(x);
                *reinterpret_cast<uint4 *>(wn + sw128(lt, col / 8 + 1)) = pack8<F16>(x + 8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- (1a) U^T += S^T (-W)^T
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dSB = sdesc_sw128(sbase + OFF_SB, 16, 1024);
            const uint64_t dWN = sdesc_sw128(sbase + OFF_WNEG, 8192, 1024);
            if (retrieval) {
#pragma unroll 1
                for (int kk = 0; kk < 8; ++kk)
                    umma_bf16(tmem + TM_U, dSB + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                              dWN + ((kk * 2048) >> 4), ID_1A, 1);
            }
            umma_commit(bar);
        }
        ok = cta_wait_mma(bar, phase, flag, p.dev_status);
        if (!ok) break;

        // ---- U^T -> bf16 A operand of (2), (3); the state's decay diag(e^{G_C}) on its columns
        {
            uint8_t *ub = smem + OFF_UB;
            float x[32];
#pragma unroll
            for (int c16 = 0; c16 < CPW / 16; ++c16) {
                const int col = CPW * wg + 16 * c16;
                float u16[16];
                tmem_ld16(tl + TM_U + col, u16);
                tmem_wait_ld();
                *reinterpret_cast<uint4 *>(ub + sw128(lt, col / 8)) = pack8<F16>(u16);
                *reinterpret_cast<uint4 *>(ub + sw128(lt, col / 8 + 1)) = pack8<F16>(u16 + 8);
            }
#pragma unroll 1
            for (int blk = BPW * wg; blk < BPW * (wg + 1); ++blk) {
                tmem_ld32(tl + TM_S + 32 * blk, x);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] *= vec[VEC_GC + 32 * blk + e];
                tmem_st32(tl + TM_S + 32 * blk, x);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- (2) S^T += U^T (K^ e^{G_C - G}), (3) Z = U^T P^T
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dUB = sdesc_sw128(sbase + OFF_UB, 16, 1024);
            const uint64_t dKD = sdesc_sw128(sbase + OFF_KD, TILE_KB, 1024);
            const uint64_t dP = sdesc_sw128(sbase + OFF_P, 16, 1024);
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_S, dUB + ((kk * 32) >> 4), dKD + ((kk * 2048) >> 4), ID_2, 1);
#pragma unroll 1
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16(tmem + TM_Z, dUB + ((kk * 32) >> 4), dP + ((kk * 32) >> 4), ID_3, kk > 0);
            umma_commit(bar);
        }
        ok = cta_wait_mma(bar, phase, flag, p.dev_status, bar_y, &phase_y);
        if (ok) y_pending = false;
        if (!ok) break;

        // ---- outputs O^T = scale (Y + Z) (lane = dv, tokens CPW wg .. CPW wg + CPW - 1), then
        //      the new state's bf16 copy (column blocks BPW wg .. BPW wg + BPW - 1)
        {
            float y[CPW], z[CPW];
            {
                // 8 tokens at a time through a warp-private [8 tokens][32 dv] scratch (the solve
                // area is free by now), then one 16-byte store per lane: lanes 4t..4t+3 write
                // token t's 64 bytes of this warp's dv
#pragma unroll
                for (int c16 = 0; c16 < CPW / 16; ++c16) {
                    float y16[16], z16[16];
                    tmem_ld16(tl + TM_Y + CPW * wg + 16 * c16, y16);
                    tmem_ld16(tl + TM_Z + CPW * wg + 16 * c16, z16);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        y[16 * c16 + e] = y16[e];
                        z[16 * c16 + e] = z16[e];
                    }
                }
                const int lane = tid & 31;
                uint8_t *ost = smem + OFF_A + 512 * warp;
                const int tt = lane >> 2, dvc = 32 * (warp & 3) + 8 * (lane & 3);
#pragma unroll
                for (int g8 = 0; g8 < CPW / 8; ++g8) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        *reinterpret_cast<uint16_t *>(ost + e * 64 + lane * 2) =
                            elem16<F16>(p.scale * (y[8 * g8 + e] + z[8 * g8 + e]));
                    __syncwarp();
                    const uint4 v = *reinterpret_cast<const uint4 *>(ost + lane * 16);
                    __syncwarp();
                    const int i = CPW * wg + 8 * g8 + tt;
                    if (i < ln && dvc < Dv) {
                        uint16_t *dst = og + ((t0 + i) * Hv + h) * (int64_t)Dv + dvc;
                        if (vvec) {
                            *reinterpret_cast<uint4 *>(dst) = v;
                        } else {
                            const uint16_t *ve = reinterpret_cast<const uint16_t *>(&v);
                            for (int e = 0; e < 8 && dvc + e < Dv; ++e) dst[e] = ve[e];
                        }
                    }
                }
            }
#pragma unroll 1
            for (int blk = BPW * wg; blk < BPW * (wg + 1); ++blk) {
                float x[32];
                tmem_ld32(tl + TM_S + 32 * blk, x);
                tmem_wait_ld();
                store_sb<F16>(smem + OFF_SB, lt, blk, x);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (ok) {
        // final state (V-major, fp32); an empty request copies its initial state through
        float x[32];
#pragma unroll 1
        for (int blk = BPW * wg; blk < BPW * (wg + 1); ++blk) {
            tmem_ld32(tl + TM_S + 32 * blk, x);
            tmem_wait_ld();
            if (lt < Dv)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int dk = 32 * blk + e;
                    if (dk < Dk) p.final_state[soff + (int64_t)lt * Dk + dk] = x[e];
                }
        }
    } else if (tid == 0) {
        // a wait ran out: give the MMAs in flight a last bounded chance before TMEM is freed
        const long long t0 = clock64();
        while (!mbar_try_wait(bar, (phase - 1) & 1))
            if (clock64() - t0 > (1ll << 24)) break;
        if (y_pending) {
            const long long t1 = clock64();
            while (!mbar_try_wait(bar_y, y_parity))
                if (clock64() - t1 > (1ll << 24)) break;
        }
    }
    // a CTA that left mid-chunk may still have the next decay tile's copies in flight
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace gdn_kd

bool prefill_kd_supported(const GdnPrefillArgs &a)
{
    return a.g_per_key && a.has_decay && a.dtype == GDN_BF16 && a.Dk >= 8 && a.Dk <= 128 &&
           a.Dv >= 8 && a.Dv <= 128;
}

cudaError_t launch_prefill_kd(const GdnPrefillArgs &a, cudaStream_t stream)
{
    using namespace gdn_kd;
    if (a.B == 0 || a.Hv == 0) return cudaSuccess;
    static DeviceOnce smem_opt_in;
    cudaError_t e = smem_opt_in.run([] {
        return cudaFuncSetAttribute(gdn_prefill_kd_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    });
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)a.B * (unsigned)a.Hv;
    gdn_prefill_kd_kernel<false><<<grid, NT, SMEM_BYTES, stream>>>(a);
    return cudaGetLastError();
}
