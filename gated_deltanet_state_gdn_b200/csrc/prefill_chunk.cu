// prefill_chunk.cu -- chunked Gated DeltaNet prefill on sm_100a tensor cores.
//
// Operation: the recurrence of "com.microsoft.GatedDeltaNet" (Description),
//   S_t = exp(g_t) S_{t-1} + k_t (beta_t (v_t - exp(g_t) S_{t-1}^T k_t))^T,
//   o_t = scale * S_t^T q_t,
// for bf16 or fp16 q/k/v with Dk, Dv <= 128 (smaller heads are read as 128-wide
// tiles zero-filled past their end, by the TMA when Dk and Dv are multiples of 8 and
// Hv % 4 == 0, else by plain loads of the TMA warp; zero padding leaves every product
// unchanged), computed 64 tokens at a time.  The
// chunk form (derived from the recurrence; the op page names a chunk-parallel
// prefill with chunk_size 64 and states that the chunk size does not change
// the result) is, for a chunk with incoming state S0 (Dk x Dv), cumulative
// log-decay G_i = sum_{l<=i} g_l, Gamma_i = exp(G_i), and (optionally) the
// L2-normalised rows k^_i = rk_i k_i, q^_i = rq_i q_i:
//   A_ij = beta_i (k^_i . k^_j) exp(G_i - G_j)   (j < i),   T = (I + A)^-1
//   W    = T diag(beta Gamma) K^,   U~ = T diag(beta) V
//   U    = U~ - W S0
//   O    = scale (diag(Gamma) Q^ S0 + P U),  P_ij = (q^_i . k^_j) exp(G_i - G_j) (j <= i)
//   S_C  = Gamma_C S0 + (diag(exp(G_C - G)) K^)^T U
// The op's update_rule variants reuse the same products: without decay g = 0;
// without the delta retrieval A = 0 (T = I) and W = 0, so U = diag(beta) V with
// beta = 1 (the rule has no beta input).  The qwen gate and the sigmoid beta
// are applied to the per-token gate values before the prefix sum.
// The norms rk, rq are never applied to the bf16 q/k tiles, so the tensor cores
// always read the caller's bytes.  With D = diag(rk), A = diag(beta rk) B D for
// the raw key products B = (K K^T) * decay, and (I + A)^-1 = D^-1 (I + A')^-1 D
// with A' = diag(beta rk^2) B: every row of A' needs only its own norm, rk_i^2 =
// 1 / (k_i . k_i + eps), read from the Gram diagonal.  Carrying U' = D U instead
// of U, the column norms land in the T' tiles and cancel elsewhere:
//   T'  = (I + A')^-1,  Tb = T' diag(beta rk),  Tbg = T' diag(beta Gamma rk^2)
//   U'  = Tb V - Tbg K S0                       (= D U)
//   S_C = Gamma_C S0 + (diag(exp(G_C - G)) K)^T U'
//   O   = scale (diag(Gamma rq) Q S0 + P' U'),  P'_ij = rq_i (q_i . k_j) exp(G_i - G_j)
// All state-dependent products are evaluated transposed (rows = value index
// dv), so every tcgen05 MMA here has M = 128:
//   (G)  [K; Q] K^T                         -> TMEM  (Gram, 128 x 64)
//   (W)  W^T  = K^T . Tbg^T                 -> TMEM
//   (U~) U^T  = V^T . Tb^T                  -> TMEM
//   (1a) U^T += S^T . (-W)^T                 (bf16 copy of S^T from TMEM)
//   (1b) Y    = S^T . Q^T
//   (2)  S^T += (U^T diag(exp(G_C - G))) . K  (fp32 accumulator stays in TMEM)
//   (3)  Z    = U^T . P'^T
//   O^T = scale (Y diag(Gamma rq) + Z)
// TMEM (512 columns): S^T [0,128) | U^T [128,192) | Y [192,256) | Z [256,320) |
// Gram [320,384) | W^T [384,448) | bf16 S^T [448,512) (A of 1a/1b, 8 columns per
// 16 dk).  After U^T is read, its columns hold the bf16 A operands of (2) and (3)
// (per 16 tokens: 8 columns of U, then 8 of the decayed U).
//
// CTA = 15 warps, one (request, value head) unit at a time, persistent over a
// longest-first unit list:
//   warps 0-3   state warpgroup: TMEM <-> bf16 operand tiles, outputs, state I/O
//   warps 4-7   prep front: gates, query norms, Gram -> A' (with the key norms) and P'
//   warps 8-11  prep back: the 64x64 unit-triangular solve and the bf16 T' tiles
//               (front and back work on consecutive chunks, ahead of the state chain)
//   warp  12    TMA producers (lane 0: q/k/g/beta tiles in three stages; lane 1: v tiles)
//   warp  13    TMEM owner; UMMA issuer of the state chain (1a, 1b, 2, 3)
//   warp  14    UMMA issuer of the prep stream (G, W, U~)
// Every wait on an mbarrier is bounded (2^31 cycles) and also ends as soon as another
// role has raised the CTA's abort flag; a wait that runs out raises the flag and sets
// GDN_DEV_TIMEOUT in the status word.  After an abort every thread still reaches the same
// barriers: each of the three 128-thread groups (state, prep front, prep back) runs one
// control flow in which a failed wait only clears `ok` (named barriers and warp-collective
// tcgen05.ld/st are reached on every path) and leaves its chunk loop through the per-chunk
// OR vote; the single-thread roles (TMA lanes, UMMA issuers) leave their loops on the flag;
// all threads then meet the CTA barrier that ends the batch and see the flag alike.  The
// teardown drains copies and MMAs still in flight (bounded) and frees TMEM.  Checked builds
// can force this path from the host (GDN_DEV_TEST_STALL).
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <cuda_fp16.h>

#include "common.cuh"
#include "seqpar.cuh"
#include "sm100.cuh"
#include "tile16.cuh"

using namespace sm100;

namespace gdn_chunk {

using gdn::in_range;
using gdn::kChecked;
using gdn_tile::a_slot;
using gdn_tile::blk_mma;
using gdn_tile::blk_store;
using gdn_tile::elem16;
using gdn_tile::pack2;
using gdn_tile::pack8;
using gdn_tile::SOLVE_BLK;
using gdn_tile::SOLVE_LD;
using gdn_tile::sw128;

constexpr int C = 64;       // chunk length (tokens)
constexpr int D = 128;      // Dk = Dv
constexpr int NTHREADS = 480;
constexpr int MAX_UNITS = 64;      // per CTA per batch of the unit list
constexpr int TMA_WARP = 12, MMA_WARP = 13, ISSUE_WARP = 14;   // warps 0-3 state, 4-11 prep
constexpr float G_FLOOR = -30.f;   // per-token log-decay floor (exp(-30) ~ 9e-14)
constexpr float LOG2E = 1.4426950408889634f;

// ---- shared-memory map (bytes from a 1024-aligned base) ----
constexpr int KQ_STAGES = 3;
constexpr uint32_t OFF_KQ0 = 0;          // KQ_STAGES x [kb][128 rows: K 0-63, Q 64-127][128 B]
constexpr uint32_t KQ_STAGE = 32768;     // bytes per KQ stage
constexpr uint32_t KQ_KB = 16384;        // k-block (64 dk) stride inside a KQ stage
constexpr uint32_t OFF_V = 98304;        // [dv half][64 rows j][128 B], 16 KB
constexpr uint32_t V_HALF = 8192;
constexpr uint32_t OFF_WNEG = 114688;    // [128 rows dk][64 i], 16 KB (MN-major B)
constexpr uint32_t OFF_P = 131072;       // KQ_STAGES x [64 rows i][64 j], 8 KB (stage = KQ stage)
constexpr uint32_t P_STAGE = 8192;
constexpr uint32_t OFF_TB = OFF_P + KQ_STAGES * P_STAGE;   // [64 rows i][64 j], 8 KB
constexpr uint32_t OFF_TBG = OFF_TB + 8192;
constexpr uint32_t SOLVE_BYTES = 16 * SOLVE_BLK * 4;   // 16 padded 16 x 16 fp32 blocks
constexpr uint32_t OFF_SOLVE0 = OFF_TBG + 8192;   // two areas of 16 blocks of 16 x 20 fp32
constexpr uint32_t OFF_SOLVE1 = OFF_SOLVE0 + SOLVE_BYTES;
constexpr uint32_t OFF_GB0 = OFF_SOLVE1 + SOLVE_BYTES;         // KQ_STAGES x (g tile 1 KB + beta tile 1 KB)
constexpr uint32_t GATE_BYTES = 2560;
constexpr uint32_t OFF_GATE = OFF_GB0 + KQ_STAGES * 2048;      // KQ_STAGES x processed gates
constexpr uint32_t OFF_UNITS = OFF_GATE + KQ_STAGES * GATE_BYTES;   // int4 x MAX_UNITS
constexpr uint32_t OFF_BARS = OFF_UNITS + MAX_UNITS * 16;
constexpr uint32_t NUM_BARS = 32;
static_assert(NUM_BARS * 8 <= 256, "barrier area");
constexpr uint32_t OFF_MISC = OFF_BARS + 256;                  // tmem base, abort flag, count
constexpr uint32_t OFF_OGR = OFF_MISC + 64;                    // Gamma_i rq_i for the outputs, 64 floats
constexpr uint32_t OFF_OST = OFF_OGR + 256;                    // output transpose, 512 B per state warp
constexpr uint32_t SMEM_USED = OFF_OST + 4 * 512;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;              // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(OFF_GB0 % 1024 == 0 && OFF_V % 1024 == 0 && OFF_WNEG % 1024 == 0 && OFF_TB % 1024 == 0 &&
              OFF_KQ0 + KQ_STAGES * KQ_STAGE <= OFF_V && OFF_V + 16384 <= OFF_WNEG, "alignment");

// gate-array offsets (floats) inside a GATE stage
constexpr int GA_G2 = 0;       // G_i * log2(e)
constexpr int GA_CF = 64;      // exp(Gend_J(i) - G_i): factor to the end of i's 16-block
constexpr int GA_BETA = 128;   // beta_i (0 beyond the request)
constexpr int GA_GAM = 192;    // exp(G_i)
constexpr int GA_DEC = 256;    // exp(G_C - G_i)
constexpr int GA_RQ = 384;     // query norm factor rq_i (1 without qk_l2norm)
constexpr int GA_GEND = 448;   // G_end of each 16-block * log2(e)  [4]
constexpr int GA_GC = 452;     // exp(G_C)
constexpr int GA_BG = 456;     // beta_i Gamma_i rk_i^2 (column scale of Tbg)
constexpr int GA_TB = 520;     // beta_i rk_i (column scale of Tb)
static_assert((GA_TB + 64) * 4 <= (int)GATE_BYTES, "gate stage size");

// barrier indices
enum {
    B_KQ_FULL = 0, B_KQ_EMPTY = 3, B_V_FULL = 6, B_V_EMPTY = 7, B_GATE_FULL = 8,
    B_GATE_EMPTY = 11, B_G_DONE = 14, B_T_READY = 15, B_W_DONE = 16, B_WNEG = 17,
    B_S_READY = 18, B_U_DONE = 19, B_E1 = 20, B_S_DONE = 21, B_Z_DONE = 22, B_Y_FREE = 23,
    B_G_FREE = 24, B_A_READY = 25, B_SOLVE_FREE = 27, B_UT_DONE = 29,
    B_DRAIN_CHAIN = 30, B_DRAIN_PREP = 31,   // abort teardown: each UMMA issuer's last commit
    B_COUNT = 32
};
static_assert(B_COUNT == (int)NUM_BARS, "barrier count");

// TMEM columns
constexpr uint32_t TM_S = 0, TM_U = 128, TM_Y = 192, TM_Z = 256, TM_G = 320, TM_W = 384, TM_SB = 448;

struct __align__(64) Params {
    CUtensorMap tm_q;     // (Dk, Hq, N) bf16 or fp16, box (64, 1, 64), 128B swizzle
    CUtensorMap tm_k;
    CUtensorMap tm_v;     // (128, Hv, N)
    CUtensorMap tm_g;     // (Hv, N) fp32, box (4, 64); encoded only with a decay input
    CUtensorMap tm_beta;  // encoded only with a beta input
    const int32_t *cu_seqlens;
    const float *initial_state;
    float *final_state;
    uint16_t *out;   // bf16 or fp16 bits, as the activations
    int32_t *dev_status;
    int64_t N;
    int32_t B, Hq, Hv;
    float scale;
    int32_t qk_l2norm;
    int32_t has_decay, has_retrieval, beta_sigmoid;   // update rule and activations
    int32_t Dk, Dv;   // head sizes (<= 128; the tiles are zero-padded to 128)
    const float *a_log, *dt_bias;                     // qwen gate when non-NULL
    // plain staging (head sizes that are not multiples of 8, or Hv % 4 != 0: rows whose
    // strides the tensor maps cannot describe): the TMA warp copies rows with ordinary loads
    int32_t stage_plain;
    const uint16_t *q, *k, *v;
    const float *g, *beta;
    // sequence-parallel split (seqpar.cuh): pass 1 or 3, the split rule's CTA count, workspace
    int32_t seq_pass, seq_G;
    float *seq_ws;
};

// --------------------------------------------------------------------------
struct Ctx {
    uint8_t *smem;
    uint32_t sbase;        // shared address of smem
    volatile int *abort_flag;
    int32_t *dev_status;

    __device__ uint32_t bar(int i) const { return sbase + OFF_BARS + 8u * i; }

    // bounded wait; returns false on timeout or when another role aborted
    __device__ bool wait(int b, uint32_t parity) const
    {
        if (mbar_try_wait(bar(b), parity)) return true;
        const long long t0 = clock64();
        while (true) {
            if (mbar_try_wait(bar(b), parity)) return true;
            if (*abort_flag) return false;
            if (clock64() - t0 > (1ll << 31)) {
                *abort_flag = 1;
                if (dev_status) atomicOr(dev_status, GDN_DEV_TIMEOUT);
                return false;
            }
        }
    }
    __device__ bool aborted() const { return *abort_flag != 0; }
};

struct Unit {
    int b, h, start, len;
};

__device__ __forceinline__ Unit load_unit(const uint8_t *smem, int k)
{
    const int4 u = reinterpret_cast<const int4 *>(smem + OFF_UNITS)[k];
    return Unit{u.x, u.y, u.z, u.w};
}

__device__ __forceinline__ int64_t clampi(int64_t x, int64_t lo, int64_t hi)
{
    return x < lo ? lo : (x > hi ? hi : x);
}

template <bool F16 = false>
__device__ __forceinline__ float sumsq8_bf16(uint4 r)
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float lo, hi;
        if constexpr (F16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            lo = f.x;
            hi = f.y;
        } else {
            lo = __uint_as_float(w[i] << 16);
            hi = __uint_as_float(w[i] & 0xffff0000u);
        }
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
    }
    return s;
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void st4(float *p, float a, float b, float c, float d)
{
    *reinterpret_cast<float4 *>(p) = make_float4(a, b, c, d);
}

// --------------------------------------------------------------------------
// Unit list: requests sorted by length (longest first), heads fastest; unit u
// goes to CTA (u mod G) on even waves and G-1-(u mod G) on odd waves.
// One TMEM lane's row of an initial state S0 (dv fixed, Dk entries, zero beyond; NULL: zero):
// its bf16 copy
// into the (1a)/(1b) A-operand columns and gC * S0 into the fp32 state columns.  Runs once per
// unit, out of line so that the per-chunk code stays compact.
template <bool GENERAL, bool F16, bool IDENT = false>
__device__ __noinline__ void load_state_tmem(const float *init, int Dk, uint32_t tl, float gC,
                                             int ident = -1)
{
#pragma unroll 1
    for (int hq = 0; hq < 2; ++hq) {
        float x[64];
        if (!GENERAL || (Dk & 3) == 0) {
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float4 v = init && (!GENERAL || 64 * hq + c < Dk) ? ld4(init + 64 * hq + c)
                                                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                x[c] = v.x; x[c + 1] = v.y; x[c + 2] = v.z; x[c + 3] = v.w;
            }
        } else {
            // rows of Dk floats with Dk % 4 != 0 are only 4-byte aligned
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = init && 64 * hq + c < Dk ? init[64 * hq + c] : 0.f;
        }
        // the identity's row `ident` (sequence-parallel transition runs; init is NULL then)
        if (IDENT && ident >= 0) {
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = 64 * hq + c == ident ? 1.f : x[c];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = pack2<F16>(x[16 * q + 2 * e], x[16 * q + 2 * e + 1]);
            tmem_st8u(tl + TM_SB + 8 * (4 * hq + q), w);
            float y[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) y[e] = x[16 * q + e] * gC;
            tmem_st16(tl + TM_S + 16 * (4 * hq + q), y);
        }
    }
}

// Few requests: every CTA runs the same greedy assignment (requests longest first; the Hv
// heads of a request go to the Hv CTAs with the least work so far, counted in chunks plus one
// per unit for the switch, ties to the lower index), so each CTA knows its own list.  Many
// requests: units in length order dealt to the CTAs wave by wave, alternating direction.
__device__ __forceinline__ bool greedy_schedule(const Params &p, int G)
{
    return p.B <= 32 && G <= 256 && p.B * ((p.Hv + G - 1) / G) <= MAX_UNITS;
}

// Units of a sequence-parallel pass (seqpar.cuh), one per CTA at most: every request in
// index order, its pseudo-requests in a fixed order, Hv heads each; CTA c takes unit c.  The
// unit's b field carries the request in bits 0-7, the segment in bits 8-11, the mode in bits
// 12-14 and whether the request is split in bit 15.
__device__ __noinline__ void build_seq_unit(const Params &p, uint8_t *smem, int *count_out)
{
    if (threadIdx.x == 0) {
        int rs[gdn_seq::MAX_REQ], rl[gdn_seq::MAX_REQ], nc[gdn_seq::MAX_REQ];
        for (int b = 0; b < p.B; ++b) {
            int64_t st, en;
            if (p.cu_seqlens) {
                st = clampi(p.cu_seqlens[b], 0, p.N);
                en = clampi(p.cu_seqlens[b + 1], 0, p.N);
            } else {
                const int64_t S = p.N / p.B;
                st = (int64_t)b * S;
                en = st + S;
            }
            rs[b] = (int)st;
            rl[b] = en > st ? (int)(en - st) : 0;
            nc[b] = (rl[b] + C - 1) / C;
        }
        const uint32_t mask = gdn_seq::split_mask(nc, p.B, p.Hv, p.seq_G);
        int4 *list = reinterpret_cast<int4 *>(smem + OFF_UNITS);
        int idx = 0, found = 0;
        for (int b = 0; b < p.B && !found; ++b) {
            const bool split = (mask >> b) & 1u;
            int s0 = 0, s1 = 0, s2 = 0;
            if (split) gdn_seq::segments(nc[b], s0, s1, s2);
            // pseudo-requests of this pass: (mode, segment, first token, tokens)
            int4 ps[3];
            int nps = 0;
            if (p.seq_pass == 1) {
                if (split) {
                    ps[nps++] = make_int4(gdn_seq::MODE_TRUE, 0, rs[b], s0 * C);
                    ps[nps++] = make_int4(gdn_seq::MODE_IDENT, 1, rs[b] + s0 * C, s1 * C);
                    ps[nps++] = make_int4(gdn_seq::MODE_ZERO, 1, rs[b] + s0 * C, s1 * C);
                } else {
                    ps[nps++] = make_int4(gdn_seq::MODE_TRUE, 0, rs[b], rl[b]);
                }
            } else if (split) {
                ps[nps++] = make_int4(gdn_seq::MODE_TRUE, 1, rs[b] + s0 * C, s1 * C);
                ps[nps++] = make_int4(gdn_seq::MODE_TRUE, 2, rs[b] + (s0 + s1) * C, rl[b] - (s0 + s1) * C);
            }
            for (int i = 0; i < nps && !found; ++i) {
                if ((int)blockIdx.x < idx + p.Hv) {
                    const int h = blockIdx.x - idx;
                    list[0] = make_int4(b | (ps[i].y << 8) | (ps[i].x << 12) | ((split ? 1 : 0) << 15), h,
                                        ps[i].z, ps[i].w);
                    found = 1;
                }
                idx += p.Hv;
            }
        }
        *count_out = found;
    }
    __syncthreads();
}

__device__ __noinline__ void build_unit_list(const Params &p, uint8_t *smem, int batch0,
                                             int *count_out)
{
    // scratch for up to 8192 ints: the two solve areas, idle between batches and written by
    // generic stores only (a TMA destination here would need a proxy fence before its next load)
    static_assert(2 * SOLVE_BYTES >= 8192 * 4 && OFF_SOLVE1 == OFF_SOLVE0 + SOLVE_BYTES, "unit scratch");
    int *ord = reinterpret_cast<int *>(smem + OFF_SOLVE0);
    const int B = p.B;
    const int tid = threadIdx.x;
    const bool sorted = B <= 8192;
    auto req_range = [&](int b, int &s, int &l) {
        int64_t st, en;
        if (p.cu_seqlens) {
            st = clampi(p.cu_seqlens[b], 0, p.N);
            en = clampi(p.cu_seqlens[b + 1], 0, p.N);
        } else {
            const int64_t S = p.N / B;
            st = (int64_t)b * S;
            en = st + S;
        }
        s = (int)st;
        l = en > st ? (int)(en - st) : 0;
    };
    // few requests: ranges read once into shared memory (starts, lengths after ord)
    const bool small = B <= 32;
    int *rs = ord + 32, *rl = ord + 64;
    if (small) {
        if (tid < B) req_range(tid, rs[tid], rl[tid]);
        __syncthreads();
    }
    if (sorted) {
        for (int b = tid; b < B; b += NTHREADS) {
            int sb, lb;
            if (small) {
                lb = rl[b];
            } else {
                req_range(b, sb, lb);
            }
            int rank = 0;
            for (int o = 0; o < B; ++o) {
                int so, lo;
                if (small) {
                    lo = rl[o];
                } else {
                    req_range(o, so, lo);
                }
                rank += (lo > lb) || (lo == lb && o < b);
            }
            ord[rank] = b;
        }
    }
    __syncthreads();
    const int G = gridDim.x;
    const int U = B * p.Hv;
    const int c = blockIdx.x;
    int4 *list = reinterpret_cast<int4 *>(smem + OFF_UNITS);
    if (greedy_schedule(p, G)) {
        // CTAs kept in order of (work so far, index), as packed 64-bit keys: a request's heads
        // go to the first Hv of the order; the order is then rebuilt by merging the untouched
        // tail with the updated head (both stay sorted), each thread placing one CTA with a
        // binary search into the other of two buffers (one barrier per step).
        long long *key = reinterpret_cast<long long *>(ord + 128);   // two buffers of G keys
        for (int i = tid; i < G; i += NTHREADS) key[i] = i;
        if (tid == 0) *count_out = 0;
        __syncthreads();
        int cur = 0;
        for (int r = 0; r < B; ++r) {
            const int b = ord[r];
            const int sb = rs[b], lb = rl[b];
            const long long cost = (long long)((lb + C - 1) / C + 1) << 32;
            for (int h0 = 0; h0 < p.Hv; h0 += G) {
                const int m = min(G, p.Hv - h0);   // CTAs taking one head of this request
                const long long *od = key + cur * 256;
                long long *nd = key + (cur ^ 1) * 256;
                long long kx = 0;
                int npos = 0;
                if (tid < G) {
                    kx = od[tid];
                    int lo, hi;
                    if (tid < m) {
                        // updated head entry: count the tail entries below its new key
                        kx += cost;
                        lo = m;
                        hi = G;
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (od[mid] < kx) lo = mid + 1; else hi = mid;
                        }
                        npos = tid + (lo - m);
                        if ((int)(kx & 0xffffffff) == c) {
                            list[*count_out] = make_int4(b, h0 + tid, sb, lb);
                            *count_out += 1;
                        }
                    } else {
                        // untouched tail entry: count the updated head entries below it
                        lo = 0;
                        hi = m;
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (od[mid] + cost < kx) lo = mid + 1; else hi = mid;
                        }
                        npos = (tid - m) + lo;
                    }
                    // nd is not od, and every read of nd's previous contents (as the old order
                    // of the step before) finished before that step's closing barrier
                    nd[npos] = kx;
                }
                __syncthreads();
                cur ^= 1;
            }
        }
        return;
    }
    int total = 0;
    const int waves = (U + G - 1) / G;
    for (int w = batch0; w < waves && total < MAX_UNITS; ++w) {
        const int u = w * G + ((w & 1) ? (G - 1 - c) : c);
        if (u < U) {
            if (tid == 0) {
                const int r = u / p.Hv;
                const int h = u - r * p.Hv;
                const int b = sorted ? ord[r] : r;
                int s, l;
                req_range(b, s, l);
                list[total] = make_int4(b, h, s, l);
            }
            ++total;
        }
    }
    *count_out = total;
}

// Block (I, J) of T' from an mma fragment (times sgn), written to the bf16 operand
// tiles Tb = T' diag(beta rk) and Tbg = T' diag(beta Gamma rk^2) (K-major, 128B-swizzled)
template <bool F16>
__device__ __forceinline__ void blk_store_tiles(const float (&acc)[2][4], float sgn, int I, int J,
                                                const float *ga, uint8_t *tb, uint8_t *tbg)
{
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        const int j = 16 * J + 8 * nh + 2 * t;
        const float2 b = *reinterpret_cast<const float2 *>(ga + GA_TB + j);
        const float2 bg = *reinterpret_cast<const float2 *>(ga + GA_BG + j);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float x0 = sgn * acc[nh][2 * h], x1 = sgn * acc[nh][2 * h + 1];
            const uint32_t off = sw128(16 * I + g + 8 * h, j >> 3) + (uint32_t)(j & 7) * 2u;
            *reinterpret_cast<uint32_t *>(tb + off) = pack2<F16>(x0 * b.x, x1 * b.y);
            *reinterpret_cast<uint32_t *>(tbg + off) = pack2<F16>(x0 * bg.x, x1 * bg.y);
        }
    }
}

// SOLVE slots (see tile16.cuh): the X products later hold T_20 T_21 T_30 T_31.

__device__ __forceinline__ int t_slot(int I, int J)
{
    // J <= I
    if (I == J) return 10 + I;
    if (I == 1) return 14;
    if (I == 3 && J == 2) return 15;
    if (I == 2) return 6 + J;
    return 8 + J;
}

// Row i of A' (TMEM quadrants 0-1: beta_i rk_i^2 (k_i . k_j) exp(G_i - G_j) for j < i, fp32
// into the solve blocks) or of P' (quadrants 2-3: rq_i (q_i . k_j) exp(G_i - G_j) for
// j <= i, bf16 tile), read 16 Gram columns at a time from TMEM.  Only the row's own norm
// enters: the key norms of the columns move into the T' tiles (see the kernel notes), and
// a key row takes its own norm from the Gram diagonal k_i . k_i, element r of its diagonal
// block.  Blocks right of the
// row's diagonal block are zero: never stored for A', zero from the start in P'.  The
// exponent of an earlier block J is split as exp(G_i - Gend_J) exp(Gend_J - G_j), both
// <= 1.  Returns rk_i for key rows (1 without the norm or for query rows).
template <bool F16>
__device__ __forceinline__ float build_row(uint32_t tl_gram, int qd, const float *ga, float *solve,
                                           uint8_t *ptile, bool retrieval, bool knorm)
{
    const int lane = threadIdx.x & 31;
    const bool isP = qd >= 2;
    const int r = lane & 15;
    const int I = 2 * (qd & 1) + (lane >> 4);
    const int i = 16 * I + r;
    const int jmax = 2 * (qd & 1) + 1;   // last diagonal block among the warp's rows
    const float G2i = ga[GA_G2 + i];
    // without the delta retrieval A' = 0, so T' = I; key rows take rk_i^2 at their diagonal
    // block, which the descending block order reaches first
    float rk = 1.f;
    float rowscale = isP ? ga[GA_RQ + i] : (retrieval ? ga[GA_BETA + i] : 0.f);
    float gend[3];
#pragma unroll
    for (int J = 0; J < 3; ++J) gend[J] = ga[GA_GEND + J];
#pragma unroll 1
    for (int J = jmax; J >= 0; --J) {
        // ---- loads (TMEM Gram columns, gate factors) before any store of this block
        float x[16], cf[16], g2[16];
        tmem_ld16(tl_gram + 16 * J, x);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 a = ld4(ga + GA_CF + 16 * J + 4 * q);
            const float4 b = ld4(ga + GA_G2 + 16 * J + 4 * q);
            cf[4 * q] = a.x; cf[4 * q + 1] = a.y; cf[4 * q + 2] = a.z; cf[4 * q + 3] = a.w;
            g2[4 * q] = b.x; g2[4 * q + 1] = b.y; g2[4 * q + 2] = b.z; g2[4 * q + 3] = b.w;
        }
        tmem_wait_ld();
        if (J > I) continue;
        if (J == I && knorm && !isP) {
            float kk = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) kk = e == r ? x[e] : kk;
            rk = 1.0f / sqrtf(kk + 1e-12f);
            rowscale *= rk * rk;
        }
        // ---- compute
        if (J < I) {
            const float f = ex2_approx(G2i - (J == 0 ? gend[0] : (J == 1 ? gend[1] : gend[2]))) * rowscale;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) x[jj] *= f * cf[jj];
        } else {
            // branch-free: every lane evaluates all 16 factors, then masks
            const int lim = isP ? r + 1 : r;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                const float e = ex2_approx(fminf(G2i - g2[jj], 0.f)) * rowscale;
                x[jj] = (jj < lim) ? x[jj] * e : 0.f;
            }
        }
        // ---- stores
        if (isP) {
            *reinterpret_cast<uint4 *>(ptile + sw128(i, 2 * J)) = pack8<F16>(x);
            *reinterpret_cast<uint4 *>(ptile + sw128(i, 2 * J + 1)) = pack8<F16>(x + 8);
        } else {
            float *row = solve + (J == I ? I : a_slot(I, J)) * SOLVE_BLK + r * SOLVE_LD;
#pragma unroll
            for (int q = 0; q < 4; ++q) st4(row + 4 * q, x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
    }
    return rk;
}

// Plain staging of one chunk's q/k (and g/beta) or v rows into the swizzled operand tiles, for
// head sizes the tensor maps cannot describe (row strides that are not multiples of 16 bytes).
// The 32 lanes of the TMA warp copy element by element; the tiles were zeroed at kernel start
// and positions past the head size are never written, so the padding stays zero exactly as
// the TMA's fill would leave it.  Tokens at or past N read as zero, as with the TMA.
__device__ __noinline__ void stage_plain_kq(const Params &p, uint8_t *kq, float *gtile, int qh, int h,
                                            int64_t t0, bool has_decay, bool has_retrieval)
{
    const int lane = threadIdx.x & 31;
    const int Dk = p.Dk;
    const int n = C * Dk;
    for (int idx = lane; idx < 2 * n; idx += 32) {
        const int which = idx >= n;              // 0: k rows, 1: q rows
        const int r = idx - which * n;
        const int i = r / Dk, e = r - i * Dk;
        const int64_t t = t0 + i;
        uint16_t x = 0;
        if (t < p.N) x = (which ? p.q : p.k)[(t * p.Hq + qh) * Dk + e];
        const uint32_t off = (e >> 6) * KQ_KB + which * 8192u + sw128(i, (e & 63) >> 3) + (uint32_t)(e & 7) * 2u;
        *reinterpret_cast<uint16_t *>(kq + off) = x;
    }
    for (int i = lane; i < C; i += 32) {
        const int64_t t = t0 + i;
        const bool in = t < p.N;
        if (has_decay) gtile[i * 4 + (h & 3)] = in ? p.g[t * p.Hv + h] : 0.f;
        if (has_retrieval) gtile[256 + i * 4 + (h & 3)] = in ? p.beta[t * p.Hv + h] : 0.f;
    }
}

__device__ __noinline__ void stage_plain_v(const Params &p, uint8_t *vt, int h, int64_t t0)
{
    const int lane = threadIdx.x & 31;
    const int Dv = p.Dv;
    for (int idx = lane; idx < C * Dv; idx += 32) {
        const int j = idx / Dv, e = idx - j * Dv;
        const int64_t t = t0 + j;
        const uint16_t x = t < p.N ? p.v[(t * p.Hv + h) * Dv + e] : (uint16_t)0;
        *reinterpret_cast<uint16_t *>(vt + (e >> 6) * V_HALF + sw128(j, (e & 63) >> 3) + (uint32_t)(e & 7) * 2u) = x;
    }
}

// Start state, final-state destination and outputs of a unit of a split pass (seqpar.cuh):
// segment 0 runs from the true initial state, its final state the start of segment 1;
// segment 1 runs from the identity (final state A1^T) and from zero (B1^T), without outputs;
// in pass 3 segments 1 and 2 run from their composed start states, segment 2's final state the
// request's.  `bfield` is the unit's b field (request, segment, mode, split bit).
__device__ __noinline__ void seq_unit_io(const Params &p, int bfield, int h, int dv, const float *&init,
                                         float *&fin, int &ident, bool &outputs_on)
{
    const gdn_seq::Workspace ws{p.seq_ws, p.B, p.Hv, D, D};
    const int ub = bfield & 255, useg = (bfield >> 8) & 15, umode = (bfield >> 12) & 7;
    const bool usplit = (bfield >> 15) & 1;
    const int64_t ro = (int64_t)dv * D;
    if (umode == gdn_seq::MODE_IDENT) {
        init = nullptr;
        ident = dv;
        fin = ws.A1(ub, h) + ro;
        outputs_on = false;
    } else if (umode == gdn_seq::MODE_ZERO) {
        init = nullptr;
        fin = ws.B1(ub, h) + ro;
        outputs_on = false;
    } else if (useg == 1) {
        init = ws.S1(ub, h) + ro;
        fin = nullptr;
    } else if (useg == 2) {
        init = ws.S2(ub, h) + ro;
    } else if (usplit) {
        fin = ws.S1(ub, h) + ro;
    }
}

// ========================================================================== kernel
// GENERAL = false: the default rule (gated_delta, no gate or beta activation), with the
// variant switches folded at compile time; GENERAL = true reads them from p.
// SEQ = true: a pass of the sequence-parallel split (default rule, bf16, 128-wide heads), one
// unit per CTA, whose mode picks its start state, where its final state goes and whether it
// writes outputs (seqpar.cuh).
template <bool GENERAL, bool F16, bool SEQ = false>
__global__ void __launch_bounds__(NTHREADS, 1) gdn_prefill_chunk_kernel(const __grid_constant__ Params p)
{
    static_assert(!SEQ || (!GENERAL && !F16), "the split runs the default bf16 instantiation");
    const bool has_decay = GENERAL ? p.has_decay != 0 : true;
    const bool has_retrieval = GENERAL ? p.has_retrieval != 0 : true;
    const bool beta_sigmoid = GENERAL ? p.beta_sigmoid != 0 : false;
    const float *const a_log = GENERAL ? p.a_log : nullptr;
    const int Dk = GENERAL ? p.Dk : D;
    const int Dv = GENERAL ? p.Dv : D;
    extern __shared__ uint8_t smem_raw[];
    // align the shared-window offset (not the generic address) to 1024 bytes: the
    // 128-byte swizzle of TMA and UMMA is a function of shared-address bits [4, 10)
    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw_base & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // layout self-check: swizzled tiles need a 1024-aligned base, tensor maps 64 bytes
    if ((sbase & 1023u) != 0 || (reinterpret_cast<uintptr_t>(&p.tm_q) & 63) != 0) {
        if (tid == 0 && p.dev_status) atomicOr(p.dev_status, GDN_DEV_INTERNAL);
        return;
    }

    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    int *count_slot = reinterpret_cast<int *>(smem + OFF_MISC + 8);
    Ctx cx{smem, sbase, abort_flag, p.dev_status};

    if (tid == 0) {
        *abort_flag = 0;
        for (int i = 0; i < (int)NUM_BARS; ++i) mbar_init(cx.bar(i), 1);
        fence_mbar_init();
    }
    if (warp == TMA_WARP && lane == 0 && !(GENERAL && p.stage_plain)) {
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
        if (has_decay) prefetch_tmap(&p.tm_g);
        if (has_retrieval) prefetch_tmap(&p.tm_beta);
    }
    if (warp == MMA_WARP) {
        tmem_alloc(sbase + OFF_MISC, 512);
        tmem_relinquish();
    }
    // P and T tiles: only the blocks on and below the diagonal are ever written
    static_assert(OFF_TB == OFF_P + KQ_STAGES * P_STAGE && OFF_TBG == OFF_TB + 8192, "tile order");
    for (int i = tid; i < (int)((OFF_TBG + 8192 - OFF_P) / 16); i += NTHREADS)
        reinterpret_cast<uint4 *>(smem + OFF_P)[i] = make_uint4(0u, 0u, 0u, 0u);
    // plain staging writes only the head's own columns: the q/k stages and the v tile start
    // zeroed, so their padding is zero as the TMA would fill it
    static_assert(OFF_KQ0 == 0 && OFF_V == KQ_STAGES * KQ_STAGE, "staging tiles are contiguous");
    if (GENERAL && p.stage_plain)
        for (int i = tid; i < (int)((OFF_V + 16384) / 16); i += NTHREADS)
            reinterpret_cast<uint4 *>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // per-role pipeline counters (persist across units and batches)
    uint32_t kq_use[KQ_STAGES] = {}, v_use = 0;               // TMA
    uint32_t c_wneg = 0, c_s = 0, c_y = 0, c_e1 = 0, c_ut = 0;       // chain issuer
    uint32_t q_kq[KQ_STAGES] = {}, q_t = 0, q_v = 0, q_w = 0, q_u = 0, q_g = 0;   // prep-stream issuer
    uint32_t p_kq[KQ_STAGES] = {}, p_gate_empty[KQ_STAGES] = {}, p_g = 0, p_sf[2] = {0, 0};   // prep front
    uint32_t p_ar[2] = {0, 0}, p_wu = 0;                              // prep back
    uint32_t s_u = 0, s_sd = 0, s_zd = 0, s_w = 0, s_gate[KQ_STAGES] = {};   // state
    uint32_t gc = 0;   // global chunk counter (same sequence in every role)

    const int G = gridDim.x;
    const int U = p.B * p.Hv;
    const int waves = SEQ ? 1 : (U + G - 1) / G;

    for (int batch0 = 0; batch0 < waves;) {
        if constexpr (SEQ)
            build_seq_unit(p, smem, count_slot);
        else
            build_unit_list(p, smem, batch0, count_slot);
        __syncthreads();
        const int nunits = *count_slot;
        int wcover = 0;
        if (SEQ || greedy_schedule(p, G)) {
            wcover = waves;   // one list holds every unit of this CTA
        } else {
            int cnt = 0;
            for (int w = batch0; w < waves; ++w) {
                const int u = w * G + ((w & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
                if (u < U) {
                    if (cnt == MAX_UNITS) break;
                    ++cnt;
                }
                ++wcover;
            }
        }

        if (warp == TMA_WARP && GENERAL && p.stage_plain) {
            // ------------------------------------------------------------ plain staging
            // the whole warp stages each chunk's q/k/g/beta stage, then its v tile, in chunk
            // order (the two streams are not independent here, which costs overlap but no
            // progress: a v tile waits only on products of earlier chunks)
            bool ok = true;
            for (int k = 0; k < nunits && ok; ++k) {
                const Unit un = load_unit(smem, k);
                const int qh = (int)(((int64_t)un.h * p.Hq) / p.Hv);
                const int nc = (un.len + C - 1) / C;
                for (int n = 0; n < nc && ok; ++n) {
                    const uint32_t ks = (gc + n) % KQ_STAGES;
                    const int64_t t0 = (int64_t)un.start + (int64_t)n * C;
                    if (kq_use[ks] > 0) ok = cx.wait(B_KQ_EMPTY + ks, (kq_use[ks] - 1) & 1);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    ++kq_use[ks];
                    stage_plain_kq(p, smem + OFF_KQ0 + ks * KQ_STAGE,
                                   reinterpret_cast<float *>(smem + OFF_GB0 + ks * 2048), qh, un.h, t0,
                                   has_decay, has_retrieval);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(cx.bar(B_KQ_FULL + ks));
                    if (v_use > 0) ok = cx.wait(B_V_EMPTY, (v_use - 1) & 1);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    ++v_use;
                    stage_plain_v(p, smem + OFF_V, un.h, t0);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(cx.bar(B_V_FULL));
                }
                gc += nc;
            }
        } else if (warp == TMA_WARP) {
            // ------------------------------------------------------------ TMA producers
            // lane 0: q/k/g/beta tiles (KQ_STAGES stages); lane 1: v tiles (one stage).  The
            // two streams are released by different consumers (the state chain, the W/U~
            // products), so neither waits behind the other.  Each also pulls a later chunk
            // of its stream into L2, so that a reload does not start cold.
            if (lane == 0) {
                // checked builds: a caller-requested stall makes the first q/k stage expect 16
                // bytes more than its copies deliver, so every wait on it runs out
                bool stall = batch0 == 0 && gdn::test_stall_requested(p.dev_status);
                for (int k = 0; k < nunits && !cx.aborted(); ++k) {
                    const Unit un = load_unit(smem, k);
                    const int qh = (int)(((int64_t)un.h * p.Hq) / p.Hv);
                    const int nc = (un.len + C - 1) / C;
                    for (int n = 0; n < nc; ++n) {
                        const uint32_t ks = (gc + n) % KQ_STAGES;
                        if (kq_use[ks] > 0 && !cx.wait(B_KQ_EMPTY + ks, (kq_use[ks] - 1) & 1)) break;
                        ++kq_use[ks];
                        const uint32_t kq = sbase + OFF_KQ0 + ks * KQ_STAGE;
                        const uint32_t gb = sbase + OFF_GB0 + ks * 2048;
                        const int t0 = un.start + n * C;
                        const uint32_t kb = cx.bar(B_KQ_FULL + ks);
                        mbar_arrive_expect_tx(kb, 32768 + (has_decay ? 1024 : 0) + (has_retrieval ? 1024 : 0) +
                                                      (stall ? 16 : 0));
                        stall = false;
                        tma_load_3d(kq, &p.tm_k, kb, 0, qh, t0);
                        tma_load_3d(kq + KQ_KB, &p.tm_k, kb, 64, qh, t0);
                        tma_load_3d(kq + 8192, &p.tm_q, kb, 0, qh, t0);
                        tma_load_3d(kq + KQ_KB + 8192, &p.tm_q, kb, 64, qh, t0);
                        if (has_decay) tma_load_2d(gb, &p.tm_g, kb, un.h & ~3, t0);
                        if (has_retrieval) tma_load_2d(gb + 1024, &p.tm_beta, kb, un.h & ~3, t0);
                        if (n + KQ_STAGES < nc) {
                            const int t2 = t0 + KQ_STAGES * C;
                            tma_prefetch_3d(&p.tm_k, 0, qh, t2);
                            tma_prefetch_3d(&p.tm_k, 64, qh, t2);
                            tma_prefetch_3d(&p.tm_q, 0, qh, t2);
                            tma_prefetch_3d(&p.tm_q, 64, qh, t2);
                            if (has_decay) tma_prefetch_2d(&p.tm_g, un.h & ~3, t2);
                            if (has_retrieval) tma_prefetch_2d(&p.tm_beta, un.h & ~3, t2);
                        }
                    }
                    gc += nc;
                }
            } else if (lane == 1) {
                for (int k = 0; k < nunits && !cx.aborted(); ++k) {
                    const Unit un = load_unit(smem, k);
                    const int nc = (un.len + C - 1) / C;
                    // a transition run from the identity takes v = 0: the tile is zeroed once
                    // and every chunk's stage completes without a copy (SEQ passes hold one unit
                    // per CTA, so nothing reloads the tile in between)
                    const bool vzero = SEQ && ((un.b >> 12) & 7) == gdn_seq::MODE_IDENT;
                    for (int n = 0; n < nc; ++n) {
                        const int t0 = un.start + n * C;
                        if (v_use > 0 && !cx.wait(B_V_EMPTY, (v_use - 1) & 1)) break;
                        ++v_use;
                        if (vzero) {
                            if (n == 0) {
                                for (int i = 0; i < 16384 / 16; ++i)
                                    reinterpret_cast<uint4 *>(smem + OFF_V)[i] = make_uint4(0u, 0u, 0u, 0u);
                                fence_proxy_async_smem();
                            }
                            mbar_arrive(cx.bar(B_V_FULL));
                            continue;
                        }
                        mbar_arrive_expect_tx(cx.bar(B_V_FULL), 16384);
                        tma_load_3d(sbase + OFF_V, &p.tm_v, cx.bar(B_V_FULL), 0, un.h, t0);
                        tma_load_3d(sbase + OFF_V + V_HALF, &p.tm_v, cx.bar(B_V_FULL), 64, un.h, t0);
                        if (n + 2 < nc) {
                            tma_prefetch_3d(&p.tm_v, 0, un.h, t0 + 2 * C);
                            tma_prefetch_3d(&p.tm_v, 64, un.h, t0 + 2 * C);
                        }
                    }
                    gc += nc;
                }
            }
        } else if (warp == MMA_WARP || warp == ISSUE_WARP) {
            // ------------------------------------------------------------ UMMA issuers
            // Two single-thread issuers, so that neither stream waits behind the other's
            // (blocking) MMA issue: the chain issuer (warp MMA_WARP: C1, C2 of each chunk,
            // in order) and the prep-stream issuer (warp ISSUE_WARP: Gram and W/U~ of each
            // chunk, in order).  Each commit tracks only its own thread's MMAs; every
            // cross-stream hazard is ordered by an mbarrier:
            //   G(x):  KQ(x) loaded, G_FREE(x-1) (A/P of x-1 built); up to one chunk
            //          ahead of WU inside a unit
            //   W(x):  T(x) ready, WNEG(x-1) (W columns converted)
            //   U~(x): V(x) loaded, Z_DONE(x-1) (the U columns hold the bf16 operands of
            //          (2)/(3) until then)
            //   C1(x): WNEG(x) (W(x) converted; the state warpgroup converts only after it
            //          saw U_DONE(x-1), so (1a) of x-1 no longer reads the -W tile),
            //          UT_DONE(x), S_READY(x); the Y part after Y_FREE(x-1)
            //   C2(x): E1(x)
            if (lane == 0) {
                constexpr uint32_t ID_G = idesc_f16kind(128, 64, 0, 0, !F16);
                constexpr uint32_t ID_W = idesc_f16kind(128, 64, 1, 0, !F16);
                constexpr uint32_t ID_U = idesc_f16kind(128, 64, 1, 0, !F16);
                constexpr uint32_t ID_1A = idesc_f16kind(128, 64, 0, 1, !F16);
                constexpr uint32_t ID_1B = idesc_f16kind(128, 64, 0, 0, !F16);
                constexpr uint32_t ID_2 = idesc_f16kind(128, 128, 0, 1, !F16);
                constexpr uint32_t ID_3 = idesc_f16kind(128, 64, 0, 0, !F16);
                // descriptor bases; a byte offset `o` inside a tile is added as (o >> 4)
                // KQ stage ks starts (ks * KQ_STAGE) >> 4 descriptor units after stage 0
                const uint64_t dKQk = sdesc_sw128(sbase + OFF_KQ0, 16, 1024);      // K-major
                const uint64_t dKQm = sdesc_sw128(sbase + OFF_KQ0, KQ_KB, 1024);   // MN-major K
                bool ok = true;
                if (warp == ISSUE_WARP) {
                    const uint64_t dV = sdesc_sw128(sbase + OFF_V, V_HALF, 1024);
                    const uint64_t dTB = sdesc_sw128(sbase + OFF_TB, 16, 1024);
                    const uint64_t dTBG = sdesc_sw128(sbase + OFF_TBG, 16, 1024);
                    // Three tasks per chunk x, each issued as soon as its inputs are ready
                    // (non-blocking tests, so none waits behind another; an issue blocks while
                    // the tensor pipe drains, so the state chain's inputs U~ and W go first and
                    // the Gram look-ahead last):
                    //   G(x):  previous Gram read by the prep (G_FREE), KQ(x) loaded; at most
                    //          one chunk ahead of W
                    //   W(x):  G(x) issued, T(x) ready, WNEG(x-1) (W columns converted)
                    //   U~(x): W(x) issued, V(x) loaded, Z_DONE(x-1) (the U columns hold the bf16
                    //          operands of (2)/(3) of x-1 until then); its commit (UT_DONE)
                    //          therefore also covers W(x)
                    // Every barrier tested here can run at most one phase ahead of its counter:
                    // its next phase depends on the task that consumes this one.
                    for (int k = 0; k < nunits && ok; ++k) {
                        const Unit un = load_unit(smem, k);
                        const int nc = (un.len + C - 1) / C;
                        int gi = 0, wi = 0, ui = 0;   // G / W / U~ issued in this unit
                        long long t_last = clock64();
                        while (ui < nc) {
                            bool did = false;
                            if (ui < wi && mbar_test_wait(cx.bar(B_V_FULL), q_v & 1) &&
                                (q_u == 0 || mbar_test_wait(cx.bar(B_Z_DONE), (q_u - 1) & 1))) {
                                ++q_v;
                                ++q_u;
                                tc_fence_after();
                                // (U~): U^T[dv][i] = sum_j V[j][dv] Tb[i][j]; A = V (MN-major), B = Tb
#pragma unroll 1
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16(tmem + TM_U, dV + ((kk * 2048) >> 4), dTB + ((kk * 32) >> 4), ID_U, kk > 0);
                                umma_commit(cx.bar(B_UT_DONE));
                                umma_commit(cx.bar(B_V_EMPTY));
                                ++ui;
                                did = true;
                            }
                            if (!did && wi < gi && mbar_test_wait(cx.bar(B_T_READY), q_t & 1) &&
                                (q_w == 0 || mbar_test_wait(cx.bar(B_WNEG), (q_w - 1) & 1))) {
                                ++q_t;
                                ++q_w;
                                const uint32_t ks = (gc + wi) % KQ_STAGES;
                                tc_fence_after();
                                // (W): W^T[dk][i] = sum_j K[j][dk] Tbg[i][j]; A = K (MN-major), B = Tbg
#pragma unroll 1
                                for (int kk = 0; kk < 4; ++kk)
                                    umma_bf16(tmem + TM_W, dKQm + ((ks * KQ_STAGE + kk * 2048) >> 4), dTBG + ((kk * 32) >> 4), ID_W, kk > 0);
                                umma_commit(cx.bar(B_W_DONE));
                                ++wi;
                                did = true;
                            }
                            if (!did && gi < nc && gi <= wi + 1) {
                                const uint32_t sg = (gc + gi) % KQ_STAGES;
                                if ((q_g == 0 || mbar_test_wait(cx.bar(B_G_FREE), (q_g - 1) & 1)) &&
                                    mbar_test_wait(cx.bar(B_KQ_FULL + sg), q_kq[sg] & 1)) {
                                    ++q_g;
                                    ++q_kq[sg];
                                    tc_fence_after();
                                    // (G): [K;Q] (128 x 128, K-major) x K^T
#pragma unroll 1
                                    for (int kk = 0; kk < 8; ++kk) {
                                        const uint32_t o = ((kk >> 2) * KQ_KB + (kk & 3) * 32) >> 4;
                                        const uint64_t d = dKQk + ((sg * KQ_STAGE) >> 4) + o;
                                        umma_bf16(tmem + TM_G, d, d, ID_G, kk > 0);
                                    }
                                    umma_commit(cx.bar(B_G_DONE));
                                    ++gi;
                                    did = true;
                                }
                            }
                            if (did) {
                                t_last = clock64();
                            } else {
                                if (cx.aborted()) { ok = false; break; }
                                if (clock64() - t_last > (1ll << 31)) {
                                    *cx.abort_flag = 1;
                                    if (p.dev_status) atomicOr(p.dev_status, GDN_DEV_TIMEOUT);
                                    ok = false;
                                    break;
                                }
                                __nanosleep(32);
                            }
                        }
                        gc += nc;
                    }
                } else {
                    const uint64_t dWNEG = sdesc_sw128(sbase + OFF_WNEG, 8192, 1024);
                    const uint64_t dP = sdesc_sw128(sbase + OFF_P, 16, 1024);
                    for (int k = 0; k < nunits && ok; ++k) {
                        const Unit un = load_unit(smem, k);
                        const int nc = (un.len + C - 1) / C;
                        for (int n = 0; n < nc && ok; ++n) {
                            const uint32_t ks = (gc + n) % KQ_STAGES;
                            // (1a) U^T += S^T (-W)^T; the bf16 S^T is the TMEM A operand (8 columns
                            //      per 16 dk)
                            ok = cx.wait(B_WNEG, c_wneg & 1);
                            ++c_wneg;
                            ok = ok && cx.wait(B_UT_DONE, c_ut & 1);
                            ++c_ut;
                            ok = ok && cx.wait(B_S_READY, c_s & 1);
                            ++c_s;
                            if (!ok) break;
                            tc_fence_after();
#pragma unroll 1
                            for (int kk = 0; kk < 8; ++kk)
                                umma_bf16_ts(tmem + TM_U, tmem + TM_SB + 8 * kk, dWNEG + ((kk * 2048) >> 4), ID_1A, 1);
                            umma_commit(cx.bar(B_U_DONE));
                            // (1b) Y = S^T Q^T, once the outputs of the previous chunk have read Y
                            if (c_y > 0) ok = cx.wait(B_Y_FREE, (c_y - 1) & 1);
                            ++c_y;
                            if (!ok) break;
                            tc_fence_after();
#pragma unroll 1
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint32_t bo = (ks * KQ_STAGE + (kk >> 2) * KQ_KB + 8192 + (kk & 3) * 32) >> 4;
                                umma_bf16_ts(tmem + TM_Y, tmem + TM_SB + 8 * kk, dKQk + bo, ID_1B, kk > 0);
                            }
                            // (2) S^T += Ud K, then (3) Z = U^T P^T
                            ok = cx.wait(B_E1, c_e1 & 1);
                            ++c_e1;
                            if (!ok) break;
                            tc_fence_after();
#pragma unroll 1
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16_ts(tmem + TM_S, tmem + TM_U + 16 * kk + 8, dKQm + ((ks * KQ_STAGE + kk * 2048) >> 4), ID_2, 1);
                            umma_commit(cx.bar(B_S_DONE));
#pragma unroll 1
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16_ts(tmem + TM_Z, tmem + TM_U + 16 * kk, dP + ((ks * P_STAGE + kk * 32) >> 4), ID_3, kk > 0);
                            umma_commit(cx.bar(B_Z_DONE));
                            umma_commit(cx.bar(B_KQ_EMPTY + ks));   // also releases P stage ks
                        }
                        gc += nc;
                    }
                }
            }
        } else if (warp >= 4) {
            // ------------------------------------------------------------ prep warpgroups
            // Two groups of four warps form a two-stage pipeline over consecutive chunks:
            //   front (warps 4-7):  gates, query norms, A' and P' from the Gram (TMEM)
            //   back  (warps 8-11): 16x16 diagonal inverses, block merges, bf16 T' tiles
            // A crosses in one of two solve areas (A_READY / SOLVE_FREE per area).
            const int pg = (warp - 4) >> 2;          // 0 front, 1 back
            const int lt = tid - 128 - 128 * pg;     // thread in the group, 0..127
            const int pw = lt >> 5;                  // warp in the group == TMEM lane quadrant
            const uint32_t tl = tmem + ((uint32_t)(32 * pw) << 16);
            const int nbar = pg ? 3 : 1;             // the group's named barrier
            bool ok = true;
            for (int k = 0; k < nunits && ok; ++k) {
                const Unit un = load_unit(smem, k);
                const int nc = (un.len + C - 1) / C;
                for (int n = 0; n < nc && ok; ++n) {
                    const uint32_t s = (gc + n) & 1;
                    float *solve = reinterpret_cast<float *>(smem + (s ? OFF_SOLVE1 : OFF_SOLVE0));
                    const uint32_t ks = (gc + n) % KQ_STAGES;   // KQ and gate stage
                    float *ga = reinterpret_cast<float *>(smem + OFF_GATE + ks * GATE_BYTES);
                    if (pg == 0) {
                        const int len_n = min(C, un.len - n * C);
                        const uint8_t *kq = smem + OFF_KQ0 + ks * KQ_STAGE;
                        const float *gtile = reinterpret_cast<const float *>(smem + OFF_GB0 + ks * 2048);
                        ok = cx.wait(B_KQ_FULL + ks, p_kq[ks] & 1);
                        ++p_kq[ks];
                        if (p_gate_empty[ks] > 0) ok = ok && cx.wait(B_GATE_EMPTY + ks, (p_gate_empty[ks] - 1) & 1);
                        ++p_gate_empty[ks];
                        if (p_sf[s] > 0) ok = ok && cx.wait(B_SOLVE_FREE + s, (p_sf[s] - 1) & 1);
                        ++p_sf[s];
                        // --- gates first (front warp 0, tokens 2l and 2l+1 per lane): floored,
                        //     masked log-decay, inclusive prefix sum, exponentials
                        if (pw == 0) {
                            const int i0 = 2 * lane, i1 = i0 + 1;
                            const int hc = un.h & 3;
                            // update rule: no decay -> g = 0; no retrieval -> beta = 1; qwen gate
                            // -exp(a_log) softplus(decay + dt_bias) and sigmoid beta in fp32
                            const bool v0 = i0 < len_n, v1 = i1 < len_n;
                            float g0 = 0.f, g1 = 0.f, b0 = 1.f, b1 = 1.f;
                            if (has_decay) {
                                g0 = gtile[i0 * 4 + hc];
                                g1 = gtile[i1 * 4 + hc];
                                if (a_log) {
                                    const float ea = expf(__ldg(a_log + un.h));
                                    const float dtb = __ldg(p.dt_bias + un.h);
                                    g0 = -ea * gdn::softplus20(g0 + dtb);
                                    g1 = -ea * gdn::softplus20(g1 + dtb);
                                }
                                g0 = fmaxf(g0, G_FLOOR);
                                g1 = fmaxf(g1, G_FLOOR);
                            }
                            if (has_retrieval) {
                                b0 = gtile[256 + i0 * 4 + hc];
                                b1 = gtile[256 + i1 * 4 + hc];
                                if (beta_sigmoid) {
                                    b0 = gdn::sigmoidf_(b0);
                                    b1 = gdn::sigmoidf_(b1);
                                }
                            }
                            g0 = v0 ? g0 : 0.f;
                            g1 = v1 ? g1 : 0.f;
                            b0 = v0 ? b0 : 0.f;
                            b1 = v1 ? b1 : 0.f;
                            float x = g0 + g1;
#pragma unroll
                            for (int o = 1; o < 32; o <<= 1) {
                                const float y = __shfl_up_sync(0xffffffffu, x, o);
                                if (lane >= o) x += y;
                            }
                            const float G2b = x * LOG2E;            // token i1
                            const float G2a = (x - g1) * LOG2E;     // token i0
                            const float gend = __shfl_sync(0xffffffffu, G2b, (lane & ~7) + 7);
                            const float gcl = __shfl_sync(0xffffffffu, G2b, 31);
                            *reinterpret_cast<float2 *>(ga + GA_G2 + i0) = make_float2(G2a, G2b);
                            *reinterpret_cast<float2 *>(ga + GA_BETA + i0) = make_float2(b0, b1);
                            *reinterpret_cast<float2 *>(ga + GA_CF + i0) =
                                make_float2(ex2_approx(gend - G2a), ex2_approx(gend - G2b));
                            *reinterpret_cast<float2 *>(ga + GA_GAM + i0) = make_float2(ex2_approx(G2a), ex2_approx(G2b));
                            *reinterpret_cast<float2 *>(ga + GA_DEC + i0) =
                                make_float2(ex2_approx(gcl - G2a), ex2_approx(gcl - G2b));
                            if ((lane & 7) == 7) ga[GA_GEND + (lane >> 3)] = G2b;
                            if (lane == 31) ga[GA_GC] = ex2_approx(G2b);
                            // published at once: the state chain waits for exp(G_C) of the next
                            // chunk, and nothing here depends on the norms
                            __syncwarp();
                            if (lane == 0) mbar_arrive(cx.bar(B_GATE_FULL + ks));
                        }
                        // --- query row norms (Q rows 64..127 of the stage): two threads per row,
                        //     chunks c and 4 + c of each k-block (distinct swizzled 16-byte
                        //     positions within every four rows: conflict-free).  Key row norms
                        //     come from the Gram diagonal inside build_row; without qk_l2norm
                        //     every factor is 1.
                        if (p.qk_l2norm) {
                            const int qrow = 64 + (lt >> 1);
                            const int hf = lt & 1;
                            float ss = 0.f;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const uint32_t off = sw128(qrow, 4 * hf + c);
                                const uint4 va = *reinterpret_cast<const uint4 *>(kq + off);
                                const uint4 vb = *reinterpret_cast<const uint4 *>(kq + KQ_KB + off);
                                ss += sumsq8_bf16<F16>(va) + sumsq8_bf16<F16>(vb);
                            }
                            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                            if (hf == 0) ga[GA_RQ + (qrow - 64)] = 1.0f / sqrtf(ss + 1e-12f);
                        } else if (lt < 64) {
                            ga[GA_RQ + lt] = 1.f;
                        }
                        named_sync(1, 128);
                        // --- Gram -> A (rows 0..63, fp32 blocks) and P (rows 64..127, bf16 tile); P
                        //     shares the KQ stage, so the (3) product that last read it completed
                        //     before this stage was reloaded (KQ_EMPTY is committed after it)
                        ok = ok && cx.wait(B_G_DONE, p_g & 1);
                        ++p_g;
                        tc_fence_after();
                        const float rk = build_row<F16>(tl + TM_G, pw, ga, solve, smem + OFF_P + ks * P_STAGE,
                                                        has_retrieval, p.qk_l2norm != 0);
                        if (pw >= 2) fence_proxy_async_smem();
                        // column scales of the T' tiles (thread lt < 64 built key row lt): W = Tbg K
                        // carries the retrieval term (zero without it), U~ = Tb V
                        if (lt < 64) {
                            const float b = ga[GA_BETA + lt];
                            ga[GA_BG + lt] = has_retrieval ? b * ga[GA_GAM + lt] * rk * rk : 0.f;
                            ga[GA_TB + lt] = b * rk;
                        }
                        tc_fence_before();
                        named_sync(1, 128);
                        if (lt == 0) {
                            mbar_arrive(cx.bar(B_G_FREE));
                            mbar_arrive(cx.bar(B_A_READY + s));
                        }
                    } else {
                        ok = cx.wait(B_A_READY + s, p_ar[s] & 1);
                        ++p_ar[s];
                        // the T tiles of the previous chunk are read by its W and U~ products
                        if (p_wu > 0) ok = ok && cx.wait(B_UT_DONE, (p_wu - 1) & 1);
                        ++p_wu;
                        // --- diagonal 16x16 inverses D_I = (I + A_II)^-1 (back threads 0..63, one column each)
                        if (lt < 64) {
                            const int I = lt >> 4, c = lt & 15;
                            const float *Ab = solve + I * SOLVE_BLK;
                            float x[16];
#pragma unroll
                            for (int r = 0; r < 16; ++r) {
                                float a[16];
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    if (4 * q < r) {
                                        const float4 v = ld4(Ab + r * SOLVE_LD + 4 * q);
                                        a[4 * q] = v.x; a[4 * q + 1] = v.y; a[4 * q + 2] = v.z; a[4 * q + 3] = v.w;
                                    }
                                }
                                float acc0 = (r == c) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
                                for (int m = 0; m < r; ++m) {
                                    if (m & 1) acc1 = fmaf(-a[m], x[m], acc1);
                                    else acc0 = fmaf(-a[m], x[m], acc0);
                                }
                                x[r] = acc0 + acc1;
                            }
                            float *Db = solve + (10 + I) * SOLVE_BLK;
#pragma unroll
                            for (int r = 0; r < 16; ++r) Db[r * SOLVE_LD + c] = x[r];
                            const int j = 16 * I + c;
                            const float bj = ga[GA_TB + j], sj = ga[GA_BG + j];
                            const uint32_t cw = (uint32_t)(j & 7) * 2u;
#pragma unroll
                            for (int r = 0; r < 16; ++r) {
                                const uint32_t off = sw128(16 * I + r, j >> 3) + cw;
                                *reinterpret_cast<uint16_t *>(smem + OFF_TB + off) = elem16<F16>(x[r] * bj);
                                *reinterpret_cast<uint16_t *>(smem + OFF_TBG + off) = elem16<F16>(x[r] * sj);
                            }
                        }
                        named_sync(3, 128);
                        // --- block merges (warp-level tf32 products):
                        //   L1: T_10 = -D_1 (A_10 D_0) (warp 0), T_32 = -D_3 (A_32 D_2) (warp 1)
                        //   X : X_pq = (A_BA T_AA)_pq -> slot 2p+q (the dead A_II blocks)
                        //   TB: T_{2+p,q} = -(T_BB X)_pq -> slot 6+2p+q (the dead A_BA blocks)
                        if (pw < 2) {
                            float *tmp = solve + (pw ? 15 : 14) * SOLVE_BLK;
                            float acc[2][4] = {};
                            blk_mma(acc, solve + (pw ? 5 : 4) * SOLVE_BLK, solve + (pw ? 12 : 10) * SOLVE_BLK);
                            blk_store(tmp, acc, 1.f);
                            __syncwarp();
                            float acc2[2][4] = {};
                            blk_mma(acc2, solve + (pw ? 13 : 11) * SOLVE_BLK, tmp);
                            __syncwarp();
                            blk_store(tmp, acc2, -1.f);
                            blk_store_tiles<F16>(acc2, -1.f, pw ? 3 : 1, pw ? 2 : 0, ga, smem + OFF_TB, smem + OFF_TBG);
                        }
                        named_sync(3, 128);
#pragma unroll 1
                        for (int ph = 0; ph < 2; ++ph) {
                            const int pp = (pw >> 1) & 1, q = pw & 1;
                            const float *X0, *Y0, *X1 = nullptr, *Y1 = nullptr;
                            int dst;
                            float sgn;
                            if (ph == 0) {
                                if (q == 0) {
                                    X0 = solve + a_slot(2 + pp, 0) * SOLVE_BLK; Y0 = solve + 10 * SOLVE_BLK;
                                    X1 = solve + a_slot(2 + pp, 1) * SOLVE_BLK; Y1 = solve + 14 * SOLVE_BLK;
                                } else {
                                    X0 = solve + a_slot(2 + pp, 1) * SOLVE_BLK; Y0 = solve + 11 * SOLVE_BLK;
                                }
                                dst = 2 * pp + q; sgn = 1.f;
                            } else {
                                if (pp == 0) {
                                    X0 = solve + 12 * SOLVE_BLK; Y0 = solve + q * SOLVE_BLK;
                                } else {
                                    X0 = solve + 15 * SOLVE_BLK; Y0 = solve + q * SOLVE_BLK;
                                    X1 = solve + 13 * SOLVE_BLK; Y1 = solve + (2 + q) * SOLVE_BLK;
                                }
                                dst = 6 + 2 * pp + q; sgn = -1.f;
                            }
                            {
                                float acc[2][4] = {};
                                const int np = X1 ? 2 : 1;
#pragma unroll 1
                                for (int t = 0; t < np; ++t) blk_mma(acc, t ? X1 : X0, t ? Y1 : Y0);
                                if (ph == 0) blk_store(solve + dst * SOLVE_BLK, acc, sgn);
                                else blk_store_tiles<F16>(acc, sgn, 2 + pp, q, ga, smem + OFF_TB, smem + OFF_TBG);
                            }
                            if (ph == 1) fence_proxy_async_smem();   // T tiles -> UMMA operands
                            named_sync(3, 128);
                        }
                        if (lt == 0) {
                            mbar_arrive(cx.bar(B_T_READY));
                            mbar_arrive(cx.bar(B_SOLVE_FREE + s));
                        }
                    }
                    ok = !named_sync_or(nbar, 128, !ok || cx.aborted());
                }
                gc += nc;
            }
        } else {
            // ------------------------------------------------------------ state warpgroup
            const int dv = tid;                 // 0..127 == TMEM lane
            const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
            // W^T of the next chunk (TMEM, lane dk) -> -W as the MN-major B tile of (1a) (row
            // dk).  The tile is free: this warpgroup already saw U_DONE of the chunk before,
            // so (1a) of that chunk has read it.
            auto convert_wneg = [&]() -> bool {
                const bool w_ok = cx.wait(B_W_DONE, s_w & 1);
                ++s_w;
                tc_fence_after();
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    float t[32];
                    tmem_ld32(tl + TM_W + 32 * q, t);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) t[e] = -t[e];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4 *>(smem + OFF_WNEG + sw128(dv, 4 * q + c)) = pack8<F16>(t + 8 * c);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_sync(2, 128);
                if (dv == 0) mbar_arrive(cx.bar(B_WNEG));
                return w_ok;
            };
            float *ogr = reinterpret_cast<float *>(smem + OFF_OGR);
            bool pre = false;   // this unit's state is already in TMEM
            for (int k = 0; k < nunits; ++k) {
                const Unit un = load_unit(smem, k);
                const int nc = (un.len + C - 1) / C;
                // SEQ units carry their request, segment, mode and split bit in the b field
                const int ub = SEQ ? (un.b & 255) : un.b;
                // this lane's state row (dv < Dv; lanes past Dv carry zero rows)
                const int64_t st_off = (((int64_t)ub * p.Hv + un.h) * Dv + dv) * Dk;
#ifdef GDN_CHECKS
                const int64_t st_n = (int64_t)p.B * p.Hv * Dv * Dk;
                const bool row_ok = (!GENERAL || dv < Dv) && in_range(st_off, Dk, st_n, p.dev_status);
#else
                const bool row_ok = !GENERAL || dv < Dv;
#endif
                const float *init = p.initial_state && row_ok ? p.initial_state + st_off : nullptr;
                float *fin = row_ok ? p.final_state + st_off : nullptr;
                int ident = -1;            // start from the identity's row dv instead of init
                bool outputs_on = true;
                if constexpr (SEQ) seq_unit_io(p, un.b, un.h, dv, init, fin, ident, outputs_on);
                if (nc == 0) {
                    if (row_ok && (!GENERAL || (Dk & 3) == 0)) {
                        for (int c = 0; c < Dk; c += 4) {
                            float4 v = init ? ld4(init + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                            *reinterpret_cast<float4 *>(fin + c) = v;
                        }
                    } else if (row_ok) {
                        for (int c = 0; c < Dk; ++c) fin[c] = init ? init[c] : 0.f;
                    }
                    continue;
                }
                bool ok = true;
                // unit start: S0 -> bf16 operand columns and gC(0) * S0 -> TMEM, unless the
                // previous unit's last chunk already did it (pre)
                if (!pre) {
                    const uint32_t gs = gc % KQ_STAGES;
                    ok = cx.wait(B_GATE_FULL + gs, s_gate[gs] & 1);
                    ++s_gate[gs];
                    const float gC = reinterpret_cast<const float *>(smem + OFF_GATE + gs * GATE_BYTES)[GA_GC];
                    load_state_tmem<GENERAL, F16, SEQ>(init, Dk, tl, gC, ident);
                    tmem_wait_st();
                    tc_fence_before();
                    ok = !named_sync_or(2, 128, !ok || cx.aborted());
                    if (dv == 0 && ok) mbar_arrive(cx.bar(B_S_READY));
                }
                // a non-empty next unit takes its state at this unit's last E2, before the last
                // outputs, so that the chain does not wait for them at the switch; its row is
                // pulled into L2 now
                const Unit nx = load_unit(smem, min(k + 1, nunits - 1));
                const bool has_next = k + 1 < nunits && nx.len > 0;
#ifdef GDN_CHECKS
                const int64_t nx_off = (((int64_t)nx.b * p.Hv + nx.h) * Dv + dv) * Dk;
                const float *next_init =
                    has_next && p.initial_state && row_ok && in_range(nx_off, Dk, st_n, p.dev_status)
                        ? p.initial_state + nx_off
                        : nullptr;
#else
                const float *next_init =
                    has_next && p.initial_state && row_ok
                        ? p.initial_state + (((int64_t)nx.b * p.Hv + nx.h) * Dv + dv) * Dk
                        : nullptr;
#endif
                if (next_init) {
                    for (int c = 0; c < Dk; c += 32) prefetch_l2(next_init + c);
                }
                for (int n = 0; n < nc && ok; ++n) {
                    const uint32_t gs = (gc + n) % KQ_STAGES, gs1 = (gc + n + 1) % KQ_STAGES;
                    const int len_n = min(C, un.len - n * C);
                    const float *ga = reinterpret_cast<const float *>(smem + OFF_GATE + gs * GATE_BYTES);
                    // the -W tile of a unit's first chunk (later ones, and the first of a unit
                    // that follows a non-empty one, are converted after E2)
                    if (n == 0 && !pre) ok = convert_wneg();
                    // ---- E1: U^T -> bf16 tiles (plain for Z, decayed and key-normed for S)
                    ok = ok && cx.wait(B_U_DONE, s_u & 1);
                    ++s_u;
                    tc_fence_after();
#pragma unroll 1
                    for (int q = 0; q < 2; ++q) {
                        float u[32];
                        tmem_ld32(tl + TM_U + 32 * q, u);
                        tmem_wait_ld();
                        // per 16 tokens: 8 columns of bf16 U (A of (3)), then 8 of the decayed U (A of (2))
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int t0 = 32 * q + 16 * h;
                            float d[16];
#pragma unroll
                            for (int e = 0; e < 16; e += 4) {
                                const float4 d4 = ld4(ga + GA_DEC + t0 + e);
                                d[e] = d4.x; d[e + 1] = d4.y; d[e + 2] = d4.z; d[e + 3] = d4.w;
                            }
                            uint32_t w[16];
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                w[e] = pack2<F16>(u[16 * h + 2 * e], u[16 * h + 2 * e + 1]);
                                w[8 + e] = pack2<F16>(u[16 * h + 2 * e] * d[2 * e], u[16 * h + 2 * e + 1] * d[2 * e + 1]);
                            }
                            tmem_st16u(tl + TM_U + t0, w);
                        }
                    }
                    tmem_wait_st();
                    if (dv < 64) ogr[dv] = ga[GA_GAM + dv] * ga[GA_RQ + dv];
                    tc_fence_before();
                    named_sync(2, 128);
                    if (dv == 0) {
                        mbar_arrive(cx.bar(B_E1));
                        mbar_arrive(cx.bar(B_GATE_EMPTY + gs));   // the outputs read ogr from here on
                    }
                    // ---- E2: new state -> bf16 operand columns (+ decay of the next chunk) or final state
                    ok = ok && cx.wait(B_S_DONE, s_sd & 1);
                    ++s_sd;
                    tc_fence_after();
                    const bool more = n + 1 < nc;
                    const bool chain = more || has_next;   // a state follows in TMEM
                    float gC1 = 1.f;
                    if (chain) {
                        ok = ok && cx.wait(B_GATE_FULL + gs1, s_gate[gs1] & 1);
                        ++s_gate[gs1];
                        gC1 = reinterpret_cast<const float *>(smem + OFF_GATE + gs1 * GATE_BYTES)[GA_GC];
                    }
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        float x[32];
                        tmem_ld32(tl + TM_S + 32 * q, x);
                        tmem_wait_ld();
                        if (more) {
                            uint32_t w[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) w[e] = pack2<F16>(x[2 * e], x[2 * e + 1]);
                            tmem_st16u(tl + TM_SB + 16 * q, w);
#pragma unroll
                            for (int e = 0; e < 32; ++e) x[e] *= gC1;
                            tmem_st32(tl + TM_S + 32 * q, x);
                        } else {
                            if (!GENERAL && fin && (!kChecked || row_ok)) {
#pragma unroll
                                for (int c = 0; c < 32; c += 4) st4(fin + 32 * q + c, x[c], x[c + 1], x[c + 2], x[c + 3]);
                            } else if (row_ok && (Dk & 3) == 0) {
                                for (int c = 0; c < 32 && 32 * q + c < Dk; c += 4)
                                    st4(fin + 32 * q + c, x[c], x[c + 1], x[c + 2], x[c + 3]);
                            } else if (row_ok) {
#pragma unroll
                                for (int c = 0; c < 32; ++c)
                                    if (32 * q + c < Dk) fin[32 * q + c] = x[c];
                            }
                        }
                    }
                    if (!more && has_next) load_state_tmem<GENERAL, F16>(next_init, Dk, tl, gC1);
                    if (chain) {
                        tmem_wait_st();
                        tc_fence_before();
                        named_sync(2, 128);
                        if (dv == 0) mbar_arrive(cx.bar(B_S_READY));
                        // the next chunk's (1a) waits on its -W tile: convert it before the outputs
                        ok = convert_wneg() && ok;
                    }
                    // ---- outputs O^T = scale (Y diag(Gamma rq) + Z): 8 tokens at a time through a
                    //      warp-private [8 tokens][32 dv] bf16 scratch, then one 16-byte store per
                    //      lane (lanes 4t..4t+3 write token t's 64 bytes of this warp's dv); rows
                    //      past len_n belong to the next request and are skipped
                    ok = ok && cx.wait(B_Z_DONE, s_zd & 1);
                    ++s_zd;
                    tc_fence_after();
                    {
                        const float sc = p.scale;
                        uint8_t *ost = smem + OFF_OST + 512 * warp;
                        const int tt = lane >> 2;   // token of this lane's 16-byte store
                        const int ocol = 32 * warp + 8 * (lane & 3);   // this lane's 8 dv
                        uint16_t *obase = p.out + ((int64_t)(un.start + n * C + tt) * p.Hv + un.h) * Dv + ocol;
                        const int64_t ostride8 = (int64_t)8 * p.Hv * Dv;
#pragma unroll 1
                        for (int q = 0; q < 4; ++q) {
                            float y[16], z[16];
                            tmem_ld16(tl + TM_Y + 16 * q, y);
                            tmem_ld16(tl + TM_Z + 16 * q, z);
                            tmem_wait_ld();
#pragma unroll
                            for (int hb = 0; hb < 2; ++hb) {
                                const float4 g0 = ld4(ogr + 16 * q + 8 * hb), g1 = ld4(ogr + 16 * q + 8 * hb + 4);
                                const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    *reinterpret_cast<uint16_t *>(ost + e * 64 + lane * 2) =
                                        elem16<F16>(sc * fmaf(gg[e], y[8 * hb + e], z[8 * hb + e]));
                                __syncwarp();
                                const uint4 v = *reinterpret_cast<const uint4 *>(ost + lane * 16);
                                __syncwarp();
                                const int i0 = 16 * q + 8 * hb;   // first token of this group
                                if (!GENERAL || (Dv & 7) == 0) {
                                    if (outputs_on && i0 + tt < len_n && (!GENERAL || ocol < Dv) &&
                                        in_range(((int64_t)(un.start + n * C + tt + i0) * p.Hv + un.h) * Dv + ocol,
                                                 8, (int64_t)p.N * p.Hv * Dv, p.dev_status))
                                        *reinterpret_cast<uint4 *>(obase + (i0 / 8) * ostride8) = v;
                                } else if (i0 + tt < len_n && ocol < Dv) {
                                    // rows of Dv elements with Dv % 8 != 0: element stores, only
                                    // the head's own columns
                                    const int ne = min(8, Dv - ocol);
                                    const uint16_t *ve = reinterpret_cast<const uint16_t *>(&v);
                                    if (in_range(((int64_t)(un.start + n * C + tt + i0) * p.Hv + un.h) * Dv + ocol,
                                                 ne, (int64_t)p.N * p.Hv * Dv, p.dev_status))
                                        for (int e = 0; e < ne; ++e) obase[(i0 / 8) * ostride8 + e] = ve[e];
                                }
                            }
                        }
                        tc_fence_before();
                        named_sync(2, 128);
                        if (dv == 0) mbar_arrive(cx.bar(B_Y_FREE));
                    }
                    ok = !named_sync_or(2, 128, !ok || cx.aborted());
                }
                gc += nc;
                pre = has_next;
                if (!ok) break;
            }
        }
        __syncthreads();
        if (cx.aborted()) break;
        batch0 += wcover;
    }

    // teardown after an abort: every role has left its loop (each wait ends on the abort flag
    // or its own bound, each group leaves through its vote) and met the barrier above.  Copies
    // and MMAs still in flight land before the shared memory and TMEM go away: each TMA lane
    // waits for the last copy of every stage it filled, each UMMA issuer commits once more and
    // waits for that commit (it arrives when all of the thread's earlier MMAs completed).  An
    // operation on its way completes within microseconds, so these waits are short (2^24
    // cycles, ~8 ms) rather than a second bound on bytes that may never come.
    if (cx.aborted()) {
        constexpr long long kDrain = 1ll << 24;
        if (warp == TMA_WARP && lane < 2) {
            for (int s = 0; s < KQ_STAGES; ++s) {
                const long long t0 = clock64();
                while (kq_use[s] > 0 && !mbar_try_wait(cx.bar(B_KQ_FULL + s), (kq_use[s] - 1) & 1))
                    if (clock64() - t0 > kDrain) break;
            }
            const long long t0 = clock64();
            while (v_use > 0 && !mbar_try_wait(cx.bar(B_V_FULL), (v_use - 1) & 1))
                if (clock64() - t0 > kDrain) break;
        }
        if ((warp == MMA_WARP || warp == ISSUE_WARP) && lane == 0) {
            const uint32_t db = cx.bar(warp == MMA_WARP ? B_DRAIN_CHAIN : B_DRAIN_PREP);
            umma_commit(db);
            const long long t0 = clock64();
            while (!mbar_try_wait(db, 0))
                if (clock64() - t0 > kDrain) break;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) tmem_dealloc(tmem, 512);
}

}  // namespace gdn_chunk

// ============================================================================ host side
namespace {

// the driver's tensor-map encoder, looked up once (thread-safe static initialisation)
PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

bool make_map_3d_16(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                    bool f16)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d_f32(CUtensorMap *m, const void *base, uint64_t d0, uint64_t d1)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {d0 * 4};
    cuuint32_t box[2] = {4, 64};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms()
{
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace

// Head sizes up to 128 of bf16 or fp16 run on the tensor cores.  Rows the tensor maps can
// describe (Dk, Dv multiples of 8, Hv % 4 == 0) are loaded by the TMA; any other size is
// staged with plain loads into the same zero-padded tiles.
bool prefill_chunked_supported(const GdnPrefillArgs &a)
{
    return (a.dtype == GDN_BF16 || a.dtype == GDN_F16) && a.Dk >= 1 && a.Dk <= 128 &&
           a.Dv >= 1 && a.Dv <= 128 && get_encode() != nullptr;
}

static bool prefill_needs_plain_staging(const GdnPrefillArgs &a)
{
    return a.Dk % 8 != 0 || a.Dv % 8 != 0 || a.Hv % 4 != 0;
}

// The split (seqpar.cuh) runs the default bf16 instantiation on 128-wide heads, for calls with
// few requests whose units fit one per SM; the device decides per request whether to split.
uint64_t prefill_split_workspace_bytes(const GdnPrefillArgs &a)
{
    if (!prefill_chunked_supported(a) || prefill_needs_plain_staging(a)) return 0;
    if (a.dtype != GDN_BF16 || a.Dk != 128 || a.Dv != 128) return 0;
    if (!a.has_decay || !a.has_retrieval || a.beta_sigmoid || a.a_log) return 0;
    if (a.B < 1 || a.B > gdn_seq::MAX_REQ || a.B * a.Hv > gdn_seq::MAX_UNITS_PER_CALL) return 0;
    if (a.B * a.Hv > num_sms()) return 0;
    return gdn_seq::workspace_bytes(a.B, a.Hv, a.Dk, a.Dv);
}

cudaError_t launch_prefill_chunked(const GdnPrefillArgs &a, cudaStream_t stream)
{
    using namespace gdn_chunk;
    if (a.B == 0) return cudaSuccess;
    static DeviceOnce smem_opt_in;
    cudaError_t attr_err = smem_opt_in.run([] {
        cudaError_t e = cudaFuncSetAttribute(gdn_prefill_chunk_kernel<false, false>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_prefill_chunk_kernel<true, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_prefill_chunk_kernel<true, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_prefill_chunk_kernel<false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        return e;
    });
    if (attr_err != cudaSuccess) return attr_err;
    Params p;
    memset(&p, 0, sizeof(p));
    const uint64_t N = (uint64_t)(a.N > 0 ? a.N : 1);
    const bool plain = prefill_needs_plain_staging(a);
    // TMA maps need a valid base even when N == 0 (no chunk is loaded then)
    if (a.N > 0 && !plain) {
        // head dims below 128 read zeros past their end (TMA fill), so every tile is a
        // zero-padded 128-wide tile and the products are unchanged
        const bool f16 = a.dtype == GDN_F16;
        if (!make_map_3d_16(&p.tm_q, a.q, a.Dk, a.Hq, N, f16) ||
            !make_map_3d_16(&p.tm_k, a.k, a.Dk, a.Hq, N, f16) ||
            !make_map_3d_16(&p.tm_v, a.v, a.Dv, a.Hv, N, f16) ||
            (a.has_decay && !make_map_2d_f32(&p.tm_g, a.g, a.Hv, N)) ||
            (a.has_retrieval && !make_map_2d_f32(&p.tm_beta, a.beta, a.Hv, N)))
            return cudaErrorInvalidValue;
    }
    p.cu_seqlens = a.cu_seqlens;
    p.initial_state = a.initial_state;
    p.final_state = a.final_state;
    p.out = static_cast<uint16_t *>(a.out);
    p.dev_status = a.dev_status;
    p.N = a.N;
    p.B = a.B;
    p.Hq = a.Hq;
    p.Hv = a.Hv;
    p.scale = a.scale;
    p.qk_l2norm = a.qk_l2norm;
    p.has_decay = a.has_decay;
    p.has_retrieval = a.has_retrieval;
    p.beta_sigmoid = a.beta_sigmoid;
    p.Dk = a.Dk;
    p.Dv = a.Dv;
    p.a_log = a.a_log;
    p.dt_bias = a.dt_bias;
    p.stage_plain = plain ? 1 : 0;
    p.q = static_cast<const uint16_t *>(a.q);
    p.k = static_cast<const uint16_t *>(a.k);
    p.v = static_cast<const uint16_t *>(a.v);
    p.g = a.g;
    p.beta = a.beta;
    const int units = a.B * a.Hv;
    const int nsm = num_sms();
    const int grid = units < nsm ? units : nsm;
    const uint64_t ws_need = prefill_split_workspace_bytes(a);
    if (ws_need > 0 && a.workspace && a.workspace_bytes >= ws_need) {
        // pass 1, composition, pass 3 (seqpar.cuh); every launch sees the same CTA count, on
        // which the split rule depends
        // (grids: at most three units per (request, head) in pass 1 and two in pass 3)
        p.seq_ws = static_cast<float *>(a.workspace);
        p.seq_G = nsm;
        p.seq_pass = 1;
        const int g1 = 3 * units < nsm ? 3 * units : nsm, g3 = 2 * units < nsm ? 2 * units : nsm;
        gdn_prefill_chunk_kernel<false, false, true><<<g1, NTHREADS, SMEM_BYTES, stream>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        e = launch_seq_compose(a, a.workspace, nsm, stream);
        if (e != cudaSuccess) return e;
        p.seq_pass = 3;
        gdn_prefill_chunk_kernel<false, false, true><<<g3, NTHREADS, SMEM_BYTES, stream>>>(p);
        return cudaGetLastError();
    }
    const bool general = !a.has_decay || !a.has_retrieval || a.beta_sigmoid || a.a_log != nullptr ||
                         a.Dk != D || a.Dv != D || plain;
    // fp16 activations run the general instantiation with fp16 operand tiles
    if (a.dtype == GDN_F16)
        gdn_prefill_chunk_kernel<true, true><<<grid, NTHREADS, SMEM_BYTES, stream>>>(p);
    else if (general)
        gdn_prefill_chunk_kernel<true, false><<<grid, NTHREADS, SMEM_BYTES, stream>>>(p);
    else
        gdn_prefill_chunk_kernel<false, false><<<grid, NTHREADS, SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}
