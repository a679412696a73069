// conv1d.cu -- causal depthwise conv1d over ragged requests with a
// slot-indexed pool of conv windows, updated in place.
//
// Operation ("max.nn.legacy.state_space.gated_delta_conv1d_fwd", description,
// Parameters, example): request b covers tokens [s, e) of x [N, conv_dim] and
// owns slot r = slot_idx[b] of the pool [max_slots, conv_dim, K-1].  Channel
// c convolves xe = (pool[r, c, 0..K-2], x[s..e-1, c]) with weight[c, 0..K-1]
// (index K-1 meets the current token); the slot then holds the last K-1
// entries of xe.
//
// HBM-bound: every input row is read once (plus K-1 look-back rows per chunk,
// mostly L2 hits), every output row written once, each request's window read
// and written once.  Work layout:
//   - a block is (request-aligned chunk of L tokens, channel tile), the tile
//     index varying fastest along the 1-D grid; a thread owns V adjacent
//     channels -- 16 bytes of a row, so a warp reads 512 contiguous bytes per
//     token -- and walks its chunk in token order with the last K-1 inputs in
//     registers, 8 rows loaded ahead when chunks are long (L >= 32);
//   - L is the largest of 128, 64, ..., 8 that still gives about two waves of
//     blocks, chosen on the host from N and conv_dim only;
//   - chunks never straddle requests: block x finds its (request, chunk) by a
//     block-wide prefix sum of ceil(len_b / L), so the host reads no device
//     data and the launch can be captured in a graph;
//   - only chunk 0 of a request touches its pool slot: it reads the old
//     window for its look-back and, after that, writes the new one, so no
//     block ever sees a half-updated slot.  Later chunks take their
//     look-back from x (L >= K-1).
#include <cuda_fp16.h>

#include <type_traits>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn_conv {

using namespace sm100;
using gdn::in_range;
using gdn::in_smem;

constexpr int kThreads = 128;
constexpr int kVecBytes = 16;  // bytes of a row per thread on the vector path
constexpr int kBatchLong = 8;  // rows loaded ahead per thread (chunks >= 32 tokens)

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <>
__device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

// NE consecutive elements starting at p: kVecBytes-wide accesses on the vector
// path (NE * sizeof(T) is then a multiple of kVecBytes and p aligned to it),
// element accesses otherwise.  Raw words are kept so that loads can be issued ahead
// of their conversion.
template <typename T, int NE, bool VEC>
struct Flat {
    using Vw = typename std::conditional<kVecBytes == 16, uint4, uint2>::type;
    static constexpr int kWords = VEC ? NE * (int)sizeof(T) / kVecBytes : NE;
    using Word = typename std::conditional<VEC, Vw, T>::type;
    Word w[kWords];

    __device__ __forceinline__ void load(const T *p)
    {
        const Word *q = reinterpret_cast<const Word *>(p);
#pragma unroll
        for (int i = 0; i < kWords; ++i) w[i] = __ldg(q + i);
    }
    __device__ __forceinline__ void to_float(float (&f)[NE]) const
    {
        const T *e = reinterpret_cast<const T *>(w);
#pragma unroll
        for (int i = 0; i < NE; ++i) f[i] = to_f<T>(e[i]);
    }
    __device__ __forceinline__ void from_float(const float (&f)[NE])
    {
        T *e = reinterpret_cast<T *>(w);
#pragma unroll
        for (int i = 0; i < NE; ++i) e[i] = from_f<T>(f[i]);
    }
    __device__ __forceinline__ void store(T *p, bool streaming) const
    {
        Word *q = reinterpret_cast<Word *>(p);
#pragma unroll
        for (int i = 0; i < kWords; ++i) {
            if (streaming)
                __stcs(q + i, w[i]);
            else
                q[i] = w[i];
        }
    }
};

// inclusive block prefix sum of one int per thread; returns the block total in *total
__device__ __forceinline__ int block_scan(int x, int *s_warp, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        const int t = s_warp[w];
        before += w < warp ? t : 0;
        all += t;
    }
    __syncthreads();  // s_warp is reused by the next call
    *total = all;
    return x + before;
}

// Block-wide: the request b and chunk index ci of this block's chunk (b = -1 past the last
// chunk; the grid is an upper bound).  Chunks are numbered request by request, request b
// owning ceil(len_b / L) of them.  Every thread of the block must call it.
__device__ __forceinline__ int2 find_chunk(const GdnConv1dArgs &a, int chunk, int L, int *s_warp,
                                           int *s_ref)
{
    const int N32 = (int)a.N;
    if (threadIdx.x == 0) s_ref[0] = -1;
    int base = 0;
    for (int b0 = 0; b0 < a.B; b0 += kThreads) {
        const int b = b0 + threadIdx.x;
        int cnt = 0;
        if (b < a.B) {
            const int s = (int)min(a.offsets[b], (uint32_t)N32);
            const int e = (int)min(a.offsets[b + 1], (uint32_t)N32);
            cnt = e > s ? (int)(((int64_t)(e - s) + L - 1) / L) : 0;
        }
        int total;
        const int incl = block_scan(cnt, s_warp, &total);  // its barriers order s_ref too
        if (cnt > 0 && chunk >= base + incl - cnt && chunk < base + incl) {
            s_ref[0] = b;
            s_ref[1] = chunk - (base + incl - cnt);
        }
        base += total;
        __syncthreads();
        if (s_ref[0] >= 0 || chunk < base) break;
    }
    __syncthreads();
    return make_int2(s_ref[0], s_ref[1]);
}

// bounded wait for phase 0 of a copy barrier; false (and GDN_DEV_TIMEOUT) when it does not
// complete within ~2^31 cycles
__device__ __forceinline__ bool wait_copies(uint32_t bar, int32_t *dev_status)
{
    if (mbar_try_wait(bar, 0)) return true;
    const long long start = clock64();
    while (!mbar_try_wait(bar, 0)) {
        if (clock64() - start > (1ll << 31)) {
            if (dev_status) atomicOr(dev_status, GDN_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Checked builds: the rows a block touches (its chunk [t0, t1), the K-1 look-back rows of a later
// chunk, the last K-1 rows of the request for a first chunk that does not reach its end), its
// channels [c, c + nc) and its window slot r all lie inside their buffers.  Every access of the
// block is inside these ranges.  Always true in other builds.
template <int W>
__device__ __forceinline__ bool rows_in_range(const GdnConv1dArgs &a, int ci, int t0, int t1, int e,
                                              int c, int nc, uint32_t r)
{
    if constexpr (!gdn::kChecked) return true;
    int lo = ci > 0 ? t0 - W : t0;
    int hi = t1;
    if (W > 0 && ci == 0 && t1 < e) {
        lo = min(lo, e - W);
        hi = e;
    }
    const int64_t cd = a.conv_dim;
    return in_range(lo, hi - lo, a.N, a.dev_status) && in_range(c, nc, cd, a.dev_status) &&
           (W == 0 || in_range(((int64_t)r * cd + c) * W, (int64_t)nc * W, (int64_t)a.max_slots * cd * W,
                               a.dev_status));
}

// Element path (rows not 16-byte aligned): every access goes through registers.
template <typename T, int K, bool VEC, int kBatch>
__global__ void __launch_bounds__(kThreads) conv1d_kernel(const GdnConv1dArgs a, const int L, const int tiles)
{
    constexpr int V = VEC ? kVecBytes / (int)sizeof(T) : 1;
    constexpr int W = K - 1;
    __shared__ int s_warp[kThreads / 32];
    __shared__ int s_ref[2];

    // ---- weights first (they do not depend on the request): V channels x K taps
    // the channel tile varies fastest along the grid, so blocks resident together cover
    // whole rows
    const int tile = (int)(blockIdx.x % (unsigned)tiles);
    const int chunk = (int)(blockIdx.x / (unsigned)tiles);
    const int c0 = (tile * kThreads + threadIdx.x) * V;
    const bool has_ch = c0 < a.conv_dim &&
                        in_range((int64_t)c0 * K, V * K, (int64_t)a.conv_dim * K, a.dev_status);
    Flat<T, V * K, VEC> fw;
    if (has_ch) fw.load(static_cast<const T *>(a.weight) + (int64_t)c0 * K);

    // ---- which (request, chunk) this block covers
    const int N32 = (int)a.N;
    const int2 ref = find_chunk(a, chunk, L, s_warp, s_ref);
    const int b = ref.x;
    if (b < 0) return;  // past the last chunk (the grid is an upper bound)
    const int ci = ref.y;
    const int s = (int)min(a.offsets[b], (uint32_t)N32);
    const int e = (int)min(a.offsets[b + 1], (uint32_t)N32);
    const uint32_t r = a.slot_idx[b];
    if (r >= (uint32_t)a.max_slots) {
        if (ci == 0 && tile == 0 && threadIdx.x == 0 && a.dev_status)
            atomicOr(a.dev_status, GDN_DEV_BAD_SLOT);
        return;
    }
    if (!has_ch) return;

    const T *__restrict__ x = static_cast<const T *>(a.x);
    T *__restrict__ out = static_cast<T *>(a.out);
    const int64_t ld = a.conv_dim;
    const int t0 = s + ci * L;
    const int t1 = min(e, t0 + L);
    if (!rows_in_range<W>(a, ci, t0, t1, e, c0, V, r)) return;

    float wf[K][V];
    {
        float f[V * K];
        fw.to_float(f);
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < K; ++j) wf[j][v] = f[v * K + j];
    }

    // ---- look-back window, oldest first
    float xw[W > 0 ? W : 1][V];
    T *const slot = W > 0 ? static_cast<T *>(a.conv_state) + ((int64_t)r * a.conv_dim + c0) * W
                          : nullptr;
    if (W > 0) {
        if (ci == 0) {
            Flat<T, V * (W > 0 ? W : 1), VEC> fs;
            fs.load(slot);
            float f[V * (W > 0 ? W : 1)];
            fs.to_float(f);
#pragma unroll
            for (int v = 0; v < V; ++v)
#pragma unroll
                for (int j = 0; j < W; ++j) xw[j][v] = f[v * W + j];
        } else {
#pragma unroll
            for (int j = 0; j < W; ++j) {
                Flat<T, V, VEC> fx;
                fx.load(x + (int64_t)(t0 - W + j) * ld + c0);
                float f[V];
                fx.to_float(f);
#pragma unroll
                for (int v = 0; v < V; ++v) xw[j][v] = f[v];
            }
        }
    }

    // ---- the chunk's tokens: full batches of kBatch rows loaded ahead, then the rest
    // one row at a time
    const T *xp = x + (int64_t)t0 * ld + c0;
    T *op = out + (int64_t)t0 * ld + c0;
    auto step = [&](const Flat<T, V, VEC> &fx) {
        float xn[V], y[V];
        fx.to_float(xn);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) acc = fmaf(wf[j][v], xw[j][v], acc);
            y[v] = fmaf(wf[W][v], xn[v], acc);
        }
#pragma unroll
        for (int j = 0; j + 1 < W; ++j)
#pragma unroll
            for (int v = 0; v < V; ++v) xw[j][v] = xw[j + 1][v];
        if (W > 0) {
#pragma unroll
            for (int v = 0; v < V; ++v) xw[W > 0 ? W - 1 : 0][v] = xn[v];
        }
        Flat<T, V, VEC> fy;
        fy.from_float(y);
        fy.store(op, true);
        op += ld;
    };
    int t = t0;
    for (; t + kBatch <= t1; t += kBatch) {
        Flat<T, V, VEC> fx[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) fx[u].load(xp + u * ld);
        xp += kBatch * ld;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) step(fx[u]);
    }
#pragma unroll 1
    for (; t < t1; ++t) {
        Flat<T, V, VEC> fx;
        fx.load(xp);
        xp += ld;
        step(fx);
    }

    // ---- new window (chunk 0 only; it has read the old one above)
    if (W > 0 && ci == 0 && a.write_state) {
        if (t1 < e) {
            // the request continues past this chunk, so it has >= L >= K-1 tokens: the
            // window is its last K-1 inputs
#pragma unroll
            for (int j = 0; j < W; ++j) {
                Flat<T, V, VEC> fx;
                fx.load(x + (int64_t)(e - W + j) * ld + c0);
                float f[V];
                fx.to_float(f);
#pragma unroll
                for (int v = 0; v < V; ++v) xw[j][v] = f[v];
            }
        }
        // else the sliding window after the last token already is the new one
        float f[V * (W > 0 ? W : 1)];
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < W; ++j) f[v * W + j] = xw[j][v];
        Flat<T, V * (W > 0 ? W : 1), VEC> fs;
        fs.from_float(f);
        fs.store(slot, false);
    }
}

// Vector path (rows 16-byte aligned, conv_dim * sizeof(T) a multiple of 16).  The chunk's
// rows of this channel tile -- plus the K-1 look-back rows when the chunk is not the
// request's first -- are staged in shared memory by bulk async copies, one per row, all
// completing on one mbarrier: up to (L + K-1) x 2 KB in flight per block, independent of
// the register budget.  Threads then read their 16 bytes per row from shared memory.
constexpr int kRowBytes = kThreads * 16;  // one row of a channel tile
constexpr int kStagedMaxL = 32;

template <typename T, int K>
__global__ void __launch_bounds__(kThreads) conv1d_staged_kernel(const GdnConv1dArgs a,
                                                                 const int L, const int tiles)
{
    constexpr int V = 16 / (int)sizeof(T);
    constexpr int W = K - 1;
    extern __shared__ __align__(128) uint8_t stage[];  // (L + W) rows of kRowBytes
    __shared__ int s_warp[kThreads / 32];
    __shared__ int s_ref[2];
    __shared__ __align__(8) uint64_t s_bar;

    const int tile = (int)(blockIdx.x % (unsigned)tiles);
    const int chunk = (int)(blockIdx.x / (unsigned)tiles);
    const int tc0 = tile * kThreads * V;  // first channel of the tile
    const int c0 = tc0 + threadIdx.x * V;
    const bool has_ch = c0 < a.conv_dim &&
                        in_range((int64_t)c0 * K, V * K, (int64_t)a.conv_dim * K, a.dev_status);
    const uint32_t bar = smem_u32(&s_bar);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    Flat<T, V * K, true> fw;
    if (has_ch) fw.load(static_cast<const T *>(a.weight) + (int64_t)c0 * K);

    const int2 ref = find_chunk(a, chunk, L, s_warp, s_ref);  // its barriers publish the init
    const int b = ref.x;
    if (b < 0) return;
    const int ci = ref.y;
    const int N32 = (int)a.N;
    const int s = (int)min(a.offsets[b], (uint32_t)N32);
    const int e = (int)min(a.offsets[b + 1], (uint32_t)N32);
    const T *__restrict__ x = static_cast<const T *>(a.x);
    const int64_t ld = a.conv_dim;
    const int t0 = s + ci * L;
    const int t1 = min(e, t0 + L);
    const int r0 = ci > 0 ? t0 - W : t0;  // first staged row
    const uint32_t row_bytes = (uint32_t)min(kThreads * V, a.conv_dim - tc0) * (uint32_t)sizeof(T);
    const uint32_t r = __ldg(a.slot_idx + b);
    if (r >= (uint32_t)a.max_slots) {
        if (ci == 0 && tile == 0 && threadIdx.x == 0 && a.dev_status)
            atomicOr(a.dev_status, GDN_DEV_BAD_SLOT);
        return;
    }
    // (checked builds) the tile's rows, channels, window slot and stage, tested block-wide
    // before any copy is issued
    if (!rows_in_range<W>(a, ci, t0, t1, e, tc0, (int)(row_bytes / sizeof(T)), r) ||
        !in_smem(stage, (uint32_t)(t1 - r0) * kRowBytes, a.dev_status))
        return;
    if (threadIdx.x == 0) {
        const int nrows = t1 - r0;
        mbar_arrive_expect_tx(bar, (uint32_t)nrows * row_bytes);
        const T *src = x + (int64_t)r0 * ld + tc0;
        const uint32_t dst = smem_u32(stage);
        for (int i = 0; i < nrows; ++i)
            bulk_load_1d(dst + (uint32_t)i * kRowBytes, src + (int64_t)i * ld, row_bytes, bar);
    }
    if (!has_ch) return;  // thread 0 always has channels, so the copies are waited for

    float wf[K][V];
    {
        float f[V * K];
        fw.to_float(f);
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < K; ++j) wf[j][v] = f[v * K + j];
    }
    float xw[W > 0 ? W : 1][V];
    T *const slot = W > 0 ? static_cast<T *>(a.conv_state) + ((int64_t)r * a.conv_dim + c0) * W
                          : nullptr;
    if (W > 0 && ci == 0) {
        Flat<T, V * (W > 0 ? W : 1), true> fs;
        fs.load(slot);
        float f[V * (W > 0 ? W : 1)];
        fs.to_float(f);
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < W; ++j) xw[j][v] = f[v * W + j];
    }
    if (!wait_copies(bar, a.dev_status)) return;

    const uint8_t *sp = stage + threadIdx.x * 16;
    auto staged = [&](int row, float (&f)[V]) {
        Flat<T, V, true> fx;
        fx.w[0] = *reinterpret_cast<const uint4 *>(sp + row * kRowBytes);
        fx.to_float(f);
    };
    if (W > 0 && ci > 0) {
#pragma unroll
        for (int j = 0; j < W; ++j) staged(j, xw[j]);
    }
    T *op = static_cast<T *>(a.out) + (int64_t)t0 * ld + c0;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        float xn[V], y[V];
        staged(t - r0, xn);
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < W; ++j) acc = fmaf(wf[j][v], xw[j][v], acc);
            y[v] = fmaf(wf[W][v], xn[v], acc);
        }
#pragma unroll
        for (int j = 0; j + 1 < W; ++j)
#pragma unroll
            for (int v = 0; v < V; ++v) xw[j][v] = xw[j + 1][v];
        if (W > 0) {
#pragma unroll
            for (int v = 0; v < V; ++v) xw[W > 0 ? W - 1 : 0][v] = xn[v];
        }
        Flat<T, V, true> fy;
        fy.from_float(y);
        fy.store(op, true);
        op += ld;
    }

    // new window (chunk 0 only; it read the old one above)
    if (W > 0 && ci == 0 && a.write_state) {
        if (t1 < e) {
            // the request continues past this chunk (so it has >= L >= K-1 tokens): the
            // window is its last K-1 inputs, read from x
#pragma unroll
            for (int j = 0; j < W; ++j) {
                Flat<T, V, true> fx;
                fx.load(x + (int64_t)(e - W + j) * ld + c0);
                fx.to_float(xw[j]);
            }
        }
        float f[V * (W > 0 ? W : 1)];
#pragma unroll
        for (int v = 0; v < V; ++v)
#pragma unroll
            for (int j = 0; j < W; ++j) f[v * W + j] = xw[j][v];
        Flat<T, V * (W > 0 ? W : 1), true> fs;
        fs.from_float(f);
        fs.store(slot, false);
    }
}

int device_sms()
{
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

// tokens per chunk: the largest of max_L, max_L / 2, ..., 8 that still gives about two
// waves of blocks on the device (L >= 8 >= K-1 always holds)
int chunk_tokens(int64_t N, int tiles, int max_L)
{
    const int64_t target = (int64_t)device_sms() * 16;
    int L = max_L;
    while (L > 8 && ((N + L - 1) / L) * tiles < target) L >>= 1;
    return L;
}

template <typename T, bool VEC, int NB>
cudaError_t launch_k(const GdnConv1dArgs &a, dim3 grid, int L, int tiles, cudaStream_t stream)
{
    switch (a.K) {
    case 1: conv1d_kernel<T, 1, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 2: conv1d_kernel<T, 2, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 3: conv1d_kernel<T, 3, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 4: conv1d_kernel<T, 4, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 5: conv1d_kernel<T, 5, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 6: conv1d_kernel<T, 6, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 7: conv1d_kernel<T, 7, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    case 8: conv1d_kernel<T, 8, VEC, NB><<<grid, kThreads, 0, stream>>>(a, L, tiles); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename T, int K>
cudaError_t launch_staged_k(const GdnConv1dArgs &a, int L, int tiles, int64_t chunks,
                            cudaStream_t stream)
{
    const size_t smem = (size_t)(L + K - 1) * kRowBytes;
    static DeviceOnce smem_opt_in;   // the largest stage any call uses
    const cudaError_t e = smem_opt_in.run([] {
        return cudaFuncSetAttribute(conv1d_staged_kernel<T, K>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (kStagedMaxL + K - 1) * kRowBytes);
    });
    if (e != cudaSuccess) return e;
    conv1d_staged_kernel<T, K><<<(unsigned)(chunks * tiles), kThreads, smem, stream>>>(a, L, tiles);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_staged(const GdnConv1dArgs &a, cudaStream_t stream)
{
    constexpr int V = 16 / (int)sizeof(T);
    const int tiles = (a.conv_dim + kThreads * V - 1) / (kThreads * V);
    const int L = chunk_tokens(a.N, tiles, kStagedMaxL);
    const int64_t chunks = (a.N + L - 1) / L + a.B;  // request-aligned chunks, upper bound
    if (chunks * tiles > 0x7fffffff) return cudaErrorInvalidConfiguration;
    switch (a.K) {
    case 1: return launch_staged_k<T, 1>(a, L, tiles, chunks, stream);
    case 2: return launch_staged_k<T, 2>(a, L, tiles, chunks, stream);
    case 3: return launch_staged_k<T, 3>(a, L, tiles, chunks, stream);
    case 4: return launch_staged_k<T, 4>(a, L, tiles, chunks, stream);
    case 5: return launch_staged_k<T, 5>(a, L, tiles, chunks, stream);
    case 6: return launch_staged_k<T, 6>(a, L, tiles, chunks, stream);
    case 7: return launch_staged_k<T, 7>(a, L, tiles, chunks, stream);
    case 8: return launch_staged_k<T, 8>(a, L, tiles, chunks, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T, bool VEC>
cudaError_t launch_t(const GdnConv1dArgs &a, cudaStream_t stream)
{
    constexpr int V = VEC ? kVecBytes / (int)sizeof(T) : 1;
    const int tiles = (a.conv_dim + kThreads * V - 1) / (kThreads * V);
    const int L = chunk_tokens(a.N, tiles, 128);
    const int64_t chunks = (a.N + L - 1) / L + a.B;  // request-aligned chunks, upper bound
    if (chunks * tiles > 0x7fffffff) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)(chunks * tiles));
    // short chunks (few tokens per request) take the batch-1 body: fewer registers, more
    // resident blocks to hide the per-block lookup latency
    return L >= 32 ? launch_k<T, VEC, kBatchLong>(a, grid, L, tiles, stream)
                   : launch_k<T, VEC, 1>(a, grid, L, tiles, stream);
}

template <typename T>
cudaError_t launch_dtype(const GdnConv1dArgs &a, bool vec, cudaStream_t stream)
{
    return vec ? launch_staged<T>(a, stream) : launch_t<T, false>(a, stream);
}

}  // namespace gdn_conv

cudaError_t launch_conv1d(const GdnConv1dArgs &a, cudaStream_t stream)
{
    using namespace gdn_conv;
    if (a.B == 0 || a.N == 0) return cudaSuccess;
    const size_t esz = a.dtype == GDN_F32 ? 4 : 2;
    auto alv = [](const void *p) { return ((uintptr_t)p & (kVecBytes - 1)) == 0; };
    const bool vec = ((size_t)a.conv_dim * esz) % kVecBytes == 0 && alv(a.x) && alv(a.out) &&
                     alv(a.weight) && (a.K == 1 || alv(a.conv_state));
    if (a.dtype == GDN_F32) return launch_dtype<float>(a, vec, stream);
    if (a.dtype == GDN_F16) return launch_dtype<__half>(a, vec, stream);
    return launch_dtype<__nv_bfloat16>(a, vec, stream);
}
