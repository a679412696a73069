// prefill_compose.cu -- the composition step of the sequence-parallel prefill split.
//
// For every split request b and value head h (the split rule of seqpar.cuh, evaluated on the
// device from cu_seqlens exactly as the chunked kernel evaluates it):
//     S2^T = S1^T A1^T + B1^T        (V-major: S2[dv][dk] = sum_j S1[dv][j] A1[j][dk] + B1[dv][dk])
// where S1 is the true start state of segment 1, A1^T and B1^T are segment 1's affine map
// (the final states of its identity and zero runs).  fp32 FMA, a 32 x 32 tile per CTA.
#include "common.cuh"
#include "seqpar.cuh"

namespace {

__device__ int request_chunks(const GdnPrefillArgs &a, int b)
{
    int64_t st, en;
    if (a.cu_seqlens) {
        st = a.cu_seqlens[b];
        en = a.cu_seqlens[b + 1];
        st = st < 0 ? 0 : (st > a.N ? a.N : st);
        en = en < 0 ? 0 : (en > a.N ? a.N : en);
    } else {
        const int64_t S = a.N / a.B;
        st = (int64_t)b * S;
        en = st + S;
    }
    const int64_t len = en > st ? en - st : 0;
    return (int)((len + gdn_seq::C - 1) / gdn_seq::C);
}

// Block (b, h, tile): a 32 x 32 tile of S2 (rows dv0.., columns dk0..) for request b, head
// h.  The tile's 32 rows of S1 and 32 columns of A1 (all j) are staged in shared memory;
// each of the 256 threads accumulates a 2 x 2 block over j in fp32.
constexpr int TS = 32;

__global__ void __launch_bounds__(256) seq_compose_kernel(const GdnPrefillArgs a, gdn_seq::Workspace ws, int G)
{
    __shared__ int nc[gdn_seq::MAX_REQ];
    __shared__ uint32_t mask;
    __shared__ float sS[TS][128 + 1];   // S1 rows dv0 .. dv0 + 31, all j
    __shared__ float sA[128][TS + 1];   // A1 rows j, columns dk0 .. dk0 + 31
    const int Dk = a.Dk, Dv = a.Dv;
    const int tv = (Dv + TS - 1) / TS, tk = (Dk + TS - 1) / TS;
    const int bh = blockIdx.x / (tv * tk), t = blockIdx.x - bh * (tv * tk);
    const int dv0 = (t / tk) * TS, dk0 = (t % tk) * TS;
    const int b = bh / a.Hv, h = bh - b * a.Hv;
    if (threadIdx.x < a.B) nc[threadIdx.x] = request_chunks(a, threadIdx.x);
    __syncthreads();
    if (threadIdx.x == 0) mask = gdn_seq::split_mask(nc, a.B, a.Hv, G);
    __syncthreads();
    if (!((mask >> b) & 1u)) return;
    const float *S1 = ws.S1(b, h), *A1 = ws.A1(b, h), *B1 = ws.B1(b, h);
    float *S2 = ws.S2(b, h);
    for (int i = threadIdx.x; i < TS * 128; i += 256) {
        const int r = i / 128, j = i % 128;
        sS[r][j] = (dv0 + r < Dv && j < Dk) ? S1[(int64_t)(dv0 + r) * Dk + j] : 0.f;
        const int jj = i / TS, c = i % TS;
        sA[jj][c] = (jj < Dk && dk0 + c < Dk) ? A1[(int64_t)jj * Dk + dk0 + c] : 0.f;
    }
    __syncthreads();
    const int r = 2 * (threadIdx.x / 16), c = 2 * (threadIdx.x % 16);
    float acc00 = 0.f, acc01 = 0.f, acc10 = 0.f, acc11 = 0.f;
#pragma unroll 8
    for (int j = 0; j < Dk; ++j) {
        const float s0 = sS[r][j], s1 = sS[r + 1][j];
        const float a0 = sA[j][c], a1 = sA[j][c + 1];
        acc00 = fmaf(s0, a0, acc00);
        acc01 = fmaf(s0, a1, acc01);
        acc10 = fmaf(s1, a0, acc10);
        acc11 = fmaf(s1, a1, acc11);
    }
    const float accs[2][2] = {{acc00, acc01}, {acc10, acc11}};
#pragma unroll
    for (int y = 0; y < 2; ++y)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int dv = dv0 + r + y, dk = dk0 + c + x;
            if (dv < Dv && dk < Dk) {
                const int64_t o = (int64_t)dv * Dk + dk;
                S2[o] = accs[y][x] + B1[o];
            }
        }
}

}  // namespace

cudaError_t launch_seq_compose(const GdnPrefillArgs &a, void *workspace, int G, cudaStream_t stream)
{
    gdn_seq::Workspace ws{static_cast<float *>(workspace), a.B, a.Hv, a.Dk, a.Dv};
    const int tiles = ((a.Dv + TS - 1) / TS) * ((a.Dk + TS - 1) / TS);
    seq_compose_kernel<<<a.B * a.Hv * tiles, 256, 0, stream>>>(a, ws, G);
    return cudaGetLastError();
}
