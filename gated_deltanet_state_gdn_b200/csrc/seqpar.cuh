// seqpar.cuh -- sequence-parallel split of long requests for the chunked prefill.
//
// The recurrence of "com.microsoft.GatedDeltaNet" (Description) is affine in the state: over
// a run of tokens, S_end = A S_start + B with A (Dk x Dk) and B (Dk x Dv) fixed by the run's
// q/k/v/g/beta (the op's Attributes table states that the result does not depend on how the
// sequence is chunked).  When a call holds too few (request, value head) units to fill the
// GPU, a long request is cut into three segments of whole chunks:
//   pass 1 (one launch of the chunked kernel, one unit per CTA):
//     segment 0 from the true initial state, with its outputs; its final state is the true
//       start state of segment 1;
//     segment 1 from the identity (with v = 0): its final state is A_1^T;
//     segment 1 from zero: its final state is B_1^T;
//   compose: start of segment 2 = (start of segment 1) A_1^T + B_1^T (V-major, fp32);
//   pass 3: segments 1 and 2 from their true start states, with their outputs; segment 2's
//     final state is the request's.
// The three passes take two segment lengths of chunk chains instead of three (the state
// chain of a unit is sequential; its period, not the tensor rate, sets a unit's time).
//
// Every CTA of both passes, the compose kernel and the host agree on the split through the
// functions below, which read only the request lengths.
#pragma once

#include <stdint.h>

namespace gdn_seq {

constexpr int C = 64;                 // chunk length (tokens)
constexpr int MAX_REQ = 8;            // calls with more requests are never split
constexpr int MIN_SEG_CHUNKS = 8;     // a split request gives each segment at least 8 chunks
constexpr int MAX_UNITS_PER_CALL = 256;  // B * Hv bound of a split call (workspace bound)

// unit modes inside a split call
enum { MODE_TRUE = 0, MODE_IDENT = 1, MODE_ZERO = 2 };

// Which requests are split.  `nc[b]` = chunks of request b (0 when empty).  A split is taken
// only when it shortens the critical path of the two passes and the first pass fits one unit
// per CTA: the k longest requests are split, k chosen to minimise
//     max(longest unsplit, ceil(nc/3) of the split ones) + max(pass-3 segments),
// against the unsplit call's longest request.  Returns the split mask (bit b).
__host__ __device__ inline uint32_t split_mask(const int *nc, int B, int Hv, int G)
{
    if (B < 1 || B > MAX_REQ || B * Hv > MAX_UNITS_PER_CALL) return 0u;
    int order[MAX_REQ];
    for (int b = 0; b < B; ++b) order[b] = b;
    for (int i = 1; i < B; ++i)   // insertion sort, longest first, ties by index
        for (int j = i; j > 0 && (nc[order[j]] > nc[order[j - 1]] ||
                                  (nc[order[j]] == nc[order[j - 1]] && order[j] < order[j - 1])); --j) {
            const int t = order[j];
            order[j] = order[j - 1];
            order[j - 1] = t;
        }
    long long best = nc[order[0]];   // no split
    int best_k = 0;
    for (int k = 1; k <= B; ++k) {
        const int shortest_split = nc[order[k - 1]];
        if (shortest_split < 3 * MIN_SEG_CHUNKS) break;
        if ((long long)(3 * k + (B - k)) * Hv > G) break;
        long long p1 = k < B ? nc[order[k]] : 0, p3 = 0;
        for (int i = 0; i < k; ++i) {
            const int n = nc[order[i]];
            const int s0 = (n + 2) / 3, s1 = (n - s0 + 1) / 2, s2 = n - s0 - s1;
            p1 = p1 > s0 ? p1 : (s0 > s1 ? s0 : s1);
            const long long m3 = s1 > s2 ? s1 : s2;
            p3 = p3 > m3 ? p3 : m3;
        }
        if (p1 + p3 < best) {
            best = p1 + p3;
            best_k = k;
        }
    }
    uint32_t mask = 0u;
    for (int i = 0; i < best_k; ++i) mask |= 1u << order[i];
    return mask;
}

// chunks of the three segments of a split request of `n` chunks
__host__ __device__ inline void segments(int n, int &s0, int &s1, int &s2)
{
    s0 = (n + 2) / 3;
    s1 = (n - s0 + 1) / 2;
    s2 = n - s0 - s1;
}

// Workspace of a split call (fp32, per request b and value head h, allocated for every
// request since the host cannot see which are split):
//   S1[b][h]  Dv x Dk  start state of segment 1 (segment 0's final state)
//   S2[b][h]  Dv x Dk  start state of segment 2
//   A1[b][h]  Dk x Dk  A_1^T (the identity run's final state, rows = the identity's rows)
//   B1[b][h]  Dv x Dk  B_1^T (the zero run's final state)
struct Workspace {
    float *base;
    int B, Hv, Dk, Dv;
    __host__ __device__ int64_t st() const { return (int64_t)Dv * Dk; }
    __host__ __device__ int64_t bh(int b, int h) const { return (int64_t)b * Hv + h; }
    __host__ __device__ int64_t per_bh() const { return 3 * st() + (int64_t)Dk * Dk; }
    __host__ __device__ float *S1(int b, int h) const { return base + bh(b, h) * per_bh(); }
    __host__ __device__ float *S2(int b, int h) const { return S1(b, h) + st(); }
    __host__ __device__ float *B1(int b, int h) const { return S1(b, h) + 2 * st(); }
    __host__ __device__ float *A1(int b, int h) const { return S1(b, h) + 3 * st(); }
};

__host__ __device__ inline uint64_t workspace_bytes(int B, int Hv, int Dk, int Dv)
{
    return (uint64_t)B * Hv * (3ull * Dv * Dk + (uint64_t)Dk * Dk) * 4ull;
}

}  // namespace gdn_seq
