// tile16.cuh -- shared-memory tile helpers of the two chunked prefill kernels
// (prefill_chunk.cu, prefill_kd.cu): the 128-byte swizzle of the UMMA operand tiles, 16-bit
// operand packing, and the 16 x 16 block products of the blocked triangular solve.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdn_tile {

// 16-byte chunk `c` of row `r` in a 128B-swizzled tile whose base is 1024-aligned
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t c)
{
    return row * 128u + ((c ^ (row & 7u)) << 4);
}

// 16-bit operand element: bf16, or fp16 (F16) for fp16 activations; every tile the tensor
// cores read has the activations' type, since an MMA takes A and B of one type
template <bool F16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    if constexpr (F16) {
        const __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<const uint32_t *>(&v);
    } else {
        return gdn::pack_bf16x2(lo, hi);
    }
}

template <bool F16>
__device__ __forceinline__ uint16_t elem16(float x)
{
    if constexpr (F16) {
        const __half v = __float2half_rn(x);
        return *reinterpret_cast<const uint16_t *>(&v);
    } else {
        const __nv_bfloat16 v = __float2bfloat16_rn(x);
        return *reinterpret_cast<const uint16_t *>(&v);
    }
}

// eight floats as one 16-byte chunk of 16-bit operand elements
template <bool F16 = false>
__device__ __forceinline__ uint4 pack8(const float *x)
{
    uint4 r;
    r.x = pack2<F16>(x[0], x[1]);
    r.y = pack2<F16>(x[2], x[3]);
    r.z = pack2<F16>(x[4], x[5]);
    r.w = pack2<F16>(x[6], x[7]);
    return r;
}

// ---- blocked solve of T = (I + A)^-1 (A strictly lower, 4 x 4 blocks of 16), on padded
// fp32 blocks of 16 rows x SOLVE_LD floats.  Slots of the 16-block solve area: 0-3 A_II,
// 4 A_10, 5 A_32, 6-9 A_20 A_21 A_30 A_31 (later the products X), 10-13 D_I = (I + A_II)^-1,
// 14 T_10, 15 T_32.
constexpr uint32_t SOLVE_LD = 20;               // padded row stride (floats)
constexpr uint32_t SOLVE_BLK = 16 * SOLVE_LD;   // floats per block

__host__ __device__ constexpr int a_slot(int I, int J)
{
    return I == 1 ? 4 : (I == 2 ? 6 + J : (J == 2 ? 5 : 8 + J));
}

// acc[nh][.] += X(16x16) * Y(16x16), tf32 inputs (the fp32 bits as they are), fragments of
// mma.m16n8k8
__device__ __forceinline__ void blk_mma(float (&acc)[2][4], const float *X, const float *Y)
{
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kh = 0; kh < 2; ++kh) {
        uint32_t a[4];
        a[0] = __float_as_uint(X[g * SOLVE_LD + 8 * kh + t]);
        a[1] = __float_as_uint(X[(g + 8) * SOLVE_LD + 8 * kh + t]);
        a[2] = __float_as_uint(X[g * SOLVE_LD + 8 * kh + t + 4]);
        a[3] = __float_as_uint(X[(g + 8) * SOLVE_LD + 8 * kh + t + 4]);
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
            uint32_t b[2];
            b[0] = __float_as_uint(Y[(8 * kh + t) * SOLVE_LD + 8 * nh + g]);
            b[1] = __float_as_uint(Y[(8 * kh + t + 4) * SOLVE_LD + 8 * nh + g]);
            sm100::mma_tf32_16x8x8(acc[nh], a, b);
        }
    }
}

// a block product's fragments (times sgn) into a padded fp32 block
__device__ __forceinline__ void blk_store(float *Z, const float (&acc)[2][4], float sgn)
{
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
        *reinterpret_cast<float2 *>(Z + g * SOLVE_LD + 8 * nh + 2 * t) =
            make_float2(sgn * acc[nh][0], sgn * acc[nh][1]);
        *reinterpret_cast<float2 *>(Z + (g + 8) * SOLVE_LD + 8 * nh + 2 * t) =
            make_float2(sgn * acc[nh][2], sgn * acc[nh][3]);
    }
}

}  // namespace gdn_tile
