// Device helpers shared by libgdn's tensor-core prefill kernels: fp16 packing
// and hi/lo splitting, 128-byte-swizzled tile stores, the blocked triangular
// inverse, and the constants of the chunk-64 / head-128 tiling.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int kC = 64;      // chunk length
constexpr int kD = 128;     // Dk = Dv
constexpr long long kWaitLimit = 1ll << 31;  // SM clocks (about a second)
constexpr float kHighPrecisionDecay = 0.2f;  // Gamma_C at or above -> extra passes
constexpr int kAS = 65;  // row stride of A (scalar, conflict-free column access)
constexpr int kTS = 68;  // row stride of T (16-byte aligned rows for float4 access)

constexpr uint32_t IDESC_KK_N64 = make_idesc_f16(128, 64, 0, 0);
constexpr uint32_t IDESC_MK_N64 = make_idesc_f16(128, 64, 1, 0);
constexpr uint32_t IDESC_KM_N64 = make_idesc_f16(128, 64, 0, 1);
constexpr uint32_t IDESC_KM_N128 = make_idesc_f16(128, 128, 0, 1);
constexpr uint32_t IDESC_KM_N192 = make_idesc_f16(128, 192, 0, 1);
constexpr uint32_t IDESC_KK_N64_BF16 = make_idesc_f16(128, 64, 0, 0, 1);

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// hi = fp16(x), lo = fp16(x - hi) for 8 values, packed as two uint4
__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 hh = __floats2half2_rn(x[2 * j], x[2 * j + 1]);
        const float2 hf = __half22float2(hh);
        h[j] = *reinterpret_cast<const uint32_t *>(&hh);
        l[j] = pack_half2(x[2 * j] - hf.x, x[2 * j + 1] - hf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(pack_half2(x[0], x[1]), pack_half2(x[2], x[3]), pack_half2(x[4], x[5]),
                      pack_half2(x[6], x[7]));
}

__device__ __forceinline__ void st_row_chunk(uint8_t *tile, uint32_t row, uint32_t chunk,
                                             uint4 val) {
    *reinterpret_cast<uint4 *>(tile + sw128(row, chunk * 16)) = val;
}

// Writes 32 consecutive values (columns c .. c+31 of row `row`) of a 128-byte
// swizzled fp16 tile as hi (and, if `with_lo`, lo) parts.
__device__ __forceinline__ void store_split32(uint8_t *hi_tile, uint8_t *lo_tile, int row, int c,
                                              const float *v, bool with_lo) {
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
        uint4 hi, lo;
        split8(v + e, hi, lo);
        st_row_chunk(hi_tile, row, (c + e) / 8, hi);
        if (with_lo) st_row_chunk(lo_tile, row, (c + e) / 8, lo);
    }
}

// One block-distance level D of the triangular inverse (see the solve phase):
//   X = sum_{m = k}^{i-1} A_im T_mk,   T_ik = -D_i X,   i = k + D,
// each thread producing four adjacent columns of one row of one block.
template <int D>
__device__ __forceinline__ void solve_level(const float *As, float *Ts, float *Xs, int tid) {
    constexpr int kBlocks = 4 - D;
    const bool act = tid < kBlocks * 64;
    const int blk = tid >> 6, r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
    const int bi = blk + D, bk = blk;
    if (act) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *arow = As + (16 * bi + r) * kAS + 16 * bk;
        const float *tcol = Ts + (16 * bk) * kTS + 16 * bk + c4;
#pragma unroll
        for (int m = 0; m < 16 * D; ++m) {
            const float a = arow[m];
            const float4 t = *reinterpret_cast<const float4 *>(tcol + m * kTS);
            acc.x = fmaf(a, t.x, acc.x); acc.y = fmaf(a, t.y, acc.y);
            acc.z = fmaf(a, t.z, acc.z); acc.w = fmaf(a, t.w, acc.w);
        }
        *reinterpret_cast<float4 *>(Xs + (blk << 8) + r * 16 + c4) = acc;
    }
    __syncthreads();
    if (act) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *drow = Ts + (16 * bi + r) * kTS + 16 * bi;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float d = drow[m];
            const float4 x = *reinterpret_cast<const float4 *>(Xs + (blk << 8) + m * 16 + c4);
            acc.x = fmaf(d, x.x, acc.x); acc.y = fmaf(d, x.y, acc.y);
            acc.z = fmaf(d, x.z, acc.z); acc.w = fmaf(d, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(Ts + (16 * bi + r) * kTS + 16 * bk + c4) =
            make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
}

// T = (I + A)^-1 for the 64 x 64 strictly lower A in As (row stride kAS), into
// Ts (row stride kTS), fp32, 256 threads.  Three steps:
//   1. the four 16 x 16 diagonal blocks D_i = (I + A_ii)^-1, by forward
//      substitution (one thread per (block, column));
//   2. T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2 (upper 32 x 32 halves);
//   3. the lower-left 32 x 32 block T_bl = -T_bot (A_bl T_top), where T_top
//      and T_bot are the two lower-triangular 32 x 32 diagonal halves.
// Each step keeps most threads busy; block-triangular zeros are skipped.  The
// entries above the diagonal blocks of Ts are left unwritten and never read.
// Xs needs 1024 floats.  Callers synchronise before (As complete) and after.
__device__ __forceinline__ void solve_tril64(const float *As, float *Ts, float *Xs, int tid) {
    if (tid < kC) {  // 1. diagonal blocks
        const int bi = tid >> 4, col = tid & 15;
        const float *Ab = As + (16 * bi) * kAS + 16 * bi;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            float a0 = (rr == col) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
            for (int ii = 0; ii + 1 < rr; ii += 2) {
                a0 -= Ab[rr * kAS + ii] * x[ii];
                a1 -= Ab[rr * kAS + ii + 1] * x[ii + 1];
            }
            if (rr & 1) a0 -= Ab[rr * kAS + rr - 1] * x[rr - 1];
            x[rr] = a0 + a1;
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) Ts[(16 * bi + rr) * kTS + 16 * bi + col] = x[rr];
    }
    __syncthreads();
    {   // 2a. X = A_{i,i-1} D_{i-1} for i = 1, 3
        const int blk = tid >> 6;            // 0, 1 active (128 threads)
        const int r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
        if (blk < 2) {
            const int bi = 2 * blk + 1, bk = bi - 1;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float *arow = As + (16 * bi + r) * kAS + 16 * bk;
            const float *tcol = Ts + (16 * bk) * kTS + 16 * bk + c4;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float a = arow[m];
                const float4 t = *reinterpret_cast<const float4 *>(tcol + m * kTS);
                acc.x = fmaf(a, t.x, acc.x); acc.y = fmaf(a, t.y, acc.y);
                acc.z = fmaf(a, t.z, acc.z); acc.w = fmaf(a, t.w, acc.w);
            }
            *reinterpret_cast<float4 *>(Xs + (blk << 8) + r * 16 + c4) = acc;
        }
    }
    __syncthreads();
    {   // 2b. T_{i,i-1} = -D_i X
        const int blk = tid >> 6;
        const int r = (tid >> 2) & 15, c4 = 4 * (tid & 3);
        if (blk < 2) {
            const int bi = 2 * blk + 1, bk = bi - 1;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            const float *drow = Ts + (16 * bi + r) * kTS + 16 * bi;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float d = drow[m];
                const float4 x = *reinterpret_cast<const float4 *>(Xs + (blk << 8) + m * 16 + c4);
                acc.x = fmaf(d, x.x, acc.x); acc.y = fmaf(d, x.y, acc.y);
                acc.z = fmaf(d, x.z, acc.z); acc.w = fmaf(d, x.w, acc.w);
            }
            *reinterpret_cast<float4 *>(Ts + (16 * bi + r) * kTS + 16 * bk + c4) =
                make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
        }
    }
    __syncthreads();
    const int r = tid >> 3, c4 = 4 * (tid & 7);  // 32 rows x 8 column groups
    {   // 3a. X = A_bl T_top   (T_top[m][c] = 0 for m < c)
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *arow = As + (32 + r) * kAS;
#pragma unroll 4
        for (int m = c4; m < 32; ++m) {
            const float a = arow[m];
            const float4 t = *reinterpret_cast<const float4 *>(Ts + m * kTS + c4);
            acc.x = fmaf(a, t.x, acc.x); acc.y = fmaf(a, t.y, acc.y);
            acc.z = fmaf(a, t.z, acc.z); acc.w = fmaf(a, t.w, acc.w);
        }
        *reinterpret_cast<float4 *>(Xs + r * 32 + c4) = acc;
    }
    __syncthreads();
    {   // 3b. T_bl = -T_bot X   (T_bot[r][m] = 0 for m > r)
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float *brow = Ts + (32 + r) * kTS + 32;
#pragma unroll 4
        for (int m = 0; m <= r; ++m) {
            const float b = brow[m];
            const float4 x = *reinterpret_cast<const float4 *>(Xs + m * 32 + c4);
            acc.x = fmaf(b, x.x, acc.x); acc.y = fmaf(b, x.y, acc.y);
            acc.z = fmaf(b, x.z, acc.z); acc.w = fmaf(b, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(Ts + (32 + r) * kTS + c4) =
            make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    __syncthreads();
}

}  // namespace tc
}  // namespace gdn
