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
// The same threshold on the chunk's summed log-decay, log(0.2), which is how
// the kernels decide it: one sum, in one fixed order, for every party that
// needs the decision of a chunk.
constexpr float kLogHighPrecisionDecay = -1.6094379f;
constexpr int kAS4 = 68; // row stride of A for solve_tril64 (16-byte aligned rows)
constexpr int kTS = 68;  // row stride of T (16-byte aligned rows for float4 access)

constexpr uint32_t IDESC_KK_N64 = make_idesc_f16(128, 64, 0, 0);
constexpr uint32_t IDESC_MK_N64 = make_idesc_f16(128, 64, 1, 0);
constexpr uint32_t IDESC_KM_N64 = make_idesc_f16(128, 64, 0, 1);
constexpr uint32_t IDESC_KM_N128 = make_idesc_f16(128, 128, 0, 1);
constexpr uint32_t IDESC_KM_N192 = make_idesc_f16(128, 192, 0, 1);
constexpr uint32_t IDESC_KK_N64_BF16 = make_idesc_f16(128, 64, 0, 0, 1);
constexpr uint32_t IDESC_MK_N64_BF16 = make_idesc_f16(128, 64, 1, 0, 1);

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

// Largest |v[i]| over N values (N a multiple of 8), as a tree of eight
// independent running maxima rather than one dependent chain.
template <int N>
__device__ __forceinline__ float max_abs(const float *v) {
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = fabsf(v[j]);
#pragma unroll
    for (int i = 8; i < N; i += 8)
#pragma unroll
        for (int j = 0; j < 8; ++j) m[j] = fmaxf(m[j], fabsf(v[i + j]));
    return fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
                 fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
}

// The same with the largest |x| folded into amax (range check of fp16 operands).
__device__ __forceinline__ uint4 pack8_track(const float *x, float &amax) {
    amax = fmaxf(amax, max_abs<8>(x));
    return pack8(x);
}

// x = hi + mid + lo with all three parts bfloat16 (exact for normal fp32 x:
// each residual has at most 16, then 8, significant bits), 8 values.
__device__ __forceinline__ void split8_bf16x3(const float *x, uint4 &hi, uint4 &mid, uint4 &lo) {
    uint32_t h[4], m[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
        const float2 hf = __bfloat1622float2(hh);
        const float r0 = x[2 * j] - hf.x, r1 = x[2 * j + 1] - hf.y;
        const __nv_bfloat162 mm = __floats2bfloat162_rn(r0, r1);
        const float2 mf = __bfloat1622float2(mm);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(r0 - mf.x, r1 - mf.y);
        h[j] = *reinterpret_cast<const uint32_t *>(&hh);
        m[j] = *reinterpret_cast<const uint32_t *>(&mm);
        l[j] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    mid = make_uint4(m[0], m[1], m[2], m[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// ---- power-of-two operand scaling ----
// A value-side fp16 operand (the state, U, U') is stored as x * 2^-e, with e
// chosen per accumulator row from that row's largest magnitude, and the MMA
// result row is multiplied back by 2^e in fp32.  Both multiplications are
// exact, so the scaling changes no bit of the arithmetic except that every
// value now lies in fp16's normal range.

// e such that amax * 2^-e lies in [2^10, 2^11), clamped so that 2^e and
// 2^-e are normal floats.  That leaves fp16 four binades of headroom above
// the largest scaled value (other operands that share the scale, such as U
// beside the state, may exceed it) and six below it before a hi / lo split
// of the largest values loses bits to subnormals.
__device__ __forceinline__ int fp16_scale_exp(float amax) {
    const int e = (int)((__float_as_uint(amax) >> 23) & 0xffu) - 127 - 10;
    return min(max(e, -126), 126);
}

// 2^e for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Largest fp16 magnitude that does not round to infinity is just below this.
constexpr float kFp16Overflow = 65520.f;

// Sum over the warp of one value per lane, by xor butterflies: every lane
// ends with the same, bit-identical total (each step adds a pair of equal
// partial sums in both lanes of the pair).
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// 2^e with e clamped to [-126, 127].
__device__ __forceinline__ float exp2c(int e) { return exp2i(min(max(e, -126), 127)); }

// The band a scaled value-side operand is kept in: its largest magnitude in
// [kScaleLo, kScaleHi).  Above it fp16 would overflow; below it the lo parts
// of a hi / lo split drift towards fp16's subnormals.
constexpr float kScaleHi = 32768.f;
constexpr float kScaleLo = 16.f;

// Bits of a scale vote: some value at or above the band, some value at or
// above its floor, some value nonzero.
__device__ __forceinline__ unsigned scale_bits(float amax) {
    return (amax >= kScaleHi ? 1u : 0u) | (amax >= kScaleLo ? 2u : 0u) | (amax > 0.f ? 4u : 0u);
}
// Whether voted bits call for a new scale: something overflowed, or nothing
// reaches the floor although something is nonzero.
__device__ __forceinline__ bool rescale_needed(unsigned bits) {
    return (bits & 1u) || ((bits & 4u) && !(bits & 2u));
}

// OR of a warp-uniform word over the CTA's 8 warps: lane 0 of each warp posts
// it to words[warp], and after the CTA barrier every thread reads all 8.  The
// barrier is part of the call; a second use of `words` must be separated from
// this one by another CTA barrier.
__device__ __forceinline__ unsigned cta_or8(unsigned x, uint32_t *words, int warp, int lane) {
    if (lane == 0) words[warp] = x;
    __syncthreads();
    const uint4 a = *reinterpret_cast<const uint4 *>(words);
    const uint4 b = *reinterpret_cast<const uint4 *>(words + 4);
    return a.x | a.y | a.z | a.w | b.x | b.y | b.z | b.w;
}

// Maximum of x (>= 0) over the CTA's 256 threads; red holds 8 floats.  Ends
// with every thread holding the result; contains one CTA barrier, and a
// second use of red must be separated from this one by another.
__device__ __forceinline__ float cta_max(float x, float *red, int warp, int lane) {
    const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(x));  // x >= 0: bit order
    if (lane == 0) red[warp] = __uint_as_float(m);
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) r = fmaxf(r, red[w]);
    return r;
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

// store_split32 with the largest |v| folded into amax.
__device__ __forceinline__ void store_split32(uint8_t *hi_tile, uint8_t *lo_tile, int row, int c,
                                              const float *v, bool with_lo, float &amax) {
    amax = fmaxf(amax, max_abs<32>(v));
    store_split32(hi_tile, lo_tile, row, c, v, with_lo);
}

// Writes 32 consecutive values of a row of three 128-byte swizzled bf16 tiles
// as the hi, mid and lo parts of an exact three-way split.
__device__ __forceinline__ void store_split32_bf16x3(uint8_t *hi_tile, uint8_t *mid_tile,
                                                     uint8_t *lo_tile, int row, int c,
                                                     const float *v) {
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
        uint4 hi, mid, lo;
        split8_bf16x3(v + e, hi, mid, lo);
        st_row_chunk(hi_tile, row, (c + e) / 8, hi);
        st_row_chunk(mid_tile, row, (c + e) / 8, mid);
        st_row_chunk(lo_tile, row, (c + e) / 8, lo);
    }
}

// ---- warp-level tf32 tensor-core products (mma.sync m16n8k8) ----

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// x = hi + lo with both parts tf32 (about 21 significant bits together)
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4],
                                                const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// D = L R for 32 x 32 fp32 matrices on one warp's 16 x 8 tile per call site:
// warp w (0..7) computes rows 16 (w >> 2) .. + 15, columns 8 (w & 3) .. + 7.
// L(r, m) = Lp[r * ls + m], R(m, c) = Rp[m * rs + c].  Three tf32 passes
// (hi hi, hi lo, lo hi, in separate accumulators) give nearly fp32 products.
// The result goes to store(r, c, value), two columns per lane and row.
template <class Store>
__device__ __forceinline__ void mm32_tf32(const float *Lp, int ls, const float *Rp, int rs,
                                          int warp, int lane, Store store) {
    const int mt = warp >> 2, nt = warp & 3, gid = lane >> 2, tig = lane & 3;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        const int r0 = 16 * mt + gid, k0 = 8 * ks + tig, c0 = 8 * nt + gid;
        uint32_t ah[4], al[4], bh[2], bl[2];
        split_tf32(Lp[r0 * ls + k0], ah[0], al[0]);
        split_tf32(Lp[(r0 + 8) * ls + k0], ah[1], al[1]);
        split_tf32(Lp[r0 * ls + k0 + 4], ah[2], al[2]);
        split_tf32(Lp[(r0 + 8) * ls + k0 + 4], ah[3], al[3]);
        split_tf32(Rp[k0 * rs + c0], bh[0], bl[0]);
        split_tf32(Rp[(k0 + 4) * rs + c0], bh[1], bl[1]);
        mma_tf32_16x8x8(d0, ah, bh);
        mma_tf32_16x8x8(d1, ah, bl);
        mma_tf32_16x8x8(d2, al, bh);
    }
    const int rr = 16 * mt + gid, cc = 8 * nt + 2 * tig;
    store(rr, cc, d0[0] + (d1[0] + d2[0]));
    store(rr, cc + 1, d0[1] + (d1[1] + d2[1]));
    store(rr + 8, cc, d0[2] + (d1[2] + d2[2]));
    store(rr + 8, cc + 1, d0[3] + (d1[3] + d2[3]));
}

// D = L R for one 16 x 8 tile with a 16-term sum: L(r, m) = Lp[r * ls + m]
// (16 x 16), R(m, c) = Rp[m * rs + c] (16 x 8), three tf32 passes; the warp's
// lanes pass the result to store(r, c, value).
template <class Store>
__device__ __forceinline__ void mm16x8_tf32(const float *Lp, int ls, const float *Rp, int rs,
                                            int lane, Store store) {
    const int gid = lane >> 2, tig = lane & 3;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        const int k0 = 8 * ks + tig;
        uint32_t ah[4], al[4], bh[2], bl[2];
        split_tf32(Lp[gid * ls + k0], ah[0], al[0]);
        split_tf32(Lp[(gid + 8) * ls + k0], ah[1], al[1]);
        split_tf32(Lp[gid * ls + k0 + 4], ah[2], al[2]);
        split_tf32(Lp[(gid + 8) * ls + k0 + 4], ah[3], al[3]);
        split_tf32(Rp[k0 * rs + gid], bh[0], bl[0]);
        split_tf32(Rp[(k0 + 4) * rs + gid], bh[1], bl[1]);
        mma_tf32_16x8x8(d0, ah, bh);
        mma_tf32_16x8x8(d1, ah, bl);
        mma_tf32_16x8x8(d2, al, bh);
    }
    store(gid, 2 * tig, d0[0] + (d1[0] + d2[0]));
    store(gid, 2 * tig + 1, d0[1] + (d1[1] + d2[1]));
    store(gid + 8, 2 * tig, d0[2] + (d1[2] + d2[2]));
    store(gid + 8, 2 * tig + 1, d0[3] + (d1[3] + d2[3]));
}

// T = (I + A)^-1 for the 64 x 64 strictly lower A in As (row stride kAS4),
// into Ts (row stride kTS), fp32, 256 threads.  Three steps:
//   1. the four 16 x 16 diagonal blocks D_i = (I + A_ii)^-1, by forward
//      substitution (lanes 0-15 of warp 4 + i, one per column of block i, so
//      the four blocks run on the four SM sub-partitions, on warps that carry
//      no other duties here); the other threads write zeros above the
//      diagonal blocks;
//   2. T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2 (the 32 x 32 halves);
//   3. the lower-left 32 x 32 block T_bl = -T_bot (A_bl T_top), where T_top and
//      T_bot are the two lower-triangular 32 x 32 diagonal halves.
// The block products of steps 2 and 3 run on warp-level tf32 tensor cores
// (three hi/lo passes, so nearly fp32).  As must hold explicit zeros on and above its diagonal
// and have 16-byte aligned rows.  Xs needs 1024 floats.  Callers synchronise
// before (As complete); the function ends with a barrier.
__device__ __forceinline__ void solve_tril64(const float *As, float *Ts, float *Xs, int tid) {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp >= 4 && lane < 16) {  // 1. diagonal block warp - 4 (one warp per block: 4 SMSPs)
        const int bi = warp - 4, col = lane;
        const float *Ab = As + (16 * bi) * kAS4 + 16 * bi;
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == col) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < 15; ++j)
#pragma unroll
            for (int i = j + 1; i < 16; ++i) x[i] -= Ab[i * kAS4 + j] * x[j];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) Ts[(16 * bi + rr) * kTS + 16 * bi + col] = x[rr];
    } else {  // zeros above the diagonal blocks: 6 blocks of 16 x 16, 8 floats per thread
        const int z = warp >= 4 ? 128 + 16 * (warp - 4) + (lane - 16) : tid;  // 0 .. 191
        const int blk = z >> 5, part = z & 31;
        // upper blocks (bi, bj), bi < bj: (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)
        const int bi = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
        const int bj = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
        const int rr = part >> 1, c8 = 8 * (part & 1);
        float *dst = Ts + (16 * bi + rr) * kTS + 16 * bj + c8;
        *reinterpret_cast<float4 *>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    // 2. (warps 0..3: block b = warp >> 1 with i = 2b + 1, k = 2b; output
    //    columns 8 (warp & 1) .. + 7), warp-level tf32 tensor cores
    if (warp < 4) {  // 2a. X = A_{i,k} D_k
        const int b2 = warp >> 1, bi = 2 * b2 + 1, bk = bi - 1, c8 = 8 * (warp & 1);
        mm16x8_tf32(As + (16 * bi) * kAS4 + 16 * bk, kAS4, Ts + (16 * bk) * kTS + 16 * bk + c8, kTS,
                    lane, [&](int r, int c, float v) { Xs[(b2 << 8) + r * 16 + c8 + c] = v; });
    }
    __syncthreads();
    if (warp < 4) {  // 2b. T_{i,k} = -D_i X
        const int b2 = warp >> 1, bi = 2 * b2 + 1, bk = bi - 1, c8 = 8 * (warp & 1);
        mm16x8_tf32(Ts + (16 * bi) * kTS + 16 * bi, kTS, Xs + (b2 << 8) + c8, 16, lane,
                    [&](int r, int c, float v) { Ts[(16 * bi + r) * kTS + 16 * bk + c8 + c] = -v; });
    }
    __syncthreads();
    // 3a. X = A_bl T_top;  3b. T_bl = -T_bot X  (warp-level tf32 tensor cores)
    mm32_tf32(As + 32 * kAS4, kAS4, Ts, kTS, warp, lane,
              [&](int r, int c, float v) { Xs[r * 32 + c] = v; });
    __syncthreads();
    mm32_tf32(Ts + 32 * kTS + 32, kTS, Xs, 32, warp, lane,
              [&](int r, int c, float v) { Ts[(32 + r) * kTS + c] = -v; });
    __syncthreads();
}

}  // namespace tc
}  // namespace gdn
