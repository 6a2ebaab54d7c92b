// One-token decode update of the gated delta rule, in place on the fp32 state.
//
// Section 三 of "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与 262K
// 长上下文": at inference every step does one fixed-size matrix update.  Per
// (sequence n, v-head h) with a = exp(g), b = beta and row i of the state:
//     r_i   = (a S_i) . k                 (recall from the decayed state)
//     u_i   = b (v_i - r_i)
//     S_i'  = a S_i + u_i k^T             (delta write)
//     o_i   = S_i' . q = a (S_i . q) + u_i (k . q)
// The state is streamed exactly once: every row is loaded, reduced against k
// and q, rewritten and stored by the same lanes, so the kernel is bound by
// HBM bandwidth on 2 * Dv * Dk * 4 bytes per (n, h).
//
// Mapping: one CTA of 8 warps per (n, h).  A row of Dk fp32 values is spread
// over LPR = Dk/4 lanes as float4 (Dk = 128: a full warp per row, 512
// contiguous bytes, fully coalesced).  Each warp keeps ROWS_IN_FLIGHT rows
// loaded before reducing them, so every lane has several independent 16-byte
// loads outstanding.  Streaming cache hints keep the once-touched state from
// displacing other data in L2.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kDecodeWarps = 8;
constexpr int kRowsInFlight = 8;

template <int DK>
struct DecodeShape {
    static constexpr int LPR = DK / 4;             // lanes per row
    static constexpr int RP = 32 / LPR;            // rows per warp pass
    static constexpr int STRIDE = kDecodeWarps * RP;
};

__device__ __forceinline__ float4 load_vec4(const void *p, int64_t idx, gdn_dtype dt) {
    if (dt == GDN_DTYPE_BF16) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + idx);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
        const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    return *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + idx);
}

template <int LPR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int DK>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    gdn_decode_kernel(DecodeArgs a) {
    using S = DecodeShape<DK>;
    const int unit = blockIdx.x;  // n * Hv + h
    const int h = unit % a.Hv;
    const int n = unit / a.Hv;
    const int j = h / (a.Hv / a.Hqk);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane / S::LPR;
    const int l = lane % S::LPR;

    const int64_t qk_off = ((int64_t)n * a.Hqk + j) * DK + 4 * l;
    const float4 kk = load_vec4(a.k, qk_off, a.dtype);
    const float4 qq = load_vec4(a.q, qk_off, a.dtype);
    const float kq = group_sum<S::LPR>(kk.x * qq.x + kk.y * qq.y + kk.z * qq.z + kk.w * qq.w);
    const float gate = a.g[(int64_t)n * a.Hv + h];
    const float dec = expf(gate);
    const float b = a.beta[(int64_t)n * a.Hv + h];

    float *st = a.state + (int64_t)unit * a.Dv * DK;
    const int64_t vo_base = (int64_t)unit * a.Dv;

    // w0 is warp-uniform, so every lane runs every shuffle below; rows past Dv
    // (possible for single row groups when Dv is not a multiple of RP) only
    // skip their loads and stores.
    for (int w0 = warp * S::RP; w0 < a.Dv; w0 += S::STRIDE * kRowsInFlight) {
        const int i0 = w0 + sub;
        float4 row[kRowsInFlight];
        float vi[kRowsInFlight];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const int i = i0 + r * S::STRIDE;
            if (i < a.Dv) {
                row[r] = __ldcs(reinterpret_cast<const float4 *>(st + (int64_t)i * DK) + l);
                vi[r] = load_io(a.v, vo_base + i, a.dtype);
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const int i = i0 + r * S::STRIDE;
            const float4 s = (i < a.Dv) ? row[r] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float sk = group_sum<S::LPR>(s.x * kk.x + s.y * kk.y + s.z * kk.z + s.w * kk.w);
            const float sq = group_sum<S::LPR>(s.x * qq.x + s.y * qq.y + s.z * qq.z + s.w * qq.w);
            if (i < a.Dv) {
                const float u = b * (vi[r] - dec * sk);
                float4 w;
                w.x = fmaf(u, kk.x, dec * s.x);
                w.y = fmaf(u, kk.y, dec * s.y);
                w.z = fmaf(u, kk.z, dec * s.z);
                w.w = fmaf(u, kk.w, dec * s.w);
                __stcs(reinterpret_cast<float4 *>(st + (int64_t)i * DK) + l, w);
                if (l == 0) store_io(a.o, vo_base + i, fmaf(u, kq, dec * sq), a.dtype);
            }
        }
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    const dim3 grid((unsigned)((int64_t)a.N * a.Hv));
    const dim3 block(kDecodeWarps * 32);
    switch (a.Dk) {
        case 16: gdn_decode_kernel<16><<<grid, block, 0, s>>>(a); break;
        case 32: gdn_decode_kernel<32><<<grid, block, 0, s>>>(a); break;
        case 64: gdn_decode_kernel<64><<<grid, block, 0, s>>>(a); break;
        case 128: gdn_decode_kernel<128><<<grid, block, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace gdn
