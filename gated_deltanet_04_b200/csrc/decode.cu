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
// Two kernels:
//  * Dk = Dv = 128 (the workload shape): a persistent kernel, one CTA per SM,
//    that streams each 64 KB head state through shared memory with bulk TMA
//    copies (3 states in flight per SM: loads of the next two overlap the
//    update of the current one, and the updated state leaves by a bulk store
//    while the next is computed).  Threads only read and write shared memory.
//    Each CTA takes a contiguous range of (n, h) units, so every SM streams
//    one contiguous stretch of the states (measured ~1% faster on B200 than
//    dealing units round-robin).  The units % grid left over are split into
//    single rows across all CTAs, so no SM runs a whole extra unit at the end.
//  * other head sizes: the direct kernel below.
//
// Direct kernel: one CTA of 8 warps per (n, h).  A row of Dk fp32 values is spread
// over LPR = Dk/4 lanes as float4 (Dk = 128: a full warp per row, 512
// contiguous bytes, fully coalesced).  Each warp keeps ROWS_IN_FLIGHT rows
// loaded before reducing them, so every lane has several independent 16-byte
// loads outstanding.  Streaming cache hints keep the once-touched state from
// displacing other data in L2.
#include "gdn_internal.cuh"
#include "sm100.cuh"

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


// ---------------------------------------------------------------- staged --

constexpr int kStStages = 3;
constexpr int kStThreads = 256;                 // 8 warps x 16 state rows
constexpr uint32_t kStUnitFloats = 128 * 128;   // one (n, h) state
constexpr uint32_t kStUnitBytes = kStUnitFloats * 4;
constexpr long long kStWaitLimit = 1ll << 31;   // SM clocks (about a second)

struct StagedSmem {
    float state[kStStages][kStUnitFloats];
    float o[2][128];
    uint64_t full[kStStages];
};
constexpr size_t kStSmemBytes = sizeof(StagedSmem) + 128;

struct UnitInputs {
    float4 k, q;
    float g, b, v;  // v: lanes 0..15 hold rows 16*warp + lane
};

__device__ __forceinline__ UnitInputs load_unit_inputs(const DecodeArgs &a, int u, int warp,
                                                       int lane) {
    UnitInputs in;
    const int h = u % a.Hv, n = u / a.Hv;
    const int j = h / (a.Hv / a.Hqk);
    const int64_t qk = ((int64_t)n * a.Hqk + j) * 128 + 4 * lane;
    in.k = load_vec4(a.k, qk, a.dtype);
    in.q = load_vec4(a.q, qk, a.dtype);
    in.g = a.g[u];
    in.b = a.beta[u];
    in.v = lane < 16 ? load_io(a.v, (int64_t)u * 128 + 16 * warp + lane, a.dtype) : 0.f;
    return in;
}

__global__ void __launch_bounds__(kStThreads, 1)
    gdn_decode_staged_kernel(DecodeArgs a, int units) {
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    StagedSmem &sm = *reinterpret_cast<StagedSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per = units / (int)gridDim.x, extra = units % (int)gridDim.x;
    const int b = blockIdx.x;
    const int first = b * per, stride = 1;
    const int count = per;  // units of this CTA: a contiguous range (grid <= units, so >= 1)
    if (count <= 0) return;

    if (tid == 0) {
        for (int s = 0; s < kStStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    int issued = 0;  // units whose state load has been issued (thread 0's view)
    if (tid == 0) {
        for (; issued < count && issued < kStStages; ++issued) {
            const int u = first + issued * stride;
            mbar_arrive_expect_tx(&sm.full[issued], kStUnitBytes);
            bulk_load(sm.state[issued], a.state + (int64_t)u * kStUnitFloats, kStUnitBytes,
                      &sm.full[issued]);
        }
    }
    // The extra = units % grid leftover units (the last ones), as single rows
    // spread over all CTAs, one row per warp at a time, while this CTA's first
    // stage loads are in flight.  Same arithmetic as the staged update below;
    // no other CTA touches these units.
    for (int r = b + (int)gridDim.x * warp; r < extra * 128; r += (int)gridDim.x * (kStThreads / 32)) {
        const int u = per * (int)gridDim.x + r / 128, i = r % 128;
        const int h = u % a.Hv, n = u / a.Hv;
        const int j = h / (a.Hv / a.Hqk);
        const int64_t qk = ((int64_t)n * a.Hqk + j) * 128 + 4 * lane;
        const float4 k4 = load_vec4(a.k, qk, a.dtype), q4 = load_vec4(a.q, qk, a.dtype);
        float *srow = a.state + (int64_t)u * kStUnitFloats + i * 128 + 4 * lane;
        const float4 row = *reinterpret_cast<const float4 *>(srow);
        const float dec = expf(a.g[u]), bb = a.beta[u];
        const float vi = load_io(a.v, (int64_t)u * 128 + i, a.dtype);
        float kq = k4.x * q4.x + k4.y * q4.y + k4.z * q4.z + k4.w * q4.w;
        float sk = row.x * k4.x + row.y * k4.y + row.z * k4.z + row.w * k4.w;
        float sq = row.x * q4.x + row.y * q4.y + row.z * q4.z + row.w * q4.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            kq += __shfl_xor_sync(0xffffffffu, kq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
        }
        const float uu = bb * (vi - dec * sk);
        float4 w;
        w.x = fmaf(uu, k4.x, dec * row.x);
        w.y = fmaf(uu, k4.y, dec * row.y);
        w.z = fmaf(uu, k4.z, dec * row.z);
        w.w = fmaf(uu, k4.w, dec * row.w);
        *reinterpret_cast<float4 *>(srow) = w;
        if (lane == 0) store_io(a.o, (int64_t)u * 128 + i, fmaf(uu, kq, dec * sq), a.dtype);
    }
    UnitInputs nxt = load_unit_inputs(a, first, warp, lane);
    bool timed_out = false;
    int li = 0;
#pragma unroll 1
    for (; li < count; ++li) {
        const int u = first + li * stride;
        const int s = li % kStStages;
        const UnitInputs cur = nxt;
        if (li + 1 < count) nxt = load_unit_inputs(a, u + stride, warp, lane);
        if (!mbar_wait_bounded(&sm.full[s], (li / kStStages) & 1, kStWaitLimit)) timed_out = true;

        const float dec = expf(cur.g);
        float kq = cur.k.x * cur.q.x + cur.k.y * cur.q.y + cur.k.z * cur.q.z + cur.k.w * cur.q.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        float *st = sm.state[s];
#pragma unroll
        for (int r0 = 0; r0 < 16; r0 += 4) {
            float4 row[4];
            float sk[4], sq[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                row[r] = *reinterpret_cast<const float4 *>(st + (16 * warp + r0 + r) * 128 + 4 * lane);
                sk[r] = row[r].x * cur.k.x + row[r].y * cur.k.y + row[r].z * cur.k.z + row[r].w * cur.k.w;
                sq[r] = row[r].x * cur.q.x + row[r].y * cur.q.y + row[r].z * cur.q.z + row[r].w * cur.q.w;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    sk[r] += __shfl_xor_sync(0xffffffffu, sk[r], off);
                    sq[r] += __shfl_xor_sync(0xffffffffu, sq[r], off);
                }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = 16 * warp + r0 + r;
                const float vi = __shfl_sync(0xffffffffu, cur.v, r0 + r);
                const float uu = cur.b * (vi - dec * sk[r]);
                float4 w;
                w.x = fmaf(uu, cur.k.x, dec * row[r].x);
                w.y = fmaf(uu, cur.k.y, dec * row[r].y);
                w.z = fmaf(uu, cur.k.z, dec * row[r].z);
                w.w = fmaf(uu, cur.k.w, dec * row[r].w);
                *reinterpret_cast<float4 *>(st + i * 128 + 4 * lane) = w;
                if (lane == 0) sm.o[li & 1][i] = fmaf(uu, kq, dec * sq[r]);
            }
        }
        fence_proxy_async_smem();  // updated state -> visible to the bulk store
        if (__syncthreads_or(timed_out ? 1 : 0)) {
            if (tid == 0) raise_error(a.err, GDN_ERR_TIMEOUT);
            break;
        }
        if (tid < 128) store_io(a.o, (int64_t)u * 128 + tid, sm.o[li & 1][tid], a.dtype);
        if (tid == 0) {
            bulk_store(a.state + (int64_t)u * kStUnitFloats, st, kStUnitBytes);
            bulk_commit();
            if (issued < count) {  // refill this stage with the unit kStStages ahead
                bulk_wait_read_all();
                const int un = first + issued * stride;
                mbar_arrive_expect_tx(&sm.full[s], kStUnitBytes);
                bulk_load(st, a.state + (int64_t)un * kStUnitFloats, kStUnitBytes, &sm.full[s]);
                ++issued;
            }
        }
    }
    if (tid == 0) {
        // loads issued but not consumed (only after a timeout): let them land
        for (int l = li; l < issued; ++l)
            mbar_wait_bounded(&sm.full[l % kStStages], (l / kStStages) & 1, kStWaitLimit);
        bulk_wait_all();
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    const int units = a.N * a.Hv;
    if (a.Dk == 128 && a.Dv == 128) {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(gdn_decode_staged_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStSmemBytes);
        if (e != cudaSuccess) return e;
        const int grid = units < sms ? units : sms;
        gdn_decode_staged_kernel<<<grid, kStThreads, kStSmemBytes, s>>>(a, units);
        return cudaGetLastError();
    }
    const dim3 grid((unsigned)units);
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
