// Front end of the DeltaNet mixer before the delta rule: the "kernel 4"
// convolution (page "Layouts híbridos: três DeltaNet, uma attention",
// section 01) on the q, k and v channels, then q and k normalised per head.
//
// Per channel c, causally along the tokens of each sequence:
//     y[t, c] = w[c, 0] x[t-3, c] + w[c, 1] x[t-2, c] + w[c, 2] x[t-1, c] + w[c, 3] x[t, c]
// with the inputs before a sequence's first token taken from a carried conv
// state (its three predecessors, oldest first) or zero; then q, k rows of each
// (token, head) divided by their Euclidean norm.  No activation: the page
// names the convolution and nothing after it.
//
// The operation is bandwidth-bound (read x once, write q/k/v once).  A warp
// owns the 128 channels of one head, 4 per lane, and slides over 128
// consecutive tokens with its filters and the last three inputs in registers,
// its input rows streaming through a per-warp cp.async double buffer.  A
// second small kernel writes the new conv state.
#include "gdn_internal.cuh"
#include "sm100.cuh"
#include "trace.cuh"

namespace gdn {
namespace {

constexpr int kFeD = 128;        // head dimension served
constexpr int kFeWarps = 8;      // warps per CTA
constexpr int kFeRun = 128;      // consecutive tokens per warp
constexpr int kFeBlk = 16;       // rows per cp.async block (two blocks buffered per warp)

struct FeTensor {
    const void *x;               // [T][H][128] io dtype
    const float *w;              // [H*128][4]
    void *y;                     // [T][H][128] io dtype
    int32_t H;
    int32_t chan0;               // first channel of this tensor in the conv state
    int32_t norm;                // normalise each (token, head) row
};

struct FeArgs {
    FeTensor t[3];               // q, k, v
    const int32_t *cu;           // [N+1] or null (one sequence)
    const float *state_in;       // [N][3][C] or null (zeros)
    float *state_out;            // [N][3][C] or null
    int32_t *err;
    int64_t T;
    int32_t N, C;                // C = 2*Hqk*128 + Hv*128
    gdn_dtype dtype;
};

__device__ __forceinline__ float4 fe_load4(const void *p, int64_t idx, gdn_dtype dt) {
    if (dt == GDN_DTYPE_BF16) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(p) + idx);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    return *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + idx);
}

__device__ __forceinline__ void fe_store4(void *p, int64_t idx, float4 v, gdn_dtype dt) {
    if (dt == GDN_DTYPE_BF16) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 raw;
        raw.x = *reinterpret_cast<const uint32_t *>(&a);
        raw.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p) + idx) = raw;
    } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(p) + idx) = v;
    }
}

// The sequence holding token t: the largest n with cu[n] <= t (cu sorted).
__device__ __forceinline__ int fe_sequence(const int32_t *cu, int N, int64_t t) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// grid: (Hqk + Hqk + Hv, ceil(T / 1024)): x walks the q heads, then the k heads,
// then the v heads, so CTAs launched together cover whole token rows.  Each of
// the CTA's 8 warps slides over kFeRun consecutive tokens of one head, keeping
// its lanes' 16 filter taps and the last three inputs in registers, so every
// input row is read from memory once.  The rows come through the warp's own
// double buffer in shared memory, kFeBlk rows at a time by cp.async, so a
// warp has the next kFeBlk rows in flight while it computes the current ones.
__device__ __forceinline__ void fe_cp_async16(void *smem, const void *gmem) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_u32(smem)),
                 "l"(reinterpret_cast<uint64_t>(gmem))
                 : "memory");
}

__global__ void __launch_bounds__(kFeWarps * 32)
    gdn_short_conv_kernel(FeArgs a) {
    extern __shared__ __align__(16) uint8_t fe_smem[];
    const int yh = blockIdx.x, Hq = a.t[0].H;
    const unsigned tb = blockIdx.y;
    const int z = yh < Hq ? 0 : yh < 2 * Hq ? 1 : 2;
    const FeTensor ft = z == 0 ? a.t[0] : z == 1 ? a.t[1] : a.t[2];
    const int h = yh - (z == 0 ? 0 : z == 1 ? Hq : 2 * Hq);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = ((int64_t)tb * kFeWarps + warp) * kFeRun;
    if (t0 >= a.T) return;
    const int64_t t1 = t0 + kFeRun < a.T ? t0 + kFeRun : a.T;
    const int c = h * kFeD + 4 * lane;  // this lane's first channel within the tensor
    const int64_t row = (int64_t)ft.H * kFeD;  // elements per token
    const int esz = a.dtype == GDN_DTYPE_BF16 ? 2 : 4;
    const int rb = kFeD * esz;                  // bytes of this head's slice of a row
    uint8_t *wbuf = fe_smem + (size_t)warp * 2 * kFeBlk * rb;  // [2][kFeBlk][rb]

    // rows t .. t + kFeBlk - 1 (those < t1) of this head into buffer k
    const int lg_parts = esz == 2 ? 4 : 5;      // log2 of the 16-byte pieces per row slice
    auto issue = [&](int64_t tstart, int k) {
        for (int idx = lane; idx < (kFeBlk << lg_parts); idx += 32) {
            const int r = idx >> lg_parts, pc = idx & ((1 << lg_parts) - 1);
            if (tstart + r < t1)
                fe_cp_async16(wbuf + ((size_t)k * kFeBlk + r) * rb + pc * 16,
                              static_cast<const uint8_t *>(ft.x) +
                                  ((tstart + r) * row + (int64_t)h * kFeD) * esz + pc * 16);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    issue(t0, 0);

    float4 w[4];  // w[i]: the 4 taps of channel c + i
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const float4 *>(ft.w + (int64_t)(c + i) * 4);

    // the sequence of t0, and the inputs before t0 (oldest first): from x,
    // from the sequence's carried conv state, or zero
    int n = a.cu ? fe_sequence(a.cu, a.N, t0) : 0;
    int64_t start = a.cu ? (int64_t)a.cu[n] : 0;
    int64_t next = a.cu ? (int64_t)a.cu[n + 1] : a.T;
    auto before = [&](int64_t tp) -> float4 {  // input at token tp < t of sequence n
        if (tp >= start && tp >= 0) return fe_load4(ft.x, tp * row + c, a.dtype);
        const int64_t back = start - tp;
        if (a.state_in && back >= 1 && back <= 3)
            return *reinterpret_cast<const float4 *>(a.state_in + ((int64_t)n * 3 + 3 - back) * a.C +
                                                     ft.chan0 + c);
        return make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 h3 = before(t0 - 3), h2 = before(t0 - 2), h1 = before(t0 - 1);  // x[t-3], x[t-2], x[t-1]
    int k = 0;
    for (int64_t tb0 = t0; tb0 < t1; tb0 += kFeBlk, k ^= 1) {
        if (tb0 + kFeBlk < t1) {  // the next block streams in while this one is computed
            issue(tb0 + kFeBlk, k ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncwarp();
        const int nr = t1 - tb0 < kFeBlk ? (int)(t1 - tb0) : kFeBlk;
        for (int r = 0; r < nr; ++r) {
            const int64_t t = tb0 + r;
            if (t >= next) {  // a new sequence starts at t (skip empty ones)
                while (n + 1 < a.N && (int64_t)a.cu[n + 1] <= t) ++n;
                start = a.cu[n];
                next = a.cu[n + 1];
                h3 = before(t - 3);
                h2 = before(t - 2);
                h1 = before(t - 1);
            }
            const float4 x0 = fe_load4(wbuf + ((size_t)k * kFeBlk + r) * rb, 4 * lane, a.dtype);
            float y[4];
            const float xs[4][4] = {{h3.x, h3.y, h3.z, h3.w}, {h2.x, h2.y, h2.z, h2.w},
                                    {h1.x, h1.y, h1.z, h1.w}, {x0.x, x0.y, x0.z, x0.w}};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                y[i] = w[i].x * xs[0][i];
                y[i] = fmaf(w[i].y, xs[1][i], y[i]);
                y[i] = fmaf(w[i].z, xs[2][i], y[i]);
                y[i] = fmaf(w[i].w, xs[3][i], y[i]);
            }
            if (ft.norm) {  // divide the (token, head) row by its norm; a zero row stays zero
                float ss = y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                if (ss > 0.f) {
                    const float inv = 1.f / sqrtf(ss);
#pragma unroll
                    for (int i = 0; i < 4; ++i) y[i] *= inv;
                }
            }
            fe_store4(ft.y, t * row + c, make_float4(y[0], y[1], y[2], y[3]), a.dtype);
            h3 = h2;
            h2 = h1;
            h1 = x0;
        }
        __syncwarp();  // this buffer is refilled by the next block's issue
    }
}

// New conv state: each sequence's last three inputs, per channel (one thread
// per (sequence, channel), reading all three before writing, so the update
// may be in place).  Also checks cu_seqlens.
__global__ void gdn_conv_state_kernel(FeArgs a) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)a.N * a.C) return;
    const int n = (int)(idx / a.C), cc = (int)(idx % a.C);
    const int64_t s = a.cu ? a.cu[n] : 0, e = a.cu ? a.cu[n + 1] : a.T;
    if (a.cu && (s < 0 || e < s || e > a.T || (n == 0 && s != 0) || (n == a.N - 1 && e != a.T))) {
        raise_error(a.err, GDN_ERR_BAD_SEQLENS);
        return;
    }
    const int z = cc < a.t[1].chan0 ? 0 : cc < a.t[2].chan0 ? 1 : 2;
    const FeTensor ft = z == 0 ? a.t[0] : z == 1 ? a.t[1] : a.t[2];
    const int ch = cc - ft.chan0;
    const int64_t L = e - s;
    float v[3];
#pragma unroll
    for (int i = 0; i < 3; ++i) {  // input i of the three after the sequence (oldest first)
        const int64_t pos = L + i - 3;  // position within the sequence; < 0: in the old state
        if (pos >= 0) {
            const int64_t off = (s + pos) * ft.H * kFeD + ch;
            v[i] = a.dtype == GDN_DTYPE_BF16
                       ? __bfloat162float(static_cast<const __nv_bfloat16 *>(ft.x)[off])
                       : static_cast<const float *>(ft.x)[off];
        } else {
            v[i] = a.state_in ? a.state_in[((int64_t)n * 3 + 3 + pos) * a.C + cc] : 0.f;
        }
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) a.state_out[((int64_t)n * 3 + i) * a.C + cc] = v[i];
}

// The fused prefill's copy of the filters: per (tensor, head) block of 128
// channels (q heads, then k heads, then v heads, the conv state's order),
// 512 floats ordered [tap k][part p][chunk cc][i] for channel 8 cc + 4 p + i,
// so that the sixteen threads convolving the sixteen 8-channel chunks of a
// row read one tap's filters as consecutive 16-byte words.
__global__ void gdn_conv_filter_kernel(const float *wq, const float *wk, const float *wv,
                                       int32_t Hqk, int32_t Hv, float *dst) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)(2 * Hqk + Hv) * 512) return;
    const int blk = (int)(idx >> 9), r = (int)(idx & 511);
    const int k = r >> 7, part = (r >> 6) & 1, cc = (r >> 2) & 15, i = r & 3;
    const float *w = blk < Hqk ? wq : blk < 2 * Hqk ? wk : wv;
    const int head = blk < Hqk ? blk : blk < 2 * Hqk ? blk - Hqk : blk - 2 * Hqk;
    dst[idx] = w[((int64_t)head * kFeD + 8 * cc + 4 * part + i) * 4 + k];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t launch_conv_filters(const float *wq, const float *wk, const float *wv, int32_t Hqk,
                                int32_t Hv, float *dst, cudaStream_t s) {
    const int64_t total = (int64_t)(2 * Hqk + Hv) * 512;
    gdn_conv_filter_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(wq, wk, wv, Hqk, Hv, dst);
    return cudaGetLastError();
}

cudaError_t launch_conv_state(const void *xq, const void *xk, const void *xv, gdn_dtype dt,
                              const float *state_in, float *state_out, const int32_t *cu,
                              int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t *err,
                              cudaStream_t s) {
    FeArgs a;
    const int32_t Cq = Hqk * kFeD;
    a.t[0] = {xq, nullptr, nullptr, Hqk, 0, 1};
    a.t[1] = {xk, nullptr, nullptr, Hqk, Cq, 1};
    a.t[2] = {xv, nullptr, nullptr, Hv, 2 * Cq, 0};
    a.cu = cu;
    a.state_in = state_in;
    a.state_out = state_out;
    a.err = err;
    a.T = T;
    a.N = N;
    a.C = 2 * Cq + Hv * kFeD;
    a.dtype = dt;
    const int64_t total = (int64_t)N * a.C;
    gdn_conv_state_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace gdn

extern "C" GDN_API gdn_status gdn_short_conv_norm(
    const void *xq, const void *xk, const void *xv, gdn_dtype io_dtype, const float *wq,
    const float *wk, const float *wv, const float *conv_state_in, float *conv_state_out,
    const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
    int32_t Dv, void *q, void *k, void *v, int32_t *dev_error_flag, void *stream) {
    GDN_TRACE("gdn_short_conv_norm");
    using gdn::aligned16;
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && N != 1) return GDN_ERR_INVALID_ARGUMENT;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    if (Dk != gdn::kFeD || Dv != gdn::kFeD) return GDN_ERR_UNSUPPORTED;
    // token blocks are the grid's y dimension (at most 65535 of 1024 tokens)
    if ((T + (int64_t)gdn::kFeWarps * gdn::kFeRun - 1) / ((int64_t)gdn::kFeWarps * gdn::kFeRun) > 65535)
        return GDN_ERR_UNSUPPORTED;
    if (T > 0 && (!xq || !xk || !xv || !wq || !wk || !wv || !q || !k || !v))
        return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {xq, xk, xv, wq, wk, wv, conv_state_in, conv_state_out, cu_seqlens,
                          q, k, v, dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    const void *outs[] = {q, k, v};
    const void *ins[] = {xq, xk, xv, wq, wk, wv, conv_state_in};
    for (const void *o : outs)
        for (const void *i : ins)
            if (o && o == i) return GDN_ERR_INVALID_ARGUMENT;
    if (q && (q == k || q == v || k == v)) return GDN_ERR_INVALID_ARGUMENT;

    gdn::FeArgs a;
    const int32_t Cq = Hqk * gdn::kFeD;
    a.t[0] = {xq, wq, q, Hqk, 0, 1};
    a.t[1] = {xk, wk, k, Hqk, Cq, 1};
    a.t[2] = {xv, wv, v, Hv, 2 * Cq, 0};
    a.cu = cu_seqlens;
    a.state_in = conv_state_in;
    a.state_out = conv_state_out;
    a.err = dev_error_flag;
    a.T = T;
    a.N = N;
    a.C = 2 * Cq + Hv * gdn::kFeD;
    a.dtype = io_dtype;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T > 0) {
        const int64_t per_cta = (int64_t)gdn::kFeWarps * gdn::kFeRun;
        const dim3 grid((unsigned)(2 * Hqk + Hv), (unsigned)((T + per_cta - 1) / per_cta));
        const size_t smem = (size_t)gdn::kFeWarps * 2 * gdn::kFeBlk * gdn::kFeD *
                            (io_dtype == GDN_DTYPE_BF16 ? 2 : 4);
        if (cudaFuncSetAttribute(gdn::gdn_short_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return GDN_ERR_CUDA;
        gdn::gdn_short_conv_kernel<<<grid, gdn::kFeWarps * 32, smem, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (conv_state_out) {
        const int64_t total = (int64_t)N * a.C;
        gdn::gdn_conv_state_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    return GDN_OK;
}
