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
// owns one (token, head) row of 128 channels, 4 per lane; a CTA's 8 warps take
// 8 consecutive tokens of one head, so the 3-token halo of each row is read
// from L1 rather than HBM.  A second small kernel writes the new conv state.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kFeD = 128;        // head dimension served
constexpr int kFeTokens = 8;     // tokens per CTA (one per warp)

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

// grid: (ceil(T / 8), Hqk + Hqk + Hv): y walks the q heads, then the k heads,
// then the v heads; block: 8 warps, one token each
__global__ void __launch_bounds__(kFeTokens * 32)
    gdn_short_conv_kernel(FeArgs a) {
    const int yh = blockIdx.y, Hq = a.t[0].H;
    const int z = yh < Hq ? 0 : yh < 2 * Hq ? 1 : 2;
    const FeTensor ft = z == 0 ? a.t[0] : z == 1 ? a.t[1] : a.t[2];
    const int h = yh - (z == 0 ? 0 : z == 1 ? Hq : 2 * Hq);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kFeTokens + warp;
    if (t >= a.T) return;
    const int n = a.cu ? fe_sequence(a.cu, a.N, t) : 0;
    const int64_t start = a.cu ? (int64_t)a.cu[n] : 0;
    const int c = h * kFeD + 4 * lane;  // this lane's first channel within the tensor

    float4 w[4];  // w[i]: the 4 taps of channel c + i
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const float4 *>(ft.w + (int64_t)(c + i) * 4);
    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // tap j reads token t - 3 + j
        const int64_t tp = t - 3 + j;
        float4 xv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (tp >= start && tp >= 0) {
            xv = fe_load4(ft.x, tp * ft.H * kFeD + c, a.dtype);
        } else if (a.state_in) {  // before the sequence: its carried inputs
            const int64_t back = start - tp;  // 1 .. 3 for a well-formed cu_seqlens
            if (back >= 1 && back <= 3)
                xv = *reinterpret_cast<const float4 *>(a.state_in + ((int64_t)n * 3 + 3 - back) * a.C +
                                                        ft.chan0 + c);
        }
        const float x4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float wj = j == 0 ? w[i].x : j == 1 ? w[i].y : j == 2 ? w[i].z : w[i].w;
            y[i] = fmaf(wj, x4[i], y[i]);
        }
    }
    if (ft.norm) {  // divide the (token, head) row by its norm; a zero row stays zero
        float ss = y[0] * y[0] + y[1] * y[1] + y[2] * y[2] + y[3] * y[3];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float nrm = sqrtf(ss);
        if (nrm > 0.f) {
#pragma unroll
            for (int i = 0; i < 4; ++i) y[i] = y[i] / nrm;
        }
    }
    fe_store4(ft.y, t * ft.H * kFeD + c, make_float4(y[0], y[1], y[2], y[3]), a.dtype);
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

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace gdn

extern "C" GDN_API gdn_status gdn_short_conv_norm(
    const void *xq, const void *xk, const void *xv, gdn_dtype io_dtype, const float *wq,
    const float *wk, const float *wv, const float *conv_state_in, float *conv_state_out,
    const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
    int32_t Dv, void *q, void *k, void *v, int32_t *dev_error_flag, void *stream) {
    using gdn::aligned16;
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && N != 1) return GDN_ERR_INVALID_ARGUMENT;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    if (Dk != gdn::kFeD || Dv != gdn::kFeD) return GDN_ERR_UNSUPPORTED;
    if (T > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
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
        const dim3 grid((unsigned)((T + gdn::kFeTokens - 1) / gdn::kFeTokens), (unsigned)(2 * Hqk + Hv));
        gdn::gdn_short_conv_kernel<<<grid, gdn::kFeTokens * 32, 0, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (conv_state_out) {
        const int64_t total = (int64_t)N * a.C;
        gdn::gdn_conv_state_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(a);
        if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    }
    return GDN_OK;
}
