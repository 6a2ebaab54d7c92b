// Exact token-recurrent prefill of the gated delta rule on CUDA cores (fp32).
//
// This kernel runs the rule of section 三 of "Qwen3.8-27B 架构深读: Gated
// DeltaNet 混合线性注意力与 262K 长上下文" one token at a time:
//     S <- a S;  r = S k;  S <- S + b (v - r) k^T;  o = S q
// or, in the page's step function order (GDN_ORDER_RECALL_FIRST), with the
// recall r = S k taken before the decay.
// It serves the head sizes and dtypes the tensor-core chunked kernel does not
// (small heads, fp32 I/O, chunk lengths other than 64), where the chunked
// form's per-chunk set-up would cost more than it saves.
//
// Rows of the state evolve independently given (k, q, a, b): row i only needs
// v_i.  So each thread owns one row S_i (Dk fp32 values in registers), a CTA
// owns up to 128 rows of one (sequence, v-head), and no thread ever talks to
// another except to share the staged token inputs.  Per token each thread
// does 3*Dk FMAs: r = S_i.k (recall from the undecayed row, scaled by a), the
// delta write, and the read-out.  Tokens are staged through shared memory in
// blocks of kTokBlock so the (k, q) loads are shared by the CTA's rows.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kTokBlock = 16;

template <int DK>
__global__ void __launch_bounds__(128)
    gdn_prefill_recurrent_kernel(PrefillArgs a, int row_blocks) {
    __shared__ float ks[kTokBlock][DK];
    __shared__ float qs[kTokBlock][DK];
    __shared__ float vs[kTokBlock][128];
    __shared__ float as_[kTokBlock], bs[kTokBlock];
    const bool recall_first = a.order == GDN_ORDER_RECALL_FIRST;  // recall before the decay

    const int rows = blockDim.x;
    const int rb = blockIdx.x % row_blocks;
    const int h = (blockIdx.x / row_blocks) % a.Hv;
    const int n = blockIdx.x / (row_blocks * a.Hv);
    const int j = h / (a.Hv / a.Hqk);
    const int i = rb * rows + threadIdx.x;
    const bool active = i < a.Dv;

    int64_t t0, t1;
    if (!seq_range(a.cu, n, a.N, a.T, a.err, t0, t1)) return;  // uniform per CTA

    float S[DK];
    const int64_t st_off = (((int64_t)n * a.Hv + h) * a.Dv + i) * DK;
#pragma unroll
    for (int d = 0; d < DK; ++d) S[d] = (active && a.s0) ? a.s0[st_off + d] : 0.f;

    for (int64_t tb = t0; tb < t1; tb += kTokBlock) {
        const int nt = (t1 - tb < kTokBlock) ? (int)(t1 - tb) : kTokBlock;
        __syncthreads();  // previous block fully consumed
        for (int x = threadIdx.x; x < nt * DK; x += rows) {
            const int tt = x / DK, d = x % DK;
            const int64_t idx = ((tb + tt) * a.Hqk + j) * DK + d;
            ks[tt][d] = load_io(a.k, idx, a.dtype);
            qs[tt][d] = load_io(a.q, idx, a.dtype);
        }
        for (int x = threadIdx.x; x < nt * rows; x += rows) {
            const int tt = x / rows, r = x % rows;
            const int ii = rb * rows + r;
            vs[tt][r] = (ii < a.Dv) ? load_io(a.v, ((tb + tt) * a.Hv + h) * a.Dv + ii, a.dtype) : 0.f;
        }
        if (threadIdx.x < nt) {
            as_[threadIdx.x] = expf(a.g[(tb + threadIdx.x) * a.Hv + h]);
            bs[threadIdx.x] = a.beta[(tb + threadIdx.x) * a.Hv + h];
        }
        __syncthreads();
        for (int tt = 0; tt < nt; ++tt) {
            const float dec = as_[tt], b = bs[tt];
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
            for (int d = 0; d < DK; d += 4) {
                p0 = fmaf(S[d + 0], ks[tt][d + 0], p0);
                p1 = fmaf(S[d + 1], ks[tt][d + 1], p1);
                p2 = fmaf(S[d + 2], ks[tt][d + 2], p2);
                p3 = fmaf(S[d + 3], ks[tt][d + 3], p3);
            }
            const float r = (recall_first ? 1.f : dec) * ((p0 + p1) + (p2 + p3));
            const float u = b * (vs[tt][threadIdx.x] - r);
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
            for (int d = 0; d < DK; d += 4) {
                S[d + 0] = fmaf(u, ks[tt][d + 0], dec * S[d + 0]);
                S[d + 1] = fmaf(u, ks[tt][d + 1], dec * S[d + 1]);
                S[d + 2] = fmaf(u, ks[tt][d + 2], dec * S[d + 2]);
                S[d + 3] = fmaf(u, ks[tt][d + 3], dec * S[d + 3]);
                o0 = fmaf(S[d + 0], qs[tt][d + 0], o0);
                o1 = fmaf(S[d + 1], qs[tt][d + 1], o1);
                o2 = fmaf(S[d + 2], qs[tt][d + 2], o2);
                o3 = fmaf(S[d + 3], qs[tt][d + 3], o3);
            }
            if (active) store_io(a.o, ((tb + tt) * a.Hv + h) * a.Dv + i, (o0 + o1) + (o2 + o3), a.dtype);
        }
    }
    if (active && a.sT) {
#pragma unroll
        for (int d = 0; d < DK; ++d) a.sT[st_off + d] = S[d];
    }
}

}  // namespace

cudaError_t launch_prefill_recurrent(const PrefillArgs &a, cudaStream_t s) {
    const int rows = a.Dv >= 128 ? 128 : ((a.Dv + 31) / 32) * 32;
    const int row_blocks = (a.Dv + rows - 1) / rows;
    const int64_t blocks = (int64_t)row_blocks * a.Hv * a.N;
    if (blocks <= 0) return cudaSuccess;
    const dim3 grid((unsigned)blocks), block(rows);
    switch (a.Dk) {
        case 16: gdn_prefill_recurrent_kernel<16><<<grid, block, 0, s>>>(a, row_blocks); break;
        case 32: gdn_prefill_recurrent_kernel<32><<<grid, block, 0, s>>>(a, row_blocks); break;
        case 64: gdn_prefill_recurrent_kernel<64><<<grid, block, 0, s>>>(a, row_blocks); break;
        case 128: gdn_prefill_recurrent_kernel<128><<<grid, block, 0, s>>>(a, row_blocks); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace gdn
