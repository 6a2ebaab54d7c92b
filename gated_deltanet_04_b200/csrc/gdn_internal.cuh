// Internal declarations shared by libgdn's translation units (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// Everything a prefill kernel needs; pointers are device pointers.
struct PrefillArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    const float *s0;        // may be null (zeros)
    const int32_t *cu;      // may be null (one sequence)
    void *o;
    float *sT;              // may be null
    int32_t *err;           // may be null
    void *ws;               // workspace (cluster kernel's L2 ring)
    int64_t T;
    int32_t N, Hqk, Hv, Dk, Dv, chunk;
    gdn_dtype dtype;
    int32_t order = GDN_ORDER_STANDARD;  // gdn_order
    // testing only (pool kernel): a unit the producers never prepare, and the
    // SM-clock limit of every spin on a hand-off flag (0: the default)
    int32_t debug_skip_unit = -1;
    int64_t debug_flag_wait = 0;
    // front end fused into the pool kernel's load stage: q, k, v above are then
    // the raw inputs of the q, k, v channels (see gdn_prefill_conv)
    bool conv = false;
    const float *cf = nullptr;  // filters as launch_conv_filters writes them
    const float *cstate_in = nullptr;                  // [N][3][C] or null (zeros)
};

struct DecodeArgs {
    const void *q, *k, *v;
    const float *g, *beta;
    void *state;            // fp32, or bfloat16 when state_bf16
    int32_t state_bf16 = 0;
    void *o;
    int32_t *err;
    int32_t N, Hqk, Hv, Dk, Dv;
    gdn_dtype dtype;
    int32_t order = GDN_ORDER_STANDARD;  // gdn_order
    // pool decode: sequence n's state is slot slot[n] of num_slots; reset[n]
    // nonzero: it starts from zeros.  slot == nullptr: the state of n is n.
    const int32_t *slot = nullptr;
    const int32_t *reset = nullptr;
    int32_t num_slots = 0;
};

// The state slot of decode sequence n (n itself without a slot array), or -1
// when slot[n] is out of range.
__device__ __forceinline__ int64_t decode_state_slot(const DecodeArgs &a, int n) {
    if (a.slot == nullptr) return n;
    const int s = a.slot[n];
    return (s >= 0 && s < a.num_slots) ? s : -1;
}
__device__ __forceinline__ bool decode_state_reset(const DecodeArgs &a, int n) {
    return a.reset != nullptr && a.reset[n] != 0;
}

// Host launchers (return cudaGetLastError() of the launch).
cudaError_t launch_prefill_recurrent(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
// Tensor-core chunked prefill, Dk = Dv = 128, bf16, chunk 64: one CTA per
// (sequence, head), or a 3-CTA cluster per (sequence, head).
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_prefill_cluster(const PrefillArgs &a, cudaStream_t s);
// Chain CTA per (sequence, head) plus producer CTAs on every other SM, one
// cooperative launch.  Falls back to launch_prefill_tc on a GPU with too few
// SMs for the units.
cudaError_t launch_prefill_pool(const PrefillArgs &a, cudaStream_t s);
// Workspace of the cluster kernel: a 4-slot ring per (sequence, head).
size_t prefill_cluster_workspace_bytes(int64_t units);
constexpr size_t kClusterWorkspaceBytesPerUnit = 430080;
// Workspace of the pool kernel: hand-off flags, then the same ring.
size_t prefill_pool_workspace_bytes(int64_t units);
// AUTO uses the pool kernel up to this many (sequence, head) units.
constexpr int64_t kPoolMaxUnits = 64;
// Whether the current device has SMs enough for the pool kernel with `units`.
bool prefill_pool_fits(int64_t units);
// The new conv state of gdn_short_conv_norm's contract (each sequence's last
// three inputs of every q, k, v channel), also checking cu_seqlens.
cudaError_t launch_conv_state(const void *xq, const void *xk, const void *xv, gdn_dtype dt,
                              const float *state_in, float *state_out, const int32_t *cu,
                              int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t *err,
                              cudaStream_t s);
// The filters wq, wk, wv ([H * 128][4] fp32 each) rearranged for the fused
// prefill into dst, conv_filter_bytes(Hqk, Hv) bytes.
cudaError_t launch_conv_filters(const float *wq, const float *wk, const float *wv, int32_t Hqk,
                                int32_t Hv, float *dst, cudaStream_t s);
constexpr size_t conv_filter_bytes(int32_t Hqk, int32_t Hv) { return (size_t)(2 * Hqk + Hv) * 2048; }

// ---------------------------------------------------------------- device --

__device__ __forceinline__ float load_io(const void *p, int64_t idx, gdn_dtype dt) {
    if (dt == GDN_DTYPE_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[idx]);
    return static_cast<const float *>(p)[idx];
}

__device__ __forceinline__ void store_io(void *p, int64_t idx, float x, gdn_dtype dt) {
    if (dt == GDN_DTYPE_BF16)
        static_cast<__nv_bfloat16 *>(p)[idx] = __float2bfloat16_rn(x);
    else
        static_cast<float *>(p)[idx] = x;
}

__device__ __forceinline__ void raise_error(int32_t *flag, int code) {
    if (flag) atomicCAS(flag, 0, code);
}

// Reads and validates sequence n's token range.  Returns false (and raises
// GDN_ERR_BAD_SEQLENS) when cu_seqlens is malformed around n; the range is
// then not to be used.  Uniform across a CTA when every thread passes the
// same n.
__device__ __forceinline__ bool seq_range(const int32_t *cu, int32_t n, int32_t N, int64_t T,
                                          int32_t *err, int64_t &t0, int64_t &t1) {
    if (cu == nullptr) {
        t0 = 0;
        t1 = T;
        return true;
    }
    t0 = cu[n];
    t1 = cu[n + 1];
    bool ok = (t0 >= 0) && (t0 <= t1) && (t1 <= T);
    if (n == 0) ok = ok && (t0 == 0);
    if (n == N - 1) ok = ok && (t1 == T);
    if (!ok) raise_error(err, GDN_ERR_BAD_SEQLENS);
    return ok;
}

}  // namespace gdn
