// gdn_prefill_slots: a prefill whose sequences start from, and end in, slots
// of the same state pool that gdn_decode_step_slots serves (continuous
// batching: page "Hybrid · kết hợp…", section 3, state updates with batch and
// reset rules).  Sequence n starts from pool[slot_idx[n]] (zeros when
// reset[n] is set: a new request) and its final state goes back there.
//
// The states are gathered into the workspace, the ordinary prefill runs in
// place on them, and they are scattered back: two copies of N * Hv * Dv * Dk
// fp32 values around the prefill, which leaves every prefill kernel as it is.
#include <cuda_runtime.h>

#include <cstdint>

#include "gdn.h"
#include "gdn_internal.cuh"
#include "trace.cuh"

namespace {

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sequence n's slot, or -1 when its index is out of range (reported once, by
// the sequence's first thread).
__device__ __forceinline__ int slot_of(const int32_t *slot_idx, int n, int num_slots,
                                       int32_t *err, bool report) {
    const int sl = slot_idx[n];
    if (sl < 0 || sl >= num_slots) {
        if (report) gdn::raise_error(err, GDN_ERR_BAD_SLOT);
        return -1;
    }
    return sl;
}

// dst[n] = reset[n] ? 0 : pool[slot_idx[n]]  (zeros for a bad slot), float4s
__global__ void gdn_slots_gather_kernel(const float4 *pool, const int32_t *slot_idx,
                                        const int32_t *reset, int num_slots, int N,
                                        int64_t per_state, float4 *dst, int32_t *err) {
    const int64_t total = (int64_t)N * per_state;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / per_state);
        const int64_t r = i - (int64_t)n * per_state;
        const int sl = slot_of(slot_idx, n, num_slots, err, r == 0);
        const bool zero = sl < 0 || (reset != nullptr && reset[n] != 0);
        dst[i] = zero ? make_float4(0.f, 0.f, 0.f, 0.f) : pool[(int64_t)sl * per_state + r];
    }
}

// pool[slot_idx[n]] = src[n]  (nothing for a bad slot)
__global__ void gdn_slots_scatter_kernel(float4 *pool, const int32_t *slot_idx, int num_slots,
                                         int N, int64_t per_state, const float4 *src) {
    const int64_t total = (int64_t)N * per_state;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int n = (int)(i / per_state);
        const int64_t r = i - (int64_t)n * per_state;
        const int sl = slot_of(slot_idx, n, num_slots, nullptr, false);
        if (sl >= 0) pool[(int64_t)sl * per_state + r] = src[i];
    }
}

unsigned grid_for(int64_t total) {
    const int64_t blocks = (total + 255) / 256;
    return (unsigned)(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
}

}  // namespace

extern "C" {

size_t gdn_prefill_slots_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                         int32_t Dv, int32_t chunk) {
    if (N <= 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0) return 0;
    return al256((size_t)N * Hv * Dv * Dk * 4) +
           gdn_prefill_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk);
}

gdn_status gdn_prefill_slots(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                             const float *g, const float *beta, float *state_pool,
                             int32_t num_slots, const int32_t *slot_idx, const int32_t *reset,
                             const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                             int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                             void *workspace, size_t workspace_bytes, int32_t *dev_error_flag,
                             void *stream) {
    GDN_TRACE("gdn_prefill_slots");
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0)
        return GDN_ERR_INVALID_ARGUMENT;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    if (num_slots <= 0 || !state_pool || !slot_idx || !workspace) return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {state_pool, slot_idx, reset, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    const size_t need = gdn_prefill_slots_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk);
    if (workspace_bytes < need) return GDN_ERR_INVALID_ARGUMENT;
    const int64_t per_state = (int64_t)Hv * Dv * Dk / 4;  // float4s; Dk is a multiple of 16
    float *states = static_cast<float *>(workspace);
    const size_t off = al256((size_t)N * Hv * Dv * Dk * 4);
    void *ws = static_cast<uint8_t *>(workspace) + off;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // what the prefill would reject, rejected before the pool is read
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARGUMENT;
    const auto dim_ok = [](int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; };
    if (!dim_ok(Dk) || !dim_ok(Dv) || chunk > 64) return GDN_ERR_UNSUPPORTED;
    const int64_t total = (int64_t)N * per_state;
    gdn_slots_gather_kernel<<<grid_for(total), 256, 0, s>>>(
        reinterpret_cast<const float4 *>(state_pool), slot_idx, reset, num_slots, N, per_state,
        reinterpret_cast<float4 *>(states), dev_error_flag);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    const gdn_status st = gdn_prefill(q, k, v, io_dtype, g, beta, states, cu_seqlens, N, T, Hqk, Hv,
                                      Dk, Dv, chunk, o, states, ws, workspace_bytes - off,
                                      dev_error_flag, stream);
    if (st != GDN_OK) return st;
    gdn_slots_scatter_kernel<<<grid_for(total), 256, 0, s>>>(
        reinterpret_cast<float4 *>(state_pool), slot_idx, num_slots, N, per_state,
        reinterpret_cast<const float4 *>(states));
    return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // extern "C"
