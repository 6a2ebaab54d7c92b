// libgdn C ABI: argument validation and kernel dispatch.  See include/gdn.h
// for the contract of every entry point.
#include <stdint.h>

#include "gdn_internal.cuh"
#include "trace.cuh"

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int32_t d) { return d == 16 || d == 32 || d == 64 || d == 128; }

bool tc_path(gdn_dtype dt, int32_t Dk, int32_t Dv, int32_t chunk) {
    return dt == GDN_DTYPE_BF16 && Dk == 128 && Dv == 128 && (chunk == 0 || chunk == 64);
}

gdn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARGUMENT: return "GDN_ERR_INVALID_ARGUMENT";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_BAD_SEQLENS: return "GDN_ERR_BAD_SEQLENS";
        case GDN_ERR_BAD_SLOT: return "GDN_ERR_BAD_SLOT";
        case GDN_ERR_RANGE: return "GDN_ERR_RANGE";
    }
    return "GDN_ERR_UNKNOWN";
}

int32_t gdn_version(void) { return 1 * 10000 + 0 * 100 + 0; }

// The kernel gdn_prefill_ex runs for these arguments (kernel AUTO resolved).
gdn_prefill_kernel resolve_kernel(gdn_prefill_kernel kernel, bool tc_ok, int64_t units) {
    if (kernel != GDN_PREFILL_AUTO) return kernel;
    if (!tc_ok) return GDN_PREFILL_RECURRENT;
    return units <= gdn::kPoolMaxUnits ? GDN_PREFILL_POOL : GDN_PREFILL_SINGLE_CTA;
}

// Scratch bytes of a resolved kernel choice.
size_t workspace_need(gdn_prefill_kernel kernel, int64_t units) {
    if (kernel == GDN_PREFILL_CLUSTER) return gdn::prefill_cluster_workspace_bytes(units);
    if (kernel == GDN_PREFILL_POOL) return gdn::prefill_pool_workspace_bytes(units);
    return 0;
}

size_t gdn_prefill_ex_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                      int32_t Dv, int32_t chunk, gdn_prefill_kernel kernel) {
    (void)T; (void)Hqk;
    if (N <= 0 || Hv <= 0) return 0;
    const bool shape_ok = Dk == 128 && Dv == 128 && (chunk == 0 || chunk == 64);
    if (!shape_ok) return 0;
    return workspace_need(resolve_kernel(kernel, shape_ok, (int64_t)N * Hv), (int64_t)N * Hv);
}

size_t gdn_prefill_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                   int32_t Dv, int32_t chunk) {
    return gdn_prefill_ex_workspace_bytes(N, T, Hqk, Hv, Dk, Dv, chunk, GDN_PREFILL_AUTO);
}

gdn_status gdn_prefill(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                       const float *g, const float *beta, const float *initial_state,
                       const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                       int32_t Dk, int32_t Dv, int32_t chunk, void *o, float *final_state,
                       void *workspace, size_t workspace_bytes, int32_t *dev_error_flag,
                       void *stream) {
    return gdn_prefill_ex(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv,
                          Dk, Dv, chunk, o, final_state, workspace, workspace_bytes,
                          dev_error_flag, stream, GDN_PREFILL_AUTO);
}

gdn_status gdn_prefill_ex(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                          const float *g, const float *beta, const float *initial_state,
                          const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                          int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                          float *final_state, void *workspace, size_t workspace_bytes,
                          int32_t *dev_error_flag, void *stream, gdn_prefill_kernel kernel) {
    return gdn_prefill_order(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv,
                             Dk, Dv, chunk, o, final_state, workspace, workspace_bytes,
                             dev_error_flag, stream, kernel, GDN_ORDER_STANDARD);
}

}  // extern "C"

namespace {

// gdn_prefill_order, plus the testing-only settings of the pool kernel (a unit
// its producers skip, and the limit of its flag spins; -1 / 0 = off).
gdn_status prefill_impl(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                        const float *g, const float *beta, const float *initial_state,
                        const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk, int32_t Hv,
                        int32_t Dk, int32_t Dv, int32_t chunk, void *o, float *final_state,
                        void *workspace, size_t workspace_bytes, int32_t *dev_error_flag,
                        void *stream, gdn_prefill_kernel kernel, gdn_order order,
                        int32_t debug_skip_unit, int64_t debug_flag_wait) {
    GDN_TRACE("gdn_prefill");
    if (kernel < GDN_PREFILL_AUTO || kernel > GDN_PREFILL_POOL) return GDN_ERR_INVALID_ARGUMENT;
    if (order != GDN_ORDER_STANDARD && order != GDN_ORDER_RECALL_FIRST) return GDN_ERR_INVALID_ARGUMENT;
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0)
        return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && N != 1) return GDN_ERR_INVALID_ARGUMENT;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, o, final_state, workspace,
                          dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    if (o && (o == q || o == k || o == v)) return GDN_ERR_INVALID_ARGUMENT;
    if (!supported_dim(Dk) || !supported_dim(Dv) || chunk > 64) return GDN_ERR_UNSUPPORTED;
    const bool tc_ok = tc_path(io_dtype, Dk, Dv, chunk);
    if ((kernel == GDN_PREFILL_CLUSTER || kernel == GDN_PREFILL_SINGLE_CTA ||
         kernel == GDN_PREFILL_POOL) && !tc_ok)
        return GDN_ERR_UNSUPPORTED;
    if (kernel == GDN_PREFILL_POOL && (int64_t)N * Hv > gdn::kPoolMaxUnits) return GDN_ERR_UNSUPPORTED;
    kernel = resolve_kernel(kernel, tc_ok, (int64_t)N * Hv);
    const size_t need = T > 0 ? workspace_need(kernel, (int64_t)N * Hv) : 0;
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return GDN_ERR_INVALID_ARGUMENT;
    if (T == 0 && final_state == nullptr) return GDN_OK;  // nothing observable to do

    gdn::PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.s0 = initial_state; a.cu = cu_seqlens;
    a.o = o; a.sT = final_state; a.err = dev_error_flag; a.ws = workspace; a.T = T; a.N = N; a.Hqk = Hqk;
    a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.chunk = chunk == 0 ? 64 : chunk; a.dtype = io_dtype;
    a.order = order;
    a.debug_skip_unit = debug_skip_unit;
    a.debug_flag_wait = debug_flag_wait;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0 || kernel == GDN_PREFILL_RECURRENT) return from_cuda(gdn::launch_prefill_recurrent(a, s));
    if (kernel == GDN_PREFILL_SINGLE_CTA) return from_cuda(gdn::launch_prefill_tc(a, s));
    if (kernel == GDN_PREFILL_POOL) return from_cuda(gdn::launch_prefill_pool(a, s));
    return from_cuda(gdn::launch_prefill_cluster(a, s));
}

}  // namespace

extern "C" {

gdn_status gdn_prefill_order(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                             const float *g, const float *beta, const float *initial_state,
                             const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                             int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                             float *final_state, void *workspace, size_t workspace_bytes,
                             int32_t *dev_error_flag, void *stream, gdn_prefill_kernel kernel,
                             gdn_order order) {
    return prefill_impl(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv, Dk,
                        Dv, chunk, o, final_state, workspace, workspace_bytes, dev_error_flag,
                        stream, kernel, order, -1, 0);
}

// gdn_prefill_conv's scratch: the pool kernel's, then (from a 256-byte
// boundary) the rearranged filters.
size_t conv_filter_offset(int64_t units) {
    return (gdn::prefill_pool_workspace_bytes(units) + 255) & ~(size_t)255;
}

size_t gdn_prefill_conv_workspace_bytes(int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                        int32_t Dv) {
    if (N <= 0 || T <= 0 || Hqk <= 0 || Hv <= 0 || Hv % Hqk != 0 || Dk != 128 || Dv != 128)
        return 0;
    const int64_t units = (int64_t)N * Hv;
    if (units > gdn::kPoolMaxUnits) return 0;
    return conv_filter_offset(units) + gdn::conv_filter_bytes(Hqk, Hv);
}

gdn_status gdn_prefill_conv(const void *xq, const void *xk, const void *xv, gdn_dtype io_dtype,
                            const float *wq, const float *wk, const float *wv,
                            const float *conv_state_in, float *conv_state_out, const float *g,
                            const float *beta, const float *initial_state,
                            const int32_t *cu_seqlens, int32_t N, int64_t T, int32_t Hqk,
                            int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                            float *final_state, void *workspace, size_t workspace_bytes,
                            int32_t *dev_error_flag, void *stream) {
    GDN_TRACE("gdn_prefill_conv");
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0)
        return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (cu_seqlens == nullptr && N != 1) return GDN_ERR_INVALID_ARGUMENT;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!xq || !xk || !xv || !wq || !wk || !wv || !g || !beta || !o))
        return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {xq, xk, xv, wq, wk, wv, conv_state_in, conv_state_out, g, beta,
                          initial_state, cu_seqlens, o, final_state, workspace, dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    const void *ins[] = {xq, xk, xv, wq, wk, wv, g, beta};
    for (const void *i : ins)
        if (i && (i == o || i == conv_state_out)) return GDN_ERR_INVALID_ARGUMENT;
    if (!tc_path(io_dtype, Dk, Dv, chunk)) return GDN_ERR_UNSUPPORTED;
    const int64_t units = (int64_t)N * Hv;
    if (units > gdn::kPoolMaxUnits || !gdn::prefill_pool_fits(units)) return GDN_ERR_UNSUPPORTED;
    const size_t need = gdn_prefill_conv_workspace_bytes(N, T, Hqk, Hv, Dk, Dv);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return GDN_ERR_INVALID_ARGUMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    float *filters = nullptr;
    if (T > 0) {
        filters = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + conv_filter_offset(units));
        const cudaError_t e = gdn::launch_conv_filters(wq, wk, wv, Hqk, Hv, filters, s);
        if (e != cudaSuccess) return GDN_ERR_CUDA;
    }
    if (T > 0 || final_state != nullptr) {
        gdn::PrefillArgs a;
        a.q = xq; a.k = xk; a.v = xv; a.g = g; a.beta = beta; a.s0 = initial_state;
        a.cu = cu_seqlens; a.o = o; a.sT = final_state; a.err = dev_error_flag; a.ws = workspace;
        a.T = T; a.N = N; a.Hqk = Hqk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv; a.chunk = 64;
        a.dtype = io_dtype;
        a.conv = true;
        a.cf = filters;
        a.cstate_in = conv_state_in;
        const cudaError_t e = T > 0 ? gdn::launch_prefill_pool(a, s) : gdn::launch_prefill_recurrent(a, s);
        if (e == cudaErrorNotSupported) return GDN_ERR_UNSUPPORTED;
        if (e != cudaSuccess) return GDN_ERR_CUDA;
    }
    // the new conv state after the prefill, which reads the old one (so the two may alias)
    if (conv_state_out)
        return from_cuda(gdn::launch_conv_state(xq, xk, xv, io_dtype, conv_state_in, conv_state_out,
                                                cu_seqlens, N, T, Hqk, Hv, dev_error_flag, s));
    return GDN_OK;
}

gdn_status gdn_debug_prefill_pool_stall(const void *q, const void *k, const void *v,
                                        gdn_dtype io_dtype, const float *g, const float *beta,
                                        const float *initial_state, const int32_t *cu_seqlens,
                                        int32_t N, int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk,
                                        int32_t Dv, int32_t chunk, void *o, float *final_state,
                                        void *workspace, size_t workspace_bytes,
                                        int32_t *dev_error_flag, void *stream, int32_t skip_unit,
                                        int64_t flag_wait_cycles) {
    if (skip_unit < 0 || flag_wait_cycles <= 0) return GDN_ERR_INVALID_ARGUMENT;
    return prefill_impl(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv, Dk,
                        Dv, chunk, o, final_state, workspace, workspace_bytes, dev_error_flag,
                        stream, GDN_PREFILL_POOL, GDN_ORDER_STANDARD, skip_unit, flag_wait_cycles);
}

gdn_status gdn_decode_step(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                           const float *g, const float *beta, float *state, int32_t N,
                           int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, void *o,
                           int32_t *dev_error_flag, void *stream) {
    return gdn_decode_step_order(q, k, v, io_dtype, g, beta, state, N, Hqk, Hv, Dk, Dv, o,
                                 dev_error_flag, stream, GDN_ORDER_STANDARD);
}

gdn_status gdn_decode_step_order(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                                 const float *g, const float *beta, float *state, int32_t N,
                                 int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, void *o,
                                 int32_t *dev_error_flag, void *stream, gdn_order order) {
    GDN_TRACE("gdn_decode_step");
    if (order != GDN_ORDER_STANDARD && order != GDN_ORDER_RECALL_FIRST) return GDN_ERR_INVALID_ARGUMENT;
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, g, beta, state, o, dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    if (o == q || o == k || o == v || o == state) return GDN_ERR_INVALID_ARGUMENT;
    if (!supported_dim(Dk)) return GDN_ERR_UNSUPPORTED;
    gdn::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.state = state; a.o = o;
    a.err = dev_error_flag; a.N = N; a.Hqk = Hqk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv;
    a.dtype = io_dtype;
    a.order = order;
    return from_cuda(gdn::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_step_slots(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                                 const float *g, const float *beta, float *state_pool,
                                 int32_t num_slots, const int32_t *slot_idx, const int32_t *reset,
                                 int32_t N, int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                 void *o, int32_t *dev_error_flag, void *stream) {
    GDN_TRACE("gdn_decode_step_slots");
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    if (num_slots <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (!q || !k || !v || !g || !beta || !state_pool || !slot_idx || !o) return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, g, beta, state_pool, slot_idx, reset, o, dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    if (o == q || o == k || o == v || o == state_pool) return GDN_ERR_INVALID_ARGUMENT;
    if (!supported_dim(Dk)) return GDN_ERR_UNSUPPORTED;
    gdn::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.state = state_pool; a.o = o;
    a.err = dev_error_flag; a.N = N; a.Hqk = Hqk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv;
    a.dtype = io_dtype;
    a.slot = slot_idx; a.reset = reset; a.num_slots = num_slots;
    return from_cuda(gdn::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode_step_bf16_state(const void *q, const void *k, const void *v,
                                      gdn_dtype io_dtype, const float *g, const float *beta,
                                      void *state, int32_t N, int32_t Hqk, int32_t Hv, int32_t Dk,
                                      int32_t Dv, void *o, int32_t *dev_error_flag, void *stream) {
    GDN_TRACE("gdn_decode_step_bf16_state");
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (N < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * Hv > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
    if (Dk != 128 || Dv != 128) return GDN_ERR_UNSUPPORTED;
    if (N == 0) return GDN_OK;
    if (!q || !k || !v || !g || !beta || !state || !o) return GDN_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, g, beta, state, o, dev_error_flag};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return GDN_ERR_INVALID_ARGUMENT;
    if (o == q || o == k || o == v || o == state) return GDN_ERR_INVALID_ARGUMENT;
    gdn::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.state = state; a.o = o;
    a.state_bf16 = 1;
    a.err = dev_error_flag; a.N = N; a.Hqk = Hqk; a.Hv = Hv; a.Dk = Dk; a.Dv = Dv;
    a.dtype = io_dtype;
    return from_cuda(gdn::launch_decode(a, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
