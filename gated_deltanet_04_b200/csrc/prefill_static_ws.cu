// gdn_prefill_static_workspace: the cluster prefill with its workspace ring in
// a file-scope device array, for callers that allocate no device memory per
// call.  The contract is in include/gdn.h.  The path below calls no device
// allocator: the array's address is looked up once per device and context,
// and the call is then forwarded to gdn_prefill_ex with that address as the workspace.
#include <cuda.h>
#include <mutex>
#include <stdint.h>

#include "gdn_internal.cuh"

namespace {

constexpr int64_t kMaxUnits = GDN_STATIC_WORKSPACE_MAX_UNITS;
constexpr size_t kRingBytes = (size_t)kMaxUnits * gdn::kClusterWorkspaceBytesPerUnit;
static_assert(kRingBytes == 20643840, "the limit stated in gdn.h");

static __device__ __align__(256) unsigned char g_static_ring[kRingBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the device address of g_static_ring and the id of the CUDA
// context it was looked up in.  A device reset creates a new primary context
// (and a new copy of the array), whose different id triggers a new lookup.
struct RingAddr {
    void *addr;
    unsigned long long ctx_id;
};
RingAddr g_ring[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// The id of the calling thread's current context (CUDA 12.0+ driver call,
// reached through the runtime's driver entry points; libgdn links no libcuda).
gdn_status current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (get_current == nullptr || get_id == nullptr) return GDN_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return GDN_ERR_CUDA;
    return get_id(ctx, id) == CUDA_SUCCESS ? GDN_OK : GDN_ERR_CUDA;
}

// The array's address on the current device, looked up on first use in the
// device's current context.  Before libgdn's first CUDA call on this thread no
// context may be current yet; the symbol lookup then binds the device's
// primary context, and its id is read afterwards.
gdn_status ring_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx) == GDN_OK;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!have_ctx || g_ring[dev].addr == nullptr || g_ring[dev].ctx_id != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ring) != cudaSuccess || p == nullptr)
            return GDN_ERR_CUDA;
        if (current_context_id(&ctx) != GDN_OK) return GDN_ERR_CUDA;
        g_ring[dev].addr = p;
        g_ring[dev].ctx_id = ctx;
    }
    *out = g_ring[dev].addr;
    return GDN_OK;
}

}  // namespace

extern "C" gdn_status gdn_prefill_static_workspace(
    const void *q, const void *k, const void *v, gdn_dtype io_dtype, const float *g,
    const float *beta, const float *initial_state, const int32_t *cu_seqlens, int32_t N, int64_t T,
    int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o, float *final_state,
    int32_t *dev_error_flag, void *stream) {
    if (N < 0 || Hv <= 0) return GDN_ERR_INVALID_ARGUMENT;
    if ((int64_t)N * Hv > kMaxUnits) return GDN_ERR_UNSUPPORTED;
    if (io_dtype != GDN_DTYPE_BF16 || Dk != 128 || Dv != 128 || !(chunk == 0 || chunk == 64))
        return GDN_ERR_UNSUPPORTED;
    if (N == 0) return T == 0 ? GDN_OK : GDN_ERR_INVALID_ARGUMENT;
    void *ring = nullptr;
    const gdn_status st = ring_address(&ring);
    if (st != GDN_OK) return st;
    return gdn_prefill_ex(q, k, v, io_dtype, g, beta, initial_state, cu_seqlens, N, T, Hqk, Hv, Dk,
                          Dv, chunk, o, final_state, ring, kRingBytes, dev_error_flag, stream,
                          GDN_PREFILL_CLUSTER);
}
