// gdn_prefill_host: the prefill of one sequence whose inputs and outputs are in
// host memory, streamed through the device in segments so that the copies in,
// the kernels and the copies out overlap.
//
// The gated delta rule carries everything one part of a sequence passes to the
// next in its state (page "Qwen3.8-27B 架构深读…", section 三: the state is
// built up over chunks), so a sequence may be run as consecutive segments, each
// a gdn_prefill call that starts from the state the previous one left.  Here
// the segments run on the caller's stream, in place on one device state buffer,
// while a copy-in stream fetches segment i + 1's q, k, v, g, beta into the
// other half of a double buffer and a copy-out stream returns segment i - 1's o.
#include <cuda_runtime.h>

#include <cstdint>

#include "gdn.h"
#include "trace.cuh"

namespace {

constexpr int64_t kDefaultSegment = 16384;

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t io_bytes(gdn_dtype dt) { return dt == GDN_DTYPE_BF16 ? 2 : 4; }

// Offsets into the device scratch.  One segment buffer holds q, k, v, o, g and
// beta of `seg` tokens; there are two of them.
struct Layout {
    size_t state, ws, ws_bytes, buf[2];
    size_t q, k, v, o, g, beta;  // offsets within a segment buffer
    size_t total;
};

Layout layout(int64_t seg, int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk,
              gdn_dtype dt) {
    Layout L;
    const size_t e = io_bytes(dt);
    L.state = 0;
    L.ws = al256((size_t)Hv * Dv * Dk * 4);
    L.ws_bytes = gdn_prefill_workspace_bytes(1, seg, Hqk, Hv, Dk, Dv, chunk);
    L.q = 0;
    L.k = L.q + al256((size_t)seg * Hqk * Dk * e);
    L.v = L.k + al256((size_t)seg * Hqk * Dk * e);
    L.o = L.v + al256((size_t)seg * Hv * Dv * e);
    L.g = L.o + al256((size_t)seg * Hv * Dv * e);
    L.beta = L.g + al256((size_t)seg * Hv * 4);
    const size_t per_buf = L.beta + al256((size_t)seg * Hv * 4);
    L.buf[0] = al256(L.ws + L.ws_bytes);
    L.buf[1] = L.buf[0] + per_buf;
    L.total = L.buf[1] + per_buf;
    return L;
}

int64_t segment_of(int64_t T, int64_t segment_tokens) {
    const int64_t s = segment_tokens == 0 ? kDefaultSegment : segment_tokens;
    return T < s ? (T > 0 ? T : 1) : s;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Streams and events of one call, released on every return path.  Releasing
// them while work that uses them is still queued is allowed: CUDA frees them
// once that work is done.
struct Pipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in_ready[2] = {nullptr, nullptr},
                done[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
    ~Pipe() {
        cudaEvent_t evs[] = {start, end, in_ready[0], in_ready[1], done[0], done[1], freed[0], freed[1]};
        for (cudaEvent_t ev : evs)
            if (ev) cudaEventDestroy(ev);
        if (in) cudaStreamDestroy(in);
        if (out) cudaStreamDestroy(out);
    }
    cudaError_t create() {
        cudaError_t e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking);
        cudaEvent_t *evs[] = {&start, &end, &in_ready[0], &in_ready[1], &done[0], &done[1], &freed[0], &freed[1]};
        for (cudaEvent_t *ev : evs)
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        return e;
    }
};

#define GDN_TRY(x)                                     \
    do {                                               \
        if ((x) != cudaSuccess) return GDN_ERR_CUDA;   \
    } while (0)

}  // namespace

extern "C" {

size_t gdn_prefill_host_scratch_bytes(int64_t T, int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv,
                                      int32_t chunk, gdn_dtype io_dtype, int64_t segment_tokens) {
    if (T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0 || segment_tokens < 0)
        return 0;
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return 0;
    return layout(segment_of(T, segment_tokens), Hqk, Hv, Dk, Dv, chunk, io_dtype).total;
}

gdn_status gdn_prefill_host(const void *q, const void *k, const void *v, gdn_dtype io_dtype,
                            const float *g, const float *beta, const float *initial_state, int64_t T,
                            int32_t Hqk, int32_t Hv, int32_t Dk, int32_t Dv, int32_t chunk, void *o,
                            float *final_state, int64_t segment_tokens, void *scratch,
                            size_t scratch_bytes, int32_t *dev_error_flag, void *stream) {
    GDN_TRACE("gdn_prefill_host");
    if (io_dtype != GDN_DTYPE_BF16 && io_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARGUMENT;
    if (T < 0 || Hqk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0 || chunk < 0) return GDN_ERR_INVALID_ARGUMENT;
    if (Hv % Hqk != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (segment_tokens < 0 || segment_tokens % 64 != 0) return GDN_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_INVALID_ARGUMENT;
    if (!scratch || !aligned16(scratch) || (dev_error_flag && !aligned16(dev_error_flag)))
        return GDN_ERR_INVALID_ARGUMENT;
    const int64_t seg = segment_of(T, segment_tokens);
    const Layout L = layout(seg, Hqk, Hv, Dk, Dv, chunk, io_dtype);
    if (scratch_bytes < L.total) return GDN_ERR_INVALID_ARGUMENT;

    uint8_t *base = static_cast<uint8_t *>(scratch);
    float *state = reinterpret_cast<float *>(base + L.state);
    void *ws = L.ws_bytes ? base + L.ws : nullptr;
    const size_t e = io_bytes(io_dtype);
    const size_t state_bytes = (size_t)Hv * Dv * Dk * 4;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (T == 0) {  // the final state is the initial one (or zeros)
        if (!final_state) return GDN_OK;
        if (initial_state)
            GDN_TRY(cudaMemcpyAsync(state, initial_state, state_bytes, cudaMemcpyHostToDevice, s));
        else
            GDN_TRY(cudaMemsetAsync(state, 0, state_bytes, s));
        GDN_TRY(cudaMemcpyAsync(final_state, state, state_bytes, cudaMemcpyDeviceToHost, s));
        return GDN_OK;
    }

    Pipe P;
    GDN_TRY(P.create());
    GDN_TRY(cudaEventRecord(P.start, s));  // everything below comes after the caller's work
    GDN_TRY(cudaStreamWaitEvent(P.in, P.start, 0));
    GDN_TRY(cudaStreamWaitEvent(P.out, P.start, 0));
    if (initial_state)
        GDN_TRY(cudaMemcpyAsync(state, initial_state, state_bytes, cudaMemcpyHostToDevice, P.in));

    const int64_t nseg = (T + seg - 1) / seg;
    const auto bytes_at = [&](const void *h, int64_t t0, size_t per_token) {
        return static_cast<const uint8_t *>(h) + (size_t)t0 * per_token;
    };
    // segment i's inputs -> buffer i & 1, after segment i - 2's o has left it
    const auto copy_in = [&](int64_t i) -> cudaError_t {
        const int b = (int)(i & 1);
        const int64_t t0 = i * seg, n = (T - t0 < seg ? T - t0 : seg);
        uint8_t *B = base + L.buf[b];
        cudaError_t r = cudaSuccess;
        if (i >= 2) r = cudaStreamWaitEvent(P.in, P.freed[b], 0);
        const size_t pq = (size_t)Hqk * Dk * e, pv = (size_t)Hv * Dv * e, pg = (size_t)Hv * 4;
        if (r == cudaSuccess) r = cudaMemcpyAsync(B + L.q, bytes_at(q, t0, pq), n * pq, cudaMemcpyHostToDevice, P.in);
        if (r == cudaSuccess) r = cudaMemcpyAsync(B + L.k, bytes_at(k, t0, pq), n * pq, cudaMemcpyHostToDevice, P.in);
        if (r == cudaSuccess) r = cudaMemcpyAsync(B + L.v, bytes_at(v, t0, pv), n * pv, cudaMemcpyHostToDevice, P.in);
        if (r == cudaSuccess) r = cudaMemcpyAsync(B + L.g, bytes_at(g, t0, pg), n * pg, cudaMemcpyHostToDevice, P.in);
        if (r == cudaSuccess)
            r = cudaMemcpyAsync(B + L.beta, bytes_at(beta, t0, pg), n * pg, cudaMemcpyHostToDevice, P.in);
        if (r == cudaSuccess) r = cudaEventRecord(P.in_ready[b], P.in);
        return r;
    };
    // segment i on the caller's stream, in place on the device state
    const auto compute = [&](int64_t i) -> gdn_status {
        const int b = (int)(i & 1);
        const int64_t t0 = i * seg, n = (T - t0 < seg ? T - t0 : seg);
        uint8_t *B = base + L.buf[b];
        if (cudaStreamWaitEvent(s, P.in_ready[b], 0) != cudaSuccess) return GDN_ERR_CUDA;
        const float *s0 = (i == 0 && !initial_state) ? nullptr : state;
        const gdn_status st = gdn_prefill(B + L.q, B + L.k, B + L.v, io_dtype,
                                          reinterpret_cast<const float *>(B + L.g),
                                          reinterpret_cast<const float *>(B + L.beta), s0, nullptr, 1,
                                          n, Hqk, Hv, Dk, Dv, chunk, B + L.o, state, ws, L.ws_bytes,
                                          dev_error_flag, s);
        if (st != GDN_OK) return st;
        return cudaEventRecord(P.done[b], s) == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
    };
    // segment i's o -> host
    const auto copy_out = [&](int64_t i) -> cudaError_t {
        const int b = (int)(i & 1);
        const int64_t t0 = i * seg, n = (T - t0 < seg ? T - t0 : seg);
        const size_t po = (size_t)Hv * Dv * e;
        cudaError_t r = cudaStreamWaitEvent(P.out, P.done[b], 0);
        if (r == cudaSuccess)
            r = cudaMemcpyAsync(static_cast<uint8_t *>(o) + (size_t)t0 * po, base + L.buf[b] + L.o,
                                n * po, cudaMemcpyDeviceToHost, P.out);
        if (r == cudaSuccess) r = cudaEventRecord(P.freed[b], P.out);
        return r;
    };

    // Issue order: segment i + 1's copy-in and kernel before segment i's
    // copy-out, so that a copy to pageable host memory, which returns only
    // when it is done, never holds back the next segment's work.
    GDN_TRY(copy_in(0));
    gdn_status st = compute(0);
    if (st != GDN_OK) return st;
    for (int64_t i = 0; i < nseg; ++i) {
        if (i + 1 < nseg) {
            GDN_TRY(copy_in(i + 1));
            st = compute(i + 1);
            if (st != GDN_OK) return st;
        }
        GDN_TRY(copy_out(i));
    }
    if (final_state) {
        GDN_TRY(cudaStreamWaitEvent(P.out, P.done[(nseg - 1) & 1], 0));
        GDN_TRY(cudaMemcpyAsync(final_state, state, state_bytes, cudaMemcpyDeviceToHost, P.out));
    }
    GDN_TRY(cudaEventRecord(P.end, P.out));
    GDN_TRY(cudaStreamWaitEvent(s, P.end, 0));  // the caller's stream sees the whole call
    return GDN_OK;
}

}  // extern "C"
