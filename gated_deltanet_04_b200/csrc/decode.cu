// One-token decode update of the gated delta rule, in place on the state.
//
// Section 三 of "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与 262K
// 长上下文": at inference every step does one fixed-size matrix update.  Per
// (sequence n, v-head h) with a = exp(g), b = beta and row i of the state:
//     r_i   = (a S_i) . k                 (recall from the decayed state; with
//                                          GDN_ORDER_RECALL_FIRST: S_i . k)
//     u_i   = b (v_i - r_i)
//     S_i'  = a S_i + u_i k^T             (delta write)
//     o_i   = S_i' . q = a (S_i . q) + u_i (k . q)
// The state is streamed exactly once: every row is loaded, reduced against k
// and q, rewritten and stored by the same lanes, so the kernel is bound by
// HBM bandwidth on 2 * Dv * Dk * sizeof(state) bytes per (n, h).
//
// Two kernels:
//  * Dk = Dv = 128 (the workload shape): a persistent kernel that streams each
//    head state through shared-memory stages with bulk TMA copies (loads of
//    the next units overlap the update of the current one; the updated state
//    leaves by a bulk store).  Threads only read and write shared memory.
//    Each CTA takes a contiguous range of (n, h) units, so every SM streams
//    one contiguous stretch of the states, and the units % grid left over are
//    split into single rows across all CTAs.  The 8 dot products of 4 rows
//    (S.k and S.q) are summed over a warp in 9 shuffles.  Templated on the
//    state type (fp32, or bfloat16 storage computed in fp32) and on pool
//    decode (slot indices and reset flags); StagedCfg gives each state type
//    its pipeline.
//  * other head sizes: the direct kernel below (fp32 state).
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
    const float rdec = a.order == GDN_ORDER_RECALL_FIRST ? 1.f : dec;  // decay of the recall
    const float b = a.beta[(int64_t)n * a.Hv + h];

    const int64_t slot = decode_state_slot(a, n);
    if (slot < 0) {  // a bad slot index: this unit writes nothing
        if (threadIdx.x == 0) raise_error(a.err, GDN_ERR_BAD_SLOT);
        return;
    }
    const bool zero = decode_state_reset(a, n);  // a new request: start from S = 0
    float *st = static_cast<float *>(a.state) + (slot * a.Hv + h) * a.Dv * DK;
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
                row[r] = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                              : __ldcs(reinterpret_cast<const float4 *>(st + (int64_t)i * DK) + l);
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
                const float u = b * (vi[r] - rdec * sk);
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

constexpr uint32_t kStUnitElems = 128 * 128;    // one (n, h) state
constexpr long long kStWaitLimit = 1ll << 31;   // SM clocks (about a second)

// State storage: fp32, or bfloat16 (computed in fp32, rounded to nearest even
// when stored).  A bfloat16 state is half the bytes, so twice as many stages
// fit in the same shared memory.
template <class StateT>
struct StagedCfg;
// kStages: states in shared memory.  kWarps: warps per CTA, 128 / kWarps state
// rows each.  kLateRefill: a stage is refilled one unit after its bulk store
// was issued (its read is done by then, so the issuing thread never waits),
// instead of right after the store has read it.  kIoInStage: a unit's k, q and
// v rows come with its stage (bulk copies on the stage's mbarrier) instead of
// per-thread loads one unit ahead.  kCtasPerSm: resident CTAs per SM.  Measured
// on B200 (48-layer step): the fp32 state is bandwidth-bound with 3 stages and
// prefers the register path (12.8 vs 13.5 ms); a bfloat16 state moves half the
// bytes and needs the never-waiting pipeline (7.4 ms; 10.0 ms with the fp32
// choices), and runs best as two 8-warp CTAs per SM whose per-unit barriers
// do not hold each other up (7.2 ms).
template <>
struct StagedCfg<float> {
    static constexpr int kStages = 3, kWarps = 16, kLateRefill = 0, kIoInStage = 0, kCtasPerSm = 1;
};
template <>
struct StagedCfg<__nv_bfloat16> {
    static constexpr int kCtasPerSm = 2;
    static constexpr int kStages = 6 / kCtasPerSm, kWarps = 16 / kCtasPerSm, kLateRefill = 1,
                         kIoInStage = 1;
};

constexpr int kSlotCache = 128;  // sequences whose slot / reset a CTA keeps in shared memory

template <class StateT>
struct StagedSmem {
    static constexpr int kStages = StagedCfg<StateT>::kStages;
    StateT state[kStages][kStUnitElems];
    uint8_t io[kStages][3][512];  // the unit's k, q and v rows (io dtype), loaded with its state
    float o[2][128];
    uint64_t full[kStages];
    int32_t slot_c[kSlotCache];   // pool decode: slots (-1: bad) of this CTA's sequences
    int32_t reset_c[kSlotCache];
};
template <class StateT>
constexpr size_t staged_smem_bytes() {
    return sizeof(StagedSmem<StateT>) + 128;
}
static_assert(staged_smem_bytes<float>() * StagedCfg<float>::kCtasPerSm <= 232448 &&
                  staged_smem_bytes<__nv_bfloat16>() * StagedCfg<__nv_bfloat16>::kCtasPerSm <= 232448,
              "stages fit the shared memory of an SM");

// Four consecutive state elements of a row, as fp32 (a lane's share of a row).
__device__ __forceinline__ float4 ld_state4(const float *p) {
    return *reinterpret_cast<const float4 *>(p);
}
__device__ __forceinline__ float4 ld_state4(const __nv_bfloat16 *p) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ void st_state4(float *p, float4 w) {
    *reinterpret_cast<float4 *>(p) = w;
}
__device__ __forceinline__ void st_state4(__nv_bfloat16 *p, float4 w) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(w.x, w.y);  // round to nearest even
    const __nv_bfloat162 hi = __floats2bfloat162_rn(w.z, w.w);
    uint2 raw;
    raw.x = *reinterpret_cast<const uint32_t *>(&lo);
    raw.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = raw;
}

// Sums, over the 32 lanes of a warp, the 8 per-lane partial values sk[0..3],
// sq[0..3] (dot products of 4 state rows with k and with q) in 9 shuffles
// instead of 8 x 5: each exchange level sends half of the values a lane still
// holds and keeps the other half (recursive halving).  After the three halving
// levels lane L holds 8-lane partial sums of one value -- S.k (L < 16) or S.q
// (L >= 16) of row (L >> 2) & 3 -- and two plain butterfly levels complete it.
__device__ __forceinline__ float reduce8_transposed(const float (&sk)[4], const float (&sq)[4],
                                                    int lane) {
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    float h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // lanes < 16 keep the S.k partials, the others S.q
        const float send = b4 ? sk[i] : sq[i];
        const float keep = b4 ? sq[i] : sk[i];
        h[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    float h2[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {  // bit 3 of the lane: rows 0, 1 or rows 2, 3
        const float send = b3 ? h[i] : h[i + 2];
        const float keep = b3 ? h[i + 2] : h[i];
        h2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b2 ? h2[0] : h2[1];  // bit 2: the even or the odd row of the pair
    float t = (b2 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    return t;
}

// Per-thread inputs of one unit (the register path): k, q as 4 values of a
// lane, gates, and v of row R*warp + lane on lanes 0 .. R-1.
struct UnitInputs {
    float4 k, q;
    float g, b, v;
};

template <int R>
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
    in.v = lane < R ? load_io(a.v, (int64_t)u * 128 + R * warp + lane, a.dtype) : 0.f;
    return in;
}

// kSlots: pool decode (slot indices, reset flags); a separate instantiation
// so the plain kernels carry none of its code.
template <class StateT, bool kSlots>
__global__ void __launch_bounds__(StagedCfg<StateT>::kWarps * 32, StagedCfg<StateT>::kCtasPerSm)
    gdn_decode_staged_kernel(DecodeArgs a, int units) {
    using namespace sm100;
    constexpr int kStStages = StagedCfg<StateT>::kStages;
    constexpr int kStThreads = StagedCfg<StateT>::kWarps * 32;
    constexpr int R = 128 / StagedCfg<StateT>::kWarps;  // state rows per warp
    constexpr bool kLate = StagedCfg<StateT>::kLateRefill != 0;
    constexpr bool kIo = StagedCfg<StateT>::kIoInStage != 0;
    constexpr uint32_t kStUnitBytes = kStUnitElems * sizeof(StateT);
    extern __shared__ uint8_t smem_raw[];
    StagedSmem<StateT> &sm = *reinterpret_cast<StagedSmem<StateT> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    StateT *state = static_cast<StateT *>(a.state);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int per = units / (int)gridDim.x, extra = units % (int)gridDim.x;
    const int b = blockIdx.x;
    const int first = b * per, stride = 1;
    const int count = per;  // units of this CTA: a contiguous range (grid <= units, so >= 1)
    if (count <= 0) return;

    // Pool decode: the slot and reset flag of every sequence this CTA's units
    // belong to, read once into shared memory (from global memory when there
    // are more than kSlotCache of them).  Slot -1 marks an index out of range.
    const int n_lo = first / a.Hv, n_span = (first + count - 1) / a.Hv - n_lo + 1;
    const bool cached = kSlots && n_span <= kSlotCache;
    if (cached)
        for (int i = tid; i < n_span; i += kStThreads) {
            sm.slot_c[i] = (int32_t)decode_state_slot(a, n_lo + i);
            sm.reset_c[i] = decode_state_reset(a, n_lo + i) ? 1 : 0;
        }
    // (the leftover rows below belong to sequences outside that range)
    auto in_cache = [&](int n) { return cached && n >= n_lo && n - n_lo < n_span; };
    auto slot_of = [&](int n) -> int64_t {
        if constexpr (!kSlots) return n;
        else return in_cache(n) ? sm.slot_c[n - n_lo] : decode_state_slot(a, n);
    };
    auto reset_of = [&](int n) -> bool {
        if constexpr (!kSlots) return false;
        else return a.reset != nullptr && (in_cache(n) ? sm.reset_c[n - n_lo] != 0 : decode_state_reset(a, n));
    };
    // where unit u's state lives (-1: a bad slot, nothing is read or written)
    auto state_off = [&](int u) -> int64_t {
        if constexpr (!kSlots) {
            return (int64_t)u * kStUnitElems;
        } else {
            const int64_t sl = slot_of(u / a.Hv);
            return sl < 0 ? -1 : (sl * a.Hv + u % a.Hv) * (int64_t)kStUnitElems;
        }
    };

    if (tid == 0) {
        for (int s = 0; s < kStStages; ++s) mbar_init(&sm.full[s], 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    // A stage holds one unit: its state (and with kIo its k, q and v rows),
    // bulk copies that complete one mbarrier (thread 0 issues them).  A unit
    // with a bad slot, or that starts from zeros, loads no state.
    const uint32_t esz = a.dtype == GDN_DTYPE_BF16 ? 2u : 4u, row_bytes = 128u * esz;
    auto issue_stage = [&](int stg, int u) {
        const int64_t off = state_off(u);
        const bool load_state = off >= 0 && !reset_of(u / a.Hv);
        if (!load_state && !kIo) {
            mbar_arrive(&sm.full[stg]);
            return;
        }
        mbar_arrive_expect_tx(&sm.full[stg],
                              (load_state ? kStUnitBytes : 0u) + (kIo ? 3u * row_bytes : 0u));
        if (load_state) bulk_load(sm.state[stg], state + off, kStUnitBytes, &sm.full[stg]);
        if constexpr (kIo) {
            const int h = u % a.Hv, n = u / a.Hv;
            const int64_t qk = ((int64_t)n * a.Hqk + h / (a.Hv / a.Hqk)) * 128;
            const uint8_t *kp = static_cast<const uint8_t *>(a.k), *qp = static_cast<const uint8_t *>(a.q);
            bulk_load(sm.io[stg][0], kp + qk * esz, row_bytes, &sm.full[stg]);
            bulk_load(sm.io[stg][1], qp + qk * esz, row_bytes, &sm.full[stg]);
            bulk_load(sm.io[stg][2], static_cast<const uint8_t *>(a.v) + (int64_t)u * 128 * esz,
                      row_bytes, &sm.full[stg]);
        }
    };
    int issued = 0;  // units whose stage load has been issued (thread 0's view)
    if (tid == 0)
        for (; issued < count && issued < kStStages; ++issued) issue_stage(issued, first + issued * stride);
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
        const int64_t off = state_off(u);
        if (off < 0) {  // a bad slot index: this unit writes nothing
            if (lane == 0) raise_error(a.err, GDN_ERR_BAD_SLOT);
            continue;
        }
        StateT *srow = state + off + i * 128 + 4 * lane;
        const float4 row = reset_of(n) ? make_float4(0.f, 0.f, 0.f, 0.f) : ld_state4(srow);
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
        const float uu = bb * (vi - (a.order == GDN_ORDER_RECALL_FIRST ? 1.f : dec) * sk);
        float4 w;
        w.x = fmaf(uu, k4.x, dec * row.x);
        w.y = fmaf(uu, k4.y, dec * row.y);
        w.z = fmaf(uu, k4.z, dec * row.z);
        w.w = fmaf(uu, k4.w, dec * row.w);
        st_state4(srow, w);
        if (lane == 0) store_io(a.o, (int64_t)u * 128 + i, fmaf(uu, kq, dec * sq), a.dtype);
    }
    // kIo: gates two units ahead in registers, the rest comes with the stage;
    // otherwise all of a unit's inputs one unit ahead in registers
    float g1 = 0.f, b1 = 0.f, g2 = 0.f, b2 = 0.f;
    UnitInputs nxt{};
    if constexpr (kIo) {
        g1 = a.g[first];
        b1 = a.beta[first];
        if (count > 1) {
            g2 = a.g[first + 1];
            b2 = a.beta[first + 1];
        }
    } else {
        nxt = load_unit_inputs<R>(a, first, warp, lane);
    }
    bool timed_out = false;
    int li = 0;
#pragma unroll 1
    for (; li < count; ++li) {
        const int u = first + li * stride;
        const int s = li % kStStages;
        float gcur, bcur;
        UnitInputs cur{};
        if constexpr (kIo) {
            gcur = g1;
            bcur = b1;
            g1 = g2;
            b1 = b2;
            if (li + 2 < count) {
                g2 = a.g[u + 2 * stride];
                b2 = a.beta[u + 2 * stride];
            }
        } else {
            cur = nxt;
            if (li + 1 < count) nxt = load_unit_inputs<R>(a, u + stride, warp, lane);
            gcur = cur.g;
            bcur = cur.b;
        }
        if (!mbar_wait_bounded(&sm.full[s], (li / kStStages) & 1, kStWaitLimit)) timed_out = true;

        const float dec = expf(gcur);
        const float rdec = a.order == GDN_ORDER_RECALL_FIRST ? 1.f : dec;  // decay of the recall
        // pool decode: a bad slot computes on a stale stage and stores nothing;
        // a reset unit starts from zeros (its stage was not loaded)
        const int64_t uoff = state_off(u);
        const bool bad = uoff < 0, zero = !bad && reset_of(u / a.Hv);
        const float4 kv = kIo ? load_vec4(sm.io[s][0], 4 * lane, a.dtype) : cur.k;
        const float4 qv = kIo ? load_vec4(sm.io[s][1], 4 * lane, a.dtype) : cur.q;
        float kq = kv.x * qv.x + kv.y * qv.y + kv.z * qv.z + kv.w * qv.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        StateT *st = sm.state[s];
#pragma unroll
        for (int r0 = 0; r0 < R; r0 += 4) {
            float4 row[4];
            float sk[4], sq[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                row[r] = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                              : ld_state4(st + (R * warp + r0 + r) * 128 + 4 * lane);
                sk[r] = row[r].x * kv.x + row[r].y * kv.y + row[r].z * kv.z + row[r].w * kv.w;
                sq[r] = row[r].x * qv.x + row[r].y * qv.y + row[r].z * qv.z + row[r].w * qv.w;
            }
            // the 8 dot products of these 4 rows, summed over the warp at once:
            // lane L ends with the full S.k (L < 16) or S.q (L >= 16) of row
            // rr = (L >> 2) & 3
            const int rr = (lane >> 2) & 3;
            const float t = reduce8_transposed(sk, sq, lane);
            // u of row rr on lanes 0..15, then to every lane
            const float vi = kIo ? load_io(sm.io[s][2], R * warp + r0 + rr, a.dtype)
                                 : __shfl_sync(0xffffffffu, cur.v, r0 + rr);
            const float u = bcur * (vi - rdec * t);
            float uu[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) uu[r] = __shfl_sync(0xffffffffu, u, 4 * r);
            const float u_o = __shfl_xor_sync(0xffffffffu, u, 16);  // lanes >= 16: u of row rr
            if (lane >= 16 && (lane & 3) == 0)
                sm.o[li & 1][R * warp + r0 + rr] = fmaf(u_o, kq, dec * t);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int i = R * warp + r0 + r;
                float4 w;
                w.x = fmaf(uu[r], kv.x, dec * row[r].x);
                w.y = fmaf(uu[r], kv.y, dec * row[r].y);
                w.z = fmaf(uu[r], kv.z, dec * row[r].z);
                w.w = fmaf(uu[r], kv.w, dec * row[r].w);
                st_state4(st + i * 128 + 4 * lane, w);
            }
        }
        fence_proxy_async_smem();  // updated state -> visible to the bulk store
        if (__syncthreads_or(timed_out ? 1 : 0)) {
            if (tid == 0) raise_error(a.err, GDN_ERR_TIMEOUT);
            break;
        }
        if (tid < 128 && !bad) store_io(a.o, (int64_t)u * 128 + tid, sm.o[li & 1][tid], a.dtype);
        if (tid == 0) {
            if (bad) raise_error(a.err, GDN_ERR_BAD_SLOT);
            else bulk_store(state + uoff, st, kStUnitBytes);
            bulk_commit();  // one group per unit (empty for a bad slot)
            if constexpr (kLate) {
                // refill the previous unit's stage: its store was issued a unit ago
                if (li >= 1 && issued < count) {
                    bulk_wait_read_all_but_one();
                    issue_stage((li + kStStages - 1) % kStStages, first + issued * stride);
                    ++issued;
                }
            } else if (issued < count) {  // refill this stage with the unit kStStages ahead
                bulk_wait_read_all();
                issue_stage(s, first + issued * stride);
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

template <class StateT, bool kSlots>
cudaError_t launch_staged(const DecodeArgs &a, int units, cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(gdn_decode_staged_kernel<StateT, kSlots>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)staged_smem_bytes<StateT>());
    if (e != cudaSuccess) return e;
    const int ctas = sms * StagedCfg<StateT>::kCtasPerSm;
    const int grid = units < ctas ? units : ctas;
    gdn_decode_staged_kernel<StateT, kSlots>
        <<<grid, StagedCfg<StateT>::kWarps * 32, staged_smem_bytes<StateT>(), s>>>(a, units);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    const int units = a.N * a.Hv;
    if (a.state_bf16) {  // bfloat16 state storage: the staged kernel only
        if (a.Dk != 128 || a.Dv != 128) return cudaErrorInvalidValue;
        return launch_staged<__nv_bfloat16, false>(a, units, s);
    }
    if (a.Dk == 128 && a.Dv == 128)
        return a.slot ? launch_staged<float, true>(a, units, s) : launch_staged<float, false>(a, units, s);
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
