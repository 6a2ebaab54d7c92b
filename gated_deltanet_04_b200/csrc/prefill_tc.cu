// Chunk-parallel prefill of the gated delta rule on sm_100a tensor cores.
//
// Rule (page "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与 262K 长上下文",
// section 三): S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T, o_t = S_t q_t,
// with training/prefill accumulating the state chunk by chunk.  Derivation of
// the chunk step used here (from the recurrence; chunk of C = 64 tokens,
// entering state S (Dv x Dk), gamma = cumsum(g) within the chunk,
// Gamma = exp(gamma), M_ri = exp(gamma_r - gamma_i) for i <= r):
//     A   = strictly-lower part of diag(b) (K K^T (.) M),   T = (I + A)^-1
//     U~  = T diag(b) V,             W = T diag(b Gamma) K
//     U   = U~ - W S^T                                (delta-rule residuals)
//     O   = diag(Gamma) Q S^T + (Q K^T (.) M) U
//     S'  = Gamma_C S + U^T diag(Gamma_C / Gamma) K
//
// Kernel design (one CTA of 8 warps per (sequence, v-head)).  TMEM lane i is
// state row i (or chunk row i); warps w and w + 4 share lane quadrant w % 4
// and split the columns of every accumulator between them.
//   * The fp32 state S lives in tensor memory as an MMA accumulator for the
//     whole sequence (no HBM round trip between chunks).  Its fp16 hi/lo
//     copies in shared memory are the A operand of the state-side products.
//   * Every product is a tcgen05.mma (M = 128, fp16 operands, fp32
//     accumulation) whose result rows are state rows or chunk rows:
//       Gram   [K;Q] K^T            -> K K^T (lanes 0-63), Q K^T (lanes 64-127)
//       U~^T = V^T (T diag b)^T      (T split into fp16 hi + lo: 2 passes)
//       W^T  = K^T (T diag(b Gamma))^T
//       S Q^T, R = S W^T             (state times chunk queries / W)
//       S   += [U'hi | U'lo] [K ; K] (U' = U diag(Gamma_C/Gamma), split)
//       O   += U^T P^T               (P = Q K^T (.) M, onto diag(Gamma) S Q^T)
//     q/k/v tiles arrive by TMA (128-byte swizzle, no multicast) and are
//     converted in place from bf16 to fp16 (exact for |x| in [6e-5, 6.5e4]).
//   * Precision: fp16 operands keep 11 significant bits.  T diag(b) and U'
//     always get a second (low-part) pass.  W and S W^T get extra passes
//     (W: 2, S W^T: 3 = hi.hi + hi.lo + lo.hi) only in chunks whose total
//     decay Gamma_C is at least 0.2: a chunk's rounding error is carried into
//     later chunks scaled by their decay, so it only accumulates when decay
//     is weak; with the threshold the fp32 state stays within 4e-5 of fp64
//     in every regime from no decay (a = 1) to the strong decay of the
//     benchmark workloads (emulated, and checked by the GPU tests).
//   * The decay factors exp(gamma_r - gamma_i) are formed as
//     Gamma_r * exp(-gamma_i) when |gamma| <= 60 over the chunk (no overflow),
//     else elementwise.
//   * T = (I + A)^-1 is solved on CUDA cores in fp32 by 16 x 16 blocks.
//   * Rows past the end of a sequence inside the last chunk are zeroed and
//     get b = g = 0, which makes them contribute nothing.
// The phases of a chunk run in order, separated by MMA commits; every wait
// on an mbarrier is bounded and reports GDN_ERR_TIMEOUT instead of hanging.
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

#ifdef GDN_TC_PHASES
// Per-phase SM clocks of thread 0 of CTA 0, accumulated in shared memory (a
// global read-modify-write per marker would stall thread 0 and distort the
// phases) and added to the global totals once, at the end.
__device__ unsigned long long gdn_tc_phase_clk[16];
static __shared__ unsigned int gdn_tc_acc_[16];
#define GDN_TC_PHASE(k)                                             \
    do {                                                            \
        if (threadIdx.x == 0 && blockIdx.x == 0) {                  \
            const long long now_ = clock64();                       \
            gdn_tc_acc_[(k)] += (unsigned int)(now_ - phase_t_);    \
            phase_t_ = now_;                                        \
        }                                                           \
    } while (0)
#define GDN_TC_PHASE_FLUSH()                                        \
    do {                                                            \
        if (threadIdx.x == 0 && blockIdx.x == 0)                    \
            for (int i_ = 0; i_ < 16; ++i_)                         \
                atomicAdd(&gdn_tc_phase_clk[i_], (unsigned long long)gdn_tc_acc_[i_]); \
    } while (0)
#else
#define GDN_TC_PHASE(k) ((void)0)
#define GDN_TC_PHASE_FLUSH() ((void)0)
#endif

namespace gdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kThreads = 256;

// ---- shared memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t OFF_KQ = 0;          // 2 halves x [K 64 rows | Q 64 rows] x 128 B
constexpr uint32_t OFF_V = 32768;       // 2 halves x 64 rows x 128 B
constexpr uint32_t OFF_S16H = 49152;    // 2 K-halves x 128 rows x 128 B   (A: S fp16 hi)
constexpr uint32_t OFF_S16L = 81920;    //                                  (A: S fp16 lo)
// One 48 KB region holds, in turn within a chunk: the triangular-solve
// scratch, then W^T (hi, lo), then U' (hi, lo) and U^T.  Each use starts
// only after the MMAs reading the previous one have completed.
constexpr uint32_t OFF_X = 114688;
constexpr uint32_t OFF_UP = OFF_X;            // hi, lo x 128 rows x 128 B  (A: U')
constexpr uint32_t OFF_U16 = OFF_X + 32768;   // 128 rows x 128 B           (A: U^T)
constexpr uint32_t OFF_WST = OFF_X;           // hi, lo x 128 rows(d) x 128 B (B: W^T, MN-major)
constexpr uint32_t OFF_AS = OFF_X;                   // float [64][kAS4]
constexpr uint32_t OFF_TS = OFF_X + 64 * kAS4 * 4;      // float [64][kTS], 16-byte aligned
constexpr uint32_t OFF_XS = OFF_TS + 64 * kTS * 4;   // float [1024] level partials
constexpr uint32_t OFF_P16 = 163840;    // 64 rows x 128 B                  (B: P, K-major)
// T diag(b) as bf16 hi / mid / lo and T diag(b Gamma) as fp16 hi / lo, each part
// 64 rows x 128 B; the parts of each are consecutive, so one B operand of
// N = 192 (or 128) rows takes all of them, each part's product landing in
// its own accumulator columns.
constexpr uint32_t OFF_TBH = 172032;    // (B: T diag b, hi)
constexpr uint32_t OFF_TBM = 180224;    // (B: T diag b, mid)
constexpr uint32_t OFF_TBL = 188416;    // (B: T diag b, lo)
constexpr uint32_t OFF_TGH = 196608;    // (B: T diag(b Gamma), hi)
constexpr uint32_t OFF_TGL = 204800;    // (B: T diag(b Gamma), lo)
constexpr uint32_t OFF_OST = OFF_TBH;   // o staging [64 tokens][128] bf16 (TB tiles are dead)
constexpr uint32_t OFF_MISC = 212992;
static_assert(OFF_XS + 1024 * 4 <= OFF_P16, "solve scratch overflows");
static_assert(OFF_TS % 16 == 0 && OFF_XS % 16 == 0, "float4 scratch must be aligned");

struct Misc {
    float gam[kC];    // cumulative log-decay within the chunk
    float Gam[kC];    // exp(gam)
    float iGam[kC];   // exp(-gam) (only when the chunk is "safe")
    float eC[kC];     // exp(gam_C - gam_r)
    float bb[kC];     // beta (0 for padding rows)
    float bG[kC];     // beta * Gamma
    uint64_t tma_bar;
    uint64_t mma_bar;
    uint32_t tmem_base;
    int32_t safe;     // |gamma| <= 60 over the chunk
    int32_t hp;       // Gamma_C >= kHighPrecisionDecay
    float gsum_next;  // sum of g over the next (or first) chunk
    alignas(16) uint32_t vote[2][8];  // per-warp vote words of the U and state epilogues
    float red[8];                     // per-warp maxima of a rescale
};
static_assert(offsetof(Misc, vote) % 16 == 0 && OFF_MISC % 16 == 0, "vote words read as uint4");
constexpr uint32_t kSmemBytes = OFF_MISC + sizeof(Misc) + 1024;  // + alignment slack

// TMEM column map (fp32 columns; 512 allocated), each region used in turn:
//   TM_S 0..127    the fp32 state
//   TM_G 128..191  the Gram; then TM_U 128..319, U~^T as the products of T diag(b)'s
//                  hi, mid and lo parts (64 columns each)
//   TM_O 320..383  S Q^T, then the chunk output
//   TM_WT 384..511 W^T as the products of T diag(b Gamma)'s hi and lo parts; then
//   TM_R 384..447  S W^T; then TM_D 384..511, the state increment dS
constexpr uint32_t TM_S = 0, TM_G = 128, TM_U = 128, TM_O = 320, TM_WT = 384, TM_R = 384,
                   TM_D = 384;
constexpr uint32_t IDESC_MK_N192_BF16 = make_idesc_f16(128, 192, 1, 0, 1);
constexpr uint32_t IDESC_MK_N128 = make_idesc_f16(128, 128, 1, 0);


struct TcParams {
    const float *g, *beta, *s0;
    const int32_t *cu;
    void *o;
    float *sT;
    int32_t *err;
    int64_t T;
    int32_t N, Hqk, Hv;
    int32_t recall_first;  // GDN_ORDER_RECALL_FIRST: recall before the decay
};

// Sum over warp 0 of one value per lane (each lane holding the sum of its
// two gates); lane 0 writes it to *dst.
__device__ __forceinline__ void warp0_sum_to(float x, float *dst) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (threadIdx.x == 0) *dst = x;
}

__global__ void __launch_bounds__(kThreads, 1)
    gdn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    Misc *ms = reinterpret_cast<Misc *>(sm + OFF_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int quad = warp & 3;          // TMEM lane quadrant
    const int half = warp >> 2;         // which half of the columns this warp handles
    const int row = quad * 32 + lane;   // TMEM lane = accumulator row
#ifdef GDN_TC_PHASES
    long long phase_t_ = clock64();
    if (threadIdx.x == 0)
        for (int i_ = 0; i_ < 16; ++i_) gdn_tc_acc_[i_] = 0u;
#endif

    const int unit = blockIdx.x;  // n * Hv + h
    const int h = unit % p.Hv;
    const int n = unit / p.Hv;
    const int j = h / (p.Hv / p.Hqk);

    int64_t t_begin, t_end;
    if (!seq_range(p.cu, n, p.N, p.T, p.err, t_begin, t_end)) return;  // uniform

    if (tid == 0) {
        mbar_init(&ms->tma_bar, 1);
        mbar_init(&ms->mma_bar, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(&ms->tmem_base, 512);
        tmem_relinquish();
    }
    // gates of the first chunk (warp 0: lane l holds tokens 2l, 2l+1), and its total decay
    float gpre0 = 0.f, gpre1 = 0.f, bpre0 = 0.f, bpre1 = 0.f;
    auto load_gates = [&](int64_t tok0) {
        gpre0 = gpre1 = bpre0 = bpre1 = 0.f;
        const int64_t t0_ = tok0 + 2 * lane, t1_ = t0_ + 1;
        if (t0_ < t_end) { gpre0 = p.g[t0_ * p.Hv + h]; bpre0 = p.beta[t0_ * p.Hv + h]; }
        if (t1_ < t_end) { gpre1 = p.g[t1_ * p.Hv + h]; bpre1 = p.beta[t1_ * p.Hv + h]; }
    };
    if (warp == 0) {
        load_gates(t_begin);
        warp0_sum_to(gpre0 + gpre1, &ms->gsum_next);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);  // + column

    // Value-side operands are held with a power-of-two scale, uniform over
    // the unit: the fp32 master state in TMEM is S * 2^-es (times the next
    // chunk's Gamma_C, applied ahead), and its fp16 hi / lo copies (the A
    // operand of S Q^T and S W^T) are split from S * 2^-es directly, so the
    // products come out scaled by 2^-es.  U and U' are held as U * 2^-eu,
    // where eu is es unless U's magnitudes leave the band [kScaleLo, kScaleHi)
    // in that scale.  Both epilogues vote on their largest scaled magnitude;
    // the rare chunk whose values left the band recomputes them in fp32 and
    // takes a new scale (fp16_scale_exp).  The scaling is exact, so no
    // value-side operand over- or underflows fp16, whatever the scale of v
    // and S0, and the results scale exactly with it.
    int es = 0, eu = 0;
    float s_up = 1.f, sd = 1.f;  // 2^es, 2^-es
    auto set_es = [&](int e) {
        es = e;
        s_up = exp2i(e);
        sd = exp2i(-e);
    };
    // this thread's 64 scaled values of a state row -> the fp16 hi (and lo) tiles
    auto split_state = [&](const float (&sv)[64], bool with_lo) {
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = sv[32 * part + x];
            store_split32(sm + OFF_S16H + half * 16384, sm + OFF_S16L + half * 16384, row,
                          32 * part, v, with_lo);
        }
    };

    // ---- initial state: Gamma_C(first chunk) * S -> TMEM accumulator; S -> fp16 hi/lo ----
    {
        const float scale0 = t_begin < t_end ? expf(ms->gsum_next) : 1.f;
        const float *src = p.s0 ? p.s0 + (((int64_t)n * p.Hv + h) * kD + row) * kD + 64 * half
                                : nullptr;
        float sv[64];
        float am = 0.f;
#pragma unroll
        for (int x = 0; x < 64; x += 4) {
            const float4 f = src ? *reinterpret_cast<const float4 *>(src + x)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            sv[x] = f.x; sv[x + 1] = f.y; sv[x + 2] = f.z; sv[x + 3] = f.w;
            am = fmaxf(am, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
        }
        am = cta_max(am, ms->red, warp, lane);
        set_es(am > 0.f ? fp16_scale_exp(am) : 0);
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] *= sd;
        split_state(sv, true);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = sv[32 * part + x] * scale0;
            tmem_st32(trow + TM_S + 64 * half + 32 * part, v);
        }
    }
    fence_proxy_async_smem();
    tmem_wait_st();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    uint32_t tma_phase = 0, mma_phase = 0;
    bool aborted = false;
    float kmax = 0.f;             // largest key-side value this thread has put into fp16
    bool range_reported = false;
    bool timed_out = false;  // this thread saw a bounded wait expire (voted on once per chunk)
    bool tma_outstanding = false;  // a tile load was issued and not yet waited for

    auto issue_tma = [&](int64_t tok0) {
        mbar_arrive_expect_tx(&ms->tma_bar, 6 * 8192);
        const int32_t t32 = (int32_t)tok0;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sm + OFF_KQ + hf * 16384, &tm_k, &ms->tma_bar, 64 * hf, j, t32);
            tma_load_3d(sm + OFF_KQ + hf * 16384 + 8192, &tm_q, &ms->tma_bar, 64 * hf, j, t32);
            tma_load_3d(sm + OFF_V + hf * 8192, &tm_v, &ms->tma_bar, 64 * hf, h, t32);
        }
    };
    // commit the MMAs issued by thread 0, then everyone waits for them
    auto mma_sync_point = [&]() {
        if (tid == 0) mma_commit(&ms->mma_bar);
        if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
        mma_phase ^= 1;
        tc_fence_after_sync();
    };
    // generic smem / TMEM writes of every thread -> visible to the MMA issuer
    auto publish = [&]() {
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    if (t_begin < t_end) {
        if (tid == 0) issue_tma(t_begin);
        tma_outstanding = true;
    }
    GDN_TC_PHASE(0);

#pragma unroll 1
    for (int64_t c0 = t_begin; c0 < t_end && !aborted; c0 += kC) {
        const int L = (int)((t_end - c0) < kC ? (t_end - c0) : kC);
        const bool has_next = c0 + kC < t_end;

        // ---- gates (warp 0, two tokens per lane): cumulative log-decay, factors, flags ----
        if (warp == 0) {
            float x1 = gpre0 + gpre1;  // inclusive scan of pair sums
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x1, off);
                if (lane >= off) x1 += y;
            }
            const float x0 = x1 - gpre1;  // gamma at token 2l
            const float gC = __shfl_sync(0xffffffffu, x1, 31);
            float m = fmaxf(fabsf(x0), fabsf(x1));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            const bool safe_ = m <= 60.f;  // every exp(+-gamma) a normal float
            const float G0 = expf(x0), G1 = expf(x1);
            const float GC = __shfl_sync(0xffffffffu, G1, 31);
            const int r0 = 2 * lane;
            ms->gam[r0] = x0;                ms->gam[r0 + 1] = x1;
            ms->Gam[r0] = G0;                ms->Gam[r0 + 1] = G1;
            if (safe_) {  // 1 / Gamma and Gamma_C / Gamma from the exponentials above
                const float i0 = 1.f / G0, i1 = 1.f / G1;
                ms->iGam[r0] = i0;           ms->iGam[r0 + 1] = i1;
                ms->eC[r0] = GC * i0;        ms->eC[r0 + 1] = GC * i1;
            } else {
                ms->iGam[r0] = 0.f;          ms->iGam[r0 + 1] = 0.f;
                ms->eC[r0] = expf(gC - x0);  ms->eC[r0 + 1] = expf(gC - x1);
            }
            ms->bb[r0] = bpre0;              ms->bb[r0 + 1] = bpre1;
            // decay of token r's recall terms (in A and W): Gamma_r, or Gamma_{r-1}
            // when the recall is taken before the decay (Gamma_{-1} = 1)
            const float xp = __shfl_up_sync(0xffffffffu, x1, 1);  // gamma at token 2l - 1
            const float Gr0 = p.recall_first ? (lane > 0 ? expf(xp) : 1.f) : G0;
            const float Gr1 = p.recall_first ? G0 : G1;
            ms->bG[r0] = bpre0 * Gr0;        ms->bG[r0 + 1] = bpre1 * Gr1;
            if (lane == 0) {
                ms->safe = safe_;
                // from the chunk's summed log-decay, the number the previous
                // chunk used to decide whether to write the state's lo part
                ms->hp = ms->gsum_next >= kLogHighPrecisionDecay;
            }
            if (has_next) load_gates(c0 + kC);  // prefetch the next chunk's gates
        }
        GDN_TC_PHASE(1);

        // ---- wait for the tiles; Gram [K;Q] K^T -> TM_G straight from the bf16 tiles
        //      (exact products either way), bf16 -> fp16 in place meanwhile ----
        if (!mbar_wait_bounded(&ms->tma_bar, tma_phase, kWaitLimit)) timed_out = true;
        tma_phase ^= 1;
        tma_outstanding = false;
        GDN_TC_PHASE(2);
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t a = sbase + OFF_KQ + (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16_ss(tmem + TM_G, make_sdesc(a, 16, 1024), make_sdesc(a, 16, 1024),
                           IDESC_KK_N64_BF16, ks > 0);
            }
            mma_commit(&ms->mma_bar);
        }
        // 16-byte chunk x of the tile region starting at `base`; row = token
        // (offset / 128 within each 8 KB box); padding rows become zeros.  K and
        // Q go to fp16 once the Gram products have read them; V stays bf16 (the
        // U~ product splits its other operand three ways in bf16).
        auto convert16 = [&](uint8_t *base, int x) {
            uint4 *ptr = reinterpret_cast<uint4 *>(base) + x;
            const int r = (x >> 3) & 63;
            uint4 val = *ptr;
            if (r >= L) {
                val = make_uint4(0u, 0u, 0u, 0u);
            } else {
                uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&w[q2]);
                    const float2 f = __bfloat1622float2(b2);
                    kmax = fmaxf(kmax, fmaxf(fabsf(f.x), fabsf(f.y)));
                    w[q2] = pack_half2(f.x, f.y);
                }
                val = make_uint4(w[0], w[1], w[2], w[3]);
            }
            *ptr = val;
        };
        if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
        mma_phase ^= 1;
        tc_fence_after_sync();
#pragma unroll
        for (int k = 0; k < 2048 / kThreads; ++k) convert16(sm + OFF_KQ, tid + k * kThreads);  // K, Q
        const bool hp = ms->hp;
        const bool safe = ms->safe;
        GDN_TC_PHASE(3);
        GDN_TC_PHASE(4);

        // ---- A (lanes 0..63) and P (lanes 64..127) from the Gram rows ----
        float *As = reinterpret_cast<float *>(sm + OFF_AS);
        float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
        float *Xs = reinterpret_cast<float *>(sm + OFF_XS);
        {
            const int r = row & 63;
            const int c = 32 * half;
            float v[32];
            tmem_ld32(trow + TM_G + c, v);
            tmem_wait_ld();
            if (safe) {  // exp(gam_r - gam_i) = Gamma_r * exp(-gam_i), no overflow
                const float sr = row < kC ? ms->bG[r] : ms->Gam[r];
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] *= sr * ms->iGam[c + x];
            } else {
                const float gr = (row < kC && p.recall_first) ? (r > 0 ? ms->gam[r - 1] : 0.f)
                                                              : ms->gam[r];
                const float sr = row < kC ? ms->bb[r] : 1.f;
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] *= sr * expf(gr - ms->gam[c + x]);
            }
            if (row < kC) {  // A = strictly lower part (16-byte stores: conflict-free at stride kAS4)
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4 *>(As + r * kAS4 + c + x) =
                        make_float4((c + x < r) ? v[x] : 0.f, (c + x + 1 < r) ? v[x + 1] : 0.f,
                                    (c + x + 2 < r) ? v[x + 2] : 0.f, (c + x + 3 < r) ? v[x + 3] : 0.f);
            } else {         // P = lower part including the diagonal
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] = (c + x <= r) ? v[x] : 0.f;
#pragma unroll
                for (int e = 0; e < 32; e += 8)
                    st_row_chunk(sm + OFF_P16, r, (c + e) / 8, pack8_track(v + e, kmax));
            }
        }
        __syncthreads();
        GDN_TC_PHASE(5);

        // ---- T = (I + A)^-1 (fp32, CUDA cores) ----
        solve_tril64(As, Ts, Xs, tid);
        GDN_TC_PHASE(6);

        // ---- B operands: rows r of T diag(b) (bf16 hi / mid / lo) and
        //      T diag(b Gamma) (fp16 hi / lo, as K) ----
        {
            const int grp = tid >> 6, r = tid & 63;
            const bool tg = grp >= 2;
            const int c = 32 * (grp & 1);
            const float *scale = tg ? ms->bG : ms->bb;
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 t4 = *reinterpret_cast<const float4 *>(Ts + r * kTS + c + e);
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = c + e + q;
                    x[e + q] = (i <= r) ? tv[q] * scale[i] : 0.f;
                }
            }
            if (tg)
                store_split32(sm + OFF_TGH, sm + OFF_TGL, r, c, x, hp, kmax);
            else
                store_split32_bf16x3(sm + OFF_TBH, sm + OFF_TBM, sm + OFF_TBL, r, c, x);
        }
        publish();
        GDN_TC_PHASE(7);

        // ---- U~^T = V^T (T diag b)^T, W^T = K^T (T diag(b Gamma))^T, S Q^T ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // bf16 V times [hi | mid | lo] of T diag(b)
                const uint64_t a = make_sdesc(sbase + OFF_V + ks * 2048, 8192, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_TBH + ks * 32, 16, 1024);
                mma_f16_ss(tmem + TM_U, a, b, IDESC_MK_N192_BF16, ks != 0);
            }
            const uint32_t idesc_w = hp ? IDESC_MK_N128 : IDESC_MK_N64;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // fp16 K times [hi | lo] of T diag(b Gamma)
                const uint64_t a = make_sdesc(sbase + OFF_KQ + ks * 2048, 16384, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_TGH + ks * 32, 16, 1024);
                mma_f16_ss(tmem + TM_WT, a, b, idesc_w, ks != 0);
            }
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a =
                    make_sdesc(sbase + OFF_S16H + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t b =
                    make_sdesc(sbase + OFF_KQ + (ks >> 2) * 16384 + 8192 + (ks & 3) * 32, 16, 1024);
                mma_f16_ss(tmem + TM_O, a, b, IDESC_KK_N64, ks > 0);
            }
        }
        mma_sync_point();
        GDN_TC_PHASE(8);

        // ---- W^T rows -> fp16 B tiles (MN-major) ----
        {
            const int c = 32 * half;
            float v[32];
            tmem_ld32(trow + TM_WT + c, v);
            if (hp) {
                float w2[32];
                tmem_ld32(trow + TM_WT + 64 + c, w2);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] += w2[x];
            }
            tmem_wait_ld();
            store_split32(sm + OFF_WST, sm + OFF_WST + 16384, row, c, v, hp, kmax);
        }
        publish();
        GDN_TC_PHASE(9);

        // ---- R = S W^T (hp: Sh Wh^T + Sh Wl^T + Sl Wh^T) ----
        if (tid == 0) {
            for (int pass = 0; pass < (hp ? 3 : 1); ++pass)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t s_off = pass == 2 ? OFF_S16L : OFF_S16H;
                    const uint32_t w_off = pass == 1 ? OFF_WST + 16384 : OFF_WST;
                    const uint64_t a = make_sdesc(
                        sbase + s_off + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                    const uint64_t b = make_sdesc(sbase + w_off + ks * 2048, 16384, 1024);
                    mma_f16_ss(tmem + TM_R, a, b, IDESC_KM_N64, (pass | ks) != 0);
                }
        }
        mma_sync_point();
        GDN_TC_PHASE(10);

        // ---- U = U~ - R (row i of U^T) in the state's scale; U' = U diag(Gamma_C/Gamma)
        //      split and U; S Q^T rows scaled by Gamma.  A vote on U's largest
        //      scaled magnitude; if it left the band, U takes a scale of its own
        //      and O follows it. ----
        {
            const int c = 32 * half;
            float u[32];
            // U~ (the sum of its three parts) into ut, R (scaled by 2^-es) into u
            auto load_ut_r = [&](float (&ut)[32]) {
                float t1[32];
                tmem_ld32(trow + TM_U + c, ut);
                tmem_ld32(trow + TM_U + 64 + c, t1);
                tmem_ld32(trow + TM_U + 128 + c, u);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) ut[x] += t1[x] + u[x];
                tmem_ld32(trow + TM_R + c, u);
                tmem_wait_ld();
            };
            auto store_u = [&]() {  // U' hi / lo and U (scaled) -> shared memory
                float up[32];
#pragma unroll
                for (int x = 0; x < 32; ++x) up[x] = u[x] * ms->eC[c + x];
                store_split32(sm + OFF_UP, sm + OFF_UP + 16384, row, c, up, true);
#pragma unroll
                for (int e = 0; e < 32; e += 8)
                    st_row_chunk(sm + OFF_U16, row, (c + e) / 8, pack8(u + e));
            };
            auto scale_o = [&](float f) {  // S Q^T rows times f Gamma
                float ov[32];
                tmem_ld32(trow + TM_O + c, ov);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) ov[x] *= f * ms->Gam[c + x];
                tmem_st32(trow + TM_O + c, ov);
            };
            float am;
            {
                float ut[32];
                load_ut_r(ut);
#pragma unroll
                for (int x = 0; x < 32; ++x) u[x] = fmaf(ut[x], sd, -u[x]);  // U 2^-es (R: 2^-es)
                am = max_abs<32>(u);
            }
            eu = es;
            store_u();
            if (warp == 0) warp0_sum_to(gpre0 + gpre1, &ms->gsum_next);  // next chunk's log-decay
            const unsigned b =
                cta_or8(__reduce_or_sync(0xffffffffu, scale_bits(am)), ms->vote[0], warp, lane);
            if (rescale_needed(b)) {  // rare: U takes its own scale
                float ut[32];
                load_ut_r(ut);  // U~ and R are still in place
#pragma unroll
                for (int x = 0; x < 32; ++x) u[x] = fmaf(-s_up, u[x], ut[x]);  // U in fp32, unscaled
                am = cta_max(max_abs<32>(u), ms->red, warp, lane);
                eu = fp16_scale_exp(am);
                const float ud = exp2i(-eu);
#pragma unroll
                for (int x = 0; x < 32; ++x) u[x] *= ud;
                store_u();
            }
            scale_o(exp2c(es - eu));
        }
        publish();
        GDN_TC_PHASE(11);

        // ---- dS = [U'hi | U'lo] [K ; K] (rows scaled by 2^-eu);  O += U^T P^T ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a =
                    make_sdesc(sbase + OFF_UP + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_KQ + (ks & 3) * 2048, 16384, 1024);
                mma_f16_ss(tmem + TM_D, a, b, IDESC_KM_N128, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = make_sdesc(sbase + OFF_U16 + ks * 32, 16, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_P16 + ks * 32, 16, 1024);
                mma_f16_ss(tmem + TM_O, a, b, IDESC_KK_N64, 1);
            }
        }
        mma_sync_point();
        // next chunk's tiles can land while we finish this one (all MMAs reading them are done)
        if (has_next) {
            if (tid == 0) issue_tma(c0 + kC);
            tma_outstanding = true;
        }
        GDN_TC_PHASE(12);

        // ---- o rows -> staging tile; new S = Gamma_C S + dS (scaled) -> fp16 hi/lo;
        //      master = S * Gamma_C(next); a vote on S's largest scaled
        //      magnitude (rescale if it left the band) ----
        {
            const int c = 32 * half;
            const float uu = exp2i(eu);  // O and dS rows come scaled by 2^-eu
            float v[32];
            tmem_ld32(trow + TM_O + c, v);
            tmem_wait_ld();
            __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(sm + OFF_OST);
#pragma unroll
            for (int x = 0; x < 32; ++x) ost[(c + x) * kD + row] = __float2bfloat16_rn(v[x] * uu);
            const float gnext = has_next ? expf(ms->gsum_next) : 1.f;
            const bool lo_next = has_next && ms->gsum_next >= kLogHighPrecisionDecay;
            const bool same = eu == es;  // uniform over the CTA
            // same: S' in the state's scale; otherwise (U took its own scale this
            // chunk) S' in fp32, unscaled, and a new scale for it
            float sv[64];
            float am;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float d[32];
                tmem_ld32(trow + TM_S + 64 * half + 32 * part, v);
                tmem_ld32(trow + TM_D + 64 * half + 32 * part, d);
                tmem_wait_ld();
                if (same) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        sv[32 * part + x] = v[x] + d[x];
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        sv[32 * part + x] = fmaf(s_up, v[x], d[x] * uu);
                    }
                }
            }
            auto rescale = [&]() {  // a new scale for the unscaled sv, from the CTA maximum
                am = cta_max(am, ms->red, warp, lane);
                set_es(am > 0.f ? fp16_scale_exp(am) : es);
#pragma unroll
                for (int x = 0; x < 64; ++x) sv[x] *= sd;
            };
            auto store_master = [&]() {  // gnext = 1 after the last chunk
#pragma unroll
                for (int part = 0; part < 2; ++part) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) v[x] = sv[32 * part + x] * gnext;
                    tmem_st32(trow + TM_S + 64 * half + 32 * part, v);
                }
            };
            am = max_abs<64>(sv);
            if (!same) rescale();
            split_state(sv, lo_next);
            store_master();
            const unsigned b = cta_or8(__reduce_or_sync(0xffffffffu, same ? scale_bits(am) : 2u),
                                       ms->vote[1], warp, lane);
            if (rescale_needed(b)) {  // rare: S' left the band
#pragma unroll
                for (int x = 0; x < 64; ++x) sv[x] *= s_up;  // exact: S' in fp32, unscaled
                am = max_abs<64>(sv);
                rescale();
                split_state(sv, lo_next);  // published by the barrier at the chunk's end
                store_master();
            }
        }
        {
            const uint4 *ost = reinterpret_cast<const uint4 *>(sm + OFF_OST);
#pragma unroll
            for (int k = 0; k < (kC * kD * 2 / 16) / kThreads; ++k) {
                const int x = tid + k * kThreads;
                const int r = x >> 4, c16 = x & 15;
                if (r < L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                                           ((c0 + r) * p.Hv + h) * (int64_t)kD) + c16;
                    *dst = ost[x];
                }
            }
        }
        // a key-side fp16 operand of this chunk (K, Q, P, T diag(b Gamma), W^T)
        // overflowed: report it once per thread (the unit's results are then
        // unspecified; the computation goes on)
        if (kmax >= kFp16Overflow && !range_reported) {
            raise_error(p.err, GDN_ERR_RANGE);
            range_reported = true;
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        if (__syncthreads_or(timed_out ? 1 : 0)) {  // a bounded wait expired: stop here
            if (tid == 0) raise_error(p.err, GDN_ERR_TIMEOUT);
            aborted = true;
        }
        tc_fence_after_sync();
        GDN_TC_PHASE(13);
    }

    // ---- final state: the master times 2^es ----
    if (!aborted && p.sT) {
        float *dst = p.sT + (((int64_t)n * p.Hv + h) * kD + row) * kD;
#pragma unroll 1
        for (int c = 64 * half; c < 64 * half + 64; c += 32) {
            float v[32];
            tmem_ld32(trow + TM_S + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; x += 4)
                *reinterpret_cast<float4 *>(dst + c + x) =
                    make_float4(v[x] * s_up, v[x + 1] * s_up, v[x + 2] * s_up, v[x + 3] * s_up);
        }
    }
    if (aborted) {
        // Give the last committed MMAs and an outstanding tile load a bounded
        // chance to drain before TMEM is freed (parities of the latest phases).
        mbar_wait_bounded(&ms->mma_bar, mma_phase ^ 1, kWaitLimit);
        if (tma_outstanding) mbar_wait_bounded(&ms->tma_bar, tma_phase, kWaitLimit);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    GDN_TC_PHASE_FLUSH();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host --

}  // namespace

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

// [T][H][128] bf16 tensor map with 64 x 1 x 64 boxes and the 128-byte swizzle,
// shared by the tensor-core prefill kernels.
bool make_tile_map_bf16_128(CUtensorMap *m, const void *base, int64_t T, int32_t H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    const cuuint32_t box[3] = {64, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same map with 8-token boxes (the tokens before a chunk, for the fused
// front end's convolution).
bool make_halo_map_bf16_128(CUtensorMap *m, const void *base, int64_t T, int32_t H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    const cuuint32_t box[3] = {64, 1, 8};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [T][H][128] bf16 tensor map for storing whole 64-token tiles of one head
// (box 128 x 1 x 64, no swizzle: the tile is [64 tokens][128] row-major).
bool make_store_map_bf16_128(CUtensorMap *m, void *base, int64_t T, int32_t H) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kD, 1, 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t s) {
    if (a.T > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are 32-bit
    CUtensorMap mq, mk, mv;
    const int64_t Tm = a.T > 0 ? a.T : 1;
    if (!make_tile_map_bf16_128(&mq, a.q, Tm, a.Hqk) || !make_tile_map_bf16_128(&mk, a.k, Tm, a.Hqk) ||
        !make_tile_map_bf16_128(&mv, a.v, Tm, a.Hv))
        return cudaErrorInvalidValue;
    TcParams p;
    p.g = a.g; p.beta = a.beta; p.s0 = a.s0; p.cu = a.cu; p.o = a.o; p.sT = a.sT; p.err = a.err;
    p.T = a.T; p.N = a.N; p.Hqk = a.Hqk; p.Hv = a.Hv;
    p.recall_first = a.order == GDN_ORDER_RECALL_FIRST;
    cudaError_t e = cudaFuncSetAttribute(gdn_prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((int64_t)a.N * a.Hv));
    gdn_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace gdn

#ifdef GDN_TC_PHASES
extern "C" GDN_API int gdn_debug_tc_phases(long long *out, int n, int reset) {
    unsigned long long host[16];
    if (cudaMemcpyFromSymbol(host, gdn_tc_phase_clk, sizeof(host)) != cudaSuccess) return -1;
    for (int i = 0; i < n && i < 16; ++i) out[i] = (long long)host[i];
    if (reset) {
        const unsigned long long zero[16] = {0};
        cudaMemcpyToSymbol(gdn_tc_phase_clk, zero, sizeof(zero));
    }
    return 0;
}
#endif
