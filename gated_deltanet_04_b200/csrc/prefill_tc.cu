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
// Kernel design (one CTA of 4 warps per (sequence, v-head); thread i <-> TMEM
// lane i <-> state row i):
//   * The fp32 state S lives in tensor memory as an MMA accumulator for the
//     whole sequence (no HBM round trip between chunks).  Its fp16 copy in
//     shared memory is the A operand of the state-side products.
//   * Every product is a tcgen05.mma (M = 128, fp16 operands, fp32
//     accumulation) whose result rows are state rows or chunk rows:
//       Gram   [K;Q] K^T            -> K K^T (lanes 0-63), Q K^T (lanes 64-127)
//       U~^T = V^T (T diag b)^T      (T split into fp16 hi + lo: 2 passes)
//       W^T  = K^T (T diag(b Gamma))^T  (2 passes)
//       S Q^T, R = S W^T             (R: S and W^T both split, 3 passes)
//       S   += [U'hi | U'lo] [K ; K] (U' = U diag(Gamma_C/Gamma), split)
//       U^T P^T                      (P = Q K^T (.) M)
//     q/k/v tiles arrive by TMA (128-byte swizzle, no multicast) and are
//     converted in place from bf16 to fp16 (exact for |x| in [6e-5, 6.5e4]).
//     fp16 operands keep 11 significant bits.  T diag(b), T diag(b Gamma) and
//     U' get a second (low-part) pass and S W^T three (hi.hi + hi.lo + lo.hi):
//     without them the rounding of the undecayed (a = 1) state accumulates
//     past 1e-4 of fp64 within a few chunks.
//   * The unit lower-triangular solve T = (I + A)^-1 runs on CUDA cores in
//     fp32 by 16 x 16 blocks.
//   * Rows past the end of a sequence inside the last chunk are zeroed and
//     get b = g = 0, which makes them contribute nothing.
// The phases of a chunk run in order, separated by MMA commits; every wait
// on an mbarrier is bounded and reports GDN_ERR_TIMEOUT instead of hanging.
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kC = 64;      // chunk length
constexpr int kD = 128;     // Dk = Dv
constexpr int kThreads = 128;
constexpr long long kWaitLimit = 1ll << 31;  // SM clocks (about a second)

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
constexpr uint32_t OFF_AS = OFF_X;                  // float [64][65]
constexpr uint32_t OFF_TS = OFF_X + 64 * 65 * 4;    // float [64][65]
constexpr uint32_t OFF_XS = OFF_TS + 64 * 65 * 4;   // float [3][16][16]
constexpr uint32_t OFF_P16 = 163840;    // 64 rows x 128 B                  (B: P, K-major)
constexpr uint32_t OFF_TBH = 172032;    // 64 rows x 128 B                  (B: T diag b, hi)
constexpr uint32_t OFF_TBL = 180224;    //                                  (B: T diag b, lo)
constexpr uint32_t OFF_TGH = 188416;    //                                  (B: T diag(b Gamma), hi)
constexpr uint32_t OFF_TGL = 196608;    //                                  (B: T diag(b Gamma), lo)
constexpr uint32_t OFF_MISC = 204800;
static_assert(OFF_XS + 3 * 256 * 4 <= OFF_P16, "solve scratch overflows");

struct Misc {
    float gam[kC];    // cumulative log-decay within the chunk
    float Gam[kC];    // exp(gam)
    float eC[kC];     // exp(gam_C - gam_r)
    float bb[kC];     // beta (0 for padding rows)
    uint64_t tma_bar;
    uint64_t mma_bar;
    uint32_t tmem_base;
    int32_t abort;
};
constexpr uint32_t kSmemBytes = OFF_MISC + sizeof(Misc) + 1024;  // + alignment slack

// TMEM column map (fp32 columns; 512 allocated)
constexpr uint32_t TM_S = 0, TM_G = 128, TM_U = 192, TM_WT = 256, TM_O = 320, TM_R = 384,
                   TM_P = 448;

constexpr uint32_t IDESC_KK_N64 = make_idesc_f16(128, 64, 0, 0);
constexpr uint32_t IDESC_MK_N64 = make_idesc_f16(128, 64, 1, 0);
constexpr uint32_t IDESC_KM_N64 = make_idesc_f16(128, 64, 0, 1);
constexpr uint32_t IDESC_KM_N128 = make_idesc_f16(128, 128, 0, 1);

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// hi = fp16(x), lo = fp16(x - hi) for 8 values, packed as two uint4
__device__ __forceinline__ void split8(const float *x, uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __half2 hh = __floats2half2_rn(x[2 * j], x[2 * j + 1]);
        const float2 hf = __half22float2(hh);
        h[j] = *reinterpret_cast<const uint32_t *>(&hh);
        l[j] = pack_half2(x[2 * j] - hf.x, x[2 * j + 1] - hf.y);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ uint4 pack8(const float *x) {
    return make_uint4(pack_half2(x[0], x[1]), pack_half2(x[2], x[3]), pack_half2(x[4], x[5]),
                      pack_half2(x[6], x[7]));
}

__device__ __forceinline__ void st_row_chunk(uint8_t *tile, uint32_t row, uint32_t chunk,
                                             uint4 val) {
    *reinterpret_cast<uint4 *>(tile + sw128(row, chunk * 16)) = val;
}

// row i, columns [c, c + 16) of S -> fp16 hi and lo A-operand tiles
__device__ __forceinline__ void store_state_split(uint8_t *sm, int i, int c, const float *v) {
    const uint32_t half = (c / 64) * 16384, ch = (c % 64) / 8;
    uint4 hi, lo;
    split8(v, hi, lo);
    st_row_chunk(sm + OFF_S16H + half, i, ch, hi);
    st_row_chunk(sm + OFF_S16L + half, i, ch, lo);
    split8(v + 8, hi, lo);
    st_row_chunk(sm + OFF_S16H + half, i, ch + 1, hi);
    st_row_chunk(sm + OFF_S16L + half, i, ch + 1, lo);
}

struct TcParams {
    const float *g, *beta, *s0;
    const int32_t *cu;
    void *o;
    float *sT;
    int32_t *err;
    int64_t T;
    int32_t N, Hqk, Hv;
    int32_t o_f32;  // o dtype: 0 = bf16, 1 = fp32
};

// Ends the CTA's work when `bad` is set on any thread: raises the status and
// returns true for every thread.
__device__ __forceinline__ bool cta_abort(bool bad, Misc *ms, int32_t *err) {
    const int any = __syncthreads_or(bad ? 1 : 0);
    if (any && threadIdx.x == 0) raise_error(err, GDN_ERR_TIMEOUT);
    return any != 0;
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

    const int unit = blockIdx.x;  // n * Hv + h
    const int h = unit % p.Hv;
    const int n = unit / p.Hv;
    const int j = h / (p.Hv / p.Hqk);

    int64_t t_begin, t_end;
    if (!seq_range(p.cu, n, p.N, p.T, p.err, t_begin, t_end)) return;  // uniform

    if (tid == 0) {
        mbar_init(&ms->tma_bar, 1);
        mbar_init(&ms->mma_bar, 1);
        ms->abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 0) {
        tmem_alloc(&ms->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = ms->tmem_base;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes
    const uint32_t trow = tmem + lane_off;                  // + column

    // ---- initial state: S (fp32) -> TMEM accumulator, fp16 copy -> S16 ----
    {
        const int i = tid;
        const float *src = p.s0 ? p.s0 + (((int64_t)n * p.Hv + h) * kD + i) * kD : nullptr;
#pragma unroll 1
        for (int c = 0; c < kD; c += 16) {
            float v[16];
#pragma unroll
            for (int x = 0; x < 16; x += 4) {
                float4 f = src ? *reinterpret_cast<const float4 *>(src + c + x)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[x] = f.x; v[x + 1] = f.y; v[x + 2] = f.z; v[x + 3] = f.w;
            }
            tmem_st16(trow + TM_S + c, v);
            store_state_split(sm, i, c, v);
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    uint32_t tma_phase = 0, mma_phase = 0;
    bool aborted = false;

    auto issue_tma = [&](int64_t tok0) {
        mbar_arrive_expect_tx(&ms->tma_bar, 6 * 8192);
        const int32_t t32 = (int32_t)tok0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_3d(sm + OFF_KQ + half * 16384, &tm_k, &ms->tma_bar, 64 * half, j, t32);
            tma_load_3d(sm + OFF_KQ + half * 16384 + 8192, &tm_q, &ms->tma_bar, 64 * half, j, t32);
            tma_load_3d(sm + OFF_V + half * 8192, &tm_v, &ms->tma_bar, 64 * half, h, t32);
        }
    };
    // commit the MMAs issued by thread 0, then everyone waits for them
    auto mma_sync_point = [&]() -> bool {
        if (tid == 0) mma_commit(&ms->mma_bar);
        const bool ok = mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit);
        mma_phase ^= 1;
        tc_fence_after_sync();
        return cta_abort(!ok, ms, p.err);
    };
    // generic smem / TMEM writes of every thread -> visible to the MMA issuer
    auto publish = [&]() {
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    if (t_begin < t_end && tid == 0) issue_tma(t_begin);

#pragma unroll 1
    for (int64_t c0 = t_begin; c0 < t_end && !aborted; c0 += kC) {
        const int L = (int)((t_end - c0) < kC ? (t_end - c0) : kC);

        // ---- gates of the chunk (threads 0..63), cumulative log-decay ----
        float gr = 0.f, br = 0.f;
        if (tid < kC && tid < L) {
            gr = p.g[(c0 + tid) * p.Hv + h];
            br = p.beta[(c0 + tid) * p.Hv + h];
        }
        if (tid < kC) {
            float x = gr;  // inclusive scan over 64 lanes (two warps)
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, x, off);
                if ((tid & 31) >= off) x += y;
            }
            ms->gam[tid] = x;  // partial (per warp)
            ms->bb[tid] = br;
        }
        __syncthreads();
        if (tid >= 32 && tid < kC) ms->gam[tid] += ms->gam[31];
        __syncthreads();
        if (tid < kC) {
            const float gm = ms->gam[tid];
            ms->Gam[tid] = expf(gm);
            ms->eC[tid] = expf(ms->gam[kC - 1] - gm);
        }

        // ---- wait for the tiles, convert bf16 -> fp16 in place, zero padding rows ----
        {
            const bool ok = mbar_wait_bounded(&ms->tma_bar, tma_phase, kWaitLimit);
            tma_phase ^= 1;
            if (cta_abort(!ok, ms, p.err)) { aborted = true; break; }
        }
        // 48 KB = 3072 chunks of 16 bytes; row = token index (offset / 128 within each 8 KB box)
#pragma unroll 4
        for (int x = tid; x < 3072; x += kThreads) {
            uint4 *ptr = reinterpret_cast<uint4 *>(sm + OFF_KQ) + x;  // KQ and V are contiguous
            const int row = (x >> 3) & 63;
            uint4 val = *ptr;
            if (row >= L) {
                val = make_uint4(0u, 0u, 0u, 0u);
            } else {
                uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162 *>(&w[q2]);
                    const float2 f = __bfloat1622float2(b2);
                    w[q2] = pack_half2(f.x, f.y);
                }
                val = make_uint4(w[0], w[1], w[2], w[3]);
            }
            *ptr = val;
        }
        publish();

        // ---- Gram: [K;Q] K^T -> TM_G ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t a = sbase + OFF_KQ + (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16_ss(tmem + TM_G, make_sdesc(a, 16, 1024), make_sdesc(a, 16, 1024),
                           IDESC_KK_N64, ks > 0);
            }
        }
        if (mma_sync_point()) { aborted = true; break; }

        // ---- A (rows 0..63) and P (rows 64..127) from the Gram rows ----
        float *As = reinterpret_cast<float *>(sm + OFF_AS);
        float *Ts = reinterpret_cast<float *>(sm + OFF_TS);
        float *Xs = reinterpret_cast<float *>(sm + OFF_XS);
        {
            const int r = tid & 63;
            const float gr_ = ms->gam[r];
            const float br_ = ms->bb[r];
#pragma unroll 1
            for (int c = 0; c < kC; c += 16) {
                float v[16];
                tmem_ld16(trow + TM_G + c, v);
                tmem_wait_ld();
                if (tid < kC) {
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int i = c + x;
                        As[r * 65 + i] = (i < r) ? br_ * v[x] * expf(gr_ - ms->gam[i]) : 0.f;
                    }
                } else {
                    float pr[16];
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int i = c + x;
                        pr[x] = (i <= r) ? v[x] * expf(gr_ - ms->gam[i]) : 0.f;
                    }
                    uint8_t *tile = sm + OFF_P16;
                    st_row_chunk(tile, r, c / 8, pack8(pr));
                    st_row_chunk(tile, r, c / 8 + 1, pack8(pr + 8));
                }
            }
        }
        __syncthreads();

        // ---- T = (I + A)^-1 by 16 x 16 blocks (fp32, CUDA cores) ----
        if (tid < kC) {  // diagonal blocks: thread = (block, column)
            const int bi = tid >> 4, col = tid & 15;
            float x[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                float acc = (rr == col) ? 1.f : 0.f;
#pragma unroll
                for (int ii = 0; ii < rr; ++ii) acc -= As[(16 * bi + rr) * 65 + 16 * bi + ii] * x[ii];
                x[rr] = acc;
            }
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) Ts[(16 * bi + rr) * 65 + 16 * bi + col] = x[rr];
        }
        __syncthreads();
#pragma unroll 1
        for (int d = 1; d < 4; ++d) {
            const int nblk = 4 - d;
            // X_blk = sum_{m = 16k}^{16i - 1} A[16i + r][m] T[m][16k + c],  i = k + d
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
                const int bi = blk + d, bk = blk;
                float acc = 0.f;
                for (int m = 16 * bk; m < 16 * bi; ++m)
                    acc += As[(16 * bi + r) * 65 + m] * Ts[m * 65 + 16 * bk + c];
                Xs[e] = acc;
            }
            __syncthreads();
            // T[16i + r][16k + c] = - sum_m T[16i + r][16i + m] X[m][c]
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
                const int bi = blk + d, bk = blk;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc += Ts[(16 * bi + r) * 65 + 16 * bi + m] * Xs[(blk << 8) + m * 16 + c];
                Ts[(16 * bi + r) * 65 + 16 * bk + c] = -acc;
            }
            __syncthreads();
        }

        // ---- B operands from T: rows r of T diag(b) and T diag(b Gamma), hi and lo ----
        {
            const int r = tid & 63;
#pragma unroll 1
            for (int c = 0; c < kC; c += 8) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = c + e;
                    const float t = (i <= r) ? Ts[r * 65 + i] : 0.f;
                    x[e] = (tid < kC) ? t * ms->bb[i] : t * ms->bb[i] * ms->Gam[i];
                }
                uint4 hi, lo;
                split8(x, hi, lo);
                st_row_chunk(sm + (tid < kC ? OFF_TBH : OFF_TGH), r, c / 8, hi);
                st_row_chunk(sm + (tid < kC ? OFF_TBL : OFF_TGL), r, c / 8, lo);
            }
        }
        publish();

        // ---- U~^T = V^T (T diag b)^T, W^T = K^T (T diag(b Gamma))^T (2 passes each), S Q^T ----
        if (tid == 0) {
#pragma unroll
            for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = make_sdesc(sbase + OFF_V + ks * 2048, 8192, 1024);
                    const uint64_t b =
                        make_sdesc(sbase + (pass ? OFF_TBL : OFF_TBH) + ks * 32, 16, 1024);
                    mma_f16_ss(tmem + TM_U, a, b, IDESC_MK_N64, (pass | ks) != 0);
                }
#pragma unroll
            for (int pass = 0; pass < 2; ++pass)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = make_sdesc(sbase + OFF_KQ + ks * 2048, 16384, 1024);
                    const uint64_t b =
                        make_sdesc(sbase + (pass ? OFF_TGL : OFF_TGH) + ks * 32, 16, 1024);
                    mma_f16_ss(tmem + TM_WT, a, b, IDESC_MK_N64, (pass | ks) != 0);
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
        if (mma_sync_point()) { aborted = true; break; }

        // ---- W^T rows -> fp16 hi/lo B tiles (MN-major); master state *= Gamma_C ----
        {
            const float gC = ms->Gam[kC - 1];
#pragma unroll 1
            for (int c = 0; c < kC; c += 16) {
                float v[16];
                tmem_ld16(trow + TM_WT + c, v);
                tmem_wait_ld();
                uint4 hi, lo;
                split8(v, hi, lo);
                st_row_chunk(sm + OFF_WST, tid, c / 8, hi);
                st_row_chunk(sm + OFF_WST + 16384, tid, c / 8, lo);
                split8(v + 8, hi, lo);
                st_row_chunk(sm + OFF_WST, tid, c / 8 + 1, hi);
                st_row_chunk(sm + OFF_WST + 16384, tid, c / 8 + 1, lo);
            }
#pragma unroll 1
            for (int c = 0; c < kD; c += 16) {
                float v[16];
                tmem_ld16(trow + TM_S + c, v);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 16; ++x) v[x] *= gC;
                tmem_st16(trow + TM_S + c, v);
            }
        }
        publish();

        // ---- R = S W^T = Sh Wh^T + Sh Wl^T + Sl Wh^T ----
        if (tid == 0) {
#pragma unroll
            for (int pass = 0; pass < 3; ++pass)
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
        if (mma_sync_point()) { aborted = true; break; }

        // ---- U = U~ - R (row i of U^T), U' = U diag(Gamma_C/Gamma) split, U fp16 ----
        {
#pragma unroll 1
            for (int c = 0; c < kC; c += 16) {
                float u0[16], r0[16], up[16];
                tmem_ld16(trow + TM_U + c, u0);
                tmem_ld16(trow + TM_R + c, r0);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    u0[x] -= r0[x];
                    up[x] = u0[x] * ms->eC[c + x];
                }
                uint4 hi, lo;
                split8(up, hi, lo);
                st_row_chunk(sm + OFF_UP, tid, c / 8, hi);
                st_row_chunk(sm + OFF_UP + 16384, tid, c / 8, lo);
                split8(up + 8, hi, lo);
                st_row_chunk(sm + OFF_UP, tid, c / 8 + 1, hi);
                st_row_chunk(sm + OFF_UP + 16384, tid, c / 8 + 1, lo);
                st_row_chunk(sm + OFF_U16, tid, c / 8, pack8(u0));
                st_row_chunk(sm + OFF_U16, tid, c / 8 + 1, pack8(u0 + 8));
            }
        }
        publish();

        // ---- S += [U'hi | U'lo] [K ; K];  U^T P^T ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a =
                    make_sdesc(sbase + OFF_UP + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_KQ + (ks & 3) * 2048, 16384, 1024);
                mma_f16_ss(tmem + TM_S, a, b, IDESC_KM_N128, 1);
            }
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = make_sdesc(sbase + OFF_U16 + ks * 32, 16, 1024);
                const uint64_t b = make_sdesc(sbase + OFF_P16 + ks * 32, 16, 1024);
                mma_f16_ss(tmem + TM_P, a, b, IDESC_KK_N64, ks > 0);
            }
        }
        if (mma_sync_point()) { aborted = true; break; }

        // next chunk's tiles can land while we finish this one (all MMAs reading them are done)
        if (tid == 0 && c0 + kC < t_end) issue_tma(c0 + kC);

        // ---- o = diag(Gamma) S Q^T + U^T P^T (transposed), new S -> fp16 hi/lo copies ----
        {
            const int i = tid;
#pragma unroll 1
            for (int c = 0; c < kC; c += 16) {
                float so[16], pu[16];
                tmem_ld16(trow + TM_O + c, so);
                tmem_ld16(trow + TM_P + c, pu);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const int r = c + x;
                    if (r < L) {
                        const float val = fmaf(ms->Gam[r], so[x], pu[x]);
                        const int64_t idx = ((c0 + r) * p.Hv + h) * (int64_t)kD + i;
                        if (p.o_f32)
                            static_cast<float *>(p.o)[idx] = val;
                        else
                            static_cast<__nv_bfloat16 *>(p.o)[idx] = __float2bfloat16_rn(val);
                    }
                }
            }
#pragma unroll 1
            for (int c = 0; c < kD; c += 16) {
                float v[16];
                tmem_ld16(trow + TM_S + c, v);
                tmem_wait_ld();
                store_state_split(sm, i, c, v);
            }
        }
        publish();
    }

    // ---- final state ----
    if (!aborted && p.sT) {
        float *dst = p.sT + (((int64_t)n * p.Hv + h) * kD + tid) * kD;
#pragma unroll 1
        for (int c = 0; c < kD; c += 16) {
            float v[16];
            tmem_ld16(trow + TM_S + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 16; x += 4)
                *reinterpret_cast<float4 *>(dst + c + x) = make_float4(v[x], v[x + 1], v[x + 2], v[x + 3]);
        }
    }
    if (aborted) {
        // give MMAs / copies still in flight a bounded chance to drain before freeing TMEM
        mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit);
        mbar_wait_bounded(&ms->tma_bar, tma_phase, kWaitLimit);
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- host --

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

// [T][H][128] bf16 tensor, boxes of 64 (features) x 1 (head) x 64 (tokens), 128-byte swizzle
bool make_map(CUtensorMap *m, const void *base, int64_t T, int32_t H) {
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

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t s) {
    if (a.T > 0x7fffffffLL) return cudaErrorInvalidValue;  // TMA coordinates are 32-bit
    CUtensorMap mq, mk, mv;
    const int64_t Tm = a.T > 0 ? a.T : 1;
    if (!make_map(&mq, a.q, Tm, a.Hqk) || !make_map(&mk, a.k, Tm, a.Hqk) ||
        !make_map(&mv, a.v, Tm, a.Hv))
        return cudaErrorInvalidValue;
    TcParams p;
    p.g = a.g; p.beta = a.beta; p.s0 = a.s0; p.cu = a.cu; p.o = a.o; p.sT = a.sT; p.err = a.err;
    p.T = a.T; p.N = a.N; p.Hqk = a.Hqk; p.Hv = a.Hv; p.o_f32 = a.dtype == GDN_DTYPE_F32;
    cudaError_t e = cudaFuncSetAttribute(gdn_prefill_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((int64_t)a.N * a.Hv));
    gdn_prefill_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace gdn
