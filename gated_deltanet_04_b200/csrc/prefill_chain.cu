// Chunk-parallel prefill of the gated delta rule split across CTAs: one
// "chain" CTA per (sequence, v-head) carries the state from chunk to chunk,
// and "producer" CTAs prepare the chunks.
//
// The math is the chunk step of the single-CTA kernel (see prefill_tc.cu):
//     A = strict-lower(diag(b)(K K^T (.) M)),   T = (I + A)^-1
//     U~ = T diag(b) V,   W = T diag(b Gamma) K,   U = U~ - W S^T
//     O = diag(Gamma) Q S^T + (Q K^T (.) M) U,   S' = Gamma_C S + U^T diag(Gamma_C/Gamma) K
// from the rule of page "Qwen3.8-27B 架构深读: Gated DeltaNet 混合线性注意力与 262K
// 长上下文", section 三.  Only U (through S) links one chunk to the next; every
// other quantity of a chunk depends on that chunk's inputs alone.
//
// Roles (one SM per CTA):
//   * the chain CTA keeps the fp32 state as a TMEM accumulator and its fp16
//     hi/lo copies as TMEM A operands, and runs only the state-dependent
//     products of each chunk: S Q^T, R = S W^T, U = U~ - R, the state update
//     S += U'^T K, O += U^T P^T, and the output stores.
//   * a producer CTA takes whole chunks: TMA tile loads, bf16 -> fp16, Gram
//     matrices, decay factors, the triangular solve, U~ and W on tensor cores.
// A finished chunk (K, Q, W^T hi/lo, U~, P, gates: one 105 KB block laid out
// exactly like a chain slot) goes through L2: the producer bulk-stores it
// into a ring of R slots per (sequence, head) in the caller's workspace (R = 4
// for the cluster kernel, 8 for the pool kernel), and the chain bulk-loads
// it into one of its two shared-memory slots while it computes the previous
// chunk.  Chunk c of a unit always uses ring slot c % R.
//
// Two ways to schedule the producers:
//   * cluster kernel: a 3-CTA cluster per unit, rank 0 the chain, ranks 1 and
//     2 producers of the even and odd chunks.  Signals are mbarriers reached
//     through distributed shared memory:
//         ready[k] (chain)    producer k's stores of its next chunk are complete
//         full[i]  (chain)    the bulk load into shared slot i has landed
//         taken    (producer) the chain has loaded this producer's last delivery
//     A producer delivers its chunk only after the chain has taken its
//     previous one, so no barrier runs more than one phase ahead of its waiter
//     (a parity wait cannot tell phase n from n + 2).  A B200 holds at most 45
//     such clusters at once, so more than 45 units run in two waves.
//   * pool kernel: a cooperative launch of one CTA per SM; CTA u < units is
//     the chain of unit u, every other CTA is a producer that takes chunks
//     from a global counter in chunk-major order (chunk 0 of every unit, then
//     chunk 1, ...).  Signals are 32-bit flags in the workspace with gpu-scope
//     release / acquire:
//         ready[u][s]  = c + 1   chunk c of unit u is in ring slot s
//         taken[u]     = c + 1   the chain of unit u has loaded chunks 0..c
//     A producer writes chunk c only after taken[u] >= c - R + 1.
//     Every wait is on a chunk of lower counter index, and a producer works
//     through its chunks in counter order, so the lowest unfinished chunk can
//     always proceed: no deadlock while every CTA is resident, which the
//     cooperative launch guarantees.
//
// Every wait is bounded; an expired wait is voted on once per chunk, reports
// GDN_ERR_TIMEOUT and ends the CTA's loop (the pool kernel also raises its
// abort flag so that every other CTA stops waiting).  No TMA load uses
// multicast.
#include "gdn_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

#ifdef GDN_TC_PHASES
// Per-phase SM clocks of thread 0: [0] the first chain CTA, [1] the first
// producer CTA.  Accumulated in shared memory (a global read-modify-write per
// marker would stall thread 0 and distort the phases) and added to the
// global totals once, at the end of the role.
__device__ unsigned long long gdn_cl_phase_clk[2][16];
static __shared__ unsigned int gdn_phase_acc_[16];
#define GDN_CL_PHASE(role, k)                                          \
    do {                                                               \
        if (threadIdx.x == 0 && phase_on_) {                           \
            const long long now_ = clock64();                          \
            gdn_phase_acc_[(k)] += (unsigned int)(now_ - phase_t_);    \
            phase_t_ = now_;                                           \
        }                                                              \
    } while (0)
#define GDN_CL_PHASE_BEGIN()                                           \
    long long phase_t_ = clock64();                                    \
    if (threadIdx.x == 0)                                              \
        for (int i_ = 0; i_ < 16; ++i_) gdn_phase_acc_[i_] = 0u;       \
    if ((threadIdx.x & 31) == 0)                                       \
        for (int s_ = 0; s_ < 4; ++s_) gdn_bar_acc_[s_][threadIdx.x >> 5] = 0u
#define GDN_CL_PHASE_END(role)                                         \
    do {                                                               \
        if (threadIdx.x == 0 && phase_on_)                             \
            for (int i_ = 0; i_ < 16; ++i_)                            \
                atomicAdd(&gdn_cl_phase_clk[(role)][i_],               \
                          (unsigned long long)gdn_phase_acc_[i_]);     \
    } while (0)
// Per-warp waiting time at selected barriers of the same two CTAs:
// [role][site][warp], accumulated by lane 0 of each warp in shared memory.
__device__ unsigned long long gdn_cl_bar_wait[2][4][8];
static __shared__ unsigned int gdn_bar_acc_[4][8];
#define GDN_BAR_T0() const long long bar_t0_ = clock64()
#define GDN_BAR_T1(site)                                                       \
    do {                                                                       \
        if (phase_on_ && (threadIdx.x & 31) == 0)                              \
            gdn_bar_acc_[(site)][threadIdx.x >> 5] += (unsigned)(clock64() - bar_t0_); \
    } while (0)
#define GDN_BAR_END(role)                                                      \
    do {                                                                       \
        if (phase_on_ && (threadIdx.x & 31) == 0)                              \
            for (int s_ = 0; s_ < 4; ++s_)                                     \
                atomicAdd(&gdn_cl_bar_wait[(role)][s_][threadIdx.x >> 5],      \
                          (unsigned long long)gdn_bar_acc_[s_][threadIdx.x >> 5]); \
    } while (0)
#else
#define GDN_CL_PHASE(role, k) ((void)0)
#define GDN_CL_PHASE_BEGIN() ((void)0)
#define GDN_CL_PHASE_END(role) ((void)0)
#define GDN_BAR_T0() ((void)0)
#define GDN_BAR_T1(site) ((void)0)
#define GDN_BAR_END(role) ((void)0)
#endif

namespace gdn {
namespace {

using namespace sm100;
using namespace tc;

constexpr int kThreads = 256;
constexpr int kCluster = 3;
// producer threads with side duties (first lanes of warps that would otherwise
// reach the end-of-chunk vote early): ring stores, ready signals and tile
// refills; the chunk counter and the ring-slot check
constexpr int kDeliverTid = 64;
constexpr int kFetchTid = 96;
constexpr int kRefillTid = 128;
constexpr int kSlotTid = 192;
// chain thread that polls the ring, loads it, signals taken chunks and stores
// output tiles (thread 0 only issues MMAs, and never waits on L2)
constexpr int kLoadTid = 32;
// chain thread that issues the output tile stores and, before each chunk's
// first CTA barrier, waits until the store issued at the chunk's start has
// read its shared slot (so the load thread, which fences before its ring
// loads, never waits behind an output store)
constexpr int kStoreTid = 64;
constexpr int kGatesWarp = 5;  // loads g, beta and computes the next chunk's gates
constexpr int kClusterRingSlots = 4;
constexpr int kPoolRingSlots = 8;

// ---- chain CTA: two hand-off slots (offsets inside a slot) ----
constexpr uint32_t SL_K16 = 0;         // K fp16: d-halves at +0 / +8192 ([64 rows][128 B], SW128)
constexpr uint32_t SL_QT = 16384;      // Q^T fp16, MN-major [128 d][128 B] (SW128)
constexpr uint32_t SL_WH = 32768;      // W^T hi, same layout
constexpr uint32_t SL_WL = 49152;      // W^T lo, same layout
// Q^T, W^T hi and W^T lo are 16 KB apart: one MN-major B operand of N = 128
// ([Q | W hi]) or N = 192 ([Q | W hi | W lo]) tokens with that atom stride.
static_assert(SL_WH - SL_QT == 16384 && SL_WL - SL_WH == 16384, "stacked B operand");
constexpr uint32_t SL_UT = 65536;      // U~^T fp32 [128 rows][64], 16-byte chunks XOR-swizzled by row
constexpr uint32_t SL_P16 = 98304;     // P fp16 [64 rows][128 B], SW128
constexpr uint32_t SL_GATES = 106496;  // GatesBlock
constexpr uint32_t SLOT_BYTES = 107520;
// reuse of a slot's region once the chain has consumed it
constexpr uint32_t SL_OST = SL_QT;     // o staging [64 tokens][128] bf16, after S Q^T
constexpr uint32_t C_MISC = 2 * SLOT_BYTES;

struct GatesBlock {
    float Gam[kC];   // exp(gamma_r)
    float eC[kC];    // exp(gamma_C - gamma_r)
    int32_t hp;      // extra precision passes for this chunk
    int32_t qs;      // Q^T arrives scaled by Gamma (so the chain need not scale O)
    int32_t hp_next; // the unit's next chunk takes them (it reads the state's lo part)
    int32_t pad;
};
static_assert(sizeof(GatesBlock) % 16 == 0, "bulk copies move multiples of 16 bytes");

struct ChainMisc {
    uint64_t full[2];
    uint64_t ready[2];
    uint64_t mma_bar;
    uint32_t tmem_base;
    alignas(16) uint32_t vote[2][8];  // per-warp vote words of E1 and E2 (read as uint4)
    float red[8];                     // per-warp maxima of a rescale
};
static_assert(offsetof(ChainMisc, vote) % 16 == 0 && C_MISC % 16 == 0, "vote words read as uint4");

// chain TMEM columns (512 allocated):
//   S    0..127   fp32 state (accumulator of nothing: read, scaled, rewritten)
//   SH 128..191   fp16 hi copy of S (A operand); SL 192..255 its lo part,
//                 whose columns 192..223 then hold U^T fp16 (A operand)
//   O  256..319   S Q^T, then the whole transposed chunk output
//   R  320..383   S W^T (S_hi W_hi [+ S_lo W_hi]); R2 384..447 S_hi W_lo;
//                 once both are read, D 320..447 takes the state increment
//   UP 448..511   U' = U diag(Gamma_C / Gamma) as fp16 hi | lo (A operand, K = 128)
constexpr uint32_t CT_S = 0, CT_SH = 128, CT_SL = 192, CT_U16 = 192, CT_O = 256, CT_R = 320,
                   CT_R2 = 384, CT_D = 320, CT_UP = 448;

// ---- producer CTA ----
// A producer work item is one chunk of one sequence for a group of nh v-heads
// that share their q/k head (nh <= 3; 1 in the cluster kernel): the K and Q
// tiles, the Gram matrices, K in fp16 and Q^T are made once per item, and
// everything else once per head, a "step".
constexpr uint32_t P_KQ = 0;            // 2 buffers (by item parity): [K|Q] d-half 0, [K|Q] d-half 1
constexpr uint32_t P_KQ_BYTES = 32768;
constexpr uint32_t P_V = 65536;         // 2 buffers (by step parity): a head's V halves, then its Q^T
constexpr uint32_t P_V_BYTES = 16384;
constexpr int kVBufs = 2;
// Each step's ring stores read their sources asynchronously while the next
// step runs; every source region is rewritten only as late in the next step
// as its use allows, and the delivery thread waits for just the store groups
// that read it right before that point:
//   P (double-buffered)    rewritten at the A / P of the step after next
//   W^T staging            rewritten by the next step's solve (T, X)
//   U~ staging             rewritten by the next step's T tiles
constexpr uint32_t P_X = 98304;         // solve scratch: A, then T and X (fp32)
constexpr uint32_t P_AS = P_X;
constexpr uint32_t P_TS = P_X + 64 * kAS4 * 4;
constexpr uint32_t P_XS = P_TS + 64 * kTS * 4;
constexpr uint32_t P_WST = P_TS;        // W^T hi / lo staging over T and X (32 KB)
constexpr uint32_t P_P16 = 148480;      // 2 buffers (by step parity) of P fp16 [64 rows][128 B], SW128
// T tiles: T diag(b) as bf16 hi / mid / lo and T diag(b Gamma) as fp16 hi / lo,
// each [64 rows][128 B], SW128.  The parts of each are consecutive, so one B
// operand of N = 192 (or 128) rows takes all of them and the MMA writes each
// part's product to its own accumulator columns.
constexpr uint32_t P_TBH = 164864, P_TBM = 173056, P_TBL = 181248, P_TGH = 189440,
                   P_TGL = 197632;
constexpr uint32_t P_UTS = P_TBH;       // then U~^T staging (same layout as SL_UT)
constexpr uint32_t P_MISC = 205824;
constexpr uint32_t P_ID = 209920;       // bf16 identity [64][128 B] (B operand of the Q^T product)
static_assert(P_V == P_KQ + 2 * P_KQ_BYTES && P_X == P_V + kVBufs * P_V_BYTES, "tile buffers");
static_assert(P_WST + 32768 <= P_P16 && P_TBH == P_P16 + 2 * 8192, "staging regions");
static_assert(P_TBM == P_TBH + 8192 && P_TBL == P_TBM + 8192 && P_TGL == P_TGH + 8192,
              "stacked B operands");
static_assert(P_UTS + 32768 <= P_TGL + 8192, "staging fits its region");
static_assert(P_XS + 1024 * 4 <= P_P16, "solve scratch overflows");
static_assert(P_TS % 16 == 0 && P_XS % 16 == 0, "float4 scratch must be aligned");
static_assert(P_P16 % 1024 == 0 && P_TBH % 1024 == 0 && P_ID % 1024 == 0 && P_V % 1024 == 0,
              "swizzled tiles start on 1 KB");

// One work item (one chunk of one sequence for nh v-heads), as a producer
// sees it; head i of the item is v-head h + i, unit unit + i.
struct Item {
    int64_t c0;       // first token
    int32_t unit, c;  // first unit (n * Hv + h); chunk index within the sequence
    int32_t h, j, L;  // first v head, q/k head, valid rows
    int32_t valid;
    int32_t Lnext;    // valid rows of the sequence's next chunk (0: none)
};

// Decay and gate factors of one chunk (double-buffered by chunk parity: the
// next chunk's are computed while this chunk's U~ / W products run).
struct ProdGates {
    float gam[kC], Gam[kC], iGam[kC], eC[kC], bb[kC], bG[kC];
    int32_t safe, hp, qs, hp_next;
};

struct ProdMisc {
    GatesBlock gst;   // gates staging of the chunk being delivered
    ProdGates gt[2];
    Item items[4];    // this CTA's chunks l .. l + 2, by l % 4
    uint64_t tma_bar[2];      // K / Q tiles of an item, by item parity
    uint64_t tma_v[kVBufs];   // V tile of a step, by step parity
    uint64_t mma_bar;
    uint64_t taken;
    uint64_t qt_bar;  // the Q^T product of the current item has landed
    uint32_t tmem_base;
};
static_assert(P_MISC + sizeof(ProdMisc) <= P_ID, "identity tile after the misc block");
// Front end fused into the load stage (kConv): 8-row halo tiles (the 8 tokens
// before a chunk, 128-byte swizzle, 1 KB each) of the raw K and Q inputs (K
// half 0, K half 1, Q half 0, Q half 1) and of the raw V input (half 0, half
// 1), and the filters of the item's k and q heads (2 KB each) and of the
// step's v head (2 KB), in launch_conv_filters' order.  One buffer each: a
// tile's convolution is over before the load of the next one is issued.
constexpr uint32_t P_HKQ = P_ID + 8192;
constexpr uint32_t P_HV = P_HKQ + 4096;
constexpr uint32_t P_FKQ = P_HV + 2048;
constexpr uint32_t P_FV = P_FKQ + 4096;
static_assert(P_HKQ % 1024 == 0 && P_HV % 1024 == 0, "swizzled halo tiles start on 1 KB");
constexpr uint32_t kProdBytes = P_FV + 2048;
constexpr uint32_t kChainBytes = C_MISC + sizeof(ChainMisc);
constexpr uint32_t kSmemBytes = (kProdBytes > kChainBytes ? kProdBytes : kChainBytes) + 1024;
static_assert(kSmemBytes <= 232448, "fits the 227 KB opt-in shared memory of a CTA");

// producer TMEM columns (512 allocated): W^T from T diag(b Gamma)'s hi part (and
// its lo part's product at + 64); the item's Q^T (kept for all its heads);
// U~^T as three products (T diag(b)'s hi, mid, lo parts) at PT_U, + 64, + 128;
// the item's Gram at PT_G, or over W^T's columns when an item has one head
// (where it is dead by the time W^T is made).  Measured: this placement of
// W^T, Q^T and U~^T runs the 262,144-token layer 1 ms faster than W^T at 128
// and Q^T at 64.
constexpr uint32_t PT_W = 0, PT_Q = 128, PT_G = 192, PT_U = 256;
constexpr uint32_t IDESC_MK_N192_BF16 = make_idesc_f16(128, 192, 1, 0, 1);
constexpr uint32_t IDESC_MK_N128 = make_idesc_f16(128, 128, 1, 0);

// pool flags: a header of kFlagHeader words ([0] the chunk counter, [1] the
// abort flag), then 8 words per unit ([0] taken, [1 + s] ready of slot s)
constexpr int kFlagHeader = 64;
constexpr int kFlagsPerUnit = 16;
static_assert(1 + kPoolRingSlots <= kFlagsPerUnit, "flag words per unit");

struct ChainParams {
    uint8_t *ring;    // [unit][ring_slots][SLOT_BYTES]
    uint32_t *flags;  // pool kernel only
    const float *g, *beta, *s0;
    const int32_t *cu;
    void *o;
    float *sT;
    int32_t *err;
    int64_t T;
    int32_t N, Hqk, Hv, units, max_chunks;
    int32_t ring_slots;  // a power of two
    int32_t recall_first;  // GDN_ORDER_RECALL_FIRST: recall before the decay
    long long flag_wait_limit;  // SM clocks a spin on a hand-off flag may last
    int32_t skip_unit;          // testing: a unit no producer prepares (-1: none)
    int32_t nh;                 // v-heads per pool producer item (divides Hv / Hqk, <= 3)
    // front end fused into the load stage: the tiles are the raw inputs of
    // the q, k, v channels, convolved (kernel 4, causal) and, for q and k,
    // normalised per (token, head) before use
    const float *cf;            // filters, as launch_conv_filters writes them
    const float *cstate;        // conv state in, [N][3][cC] (oldest first), or null (zeros)
    int32_t cC;                 // conv-state channels: q (Hqk 128), k (Hqk 128), v (Hv 128)
};

__device__ __forceinline__ uint8_t *ring_slot(const ChainParams &p, int unit, int c) {
    return p.ring + ((size_t)unit * p.ring_slots + (c & (p.ring_slots - 1))) * SLOT_BYTES;
}

__device__ __forceinline__ uint32_t *unit_flags(const ChainParams &p, int unit) {
    return p.flags + kFlagHeader + kFlagsPerUnit * unit;
}

__device__ __forceinline__ void pool_abort(const ChainParams &p) {
    atomicExch(p.flags + 1, 1u);
}

// byte offset of 16-byte chunk q of row i in a [128][64] fp32 U~ tile
__device__ __forceinline__ uint32_t ut_off(int i, int q) {
    return (uint32_t)i * 256u + (uint32_t)((q ^ (i & 15)) << 4);
}

// The item at index i of the pool kernel's chunk-major order: chunk i / G of
// the item's nh units, G = units / nh items per chunk (valid == 0 once the
// order is exhausted).  `skip` is set when index i names no chunk (a shorter
// or malformed sequence): the caller then takes another index.
__device__ Item pool_item(const ChainParams &p, uint32_t i, bool &skip) {
    Item it;
    it.valid = 0;
    skip = false;
    const uint32_t per_chunk = (uint32_t)(p.units / p.nh);
    const int c = (int)(i / per_chunk);
    const int unit = (int)(i % per_chunk) * p.nh;
    if (c >= p.max_chunks) return it;
    if (p.skip_unit >= unit && p.skip_unit < unit + p.nh) {  // testing: a chain starves
        skip = true;
        return it;
    }
    const int n = unit / p.Hv;
    int64_t t0, t1;
    if (!seq_range(p.cu, n, p.N, p.T, nullptr, t0, t1)) {  // the chain reports it
        skip = true;
        return it;
    }
    const int64_t c0 = t0 + (int64_t)kC * c;
    if (c0 >= t1) {  // a shorter sequence
        skip = true;
        return it;
    }
    it.c0 = c0;
    it.unit = unit;
    it.c = c;
    it.h = unit % p.Hv;
    it.j = it.h / (p.Hv / p.Hqk);
    it.L = (int)((t1 - c0) < kC ? (t1 - c0) : kC);
    const int64_t rest = t1 - c0 - kC;
    it.Lnext = (int)(rest <= 0 ? 0 : (rest < kC ? rest : kC));
    it.valid = 1;
    return it;
}

// The next chunk of the order that exists, from index `first` on (invalid once
// the order is exhausted or the abort flag is up).  One thread calls it.
__device__ Item pool_fetch(const ChainParams &p, uint32_t first) {
    uint32_t i = first;
    for (;;) {
        bool skip;
        const Item it = pool_item(p, i, skip);
        if (!skip) return it;
        if (ld_relaxed_gpu(p.flags + 1) != 0u) return Item{0, 0, 0, 0, 0, 0, 0, 0};
        i = atomicAdd(p.flags, 1u);
    }
}

// ------------------------------------------------------------- producer --

// kPool: the pool kernel (items from the global counter, p.nh heads each);
// otherwise producer k of a cluster, whose items are chunks k, k + 2, ... of
// `unit` (one head).  Item l's head i is step s = l * nh + i.
// kConv: the front end is fused into the load stage (pool kernel only): tm_q,
// tm_k, tm_v map the raw inputs of the q, k, v channels and tm_hq, tm_hk,
// tm_hv the same inputs in 8-token boxes, for the tokens before a chunk.
template <bool kPool, int kNh, bool kConv = false>
__device__ void producer_role(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                              const CUtensorMap *tm_v, const ChainParams &p, int unit, int k,
                              int h, int j, int64_t t_begin, int64_t t_end, int nch,
                              const CUtensorMap *tm_hq = nullptr,
                              const CUtensorMap *tm_hk = nullptr,
                              const CUtensorMap *tm_hv = nullptr) {
    ProdMisc *ms = reinterpret_cast<ProdMisc *>(sm + P_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2, row = quad * 32 + lane;
    const uint32_t tmem = ms->tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    // cluster: the chain CTA's ready barrier for this producer (rank 0)
    const uint32_t c_ready =
        kPool ? 0u : mapa_shared(sbase + C_MISC + (uint32_t)offsetof(ChainMisc, ready) + 8u * k, 0);

    // pool: the counter index of the chunk after next, taken at the start of a
    // chunk so that its L2 round trip is over by the time it is decoded
    uint32_t pre_index = 0;
    auto fetch = [&](int l) -> Item {
        if constexpr (kPool) {
            if (l < 2) {
                if (ld_relaxed_gpu(p.flags + 1) != 0u) return Item{0, 0, 0, 0, 0, 0, 0, 0};
                return pool_fetch(p, atomicAdd(p.flags, 1u));
            }
            return pool_fetch(p, pre_index);
        } else {
            Item it;
            const int c = k + 2 * l;
            it.valid = c < nch;
            it.c0 = t_begin + (int64_t)kC * c;
            it.unit = unit;
            it.c = c;
            it.h = h;
            it.j = j;
            it.L = (int)((t_end - it.c0) < kC ? (t_end - it.c0) : kC);
            const int64_t rest = t_end - it.c0 - kC;
            it.Lnext = (int)(rest <= 0 ? 0 : (rest < kC ? rest : kC));
            return it;
        }
    };

    constexpr int nh = kNh;  // heads per item (p.nh in the pool kernel)
    constexpr uint32_t pt_g = kNh == 1 ? PT_W : PT_G;
    uint32_t mma_phase = 0;
    bool timed_out = false;
    float kmax = 0.f;             // largest key-side value this thread has put into fp16
    bool range_reported = false;
    float gpre0 = 0.f, gpre1 = 0.f, bpre0 = 0.f, bpre1 = 0.f;  // gates warp: next chunk's g, beta
    float gnx0 = 0.f, gnx1 = 0.f;  // ... and g of the chunk after it in the same unit
    // g, beta of head hh (0 .. nh - 1) of item `it`, and g of the sequence's next chunk
    auto load_gates = [&](const Item &it, int hh) {
        gpre0 = gpre1 = bpre0 = bpre1 = gnx0 = gnx1 = 0.f;
        const int hv = it.h + hh;
        const int64_t t0_ = it.c0 + 2 * lane, t1_ = t0_ + 1, te = it.c0 + it.L;
        if (t0_ < te) { gpre0 = p.g[t0_ * p.Hv + hv]; bpre0 = p.beta[t0_ * p.Hv + hv]; }
        if (t1_ < te) { gpre1 = p.g[t1_ * p.Hv + hv]; bpre1 = p.beta[t1_ * p.Hv + hv]; }
        const int64_t tn = te + 2 * lane, ten = te + it.Lnext;
        if (tn < ten) gnx0 = p.g[tn * p.Hv + hv];
        if (tn + 1 < ten) gnx1 = p.g[(tn + 1) * p.Hv + hv];
    };
    // K and Q tiles of item `it` into K / Q buffer b (by item parity); with the
    // fused front end also the 8 tokens before the chunk (the coordinate may be
    // negative: the load fills zeros there)
    auto issue_kq = [&](int b, const Item &it) {
        uint8_t *dst = sm + P_KQ + b * P_KQ_BYTES;
        mbar_arrive_expect_tx(&ms->tma_bar[b], kConv ? 4 * 8192 + 4 * 1024 + 4096 : 4 * 8192);
        const int32_t t32 = (int32_t)it.c0;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(dst + hf * 16384, tm_k, &ms->tma_bar[b], 64 * hf, it.j, t32);
            tma_load_3d(dst + hf * 16384 + 8192, tm_q, &ms->tma_bar[b], 64 * hf, it.j, t32);
            if constexpr (kConv) {
                uint8_t *hd = sm + P_HKQ;
                tma_load_3d(hd + hf * 1024, tm_hk, &ms->tma_bar[b], 64 * hf, it.j, t32 - 8);
                tma_load_3d(hd + 2048 + hf * 1024, tm_hq, &ms->tma_bar[b], 64 * hf, it.j, t32 - 8);
            }
        }
        if constexpr (kConv) {  // k head's filters, then q head's
            bulk_load(sm + P_FKQ, p.cf + (int64_t)(p.Hqk + it.j) * 512, 2048, &ms->tma_bar[b]);
            bulk_load(sm + P_FKQ + 2048, p.cf + (int64_t)it.j * 512, 2048, &ms->tma_bar[b]);
        }
    };
    // V tile of head hh of item `it` into V buffer b (by step parity), and its halo
    auto issue_v = [&](int b, const Item &it, int hh) {
        uint8_t *dst = sm + P_V + b * P_V_BYTES;
        mbar_arrive_expect_tx(&ms->tma_v[b], kConv ? 2 * 8192 + 2 * 1024 + 2048 : 2 * 8192);
        const int32_t t32 = (int32_t)it.c0;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(dst + hf * 8192, tm_v, &ms->tma_v[b], 64 * hf, it.h + hh, t32);
            if constexpr (kConv)
                tma_load_3d(sm + P_HV + hf * 1024, tm_hv, &ms->tma_v[b], 64 * hf, it.h + hh,
                            t32 - 8);
        }
        if constexpr (kConv)
            bulk_load(sm + P_FV, p.cf + (int64_t)(2 * p.Hqk + it.h + hh) * 512, 2048, &ms->tma_v[b]);
    };
    // Fused front end: the "kernel 4" causal convolution of one [64 tokens][128]
    // bf16 tile (two 64-feature halves `half0` and `half0` + hstride, 128-byte
    // swizzle), in place, rounded to bf16 once; with `norm`, each token row is
    // divided by its norm first (a zero row stays zero).  Thread (16-byte chunk
    // cch of 8 features, rows 4 rb .. 4 rb + 3) reads its rows and the three
    // before them and works on channel pairs with the two-wide fp32 FMA; the
    // rows before the chunk come from the halo tile (rows 5 .. 7 of the 8
    // tokens before the chunk) or, for a sequence's first chunk, from the
    // carried conv state (or zeros).  `filt`: the head's filters in shared
    // memory (launch_conv_filters' order); `sch`: the conv state's channel of
    // the tile's channel 0.  Every thread reads before anyone writes (one CTA
    // barrier inside).
    auto conv_tile = [&](uint8_t *half0, uint32_t hstride, const uint8_t *halo0, uint32_t halostride,
                         const uint8_t *filt, int sch, const Item &it, bool norm) {
        const int cch = tid & 15, rb = tid >> 4;
        const int hf = cch >> 3, cb = (cch & 7) * 16;
        uint8_t *tile = half0 + hf * hstride;
        const uint8_t *halo = halo0 + hf * halostride;
        float2 x[7][4];  // rows 4 rb - 3 .. 4 rb + 3; channel pairs
#pragma unroll
        for (int i = 0; i < 7; ++i) {
            const int rr = 4 * rb - 3 + i;
            if (rr >= 0 || it.c > 0) {
                const uint4 u = *reinterpret_cast<const uint4 *>(rr >= 0 ? tile + sw128(rr, cb)
                                                                         : halo + sw128(rr + 8, cb));
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    x[i][e] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&wv[e]));
            } else if (p.cstate != nullptr) {  // a sequence's first chunk
                const float *st = p.cstate + ((int64_t)(it.unit / p.Hv) * 3 + rr + 3) * p.cC + sch + 8 * cch;
#pragma unroll
                for (int e = 0; e < 4; ++e) x[i][e] = make_float2(st[2 * e], st[2 * e + 1]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[i][e] = make_float2(0.f, 0.f);
            }
        }
        float2 y[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // tap k multiplies row t - 3 + k
            const float4 w0 = *reinterpret_cast<const float4 *>(filt + k * 512 + cch * 16);
            const float4 w1 = *reinterpret_cast<const float4 *>(filt + k * 512 + 256 + cch * 16);
            const float2 wk[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w),
                                  make_float2(w1.x, w1.y), make_float2(w1.z, w1.w)};
#pragma unroll
            for (int jr = 0; jr < 4; ++jr)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    y[jr][e] = k == 0 ? fmul2(wk[e], x[jr][e]) : ffma2(wk[e], x[jr + k][e], y[jr][e]);
        }
        float2 inv[4];
#pragma unroll
        for (int jr = 0; jr < 4; ++jr) inv[jr] = make_float2(1.f, 1.f);
        if (norm) {  // the 16 lanes of a row (lanes 16 (rb & 1) .. + 15) hold its 128 features
#pragma unroll
            for (int jr = 0; jr < 4; ++jr) {
                float2 s2 = fmul2(y[jr][0], y[jr][0]);
#pragma unroll
                for (int e = 1; e < 4; ++e) s2 = ffma2(y[jr][e], y[jr][e], s2);
                float ss = s2.x + s2.y;
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float iv = ss > 0.f ? 1.f / sqrtf(ss) : 1.f;
                inv[jr] = make_float2(iv, iv);
            }
        }
        __syncthreads();  // every read of the tile is done
#pragma unroll
        for (int jr = 0; jr < 4; ++jr) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 o2 = fmul2(y[jr][e], inv[jr]);
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(o2.x, o2.y);
                wv[e] = *reinterpret_cast<const uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(tile + sw128(4 * rb + jr, cb)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    };
    auto mma_sync_point = [&]() {
        if (tid == 0) mma_commit(&ms->mma_bar);
        if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
        mma_phase ^= 1;
        tc_fence_after_sync();
    };
    auto publish = [&]() {
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };

    // The delivery thread's chunks whose ring stores are in flight and not yet
    // reported ready: the last one delivered (pending) and, in the pool kernel,
    // the one before it (older).  valid == 0: none.
    Item pending, older;
    pending.valid = 0;
    older.valid = 0;
    auto signal_ready = [&](const Item &d) {  // its stores have completed
        if constexpr (kPool)
            st_release_gpu(unit_flags(p, d.unit) + 1 + (d.c & (p.ring_slots - 1)),
                           (uint32_t)(d.c + 1));
        else
            mbar_arrive_remote(c_ready);
    };
    auto flush_delivery = [&]() {  // delivery thread only: every delivery held
        if (!pending.valid && !older.valid) return;
        bulk_wait_all();              // written to global memory
        fence_proxy_async_global();   // ... ordered before the signals below
        if (older.valid) signal_ready(older);
        if (pending.valid) signal_ready(pending);
        older.valid = 0;
        pending.valid = 0;
    };
    // Pool kernel: the delivery before the last one, whose stores landed long
    // ago (two bulk groups per delivery: the last delivery's may still be in
    // flight).  Signalling one chunk late keeps the wait for the 105 KB of
    // stores to land off the producer's path; the ring's depth absorbs the
    // extra latency.
    auto flush_older = [&]() {
        if (!older.valid) return;
        bulk_wait_all_but_two();
        fence_proxy_async_global();
        signal_ready(older);
        older.valid = 0;
    };

    // Gates of a chunk from the g, beta values in gpre / bpre (the gates warp, two
    // tokens per lane): cumulative log-decay gamma, Gamma = exp(gamma), the
    // factors of A, P, W and U', and the precision choice.
    auto compute_gates = [&](ProdGates &gt) {
        float x1 = gpre0 + gpre1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, x1, off);
            if (lane >= off) x1 += y;
        }
        const float x0 = x1 - gpre1;
        const float gC = __shfl_sync(0xffffffffu, x1, 31);
        float m = fmaxf(fabsf(x0), fabsf(x1)), top = fmaxf(x0, x1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, off));
        }
        const bool safe_ = m <= 60.f;  // every exp(+-gamma) a normal float
        const float G0 = expf(x0), G1 = expf(x1);
        const float GC = __shfl_sync(0xffffffffu, G1, 31);
        const int r0 = 2 * lane;
        gt.gam[r0] = x0;                gt.gam[r0 + 1] = x1;
        gt.Gam[r0] = G0;                gt.Gam[r0 + 1] = G1;
        if (safe_) {  // 1 / Gamma and Gamma_C / Gamma from the exponentials above
            const float i0 = 1.f / G0, i1 = 1.f / G1;
            gt.iGam[r0] = i0;           gt.iGam[r0 + 1] = i1;
            gt.eC[r0] = GC * i0;        gt.eC[r0 + 1] = GC * i1;
        } else {
            gt.iGam[r0] = 0.f;          gt.iGam[r0 + 1] = 0.f;
            gt.eC[r0] = expf(gC - x0);  gt.eC[r0 + 1] = expf(gC - x1);
        }
        gt.bb[r0] = bpre0;              gt.bb[r0 + 1] = bpre1;
        // decay of token r's recall terms (in A and W): Gamma_r, or Gamma_{r-1}
        // when the recall is taken before the decay (Gamma_{-1} = 1)
        const float xp = __shfl_up_sync(0xffffffffu, x1, 1);  // gamma at token 2l - 1
        const float Gr0 = p.recall_first ? (lane > 0 ? expf(xp) : 1.f) : G0;
        const float Gr1 = p.recall_first ? G0 : G1;
        gt.bG[r0] = bpre0 * Gr0;        gt.bG[r0 + 1] = bpre1 * Gr1;
        // the precision choice of this chunk and of the unit's next one, from the
        // same sum in the same order as the next chunk's own producer takes it
        const float gsum = warp_sum(gpre0 + gpre1), gsum_next = warp_sum(gnx0 + gnx1);
        if (lane == 0) {
            gt.safe = safe_;
            gt.hp = gsum >= kLogHighPrecisionDecay;
            gt.hp_next = gsum_next >= kLogHighPrecisionDecay;
            // Q^T is scaled by Gamma <= 1 only: Gamma q then cannot overflow fp16
            gt.qs = safe_ && top <= 0.f;
        }
    };

    // Items l and l + 1 are known when item l starts (item l + 2 is fetched
    // during the U~ / W products of its first step).  The K / Q tiles of item
    // 0 and the V tile of step 0 are loaded here; those of item l + 1 during
    // the U~ / W products of item l's last step, and the V tile of step s + 1
    // during those of step s (its buffer held step s - 2's, whose stores have
    // read it by then).
    if (tid == kFetchTid) {
        for (int l = 0; l < 2; ++l) ms->items[l] = fetch(l);
        if (ms->items[0].valid) {
            issue_kq(0, ms->items[0]);
            issue_v(0, ms->items[0], 0);
        }
    }
    // the bf16 identity, K-major with the 128-byte swizzle: row n holds 1 at k = n
    for (int x = tid; x < 512; x += kThreads) {  // 512 chunks of 16 bytes
        const int n = x >> 3, ch = x & 7;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if ((n >> 3) == ch) {
            uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
            wp[(n & 7) >> 1] = (n & 1) ? 0x3f800000u : 0x00003f80u;  // bf16 1.0 in the right half
        }
        st_row_chunk(sm + P_ID, n, ch, w);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (warp == kGatesWarp && ms->items[0].valid) {
        load_gates(ms->items[0], 0);
        compute_gates(ms->gt[0]);
    }
    __syncthreads();
#ifdef GDN_TC_PHASES
    const bool phase_on_ = blockIdx.x == (kPool ? (unsigned)p.units : 1u);
#endif
    GDN_CL_PHASE_BEGIN();
    int s = 0, l = 0, hi = 0;  // step, its item and head within the item
    bool broke = false;
    int v_loaded = 1;  // steps whose V tile load has been issued
    int kq_loaded = 1; // items whose K / Q tile load has been issued
#pragma unroll 1
    for (;; ++s) {
        l = s / nh;
        hi = s - l * nh;
        const Item item = ms->items[l & 3];
        if (!item.valid) break;
        Item it = item;  // this step's head: v-head item.h + hi, unit item.unit + hi
        it.h += hi;
        it.unit += hi;
        const int L = it.L;
        const int buf = l & 1;
        const int vb = s % kVBufs;
        const ProdGates &gt = ms->gt[s & 1];

        // the next step's g, beta: in flight until its gates are computed
        if (warp == kGatesWarp) {
            const int ln = (s + 1) / nh, hn = (s + 1) - ln * nh;
            const Item nx = ms->items[ln & 3];
            if (nx.valid) load_gates(nx, hn);
        }
        // pool: the index of item l + 2 (first step of an item) and an early
        // look at this step's ring slot, both consumed later in the step
        uint32_t early_taken = 0;
        if constexpr (kPool) {
            if (tid == kFetchTid && hi == 0) pre_index = atomicAdd(p.flags, 1u);
            if (tid == kDeliverTid && it.c >= p.ring_slots)
                early_taken = ld_relaxed_gpu(unit_flags(p, it.unit));
        }
        GDN_CL_PHASE(1, 0);  // gates
        GDN_CL_PHASE(1, 1);  // (no wait)
        uint8_t *kqv = sm + P_KQ + buf * P_KQ_BYTES;
        const uint32_t skqv = sbase + P_KQ + buf * P_KQ_BYTES;
        uint8_t *vt = sm + P_V + vb * P_V_BYTES;
        const uint32_t svt = sbase + P_V + vb * P_V_BYTES;
        // ---- first step of an item: K / Q tiles, the Gram [K;Q] K^T straight from
        //      the bf16 tiles (exact products either way), K to fp16 ----
        if (hi == 0) {
        if (!mbar_wait_bounded(&ms->tma_bar[buf], (l >> 1) & 1, kWaitLimit)) timed_out = true;
        GDN_CL_PHASE(1, 2);  // wait: tiles
        if constexpr (kConv) {
            // the item's raw k and q tiles -> convolved, each (token, head) row
            // normalised, rounded to bf16 once, in place
            conv_tile(kqv, 16384, sm + P_HKQ, 1024, sm + P_FKQ, p.Hqk * kD + item.j * kD, item, true);
            conv_tile(kqv + 8192, 16384, sm + P_HKQ + 2048, 1024, sm + P_FKQ + 2048, item.j * kD,
                      item, true);
            fence_proxy_async_smem();  // -> visible to the Gram and Q^T products
            __syncthreads();
        }
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t a = skqv + (ks >> 2) * 16384 + (ks & 3) * 32;
                mma_f16_ss(tmem + pt_g, make_sdesc(a, 16, 1024), make_sdesc(a, 16, 1024),
                           IDESC_KK_N64_BF16, ks > 0);
            }
            mma_commit(&ms->mma_bar);
        }
        // K goes from bf16 to fp16 in place (padding rows zeroed) once the Gram
        // products have read it: the chain's state update takes it in fp16.
        // V stays bf16 (the U~ product splits its other operand three ways in
        // bf16), and Q goes to fp16 in the Q^T transpose.
        auto convert16 = [&](uint8_t *base, int x) {  // 16-byte chunk x of a [64][128 B] tile
            uint4 *ptr = reinterpret_cast<uint4 *>(base) + x;
            const int r = x >> 3;
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
        // A / P rewrites the P buffer that the step before last's first store
        // group read: wait until it has been read (the last step's groups may
        // still be reading).
        if (tid == kDeliverTid) bulk_wait_read_all_but_two();
        {
            GDN_BAR_T0();
            __syncthreads();
            GDN_BAR_T1(1);
        }
#pragma unroll
        for (int q = 0; q < 1024 / kThreads; ++q) {
            const int x = tid + q * kThreads;  // K halves: 2 x 512 chunks
            convert16(kqv + (x >> 9) * 16384, x & 511);
        }
        } else {
        // a later step of the item: only the store-group wait above
        if (tid == kDeliverTid) bulk_wait_read_all_but_two();
        {
            GDN_BAR_T0();
            __syncthreads();
            GDN_BAR_T1(1);
        }
        }
        const bool hp = gt.hp;
        const bool safe = gt.safe;
        GDN_CL_PHASE(1, 3);  // Gram + convert
        GDN_CL_PHASE(1, 4);  // (merged)

        // ---- A (lanes 0..63) and P (lanes 64..127) ----
        float *As = reinterpret_cast<float *>(sm + P_AS);
        float *Ts = reinterpret_cast<float *>(sm + P_TS);
        float *Xs = reinterpret_cast<float *>(sm + P_XS);
        {
            const int r = row & 63;
            const int c = 32 * half;
            float v[32];
            tmem_ld32(trow + pt_g + c, v);
            tmem_wait_ld();
            if (safe) {
                const float sr = row < kC ? gt.bG[r] : gt.Gam[r];
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] *= sr * gt.iGam[c + x];
            } else {
                const float gr = (row < kC && p.recall_first) ? (r > 0 ? gt.gam[r - 1] : 0.f)
                                                              : gt.gam[r];
                const float sr = row < kC ? gt.bb[r] : 1.f;
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] *= sr * expf(gr - gt.gam[c + x]);
            }
            if (row < kC) {
#pragma unroll
                for (int x = 0; x < 32; x += 4)  // 16-byte stores: conflict-free at stride kAS4
                    *reinterpret_cast<float4 *>(As + r * kAS4 + c + x) =
                        make_float4((c + x < r) ? v[x] : 0.f, (c + x + 1 < r) ? v[x + 1] : 0.f,
                                    (c + x + 2 < r) ? v[x + 2] : 0.f, (c + x + 3 < r) ? v[x + 3] : 0.f);
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] = (c + x <= r) ? v[x] : 0.f;
#pragma unroll
                for (int e = 0; e < 32; e += 8)
                    st_row_chunk(sm + P_P16 + (s & 1) * 8192, r, (c + e) / 8,
                                 pack8_track(v + e, kmax));
            }
        }
        // the solve rewrites the last step's W^T staging (its first store group)
        if (tid == kDeliverTid) bulk_wait_read_all_but_one();
        __syncthreads();
        GDN_CL_PHASE(1, 5);  // A / P

        // ---- Q^T = Q^T I on the tensor cores while the solve runs (exact: bf16 x 1),
        //      once per item ----
        if (tid == 0 && hi == 0) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16_ss(tmem + PT_Q, make_sdesc(skqv + 8192 + ks * 2048, 16384, 1024),
                           make_sdesc(sbase + P_ID + ks * 32, 16, 1024), IDESC_MK_N64_BF16, ks > 0);
            mma_commit(&ms->qt_bar);
        }

        // ---- T = (I + A)^-1 ----
        solve_tril64(As, Ts, Xs, tid);
        // The T tiles below overwrite the last step's U~ staging: its stores
        // must have read it.  (Waiting for those stores to land, and signalling
        // the chunk ready, comes later, in the U~ / W window.)
        if (tid == kDeliverTid) bulk_wait_read_all();
        {
            GDN_BAR_T0();
            __syncthreads();
            GDN_BAR_T1(2);
        }
        GDN_CL_PHASE(1, 6);  // solve

        // ---- rows of T diag(b) (bf16 hi / mid / lo: exact, and V needs no
        //      conversion) and T diag(b Gamma) (fp16 hi / lo, as K): thread
        //      (row r, quarter cq) does columns 16 cq .. 16 cq + 15 of both ----
        {
            const int r = tid & 63, cq = tid >> 6;
            float tb[16], tg[16];
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 t4 = *reinterpret_cast<const float4 *>(Ts + r * kTS + 16 * cq + e);
                const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = 16 * cq + e + q;
                    tb[e + q] = (i <= r) ? tv[q] * gt.bb[i] : 0.f;
                    tg[e + q] = (i <= r) ? tv[q] * gt.bG[i] : 0.f;
                }
            }
            kmax = fmaxf(kmax, max_abs<16>(tg));
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
                uint4 hi, mid, lo;
                split8_bf16x3(tb + e, hi, mid, lo);
                const int ch = (16 * cq + e) / 8;
                st_row_chunk(sm + P_TBH, r, ch, hi);
                st_row_chunk(sm + P_TBM, r, ch, mid);
                st_row_chunk(sm + P_TBL, r, ch, lo);
                split8(tg + e, hi, lo);
                st_row_chunk(sm + P_TGH, r, ch, hi);
                if (hp) st_row_chunk(sm + P_TGL, r, ch, lo);
            }
        }
        if constexpr (kConv) {
            // this head's raw v tile -> convolved, rounded to bf16 in place
            if (!mbar_wait_bounded(&ms->tma_v[vb], (s / kVBufs) & 1, kWaitLimit)) timed_out = true;
            conv_tile(vt, 8192, sm + P_HV, 1024, sm + P_FV, 2 * p.Hqk * kD + it.h * kD, it, false);
        }
        {
            GDN_BAR_T0();
            publish();
            GDN_BAR_T1(3);
        }
        GDN_CL_PHASE(1, 7);  // T tiles

        // ---- U~^T = V^T (T diag b)^T,  W^T = K^T (T diag(b Gamma))^T ----
        if (tid == 0) {
            if (!mbar_wait_bounded(&ms->tma_v[vb], (s / kVBufs) & 1, kWaitLimit)) timed_out = true;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // bf16 V times [hi | mid | lo] of T diag(b)
                const uint64_t a = make_sdesc(svt + ks * 2048, 8192, 1024);
                const uint64_t b = make_sdesc(sbase + P_TBH + ks * 32, 16, 1024);
                mma_f16_ss(tmem + PT_U, a, b, IDESC_MK_N192_BF16, ks != 0);
            }
            const uint32_t idesc_w = hp ? IDESC_MK_N128 : IDESC_MK_N64;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {  // fp16 K times [hi | lo] of T diag(b Gamma)
                const uint64_t a = make_sdesc(skqv + ks * 2048, 16384, 1024);
                const uint64_t b = make_sdesc(sbase + P_TGH + ks * 32, 16, 1024);
                mma_f16_ss(tmem + PT_W, a, b, idesc_w, ks != 0);
            }
            mma_commit(&ms->mma_bar);
        }
        if (warp == kGatesWarp) {
            const int ln = (s + 1) / nh;
            if (ms->items[ln & 3].valid) compute_gates(ms->gt[(s + 1) & 1]);
        }
        // side duties while these products run
        if (tid == kRefillTid) {  // tile loads into buffers whose stores have read them
            const int ln = (s + 1) / nh, hn = (s + 1) - ln * nh;
            const Item nv = ms->items[ln & 3];
            if (nv.valid) {  // step s + 1's V tile
                issue_v((s + 1) % kVBufs, nv, hn);
                v_loaded = s + 2;
            }
            const Item nk = ms->items[(l + 1) & 3];
            if (hi == nh - 1 && nk.valid) {  // item l + 1's K / Q tiles
                issue_kq((l + 1) & 1, nk);
                kq_loaded = l + 2;
            }
        }
        if (tid == kFetchTid && hi == 0) ms->items[(l + 2) & 3] = fetch(l + 2);  // decode item l + 2
        if constexpr (kPool) {
            if (tid == kDeliverTid) {  // earlier deliveries -> ready; this chunk's ring slot free
                const uint32_t need = (uint32_t)(it.c - p.ring_slots + 1);
                // a free slot seen early needs no fence: the stores that refill it
                // depend on that observation, and the chain publishes it only after
                // its load of the slot has completed
                if (it.c >= p.ring_slots && early_taken < need) {
                    // about to wait on a chain: first report every delivery held,
                    // so that no producer waits while holding one back
                    flush_delivery();
                    if (!wait_flag_geq(unit_flags(p, it.unit), need, p.flags + 1,
                                       p.flag_wait_limit))
                        timed_out = true;
                } else {
                    flush_older();
                }
            }
        } else {
            if (tid == kDeliverTid) flush_delivery();  // the previous chunk, landed -> ready
            if (tid == kSlotTid) {  // make sure this chunk's ring slot is free
                if (l >= 1 && !mbar_wait_cluster_bounded(&ms->taken, (l - 1) & 1, kWaitLimit))
                    timed_out = true;
            }
        }
        if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
        mma_phase ^= 1;
        tc_fence_after_sync();
        GDN_CL_PHASE(1, 8);  // U~ / W MMAs

        // ---- staging: W^T hi/lo (MN-major), U~^T (swizzled fp32), gates, Q^T ----
        {
            const int c = 32 * half;
            float v[32];
            tmem_ld32(trow + PT_W + c, v);
            if (hp) {
                float w2[32];
                tmem_ld32(trow + PT_W + 64 + c, w2);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] += w2[x];
            }
            tmem_wait_ld();
            store_split32(sm + P_WST, sm + P_WST + 16384, row, c, v, hp, kmax);
            {
                float u1[32], u2[32];
                tmem_ld32(trow + PT_U + c, v);
                tmem_ld32(trow + PT_U + 64 + c, u1);
                tmem_ld32(trow + PT_U + 128 + c, u2);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] += u1[x] + u2[x];
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4 *>(sm + P_UTS + ut_off(row, c / 4 + q)) =
                    make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            if (tid < kC) {
                ms->gst.Gam[tid] = gt.Gam[tid];
                ms->gst.eC[tid] = gt.eC[tid];
            }
            if (tid == 0) {
                ms->gst.hp = hp;
                ms->gst.qs = gt.qs;
                ms->gst.hp_next = gt.hp_next;
            }
        }
        {   // Q^T fp16 (MN-major: row d holds 64 tokens) from TMEM into this step's V
            // buffer, which the U~ product has finished reading; scaled by this
            // head's Gamma when the gates allow (qs); tokens past L zeroed
            if (!mbar_wait_bounded(&ms->qt_bar, l & 1, kWaitLimit)) timed_out = true;
            tc_fence_after_sync();
            const int c = 32 * half;
            float v[32];
            tmem_ld32(trow + PT_Q + c, v);
            tmem_wait_ld();
            const bool qs = gt.qs;
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const float sc = qs ? gt.Gam[c + x] : 1.f;
                v[x] = (c + x < L) ? v[x] * sc : 0.f;
            }
#pragma unroll
            for (int e = 0; e < 32; e += 8)
                st_row_chunk(vt, row, (c + e) / 8, pack8_track(v + e, kmax));
        }
        fence_proxy_async_smem();  // staged data -> visible to the bulk copies
        // a key-side fp16 operand of this chunk (K, Q^T, P, T diag(b Gamma), W^T)
        // overflowed: report it once per thread (the unit's results are then
        // unspecified; the computation goes on)
        if (kmax >= kFp16Overflow && !range_reported) {
            raise_error(p.err, GDN_ERR_RANGE);
            range_reported = true;
        }
        GDN_CL_PHASE(1, 9);  // staging

        // ---- deliver with asynchronous stores (the ring slot is free: see above) ----
        GDN_BAR_T0();
        const int voted_ = __syncthreads_or(timed_out ? 1 : 0);
        GDN_BAR_T1(0);
        if (voted_) {
            if (tid == 0) {
                raise_error(p.err, GDN_ERR_TIMEOUT);
                if constexpr (kPool) pool_abort(p);
            }
            broke = true;
            break;
        }
        GDN_CL_PHASE(1, 10);  // wait: ring slot free
        if (tid == kDeliverTid) {
            uint8_t *dst = ring_slot(p, it.unit, it.c);
            fence_proxy_async_global();  // the chain's reads of this slot precede our writes
            // group 1: what the next chunk rewrites first (read before its A / P)
            bulk_store(dst + SL_WH, sm + P_WST, hp ? 32768 : 16384);
            bulk_store(dst + SL_P16, sm + P_P16 + (s & 1) * 8192, 8192);
            bulk_store(dst + SL_GATES, &ms->gst, (uint32_t)sizeof(GatesBlock));
            bulk_commit();
            // group 2: U~ (in the T tiles' space), K (in the item's K / Q buffer)
            // and Q^T (in the step's V buffer)
            bulk_store(dst + SL_UT, sm + P_UTS, 32768);
            bulk_store(dst + SL_K16, kqv, 8192);
            bulk_store(dst + SL_K16 + 8192, kqv + 16384, 8192);
            bulk_store(dst + SL_QT, vt, 16384);
            bulk_commit();
            older = pending;  // pool: signalled during the next chunk (cluster: already)
            pending = it;
        }
        GDN_CL_PHASE(1, 11);  // deliver (issue)
    }
    if (tid == kDeliverTid) flush_delivery();  // the last chunk delivered
    GDN_CL_PHASE_END(1);
    GDN_BAR_END(1);
    // Tile loads issued for steps or items this loop never reached must land
    // before this CTA's shared memory can go away (after a timeout; on a
    // normal exit nothing is in flight).
    if (broke) {  // (waiting again on a phase that completed returns at once)
        for (int ss = s; ss < v_loaded; ++ss)
            mbar_wait_bounded(&ms->tma_v[ss % kVBufs], (ss / kVBufs) & 1, kWaitLimit);
        for (int ll = l; ll < kq_loaded; ++ll)
            mbar_wait_bounded(&ms->tma_bar[ll & 1], (ll >> 1) & 1, kWaitLimit);
    }
}

// ---------------------------------------------------------------- chain --

template <bool kPool>
__device__ void chain_role(uint8_t *sm, const CUtensorMap *tm_o, const ChainParams &p, int unit,
                           int n, int h, int64_t t_begin, int64_t t_end, int nch) {
    ChainMisc *ms = reinterpret_cast<ChainMisc *>(sm + C_MISC);
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2, row = quad * 32 + lane;
    const uint32_t tmem = ms->tmem_base;
    const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
    // cluster: producer-CTA "taken" barriers (rank 1 + k)
    const uint32_t prod_taken_local = sbase + P_MISC + (uint32_t)offsetof(ProdMisc, taken);
    uint32_t *uflags = kPool ? unit_flags(p, unit) : nullptr;
    (void)warp;

    // Value-side operands are held with a power-of-two scale, uniform over
    // the unit: the fp32 master state in TMEM is S * 2^-es, and its fp16 hi /
    // lo copies (the A operand of S [Q^T | W^T]) are split from it directly,
    // so the products come out scaled by 2^-es.  U and U' are held as
    // U * 2^-eu, where eu is es unless U's magnitudes leave the band
    // [kScaleLo, kScaleHi) in that scale.  Every epilogue votes on its
    // largest scaled magnitude; the rare chunk whose values left the band
    // recomputes them in fp32 and takes a new scale (fp16_scale_exp).  The
    // scaling is exact, so no value-side operand over- or underflows fp16,
    // whatever the scale of v and S0, and the results scale exactly with it.
    int es = 0, eu = 0;
    float s_up = 1.f, sd = 1.f;  // 2^es, 2^-es
    auto set_es = [&](int e) {
        es = e;
        s_up = exp2i(e);
        sd = exp2i(-e);
    };
    // 64 values of this thread's state row (scaled) -> the hi (and lo) TMEM
    // operands; the lo part only when the next chunk's products read it
    auto split_state = [&](const float (&sv)[64], bool with_lo) {
        uint32_t hi[32];
        if (with_lo) {
            uint32_t lo[32];
#pragma unroll
            for (int x = 0; x < 64; x += 2) {
                const __half2 hh = __floats2half2_rn(sv[x], sv[x + 1]);
                const float2 hf = __half22float2(hh);
                hi[x / 2] = *reinterpret_cast<const uint32_t *>(&hh);
                lo[x / 2] = pack_half2(sv[x] - hf.x, sv[x + 1] - hf.y);
            }
            tmem_st32u(trow + CT_SL + 32 * half, lo);
        } else {
#pragma unroll
            for (int x = 0; x < 64; x += 2) hi[x / 2] = pack_half2(sv[x], sv[x + 1]);
        }
        tmem_st32u(trow + CT_SH + 32 * half, hi);
    };
    auto store_state = [&](const float (&sv)[64]) {  // the scaled fp32 master
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float v[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = sv[32 * part + x];
            tmem_st32(trow + CT_S + 64 * half + 32 * part, v);
        }
    };

    // ---- initial state: scaled fp32 -> TMEM accumulator, fp16 hi/lo -> TMEM A operands ----
    {
        const float *src = p.s0 ? p.s0 + (((int64_t)n * p.Hv + h) * kD + row) * kD + 64 * half : nullptr;
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
        store_state(sv);
        split_state(sv, true);
        tmem_wait_st();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    uint32_t mma_phase = 0;
    bool timed_out = false, aborted = false;
    auto mma_sync_point = [&]() {
        if (tid == 0) mma_commit(&ms->mma_bar);
        if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
        mma_phase ^= 1;
        tc_fence_after_sync();
    };
    auto publish = [&]() {
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before_sync();
        __syncthreads();
        tc_fence_after_sync();
    };
    // Has chunk cc reached the ring?  (load thread)  The pool kernel reads the
    // flag with a relaxed load whose value is only examined on a later call,
    // so the L2 round trip overlaps other work; an observed flag is turned
    // into an acquire by reading it again with an acquire load (a gpu-scope
    // fence there held the load thread, and the barrier after it, for over a
    // thousand cycles).
    uint32_t polled = 0;
    int polled_for = -1;  // the chunk whose flag `polled` holds
    auto read_flag = [&](int cc) {
        if constexpr (kPool) {
            polled = ld_relaxed_gpu(uflags + 1 + (cc & (p.ring_slots - 1)));
            polled_for = cc;
        }
    };
    auto ready_try = [&](int cc) -> bool {
        if constexpr (kPool) {
            if (polled_for == cc && polled >= (uint32_t)(cc + 1)) {
                // acquire: re-read the flag (it only grows) with an acquire load,
                // which costs far less than a gpu-scope fence
                (void)ld_acquire_gpu(uflags + 1 + (cc & (p.ring_slots - 1)));
                polled_for = -1;
                return true;
            }
            read_flag(cc);
            return false;
        } else {
            return mbar_try_wait_cluster(&ms->ready[cc & 1], ((cc >> 1) & 1));
        }
    };
    auto ready_wait = [&](int cc) -> bool {
        if constexpr (kPool)
            return wait_flag_geq(uflags + 1 + (cc & (p.ring_slots - 1)), (uint32_t)(cc + 1), p.flags + 1,
                                 p.flag_wait_limit);
        else
            return mbar_wait_cluster_bounded(&ms->ready[cc & 1], (cc >> 1) & 1, kWaitLimit);
    };

#ifdef GDN_TC_PHASES
    const bool phase_on_ = blockIdx.x == 0;
#endif
    GDN_CL_PHASE_BEGIN();
    // The load thread loads chunk c + 1 from the ring into shared slot (c + 1) & 1 as
    // soon as it is reported ready, while chunk c is processed; the shared
    // slot held chunk c - 1, which is finished.
    int loaded = 0;  // chunks whose load has been issued
    // (the output tile store from this shared slot has read it: the store
    // thread waited for that before an earlier CTA barrier)
    auto issue_load = [&](int cc) {  // four copies, which the copy engine can overlap
        fence_proxy_async_global();  // the producer's stores, acquired, precede our bulk load
        uint64_t *bar = &ms->full[cc & 1];
        mbar_arrive_expect_tx(bar, SLOT_BYTES);
        uint8_t *dst = sm + (cc & 1) * SLOT_BYTES;
        const uint8_t *src = ring_slot(p, unit, cc);
        bulk_load(dst, src, SL_WH, bar);                                   // K, Q^T
        bulk_load(dst + SL_WH, src + SL_WH, SL_UT - SL_WH, bar);           // W^T hi, lo
        bulk_load(dst + SL_UT, src + SL_UT, SL_P16 - SL_UT, bar);          // U~^T
        bulk_load(dst + SL_P16, src + SL_P16, SLOT_BYTES - SL_P16, bar);   // P, gates
    };
    // cur: the chunk in progress; the shared slot of chunk cur + 1 is free.
    // Loads chunk cur + 1 once it is ready; when it is loaded already, starts
    // reading the flag of chunk cur + 2 (its slot frees up with chunk cur).
    auto poll_next = [&](int cur) {
        if (tid != kLoadTid) return;
        if (loaded == cur + 1 && cur + 1 < nch) {
            if (ready_try(cur + 1)) {
                issue_load(cur + 1);
                loaded = cur + 2;
            }
        } else if (loaded == cur + 2 && cur + 2 < nch && polled_for != cur + 2) {
            read_flag(cur + 2);
        }
    };
    // Only starts reading chunk cur + 1's flag (no fence, no load).
    auto poll_read = [&](int cur) {
        if (tid == kLoadTid && loaded == cur + 1 && cur + 1 < nch) read_flag(cur + 1);
    };
    // Chunk cc's output from its staging area (the consumed Q^T region of its
    // shared slot) to global memory: a full chunk as one tile store issued by
    // the store thread (which waits for it to read the slot before the next
    // CTA barrier: the slot is reloaded after that); the last, partial chunk
    // of a sequence with 16-byte stores of warps 2..7, so nothing past the
    // sequence is written.  Warps 0 and 1 take no part in either: the MMA
    // thread and the load thread fence, and a fence waits for the issuing
    // thread's own outstanding stores.
    auto store_o = [&](int cc) {
        const int64_t cc0 = t_begin + (int64_t)kC * cc;
        const int cL = (int)((t_end - cc0) < kC ? (t_end - cc0) : kC);
        const uint8_t *ostb = sm + (cc & 1) * SLOT_BYTES + SL_OST;
        if (cL == kC) {
            if (tid == kStoreTid) {
                tma_store_3d(tm_o, ostb, 0, h, (int32_t)cc0);
                bulk_commit();
            }
            return;
        }
        if (warp <= 1) return;
        const uint4 *ost = reinterpret_cast<const uint4 *>(ostb);
        constexpr int kStorers = kThreads - 64;
#pragma unroll
        for (int q = 0; q < (kC * kD * 2 / 16 + kStorers - 1) / kStorers; ++q) {
            const int x = (tid - 64) + q * kStorers;
            const int r = x >> 4, c16 = x & 15;
            if (x < kC * kD * 2 / 16 && r < cL) {
                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.o) +
                                                       ((cc0 + r) * p.Hv + h) * (int64_t)kD) + c16;
                *dst = ost[x];
            }
        }
    };
    int c = 0;
#pragma unroll 1
    for (; c < nch && !aborted; ++c) {
        const int k = c & 1;
        uint8_t *slot = sm + k * SLOT_BYTES;
        const uint32_t sslot = sbase + k * SLOT_BYTES;
        bool have = true;
        if (tid == kLoadTid && loaded == c) {  // not prefetched: wait for the producer, then load
            if (ready_wait(c)) {
                issue_load(c);
                loaded = c + 1;
            } else {
                // Nothing will land: complete the slot's phase by hand so that no
                // thread waits for it; the vote at the end of the chunk aborts.
                timed_out = true;
                have = false;
                mbar_arrive(&ms->full[k]);
            }
        }
        {
            GDN_BAR_T0();
            if (!mbar_wait_bounded(&ms->full[k], (c >> 1) & 1, kWaitLimit)) timed_out = true;
            GDN_BAR_T1(3);
        }
        GDN_CL_PHASE(0, 0);  // wait: delivery
        if (tid == kLoadTid && have) {  // the chunk is out of the ring: its slot may be refilled
            if constexpr (kPool)
                st_relaxed_gpu(uflags, (uint32_t)(c + 1));
            else
                mbar_arrive_remote(mapa_shared(prod_taken_local, 1 + k));
        }
        const GatesBlock *gb = reinterpret_cast<const GatesBlock *>(slot + SL_GATES);
        const bool hp = gb->hp != 0;
        const float gC = gb->Gam[kC - 1];

        // ---- [O | R | R2] = S_hi [Q^T | W^T hi | W^T lo]  (+ S_lo W^T hi into R) ----
        if (tid == 0) {
            tc_fence_after_sync();
            const uint32_t idesc = hp ? IDESC_KM_N192 : IDESC_KM_N128;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_f16_ts(tmem + CT_O, tmem + CT_SH + 8 * ks,
                           make_sdesc(sslot + SL_QT + ks * 2048, 16384, 1024), idesc, ks > 0);
            if (hp) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_f16_ts(tmem + CT_R, tmem + CT_SL + 8 * ks,
                               make_sdesc(sslot + SL_WH + ks * 2048, 16384, 1024), IDESC_KM_N64, 1);
            }
            mma_commit(&ms->mma_bar);
        }
        // the previous chunk's output, staged in its shared slot, goes out while
        // these products run; its slot may be refilled after the next barrier
        if (c > 0) store_o(c - 1);
        fence_proxy_async_smem();
        GDN_CL_PHASE(0, 1);  // issue S Q^T, R
        {
            GDN_BAR_T0();
            if (!mbar_wait_bounded(&ms->mma_bar, mma_phase, kWaitLimit)) timed_out = true;
            GDN_BAR_T1(2);
        }
        mma_phase ^= 1;
        tc_fence_after_sync();
        GDN_CL_PHASE(0, 2);  // wait: S Q^T, R

        // ---- U = U~ - R in the state's scale; U', U -> TMEM; O *= Gamma unless
        //      Q^T came scaled.  A vote on U's largest scaled magnitude; if it
        //      left the band, U takes a scale of its own and O follows it. ----
        {
            const int c32 = 32 * half;
            const bool qs = gb->qs != 0;
            float v[32];
            // R (scaled by 2^-es) into v, U~ (unscaled) into ut
            auto load_r_ut = [&](float (&ut)[32]) {
                tmem_ld32(trow + CT_R + c32, v);
                tmem_wait_ld();
                if (hp) {
                    float r2[32];
                    tmem_ld32(trow + CT_R2 + c32, r2);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) v[x] += r2[x];
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 f =
                        *reinterpret_cast<const float4 *>(slot + SL_UT + ut_off(row, c32 / 4 + q));
                    ut[4 * q] = f.x; ut[4 * q + 1] = f.y; ut[4 * q + 2] = f.z; ut[4 * q + 3] = f.w;
                }
            };
            // U (scaled) -> U' = U diag(Gamma_C / Gamma) as fp16 hi / lo, and U as fp16
            auto store_u = [&]() {
                uint32_t uh[16], ul[16], u16[16];
#pragma unroll
                for (int x = 0; x < 32; x += 2) {
                    const float p0 = v[x] * gb->eC[c32 + x], p1 = v[x + 1] * gb->eC[c32 + x + 1];
                    const __half2 hh = __floats2half2_rn(p0, p1);
                    const float2 hf = __half22float2(hh);
                    uh[x / 2] = *reinterpret_cast<const uint32_t *>(&hh);
                    ul[x / 2] = pack_half2(p0 - hf.x, p1 - hf.y);
                    u16[x / 2] = pack_half2(v[x], v[x + 1]);
                }
                tmem_st16u(trow + CT_UP + c32 / 2, uh);
                tmem_st16u(trow + CT_UP + 32 + c32 / 2, ul);
                tmem_st16u(trow + CT_U16 + c32 / 2, u16);
            };
            // O (S Q^T) times f, and times Gamma unless Q^T came scaled
            auto scale_o = [&](float f, bool with_gamma) {
                float ov[32];
                tmem_ld32(trow + CT_O + c32, ov);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) ov[x] *= with_gamma ? f * gb->Gam[c32 + x] : f;
                tmem_st32(trow + CT_O + c32, ov);
            };
            float am;
            {
                float ut[32];
                load_r_ut(ut);
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] = fmaf(ut[x], sd, -v[x]);  // U 2^-es (R: 2^-es)
                am = max_abs<32>(v);
            }
            eu = es;
            store_u();
            if (!qs) scale_o(1.f, true);
            if (tid == kStoreTid) bulk_wait_read_all();  // the chunk's output store has read its slot
            tmem_wait_st();
            tc_fence_before_sync();
            GDN_BAR_T0();
            const unsigned b =
                cta_or8(__reduce_or_sync(0xffffffffu, scale_bits(am)), ms->vote[0], warp, lane);
            GDN_BAR_T1(0);
            if (rescale_needed(b)) {  // rare: U takes its own scale, O moves to it
                tc_fence_after_sync();
                float ut[32];
                load_r_ut(ut);  // R and U~ are still in place
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] = fmaf(-s_up, v[x], ut[x]);  // U in fp32, unscaled
                am = cta_max(max_abs<32>(v), ms->red, warp, lane);
                eu = fp16_scale_exp(am);
                const float ud = exp2i(-eu);
#pragma unroll
                for (int x = 0; x < 32; ++x) v[x] *= ud;
                store_u();
                scale_o(exp2c(es - eu), false);
                tmem_wait_st();
                tc_fence_before_sync();
                __syncthreads();
            }
        }
        tc_fence_after_sync();
        poll_read(c);  // the load itself is issued under the next products
        GDN_CL_PHASE(0, 3);  // O scale, U, U'

        // ---- dS = [U'hi | U'lo] [K ; K];  O += U^T P^T  (A operands from TMEM) ----
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_f16_ts(tmem + CT_D, tmem + CT_UP + 8 * ks,
                           make_sdesc(sslot + SL_K16 + (ks & 3) * 2048, 8192, 1024), IDESC_KM_N128,
                           ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_f16_ts(tmem + CT_O, tmem + CT_U16 + 8 * ks,
                           make_sdesc(sslot + SL_P16 + ks * 32, 16, 1024), IDESC_KK_N64, 1);
        }
        poll_next(c);
        mma_sync_point();
        GDN_CL_PHASE(0, 4);  // state update + P MMAs

        // ---- o -> staging (stored during the next chunk); S' = Gamma_C S + dS in
        //      the state's scale and its fp16 hi/lo TMEM operands; the vote
        //      (timeout, and S' leaving the band) ----
        {
            const int c32 = 32 * half;
            const float uu = exp2i(eu);  // O and dS come scaled by 2^-eu
            float v[32];
            tmem_ld32(trow + CT_O + c32, v);
            tmem_wait_ld();
            __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(slot + SL_OST);
#pragma unroll
            for (int x = 0; x < 32; ++x) ost[(c32 + x) * kD + row] = __float2bfloat16_rn(v[x] * uu);
            float sv[64];
            float am;
            const bool same = eu == es;  // uniform over the CTA
            // same: S' in the state's scale; otherwise (U took its own scale this
            // chunk) S' in fp32, unscaled, and a new scale for it
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float d[32];
                tmem_ld32(trow + CT_S + 64 * half + 32 * part, v);
                tmem_ld32(trow + CT_D + 64 * half + 32 * part, d);
                tmem_wait_ld();
                if (same) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        sv[32 * part + x] = fmaf(gC, v[x], d[x]);
                    }
                } else {
                    const float fs = gC * s_up;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        sv[32 * part + x] = fmaf(fs, v[x], d[x] * uu);
                    }
                }
            }
            // a new scale for the unscaled sv: set es from the CTA maximum and apply it
            auto rescale = [&]() {
                am = cta_max(am, ms->red, warp, lane);
                set_es(am > 0.f ? fp16_scale_exp(am) : es);
#pragma unroll
                for (int x = 0; x < 64; ++x) sv[x] *= sd;
            };
            am = max_abs<64>(sv);
            if (!same) rescale();
            const bool lo_next = gb->hp_next != 0;
            store_state(sv);
            split_state(sv, lo_next);
            poll_next(c);
            GDN_CL_PHASE(0, 5);  // o staging, S copies
            fence_proxy_async_smem();  // our writes to the slot precede the next bulk load into it
            tmem_wait_st();
            tc_fence_before_sync();
            GDN_BAR_T0();
            const unsigned b = cta_or8(
                __reduce_or_sync(0xffffffffu, (same ? scale_bits(am) : 2u) | (timed_out ? 8u : 0u)),
                ms->vote[1], warp, lane);
            GDN_BAR_T1(1);
            tc_fence_after_sync();
            if (b & 8u) {
                if (tid == 0) {
                    raise_error(p.err, GDN_ERR_TIMEOUT);
                    if constexpr (kPool) pool_abort(p);
                }
                aborted = true;
            } else if (rescale_needed(b)) {  // rare: S' left the band
#pragma unroll
                for (int x = 0; x < 64; ++x) sv[x] *= s_up;  // exact: S' in fp32, unscaled
                am = max_abs<64>(sv);
                rescale();
                store_state(sv);
                split_state(sv, lo_next);
                tmem_wait_st();
                tc_fence_before_sync();
                __syncthreads();
                tc_fence_after_sync();
            }
        }
        GDN_CL_PHASE(0, 6);  // vote, free the slot
    }

    if (!aborted && p.sT) {  // the master times 2^es
        float *dst = p.sT + (((int64_t)n * p.Hv + h) * kD + row) * kD;
#pragma unroll 1
        for (int cc = 64 * half; cc < 64 * half + 64; cc += 32) {
            float v[32];
            tmem_ld32(trow + CT_S + cc, v);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; x += 4)
                *reinterpret_cast<float4 *>(dst + cc + x) =
                    make_float4(v[x] * s_up, v[x + 1] * s_up, v[x + 2] * s_up, v[x + 3] * s_up);
        }
    }
    if (!aborted && nch > 0) store_o(nch - 1);  // the last chunk's output
    if (tid == kStoreTid) bulk_wait_all();  // every output tile store has landed
    GDN_CL_PHASE_END(0);
    GDN_BAR_END(0);
    if (aborted) {
        // A prefetch still landing in shared memory must finish (c is one past
        // the chunk that voted; every earlier load has been waited for).
        for (int cc = c; cc < loaded; ++cc)
            mbar_wait_bounded(&ms->full[cc & 1], (cc >> 1) & 1, kWaitLimit);
        mbar_wait_bounded(&ms->mma_bar, mma_phase ^ 1, kWaitLimit);
    }
}

// Barrier set-up and TMEM allocation of either role.
__device__ __forceinline__ uint32_t *setup_role(uint8_t *sm, bool chain, uint32_t &ncols,
                                                const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                                const CUtensorMap *tm_v) {
    const int tid = threadIdx.x;
    uint32_t *tmem_slot;
    if (chain) {
        ChainMisc *ms = reinterpret_cast<ChainMisc *>(sm + C_MISC);
        tmem_slot = &ms->tmem_base;
        ncols = 512;
        if (tid == 0) {
            mbar_init(&ms->full[0], 1);
            mbar_init(&ms->full[1], 1);
            mbar_init(&ms->ready[0], 1);
            mbar_init(&ms->ready[1], 1);
            mbar_init(&ms->mma_bar, 1);
            fence_mbarrier_init();
        }
    } else {
        ProdMisc *ms = reinterpret_cast<ProdMisc *>(sm + P_MISC);
        tmem_slot = &ms->tmem_base;
        ncols = 512;
        if (tid == 0) {
            mbar_init(&ms->tma_bar[0], 1);
            mbar_init(&ms->tma_bar[1], 1);
            for (int b = 0; b < kVBufs; ++b) mbar_init(&ms->tma_v[b], 1);
            mbar_init(&ms->mma_bar, 1);
            mbar_init(&ms->taken, 1);
            mbar_init(&ms->qt_bar, 1);
            fence_mbarrier_init();
            tma_prefetch_desc(tm_q);
            tma_prefetch_desc(tm_k);
            tma_prefetch_desc(tm_v);
        }
    }
    if ((tid >> 5) == 0) {
        tmem_alloc(tmem_slot, ncols);
        tmem_relinquish();
    }
    return tmem_slot;
}

__device__ __forceinline__ uint8_t *aligned_smem(uint8_t *raw) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    gdn_prefill_cluster_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_o, ChainParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_smem(smem_raw);
    const int rank = (int)cluster_ctarank();
    const int unit = blockIdx.x / kCluster;  // n * Hv + h
    const int h = unit % p.Hv;
    const int n = unit / p.Hv;
    const int j = h / (p.Hv / p.Hqk);

    int64_t t_begin, t_end;
    if (!seq_range(p.cu, n, p.N, p.T, p.err, t_begin, t_end)) return;  // uniform per cluster
    const int nch = (int)((t_end - t_begin + kC - 1) / kC);

    uint32_t ncols;
    uint32_t *tmem_slot = setup_role(sm, rank == 0, ncols, &tm_q, &tm_k, &tm_v);
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // every CTA's barriers exist before anyone signals them
    tc_fence_after_sync();

    if (rank == 0)
        chain_role<false>(sm, &tm_o, p, unit, n, h, t_begin, t_end, nch);
    else
        producer_role<false, 1>(sm, &tm_q, &tm_k, &tm_v, p, unit, rank - 1, h, j, t_begin, t_end,
                                nch);

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(*tmem_slot, ncols);
    cluster_sync();  // nobody's shared memory goes away while another CTA may address it
}

// kNh: v-heads per producer item (p.nh).  kConv: the front end fused into the
// load stage (tm_q, tm_k, tm_v map the raw channel inputs; tm_hq, tm_hk, tm_hv
// the same in 8-token boxes); otherwise the halo maps are unused.
template <int kNh, bool kConv>
__global__ void __launch_bounds__(kThreads, 1)
    gdn_prefill_pool_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ CUtensorMap tm_o,
                            const __grid_constant__ CUtensorMap tm_hq,
                            const __grid_constant__ CUtensorMap tm_hk,
                            const __grid_constant__ CUtensorMap tm_hv, ChainParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = aligned_smem(smem_raw);
    const bool chain = (int)blockIdx.x < p.units;
    int unit = 0, n = 0, h = 0, nch = 0;
    int64_t t_begin = 0, t_end = 0;
    if (chain) {
        unit = blockIdx.x;
        h = unit % p.Hv;
        n = unit / p.Hv;
        if (!seq_range(p.cu, n, p.N, p.T, p.err, t_begin, t_end)) return;  // producers skip it too
        nch = (int)((t_end - t_begin + kC - 1) / kC);
    }
    uint32_t ncols;
    uint32_t *tmem_slot = setup_role(sm, chain, ncols, &tm_q, &tm_k, &tm_v);
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();

    if (chain)
        chain_role<true>(sm, &tm_o, p, unit, n, h, t_begin, t_end, nch);
    else
        producer_role<true, kNh, kConv>(sm, &tm_q, &tm_k, &tm_v, p, 0, 0, 0, 0, 0, 0, 0, &tm_hq,
                                        &tm_hk, &tm_hv);

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if ((threadIdx.x >> 5) == 0) tmem_dealloc(*tmem_slot, ncols);
}

size_t pool_flag_bytes(int64_t units) {
    const size_t b = (size_t)(kFlagHeader + kFlagsPerUnit * units) * sizeof(uint32_t);
    return (b + 1023) & ~size_t(1023);
}

bool fill_params(const PrefillArgs &a, ChainParams &p, CUtensorMap &mq, CUtensorMap &mk,
                 CUtensorMap &mv, CUtensorMap &mo);

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

}  // namespace

static_assert(kClusterRingSlots * SLOT_BYTES == kClusterWorkspaceBytesPerUnit, "ring size per unit");

size_t prefill_cluster_workspace_bytes(int64_t units) {
    return (size_t)units * kClusterRingSlots * SLOT_BYTES;
}

size_t prefill_pool_workspace_bytes(int64_t units) {
    return pool_flag_bytes(units) + (size_t)units * kPoolRingSlots * SLOT_BYTES;
}

bool prefill_pool_fits(int64_t units) {
    const int sms = sm_count();
    return units >= 1 && units <= kPoolMaxUnits && units + 16 <= sms;
}

bool make_tile_map_bf16_128(CUtensorMap *m, const void *base, int64_t T, int32_t H);
bool make_halo_map_bf16_128(CUtensorMap *m, const void *base, int64_t T, int32_t H);
bool make_store_map_bf16_128(CUtensorMap *m, void *base, int64_t T, int32_t H);

namespace {
bool fill_params(const PrefillArgs &a, ChainParams &p, CUtensorMap &mq, CUtensorMap &mk,
                 CUtensorMap &mv, CUtensorMap &mo) {
    if (a.T > 0x7fffffffLL || a.ws == nullptr) return false;
    const int64_t Tm = a.T > 0 ? a.T : 1;
    if (!make_tile_map_bf16_128(&mq, a.q, Tm, a.Hqk) || !make_tile_map_bf16_128(&mk, a.k, Tm, a.Hqk) ||
        !make_tile_map_bf16_128(&mv, a.v, Tm, a.Hv) || !make_store_map_bf16_128(&mo, a.o, Tm, a.Hv))
        return false;
    p.ring = static_cast<uint8_t *>(a.ws);
    p.flags = nullptr;
    p.g = a.g; p.beta = a.beta; p.s0 = a.s0; p.cu = a.cu; p.o = a.o; p.sT = a.sT; p.err = a.err;
    p.T = a.T; p.N = a.N; p.Hqk = a.Hqk; p.Hv = a.Hv;
    p.units = a.N * a.Hv;
    p.max_chunks = (int)((a.T + kC - 1) / kC);
    p.ring_slots = kClusterRingSlots;
    p.recall_first = a.order == GDN_ORDER_RECALL_FIRST;
    p.flag_wait_limit = kWaitLimit;
    p.skip_unit = -1;
    // heads per pool producer item: the largest of 3, 2, 1 that divides the
    // v-heads per q/k head
    const int G = a.Hv / a.Hqk;
    p.nh = G % 3 == 0 ? 3 : (G % 2 == 0 ? 2 : 1);
    p.cf = a.cf;
    p.cstate = a.cstate_in;
    p.cC = 2 * a.Hqk * kD + a.Hv * kD;
    return true;
}
}  // namespace

cudaError_t launch_prefill_cluster(const PrefillArgs &a, cudaStream_t s) {
    ChainParams p;
    CUtensorMap mq, mk, mv, mo;
    if (!fill_params(a, p, mq, mk, mv, mo)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gdn_prefill_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((int64_t)a.N * a.Hv * kCluster));
    gdn_prefill_cluster_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
}

cudaError_t launch_prefill_pool(const PrefillArgs &a, cudaStream_t s) {
    ChainParams p;
    CUtensorMap mq, mk, mv, mo;
    if (!fill_params(a, p, mq, mk, mv, mo)) return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (!prefill_pool_fits(p.units) || sms <= 0) {
        if (a.conv) return cudaErrorNotSupported;  // the fused front end runs in the pool kernel only
        return launch_prefill_tc(a, s);
    }
    const size_t fb = pool_flag_bytes(p.units);
    p.flags = static_cast<uint32_t *>(a.ws);
    p.ring = static_cast<uint8_t *>(a.ws) + fb;
    p.ring_slots = kPoolRingSlots;
    if (a.debug_flag_wait > 0) p.flag_wait_limit = a.debug_flag_wait;
    p.skip_unit = a.debug_skip_unit;
    // the chunk counter, abort flag and hand-off flags start at zero
    cudaError_t e = cudaMemsetAsync(a.ws, 0, fb, s);
    if (e != cudaSuccess) return e;
    CUtensorMap hq = mq, hk = mk, hv = mv;  // halo maps (the fused front end only)
    if (a.conv && (!make_halo_map_bf16_128(&hq, a.q, a.T > 0 ? a.T : 1, a.Hqk) ||
                   !make_halo_map_bf16_128(&hk, a.k, a.T > 0 ? a.T : 1, a.Hqk) ||
                   !make_halo_map_bf16_128(&hv, a.v, a.T > 0 ? a.T : 1, a.Hv)))
        return cudaErrorInvalidValue;
    auto kern = a.conv ? (p.nh == 3 ? gdn_prefill_pool_kernel<3, true>
                                    : (p.nh == 2 ? gdn_prefill_pool_kernel<2, true>
                                                 : gdn_prefill_pool_kernel<1, true>))
                       : (p.nh == 3 ? gdn_prefill_pool_kernel<3, false>
                                    : (p.nh == 2 ? gdn_prefill_pool_kernel<2, false>
                                                 : gdn_prefill_pool_kernel<1, false>));
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once, or no launch
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, mo, hq, hk, hv, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace gdn

#ifdef GDN_TC_PHASES
extern "C" GDN_API int gdn_debug_bar_waits(long long *out, int reset) {
    unsigned long long host[64];
    if (cudaMemcpyFromSymbol(host, gdn_cl_bar_wait, sizeof(host)) != cudaSuccess) return -1;
    for (int i = 0; i < 64; ++i) out[i] = (long long)host[i];
    if (reset) {
        const unsigned long long zero[64] = {0};
        cudaMemcpyToSymbol(gdn_cl_bar_wait, zero, sizeof(zero));
    }
    return 0;
}

extern "C" GDN_API int gdn_debug_cluster_phases(long long *out, int reset) {
    unsigned long long host[32];
    if (cudaMemcpyFromSymbol(host, gdn_cl_phase_clk, sizeof(host)) != cudaSuccess) return -1;
    for (int i = 0; i < 32; ++i) out[i] = (long long)host[i];
    if (reset) {
        const unsigned long long zero[32] = {0};
        cudaMemcpyToSymbol(gdn_cl_phase_clk, zero, sizeof(zero));
    }
    return 0;
}
#endif
