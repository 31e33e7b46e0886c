// attn_tc.cu -- bf16 block attention on sm_100a tensor cores (tcgen05 + TMEM + TMA),
// run either as one block (cp_block_attn_fwd) or as the whole ring schedule.
//
// What one CTA computes ("上下文并行与 Ring Attention", hs-black.github.io):
//   two 128-row query tiles of one rank and one query head.  For each ring step r
//   the CTA takes the K/V block of rank (i - r) mod N (section Ring Attention) and
//   runs the online-softmax recurrence of section 分块注意力 over its key tiles:
//   running max m, running sum l = sum e^{x - m}, unnormalised O.  Folding the next
//   key tile (or the next ring step's block) into (m, l, O) is the LSE merge of that
//   section in the incremental form the page attributes to FlashAttention; at the
//   end o = O / l and lse = m + log l.  Key tiles the causal mask hides completely
//   are skipped whole (figure caption of section Ring Attention).
//
// Roles (384 threads, three warpgroups):
//   warps 0-3  softmax of query tile 0 (thread t owns row t = TMEM lane t)
//   warps 4-7  softmax of query tile 1
//   warp 8     TMA producer: Q0, Q1 once, then K and V tiles (2 stages each)
//   warp 9     TMEM owner (512 columns) and single-thread MMA issuer
//   warps 10-11 idle
// The third warpgroup hands most of its registers to the softmax warpgroups
// (setmaxnreg: 88 vs 208 per thread; 2*128*208 + 128*88 = 384*168, the launch
// allocation).
// TMEM columns: S_j = [128 j, 128 j + 128) holds the fp32 scores of query tile j;
// the softmax overwrites columns [0, 64) of S_j with bf16 probabilities P_j, which
// the PV MMA reads as its A operand; O_j = [256 + d j, 256 + d (j + 1)).
// The MMA warp interleaves the two tiles (PV_0(n), S_0(n+1), PV_1(n), S_1(n+1), ...)
// so the tensor core works on one tile while the other tile's softmax runs.  P is
// handed over in two halves of 64 keys, each with its own barrier, so the first
// half of PV runs while the softmax computes the second half of P; S_j(n+1) can
// only follow PV_j(n), because it overwrites the columns that hold P_j(n).
//
// Softmax details: scores are handled in the log2 domain (scale * log2 e folded
// into one FMA); the max used in the exponent is raised only when a row's max
// grows by more than 8 (log2 units), and O and l always refer to the max in use,
// so the result is exact up to rounding while most tiles skip the O rescale.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include <algorithm>

#include "kernels.h"
#include "ptx.cuh"
#include "exp2_poly.h"

namespace cpattn {
namespace {

constexpr int BM = 128;  // query rows per tile (TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int NQ = 2;    // query tiles per CTA
#ifndef CP_ATTN_NSK
#define CP_ATTN_NSK 2
#endif
#ifndef CP_ATTN_NSV
#define CP_ATTN_NSV 2
#endif
// P through shared memory (below): the two P buffers take the second V stage's room.
#ifndef CP_ATTN_P_SMEM
#define CP_ATTN_P_SMEM 0
#endif
constexpr int NSK = CP_ATTN_NSK;  // K stages
constexpr int NSV = CP_ATTN_P_SMEM ? 1 : CP_ATTN_NSV;  // V stages
constexpr int NTHREADS = 384;
#ifndef CP_ATTN_REGS_SOFTMAX
#define CP_ATTN_REGS_SOFTMAX (CP_ATTN_P_SMEM ? 200 : 208)
#endif
constexpr int REGS_SOFTMAX = CP_ATTN_REGS_SOFTMAX;
constexpr int REGS_OTHER = (NTHREADS * 168 - 2 * 128 * REGS_SOFTMAX) / 128;  // the rest of the launch's registers
static_assert(REGS_OTHER >= 24 && REGS_OTHER % 8 == 0, "register split");
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// In tiles without masking, pair i of every 16 probability pairs is computed on
// the FMA pipe (exp2_fma) when i % kEmuMod == kEmuMod - 1, the rest on the MUFU
// pipe (ex2.approx); 0 disables.  Balances the two pipes.
#ifndef CP_EXP2_EMU_MOD
#define CP_EXP2_EMU_MOD 0
#endif
constexpr int kEmuMod = CP_EXP2_EMU_MOD;
// P handed to the MMA warp in two halves of 64 keys (1) or whole (0).
#ifndef CP_ATTN_SPLIT_P
#define CP_ATTN_SPLIT_P 0
#endif
constexpr bool kSplitP = CP_ATTN_SPLIT_P != 0;
// The two softmax warpgroups take turns for their exponential phases (1) or run
// freely (0).  Turns are handed over on named barriers kTurn0 / kTurn1 (the
// teardown uses barrier 1).
#ifndef CP_ATTN_PINGPONG
#define CP_ATTN_PINGPONG 0
#endif
constexpr bool kPingPong = CP_ATTN_PINGPONG != 0;
constexpr int kTurn0 = 2, kTurn1 = 3;
// Persistent grids (one CTA per SM walking the work items) for the document-mask
// instantiation and for the ring's.
#ifndef CP_ATTN_DOC_PERSIST
#define CP_ATTN_DOC_PERSIST 0
#endif
#ifndef CP_ATTN_RING_PERSIST
#define CP_ATTN_RING_PERSIST 0
#endif
constexpr bool kDocPersist = CP_ATTN_DOC_PERSIST != 0;
// Query tiles per CTA of the document-mask instantiation: 1 (two CTAs per SM) or 2
// (the ring's CTA).  The persistent grid is written for two.
#ifndef CP_ATTN_DOC_NQ
#define CP_ATTN_DOC_NQ 1
#endif
constexpr int kDocNQ = kDocPersist ? 2 : CP_ATTN_DOC_NQ;
// Register split of the one-tile CTA (128 per thread at launch, two CTAs per SM): the
// softmax warpgroup's share; the producer / MMA warpgroup gets 256 minus it (200 / 56
// spills 40 bytes in the producer / MMA roles, the least of 176–200).
#ifndef CP_ATTN_DOC1_REGS
#define CP_ATTN_DOC1_REGS 200
#endif
// S computed in two halves of 64 keys into a two-slot ring per query tile (1): the
// next key tile's first half only waits for the PV of this tile's first half, so a
// softmax warpgroup always has the other half's scores ready; or S whole (0).
#ifndef CP_ATTN_HALF_S
#define CP_ATTN_HALF_S 0
#endif
constexpr bool kHalfS = CP_ATTN_HALF_S != 0;
constexpr int NH = kHalfS ? 2 : 1;  // S parts per key tile
constexpr int HW = BN / NH;         // keys per S part
static_assert(!(kHalfS && CP_ATTN_SPLIT_P), "split P hand-over applies to whole S only");
static_assert(!(kHalfS && CP_ATTN_PINGPONG), "turn-taking is written for whole S");
constexpr bool kRingPersist = CP_ATTN_RING_PERSIST != 0;
// Query tiles per CTA of the ring instantiation (2, or 1 as the document one).
#ifndef CP_ATTN_RING_NQ
#define CP_ATTN_RING_NQ 2
#endif
constexpr int kRingNQ = kRingPersist ? 2 : CP_ATTN_RING_NQ;
// A turn starts before the S load (0) or after the row max (1: the loads and row
// maxima of the two tiles overlap, at the cost of more live registers).
#ifndef CP_ATTN_TURN_LATE
#define CP_ATTN_TURN_LATE 0
#endif
constexpr bool kTurnLate = CP_ATTN_TURN_LATE != 0;
// One-item CTAs (the grid covers every work item):
//   CP_ATTN_EARLY_Q   the producer starts the Q load right after the barrier set-up,
//                     before the tile walk is worked out;
//   CP_ATTN_PREFETCH_Q the item one wave later gets its Q prefetched into L2;
//   CP_ATTN_STAGGER   query tile 1 starts its first key tile after tile 0's first P;
//   CP_ATTN_TMA_O     bf16 output tiles leave through shared memory and a TMA store.
#ifndef CP_ATTN_EARLY_Q
#define CP_ATTN_EARLY_Q 1
#endif
#ifndef CP_ATTN_PREFETCH_Q
#define CP_ATTN_PREFETCH_Q 0
#endif
#ifndef CP_ATTN_STAGGER
#define CP_ATTN_STAGGER 0
#endif
#ifndef CP_ATTN_TMA_O
#define CP_ATTN_TMA_O 1
#endif
constexpr bool kEarlyQ = CP_ATTN_EARLY_Q != 0;
constexpr bool kPrefetchQ = CP_ATTN_PREFETCH_Q != 0;
constexpr bool kStagger = CP_ATTN_STAGGER != 0;
constexpr bool kTmaO = CP_ATTN_TMA_O != 0;
// Where P (the bf16 probabilities) goes.  0: over the tile's own S columns in TMEM,
// PV a TS product, two V stages; the next S waits for this tile's PV.  1: a
// shared-memory buffer per query tile (a write waits for the tile's previous PV), PV
// an SS product, one V stage; the scores' TMEM columns are free once the softmax has
// read them, so the next key tile's S is issued then, while this tile's exponentials
// still run.  Measured slower: an SS product at full rate reads 128 bytes per clock,
// all of shared memory's bandwidth, and the softmax's P stores wait behind it.
constexpr bool kPSmem = CP_ATTN_P_SMEM != 0;
static_assert(!kPSmem || (!kHalfS && !kSplitP && !kPingPong && !kStagger && !kDocPersist && !kRingPersist),
              "the shared-memory P hand-over is written for whole S, free-running warpgroups and one-item CTAs");
// Key tiles after a query tile's first in a work item start their exponentials on
// the first 32 score columns while the other 96 are still being read out of TMEM
// (1), instead of after the whole row's max (0).  Written for whole P hand-over,
// free-running warpgroups and exponentials on the MUFU pipe only.
#ifndef CP_ATTN_CHUNKED_EXP
#define CP_ATTN_CHUNKED_EXP 0
#endif
constexpr bool kChunkedExp = CP_ATTN_CHUNKED_EXP != 0 && !kSplitP && !kPingPong && kEmuMod == 0 && !kPSmem;
// Grid order of the ring instantiation: (batch, kv head) outermost, the order table's
// entries within it and the query heads of the kv head's group innermost (1), so the
// CTAs resident at one time read one kv head's K/V blocks and these stay in L2; or
// the order table outermost with every (batch, query head) innermost (0).  The
// document instantiation keeps the latter: its gathered K/V fits in L2 anyway and
// its very unequal items balance better heaviest first across all heads.
#ifndef CP_ATTN_KV_MAJOR
#define CP_ATTN_KV_MAJOR 1
#endif
constexpr bool kKvMajor = CP_ATTN_KV_MAJOR != 0;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

// Shared memory, barriers, TMEM and threads of a CTA with NQT query tiles: two (the
// ring: the two tiles' chains interleave on the tensor pipe, one CTA per SM) or one
// (documents: one K and one V stage, 256 TMEM columns and 256 threads, so two CTAs
// share an SM and one's set-up, first loads and epilogue overlap the other's tiles).
template <int D, int NQT = NQ>
struct Cfg {
    static constexpr int NSK_ = NQT == 1 ? 1 : NSK;
    static constexpr int NSV_ = NQT == 1 ? 1 : NSV;
    static constexpr int NTHR = 128 * (NQT + 1);    // softmax warpgroups + producer / MMA warpgroup
    static constexpr int CTAS_PER_SM = NQT == 1 ? 2 : 1;
    static constexpr int REGS_SM = NQT == 1 ? CP_ATTN_DOC1_REGS : REGS_SOFTMAX;  // softmax warpgroups
    static constexpr int REGS_OT = NQT == 1 ? 256 - CP_ATTN_DOC1_REGS : REGS_OTHER;  // producer / MMA
    static_assert(NQT * 128 * REGS_SM + 128 * REGS_OT <= NTHR * (65536 / (NTHR * CTAS_PER_SM) / 8 * 8),
                  "register split exceeds the launch's registers");
    static constexpr int SUB = BM * 128;     // one 64-column swizzle block (16 KB)
    static constexpr int TILE = BM * D * 2;  // a 128 x D bf16 tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + NQT * TILE;
    static constexpr int OFF_V = OFF_K + NSK_ * TILE;
    static constexpr int PTILE = BM * BN * 2;         // P of one query tile (kPSmem)
    static constexpr int OFF_P = OFF_V + NSV_ * TILE;
    static constexpr int OFF_BAR = OFF_P + (kPSmem ? NQT * PTILE : 0);
    enum {
        B_Q = 0,
        B_KF = 1,
        B_KE = B_KF + NSK_,
        B_VF = B_KE + NSK_,
        B_VE = B_VF + NSV_,
        B_SF = B_VE + NSV_,  // per query tile and S part: index 2 j + part
        B_PF = B_SF + 2 * NQT,  // P of keys [0, 64) of the tile stored (per query tile)
        B_PH = B_PF + NQT,   // P stored: whole S, keys [64, 128) with the split hand-over, or S
                             // part h (index 2 j + h; one barrier per part, so the softmax
                             // never runs two phases ahead of the MMA warp on one barrier)
        B_PV = B_PH + 2 * NQT,  // PV of S part h done (index 2 j + h), one barrier per part
        B_OF = B_PV + 2 * NQT,   // O of query tile j read out by its epilogue (per query tile)
        B_QE = B_OF + NQT,   // Q buffer free: the work item's last S products are done
        B_STAG = B_QE + 1,   // query tile 0's first P is stored (tile 1 starts after it)
        B_SC = B_STAG + 1,   // kPSmem: query tile j's scores are read out of TMEM (per tile)
        B_DONE = B_SC + NQT,
        NBAR = B_DONE + 1
    };
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;  // + alignment slack
    static_assert(SMEM <= 232448, "shared memory per CTA exceeds 227 KB");
    static_assert(CTAS_PER_SM == 1 || CTAS_PER_SM * (SMEM + 1024) <= 233472, "two CTAs do not fit an SM");
    static constexpr int T_O = 128 * NQT;                // O columns after the S columns
    static constexpr uint32_t TMEM_COLS = NQT == 1 ? 256 : 512;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, HW, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
};

// Document start of position pos (one load from the per-position table).
__device__ __forceinline__ int doc_start_of(const AttnParams &p, int pos)
{
    if (!bounds_ok(pos >= 0 && pos < p.seq_len, p.status, 104)) return 0;
    return __ldg(p.doc_pos_start + pos);
}

// First key tile t of a block (kv_len keys, ranges k, tiles of BN) whose key at
// index min(t * BN + off, kv_len - 1) has a position >= x.
__device__ __forceinline__ int first_tile_from(const Range32 &k, int kv_len, int off, int x)
{
    const int n_kt = (int)((kv_len + BN - 1) / BN);
    if (k.len1 == 0 && k.stride > 0) {
        // one segment, positions start0 + i stride: the first index i* at or past x; a
        // tile qualifies once its probe index (clamped to kv_len - 1) reaches i*
        const int istar = x <= k.start0 ? 0 : k.stride == 1 ? x - k.start0 : (x - k.start0 + k.stride - 1) / k.stride;
        if (istar > kv_len - 1) return n_kt;
        const int t1 = istar - off <= 0 ? 0 : (istar - off + BN - 1) / BN;
        const int tc = kv_len - off <= 0 ? 0 : (kv_len - off + BN - 1) / BN;
        return min(min(t1, tc), n_kt);
    }
    int lo = 0, hi = n_kt;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int t = mid * BN + off;
        if (t > kv_len - 1) t = kv_len - 1;
        if (range_pos(k, t) < x) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// Key-tile sequence of one CTA: every (ring step, key tile) that at least one of the
// two query tiles must visit, in order.  All roles walk the same sequence; tile n is
// visited by query tile j iff kt_beg[j] <= kt < kt_end[j] of its step, and needs the
// element mask unless kt_fb[j] <= kt < kt_full[j].  Without documents kt_beg = kt_fb
// = 0.  With the document mask the keys a query tile sees span from the document
// start of its first row to its last row, and every row sees the keys from the
// document start of its last row to its first row (positions increase with the
// local index, so both are runs of whole tiles).
template <bool DOC, int NQT = NQ>
struct TileSeq {
    Range32 qr;
    int rank;
    int q_lo0;
    bool q_ok1;  // query tile 1 holds rows (tile 0 always does)
    int step, kt, kt_end_all;
    int kt_full0, kt_full1, kt_end0, kt_end1;
    int kt_beg0, kt_beg1, kt_fb0, kt_fb1, kt_beg_all;
    int ds_min0, ds_max0, ds_min1, ds_max1;  // document starts of the tiles' first / last rows
    int src;
    Range32 kr;

    __device__ __forceinline__ void init(const AttnParams &pp, const Range32 &q, int rk, int qlo0)
    {
        qr = q;
        rank = rk;
        q_lo0 = qlo0;
        q_ok1 = NQT > 1 && qlo0 + BM < pp.q_len;
        step = pp.step_begin - 1;
        kt = 0;
        kt_end_all = 0;
        kt_beg0 = kt_beg1 = kt_fb0 = kt_fb1 = kt_beg_all = 0;
        ds_min0 = ds_max0 = ds_min1 = ds_max1 = 0;
        if (DOC) {
            const int last = pp.q_len - 1;
            ds_min0 = doc_start_of(pp, range_pos(q, qlo0));
            ds_max0 = doc_start_of(pp, range_pos(q, qlo0 + BM - 1 < last ? qlo0 + BM - 1 : last));
            if (q_ok1) {
                ds_min1 = doc_start_of(pp, range_pos(q, qlo0 + BM));
                ds_max1 = doc_start_of(pp, range_pos(q, qlo0 + 2 * BM - 1 < last ? qlo0 + 2 * BM - 1 : last));
            }
        }
    }
    // With documents the two query tiles (far apart in position under the zig-zag
    // layout) can need two disjoint runs of key tiles; tiles in between, needed by
    // neither, are skipped, so every tile of the sequence has a reader (the K/V stage
    // bookkeeping of the producer and the MMA warp relies on it).
    __device__ __forceinline__ void skip_gap()
    {
        if (!DOC || need(0) || need(1)) return;
        int nk = kt_end_all;
        if (kt < kt_beg0 && kt_beg0 < kt_end0 && kt_beg0 < nk) nk = kt_beg0;
        if (q_ok1 && kt < kt_beg1 && kt_beg1 < kt_end1 && kt_beg1 < nk) nk = kt_beg1;
        kt = nk;
    }
    __device__ __forceinline__ bool next(const AttnParams &p)
    {
        ++kt;
        skip_gap();
        while (kt >= kt_end_all) {
            ++step;
            if (step >= p.step_end) return false;
            const int N = p.n_ranks;
            src = ((rank - step) % N + N) % N;
            kr = (p.use_layout && !p.kv_explicit) ? layout_range_t<int>(p.layout, N, (int)p.seq_len, src)
                                                    : to_range32(p.kv_range);
            kv_tile_bounds<int>(qr, p.q_len, q_lo0, BM, kr, p.kv_len, BN, p.causal != 0, &kt_full0, &kt_end0);
            kt_full1 = kt_end1 = 0;
            if (q_ok1)
                kv_tile_bounds<int>(qr, p.q_len, q_lo0 + BM, BM, kr, p.kv_len, BN, p.causal != 0, &kt_full1,
                                        &kt_end1);
            if (DOC) {
                kt_beg0 = first_tile_from(kr, p.kv_len, BN - 1, ds_min0);
                kt_fb0 = first_tile_from(kr, p.kv_len, 0, ds_max0);
                kt_beg1 = q_ok1 ? first_tile_from(kr, p.kv_len, BN - 1, ds_min1) : kt_end1;
                kt_fb1 = q_ok1 ? first_tile_from(kr, p.kv_len, 0, ds_max1) : kt_end1;
                kt_beg_all = kt_beg0 < kt_beg1 ? kt_beg0 : kt_beg1;
            }
            kt_end_all = kt_end0 > kt_end1 ? kt_end0 : kt_end1;
            kt = kt_beg_all;
            skip_gap();
        }
        return true;
    }
    __device__ __forceinline__ bool need(int j) const
    {
        return kt < (j ? kt_end1 : kt_end0) && (!DOC || kt >= (j ? kt_beg1 : kt_beg0));
    }
    __device__ __forceinline__ bool partial(int j) const
    {
        return kt >= (j ? kt_full1 : kt_full0) || (DOC && kt < (j ? kt_fb1 : kt_fb0));
    }
};

__device__ __forceinline__ void store_row_chunk(void *o, int dtype, int64_t off, const float *v)
{
    // 32 consecutive values of one output row
    if (dtype == DT_BF16) {
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(o) + off);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
            w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
            w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
            w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
            dst[i] = w;
        }
    } else {
        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(o) + off);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i + 0], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
}

template <int D, bool DOC, bool PERSIST, int NQT>
__global__ void __launch_bounds__(128 * (NQT + 1), NQT == 1 ? 2 : 1)
    attn_tc_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_o, int o_tma, int next_stride)
{
    using C = Cfg<D, NQT>;
    // this instantiation's shape (the namespace-level names are the two-tile CTA's)
    constexpr int NQ = NQT, NSK = C::NSK_, NSV = C::NSV_, NTHREADS = C::NTHR;
    constexpr int WARP_LOAD = 4 * NQT, WARP_MMA = 4 * NQT + 1;
    constexpr int REGS_SOFTMAX = C::REGS_SM, REGS_OTHER = C::REGS_OT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work items: item = (order entry e, batch, head), e = (rank, query-tile pair)
    // from the order table.  A CTA takes items blockIdx.x, blockIdx.x + gridDim.x, ...
    // (one item when the grid covers them all; a persistent grid walks several, its
    // barrier phases, K/V stages and TMEM carrying over from item to item).
    const int bh_count = p.b * p.hq;
    const int n_items = p.n_ranks * p.n_qt * bh_count;
    struct Item {
        int rank, qp, h, bb, hk, q_lo0;
        Range32 qr;
    };
    const int n_entries = p.n_ranks * p.n_qt;
    auto decode = [&](int item) {
        Item it;
        int bh, e;
        if (kKvMajor && !DOC) {
            // item = ((bb * hkv + hk) * n_entries + e) * group + g, query head hk * group + g
            const int g = item % p.group;
            const int rest = item / p.group;
            e = rest % n_entries;
            const int bkv = rest / n_entries;
            bh = (bkv / p.hkv) * p.hq + (bkv % p.hkv) * p.group + g;
        } else {
            bh = item % bh_count;
            e = item / bh_count;
        }
        if (p.order_len) {
            it.rank = (int)(p.order[e] >> 16);
            it.qp = (int)(p.order[e] & 0xffffu);
        } else {
            it.rank = e / p.n_qt;
            it.qp = e % p.n_qt;
        }
        it.h = bh % p.hq;
        it.bb = bh / p.hq;
        it.hk = it.h / p.group;
        it.q_lo0 = it.qp * (NQ * BM);
        it.qr = p.use_layout ? layout_range_t<int>(p.layout, p.n_ranks, (int)p.seq_len, it.rank) : to_range32(p.q_range);
        return it;
    };
    // tensor rows the maps and outputs cover (for the debug build's bounds checks)
    const int64_t q_rows_all = p.q_row_step ? (int64_t)p.n_ranks * p.q_row_step : p.q_len;
    const int64_t kv_rows_all = p.kv_row_step ? (int64_t)p.n_ranks * p.kv_row_step : p.kv_len;
    (void)q_rows_all;
    (void)kv_rows_all;

    // Q tiles of an item into the Q buffer (both tiles when the second holds rows)
    auto issue_q = [&](const Item &it) {
        const int q_row = (int)(it.rank * p.q_row_step) + it.q_lo0;
        const int nq = (NQ > 1 && it.q_lo0 + BM < p.q_len) ? 2 : 1;
        mbar_expect_tx(bar(C::B_Q), nq * C::TILE);
        for (int j = 0; j < nq; ++j)
            for (int kb = 0; kb < D / 64; ++kb)
                if (bounds_ok(q_row + j * BM >= 0 && q_row + j * BM < q_rows_all && it.h < p.hq && it.bb < p.b,
                              p.status, 101))
                    tma_load_4d(s_base + C::OFF_Q + j * C::TILE + kb * C::SUB, &tm_q, bar(C::B_Q), kb * 64, it.h,
                                q_row + j * BM, it.bb);
    };

    // ---- setup: barriers (by the producer thread, which then starts the Q load of a
    // one-item CTA at once, before the tile walk is worked out), TMEM
    if (warp == WARP_LOAD && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        mbar_init(bar(C::B_Q), 1);
        for (int i = 0; i < NSK; ++i) { mbar_init(bar(C::B_KF + i), 1); mbar_init(bar(C::B_KE + i), 1); }
        for (int i = 0; i < NSV; ++i) { mbar_init(bar(C::B_VF + i), 1); mbar_init(bar(C::B_VE + i), 1); }
        for (int j = 0; j < NQ; ++j) {
            mbar_init(bar(C::B_SF + 2 * j), 1);
            mbar_init(bar(C::B_SF + 2 * j + 1), 1);
            mbar_init(bar(C::B_PF + j), BM / 32);  // one arrival per softmax warp
            mbar_init(bar(C::B_PH + 2 * j), BM / 32);
            mbar_init(bar(C::B_PH + 2 * j + 1), BM / 32);
            mbar_init(bar(C::B_PV + 2 * j), 1);
            mbar_init(bar(C::B_PV + 2 * j + 1), 1);
            mbar_init(bar(C::B_OF + j), BM / 32);
        }
        mbar_init(bar(C::B_QE), 1);
        mbar_init(bar(C::B_STAG), BM / 32);
        for (int j = 0; j < NQ; ++j) {
            mbar_init(bar(C::B_SC + j), BM / 32);
        }
        mbar_init(bar(C::B_DONE), 1);
        *abort_flag = 0;
        mbar_fence_init();
        if (!PERSIST && kEarlyQ) issue_q(decode(blockIdx.x));
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    // Every role ends in teardown(): all TMEM traffic done, CTA-wide named barrier,
    // then the owner warp frees TMEM.  The roles never merge back into common code,
    // so each keeps the register budget setmaxnreg gave it.
    auto teardown = [&]() {
        __syncwarp();
        tc_fence_before();
        asm volatile("barrier.sync 1, %0;" ::"n"(NTHREADS) : "memory");
        if (warp == WARP_MMA) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tbase, C::TMEM_COLS);
        }
    };

    if (warp >= 4 * NQ) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_OTHER));
    if (warp == WARP_LOAD) {
        // ================================================================ producer
        if (lane == 0) {
            WaitCtx w{abort_flag, p.status, 1};
            int n = 0;   // K/V tiles loaded, over all work items
            int qi = (PERSIST || !kEarlyQ) ? 0 : 1;  // Q loads issued (early: at set-up)
            bool stop = false;
            for (int item = blockIdx.x; item < n_items && !stop; item += gridDim.x) {
                const Item it = decode(item);
                TileSeq<DOC, NQT> seq;
                seq.init(p, it.qr, it.rank, it.q_lo0);
                bool first = PERSIST || !kEarlyQ;
                while (seq.next(p)) {
                    if (first) {
                        // the previous item's S products have read its Q
                        if (!mbar_wait(bar(C::B_QE), (qi & 1) ^ 1, w)) { stop = true; break; }
                        issue_q(it);
                        first = false;
                        ++qi;
                    }
                    int kv_row = (int)(seq.src * p.kv_row_step) + seq.kt * BN;
                    if (p.kv_map_h > 0) kv_row = zigzag_row<int>(kv_row, p.kv_map_h, p.n_ranks);
                    const int sk = n % NSK, sv = n % NSV;
                    if (!mbar_wait(bar(C::B_KE + sk), ((n / NSK) & 1) ^ 1, w)) { stop = true; break; }
                    mbar_expect_tx(bar(C::B_KF + sk), C::TILE);
                    const bool kv_ok = bounds_ok(kv_row >= 0 && kv_row < kv_rows_all && it.hk < p.hkv && it.bb < p.b,
                                                 p.status, 102);
                    for (int kb = 0; kb < D / 64 && kv_ok; ++kb)
                        tma_load_4d(s_base + C::OFF_K + sk * C::TILE + kb * C::SUB, &tm_k, bar(C::B_KF + sk),
                                    kb * 64, it.hk, kv_row, it.bb);
                    if (!mbar_wait(bar(C::B_VE + sv), ((n / NSV) & 1) ^ 1, w)) { stop = true; break; }
                    mbar_expect_tx(bar(C::B_VF + sv), C::TILE);
                    for (int kb = 0; kb < D / 64 && kv_ok; ++kb)
                        tma_load_4d(s_base + C::OFF_V + sv * C::TILE + kb * C::SUB, &tm_v, bar(C::B_VF + sv),
                                    kb * 64, it.hk, kv_row, it.bb);
                    ++n;
                    if (!PERSIST && kPrefetchQ && n == 1 && next_stride > 0 && blockIdx.x + next_stride < n_items) {
                        // the item about to start on the SM that frees up next: its Q into L2
                        const Item nx = decode(blockIdx.x + next_stride);
                        const int nq_row = (int)(nx.rank * p.q_row_step) + nx.q_lo0;
                        for (int j = 0; j < ((NQ > 1 && nx.q_lo0 + BM < p.q_len) ? 2 : 1); ++j)
                            for (int kb = 0; kb < D / 64; ++kb)
                                if (nq_row + j * BM < q_rows_all)
                                    tma_prefetch_l2_4d(&tm_q, kb * 64, nx.h, nq_row + j * BM, nx.bb);
                    }
                }
                if (!PERSIST) {
                    // an item without key tiles never consumes its Q: let the load land
                    if (n == 0 && kEarlyQ) {
                        const uint64_t t0 = global_timer_ns();
                        while (!mbar_try_wait(bar(C::B_Q), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
                    }
                    break;
                }
            }
            if (*abort_flag && n > 0) {
                // let the loads already issued land in shared memory before the CTA leaves
                for (int i = (n > NSK ? n - NSK : 0); i < n; ++i) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::B_KF + i % NSK), (i / NSK) & 1) &&
                           global_timer_ns() - t0 < kWaitLimitNs) {}
                }
                for (int i = (n > NSV ? n - NSV : 0); i < n; ++i) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::B_VF + i % NSV), (i / NSV) & 1) &&
                           global_timer_ns() - t0 < kWaitLimitNs) {}
                }
                if (qi > 0) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::B_Q), (qi - 1) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {}
                }
            }
        }
    } else if (warp == WARP_MMA) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            WaitCtx w{abort_flag, p.status, 3};
            int pc0 = 0, pc1 = 0;  // PV products issued per query tile, over all work items
            int oi0 = 0, oi1 = 0;  // work items whose O of query tile j was accumulated
            int n = 0;             // key tiles consumed, over all work items (K/V stages)
            int qi = 0;            // work items that visit key tiles (Q loads)
            // S of query tile j against keys [HW h, HW (h + 1)) of key tile m, into the
            // tile's S columns for part h
            auto issue_s = [&](int j, int m, int h) {
                const int sk = m % NSK;
                const uint32_t d_tmem = tbase + (uint32_t)(j * 128 + h * HW);
                const uint32_t qa = s_base + C::OFF_Q + j * C::TILE;
                const uint32_t kb_ = s_base + C::OFF_K + sk * C::TILE + (uint32_t)(h * HW * 128);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * C::SUB + (k & 3) * 32;
                    mma_ss(d_tmem, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(kb_ + off, 16, 1024),
                           C::IDESC_QK, k > 0 ? 1u : 0u);
                }
                tc_commit(bar(C::B_SF + 2 * j + h));
            };
            bool ok = true;
            if constexpr (kPSmem) {
                // ---- P through shared memory (one work item per CTA).  Per key tile n:
                // the S products of tile n + 1 go out first, each once its query tile's
                // softmax has read the previous scores; then the PV products of tile n,
                // each once its P is stored.
                const int item = blockIdx.x;
                TileSeq<DOC, NQT> seq;
                bool have = false;
                if (item < n_items) {
                    const Item it = decode(item);
                    seq.init(p, it.qr, it.rank, it.q_lo0);
                    have = seq.next(p);
                }
                if (have) {
                    ok = mbar_wait(bar(C::B_Q), 0, w) && mbar_wait(bar(C::B_KF), 0, w);
                    if (ok) {
                        tc_fence_after();
                        int si0 = 0, si1 = 0;  // S products issued per query tile
                        int pc0 = 0, pc1 = 0;  // PV products issued per query tile
                        for (int j = 0; j < NQ; ++j)
                            if (seq.need(j)) {
                                issue_s(j, 0, 0);
                                ++(j ? si1 : si0);
                            }
                        tc_commit(bar(C::B_KE));
                        while (have && ok) {
                            const bool need_n0 = seq.need(0), need_n1 = seq.need(1);
                            const bool have_next = seq.next(p);  // seq now describes tile n + 1
                            if (!have_next) tc_commit(bar(C::B_QE));  // the item's last S products are issued
                            if (have_next) {
                                if (!mbar_wait(bar(C::B_KF + (n + 1) % NSK), ((n + 1) / NSK) & 1, w)) { ok = false; break; }
                                for (int j = 0; j < NQ && ok; ++j) {
                                    if (!seq.need(j)) continue;
                                    int &si = j ? si1 : si0;
                                    // the softmax has read this tile's previous scores
                                    if (si > 0 && !mbar_wait(bar(C::B_SC + j), (si - 1) & 1, w)) { ok = false; break; }
                                    tc_fence_after();
                                    issue_s(j, n + 1, 0);
                                    ++si;
                                }
                                if (!ok) break;
                                tc_commit(bar(C::B_KE + (n + 1) % NSK));
                            }
                            const int sv = n % NSV;
                            if (!mbar_wait(bar(C::B_VF + sv), (n / NSV) & 1, w)) { ok = false; break; }
                            const uint32_t vb = s_base + C::OFF_V + sv * C::TILE;
                            for (int j = 0; j < NQ && ok; ++j) {
                                if (!(j ? need_n1 : need_n0)) continue;
                                int &pc = j ? pc1 : pc0;
                                if (!mbar_wait(bar(C::B_PH + 2 * j), pc & 1, w)) { ok = false; break; }
                                tc_fence_after();
                                const uint32_t o_tmem = tbase + C::T_O + (uint32_t)(j * D);
                                const uint32_t pa = s_base + C::OFF_P + j * C::PTILE;
#pragma unroll
                                for (int k = 0; k < BN / 16; ++k) {
                                    const uint32_t off = (k >> 2) * C::SUB + (k & 3) * 32;
                                    mma_ss(o_tmem, smem_desc_sw128(pa + off, 16, 1024),
                                           smem_desc_sw128(vb + k * 2048, C::SUB, 1024), C::IDESC_PV,
                                           (k > 0 || pc > 0) ? 1u : 0u);
                                }
                                tc_commit(bar(C::B_PV + 2 * j));
                                ++pc;
                            }
                            if (!ok) break;
                            tc_commit(bar(C::B_VE + sv));
                            ++n;
                            have = have_next;
                        }
                    }
                }
            } else {
            for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
                const Item it = decode(item);
                TileSeq<DOC, NQT> seq;
                seq.init(p, it.qr, it.rank, it.q_lo0);
                bool have = seq.next(p);
                if (!have) {
                    if (!PERSIST) break;
                    continue;
                }
                ok = mbar_wait(bar(C::B_Q), qi & 1, w) && mbar_wait(bar(C::B_KF + n % NSK), (n / NSK) & 1, w);
                if (!ok) break;
                tc_fence_after();
                for (int h = 0; h < NH; ++h)
                    for (int j = 0; j < NQ; ++j)
                        if (seq.need(j)) issue_s(j, n, h);
                tc_commit(bar(C::B_KE + n % NSK));
                bool pv0 = false, pv1 = false;  // query tile j has a PV product in this item
                while (have && ok) {
                    const bool need_n0 = seq.need(0), need_n1 = seq.need(1);
                    const bool have_next = seq.next(p);  // seq now describes tile n + 1
                    if (!have_next) tc_commit(bar(C::B_QE));  // the item's last S products are issued
                    const int sv = n % NSV;
                    if (!mbar_wait(bar(C::B_VF + sv), (n / NSV) & 1, w)) { ok = false; break; }
                    bool k_ready = false;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
#pragma unroll
                    for (int j = 0; j < NQ; ++j) {
                        int &pc = j ? pc1 : pc0;
                        bool &pv = j ? pv1 : pv0;
                        const int oi = j ? oi1 : oi0;
                        if (j ? need_n1 : need_n0) {
                            const uint32_t p_tmem = tbase + (uint32_t)(j * 128 + h * HW);
                            const uint32_t vb = s_base + C::OFF_V + sv * C::TILE;
                            const uint32_t o_tmem = tbase + C::T_O + (uint32_t)(j * D);
                            // the first product of an item overwrites O: the previous item's
                            // epilogue must have read it out
                            if (!pv && oi > 0 && !mbar_wait(bar(C::B_OF + j), (oi - 1) & 1, w)) { ok = false; break; }
                            if (kSplitP) {
                                // PV in two halves of 64 keys: the first half runs while the
                                // softmax still computes the probabilities of the second
                                if (!mbar_wait(bar(C::B_PF + j), pc & 1, w)) { ok = false; break; }
                                tc_fence_after();
#pragma unroll
                                for (int k = 0; k < BN / 32; ++k)
                                    mma_ts(o_tmem, p_tmem + k * 8, smem_desc_sw128(vb + k * 2048, C::SUB, 1024),
                                           C::IDESC_PV, (k > 0 || pv) ? 1u : 0u);
                            }
                            // part h of every key tile has its own barrier: phase = tiles so far
                            if (!mbar_wait(bar(C::B_PH + 2 * j + h), (pc / NH) & 1, w)) { ok = false; break; }
                            tc_fence_after();
                            // keys [HW h, HW (h + 1)) of the tile: P columns from the part's
                            // first, V rows from 16-key step HW h / 16 on
#pragma unroll
                            for (int k = kSplitP ? BN / 32 : 0; k < HW / 16; ++k)
                                mma_ts(o_tmem, p_tmem + k * 8,
                                       smem_desc_sw128(vb + (h * (HW / 16) + k) * 2048, C::SUB, 1024), C::IDESC_PV,
                                       (k > 0 || pv) ? 1u : 0u);
                            tc_commit(bar(C::B_PV + 2 * j + h));
                            ++pc;
                            pv = true;
                        }
                        if (have_next && seq.need(j)) {
                            if (!k_ready) {
                                if (!mbar_wait(bar(C::B_KF + (n + 1) % NSK), ((n + 1) / NSK) & 1, w)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_s(j, n + 1, h);
                        }
                    }
                    if (!ok) break;
                    }
                    if (!ok) break;
                    tc_commit(bar(C::B_VE + sv));
                    if (have_next) tc_commit(bar(C::B_KE + (n + 1) % NSK));
                    ++n;
                    have = have_next;
                }
                if (pv0) ++oi0;
                if (pv1) ++oi1;
                ++qi;
                if (!PERSIST) break;
            }
            }
            // drain: every MMA issued above has finished before TMEM is released
            tc_commit(bar(C::B_DONE));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
    }
        teardown();
        return;
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
        // ================================================================ softmax warps 0-7
        const int j = warp >> 2;        // query tile of this warpgroup
        const int wl = warp & 3;        // TMEM lane quadrant
        const int r_in = wl * 32 + lane;  // row within the query tile
        WaitCtx w{abort_flag, p.status, 5 + j};
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const uint32_t s_tmem = tbase + lane_off + (uint32_t)(j * 128);
        const uint32_t o_tmem = tbase + lane_off + C::T_O + (uint32_t)(j * D);
        // this row's P in the shared buffer (kPSmem): 8-row atoms of 1024 bytes
        const uint32_t p_row = s_base + C::OFF_P + (uint32_t)(j * C::PTILE + (r_in >> 3) * 1024 + (r_in & 7) * 128);
        (void)p_row;
        const float sl2 = p.scale_log2;
        int cs = 0;           // S tiles of this query tile consumed, over all work items
        bool aborted = false;

        // one work item: its tiles' softmax and its epilogue
        auto run_item = [&](int item) {
        const Item it = decode(item);
        const int rank = it.rank, h = it.h, bb = it.bb, q_lo0 = it.q_lo0;
        const Range32 qr = it.qr;
        const int row = q_lo0 + j * BM + r_in;  // local query index in the rank's block
        const bool row_in = row < p.q_len;
        const int pos_q = range_pos(qr, row_in ? row : (p.q_len > 0 ? p.q_len - 1 : 0));
        const int ds_row = DOC ? doc_start_of(p, pos_q) : 0;

        float m = -INFINITY;  // max used in the exponent (log2 units)
        float l = 0.f;        // running sum
        int c = 0;            // tiles processed by this query tile in this item

        TileSeq<DOC, NQT> seq;
        seq.init(p, qr, rank, q_lo0);
        // Both softmax warpgroups walk the CTA's whole key-tile sequence (the union of
        // what the two query tiles visit).  With kPingPong their exponential phases
        // take turns (tile 0 first at every entry), so each has the MUFU pipe to
        // itself while the tensor core runs the other tile's products; a warpgroup
        // with nothing to do at an entry still takes and hands over its turn, and a
        // warpgroup that gave up (bounded wait expired) keeps taking its turns
        // without work, so the hand-overs always pair up.
        // ---- mask of a partial tile: keys [beg, cnt) of the tile are visible to this row
        // (positions increase with the local key index, so the visible keys form an
        // interval: up to the row's position, from its document's start)
        auto mask_bounds = [&](const TileSeq<DOC, NQT> &sq, int &cnt, int &beg) {
            const int k0 = sq.kt * BN;
            cnt = p.kv_len - k0;
            if (cnt > BN) cnt = BN;
            const Range32 &kr = sq.kr;
            const bool seg0 = kr.len1 == 0 || k0 + cnt - 1 < kr.len0;
            if (kr.stride > 0 && (seg0 || k0 >= kr.len0)) {
                // the tile's keys lie in one segment: positions base + i stride
                const int base = seg0 ? kr.start0 : kr.start1 - kr.len0 * kr.stride;
                if (p.causal) {
                    const int ilast = pos_q < base ? -1 : kr.stride == 1 ? pos_q - base : (pos_q - base) / kr.stride;
                    cnt = min(max(ilast - k0 + 1, 0), cnt);
                }
                beg = 0;
                if (DOC) {
                    const int istar = ds_row <= base     ? 0
                                      : kr.stride == 1 ? ds_row - base
                                                       : (ds_row - base + kr.stride - 1) / kr.stride;
                    beg = min(max(istar - k0, 0), cnt);
                }
                return;
            }
            if (p.causal) {
                int lo = 0, hi = cnt;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (range_pos(sq.kr, k0 + mid) <= pos_q) lo = mid + 1; else hi = mid;
                }
                cnt = lo;
            }
            beg = 0;
            if (DOC) {
                int lo = 0, hi = cnt;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (range_pos(sq.kr, k0 + mid) < ds_row) lo = mid + 1; else hi = mid;
                }
                beg = lo;
            }
        };
        int nseq = 0;
        if (!kHalfS) {
        while (seq.next(p)) {
            bool mine = seq.need(j) && !aborted;
            // a one-item CTA: when both query tiles start on the first key tile, tile 1
            // begins after tile 0's first P is stored, so the two exponential phases
            // alternate from the start instead of sharing the MUFU pipe
            const bool stagger = kStagger && !PERSIST && nseq == 0 && seq.need(0);
            if (stagger && j == 1 && mine) {
                const bool okw = mbar_wait(bar(C::B_STAG), 0, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; mine = false; }
            }
            if (mine) {
                const bool okw = mbar_wait(bar(C::B_SF + 2 * j), cs & 1, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; mine = false; }
            }
            float s[BN];
            float f_rescale = 1.f, mu = 0.f;
            bool rescale = false;
            const bool chunked = kChunkedExp && mine && c > 0;
            if (chunked) {
                // ---- a tile after the first: the exponent's max m is known before the
                // scores arrive, so the exponentials of columns [0, 32) start while
                // columns [32, 128) are still in flight from TMEM.  A chunk whose max
                // exceeds m by more than the threshold (rare once the running max has
                // settled) raises m to the max of the chunks from it on (no earlier chunk
                // can exceed that), then rescales the probabilities already stored, the
                // row sums, and O before P is handed over.
                tc_fence_after();
                tmem_ld32f_nowait(s_tmem, s);
                tmem_wait_ld_dep32(s);
                tmem_ld32f_nowait(s_tmem + 32, s + 32);
                tmem_ld64f_nowait(s_tmem + 64, s + 64);
                const bool part = seq.partial(j);
                int cnt = BN, beg = 0;
                if (part) {
                    mask_bounds(seq, cnt, beg);
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc)
                        if (cc >= cnt || (DOC && cc < beg)) s[cc] = -INFINITY;
                }
                bool rest = false;  // columns [32, 128) arrived (and masked)
                auto take_rest = [&]() {
                    tmem_wait_ld_dep32(s + 32);
                    reg_dep64(s + 64);
                    if (part) {
#pragma unroll
                        for (int cc = 32; cc < BN; ++cc)
                            if (cc >= cnt || (DOC && cc < beg)) s[cc] = -INFINITY;
                    }
                    rest = true;
                };
                mu = (m == -INFINITY) ? 0.f : m;
                bool okr = true;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    if (q4 == 1 && !rest) take_rest();
                    // max of this chunk: two chains of 3-input max
                    float c0m = s[32 * q4], c1m = s[32 * q4 + 1];
#pragma unroll
                    for (int cc = 2; cc < 30; cc += 4) {
                        c0m = fmax3(c0m, s[32 * q4 + cc], s[32 * q4 + cc + 1]);
                        c1m = fmax3(c1m, s[32 * q4 + cc + 2], s[32 * q4 + cc + 3]);
                    }
                    const float cmx = fmax3(c0m, c1m, fmaxf(s[32 * q4 + 30], s[32 * q4 + 31])) * sl2;
                    if (__any_sync(0xffffffffu, cmx > m + kRescaleThreshold)) {
                        if (!rest) take_rest();
                        float r0 = cmx, r1 = -INFINITY;
#pragma unroll
                        for (int cc = 32 * (q4 + 1); cc < BN; cc += 2) {
                            r0 = fmaxf(r0, s[cc] * sl2);
                            r1 = fmaxf(r1, s[cc + 1] * sl2);
                        }
                        const float m_new = fmaxf(m, fmaxf(r0, r1));
                        const float f = (m_new == m) ? 1.f : ex2_approx(m - m_new);
                        if (q4 > 0) {
                            // probabilities of columns [0, 32 q4) are in TMEM (bf16): scale them
                            tmem_wait_st();
#pragma unroll
                            for (int qq = 0; qq < q4; ++qq) {
                                uint32_t pr[16];
                                tmem_ld16(s_tmem + 16 * qq, pr);
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    pr[i] = pack_bf16x2(__uint_as_float(pr[i] << 16) * f,
                                                        __uint_as_float(pr[i] & 0xffff0000u) * f);
                                tmem_st16(s_tmem + 16 * qq, pr);
                            }
                        }
                        acc0 = f2_fma(acc0, f2_pack(f, f), f2_pack(0.f, 0.f));
                        acc1 = f2_fma(acc1, f2_pack(f, f), f2_pack(0.f, 0.f));
                        l *= f;
                        f_rescale = f;
                        m = m_new;
                        mu = (m == -INFINITY) ? 0.f : m;
                        rescale = true;
                    }
                    const uint64_t nmux2 = f2_pack(-mu, -mu);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float e0, e1;
                        f2_unpack(f2_fma(f2_pack(s[32 * q4 + 2 * i], s[32 * q4 + 2 * i + 1]), sl2x2, nmux2), e0, e1);
                        e0 = ex2_approx(e0);
                        e1 = ex2_approx(e1);
                        const uint64_t e01 = f2_pack(e0, e1);
                        if (i & 1) acc1 = f2_add(acc1, e01); else acc0 = f2_add(acc0, e01);
                        pk[i] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(s_tmem + 16 * q4, pk);
                    if (q4 == 3 && rescale) {
                        // O must hold every earlier tile's P V before it is rescaled
                        const bool okw = mbar_wait(bar(C::B_PV + 2 * j), (cs - 1) & 1, w);
                        okr = !__any_sync(0xffffffffu, !okw);
                        if (okr) {
                            tc_fence_after();
#pragma unroll
                            for (int c0 = 0; c0 < D; c0 += 32) {
                                uint32_t r[32];
                                tmem_ld32(o_tmem + c0, r);
#pragma unroll
                                for (int cc = 0; cc < 32; ++cc)
                                    r[cc] = __float_as_uint(__uint_as_float(r[cc]) * f_rescale);
                                tmem_st32(o_tmem + c0, r);
                            }
                        }
                    }
                    if (q4 == 3) {
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0 && okr) mbar_arrive(bar(C::B_PH + 2 * j));
                    }
                }
                float a0, a1, a2, a3;
                f2_unpack(acc0, a0, a1);
                f2_unpack(acc1, a2, a3);
                l += (a0 + a1) + (a2 + a3);
                if (okr) {
                    ++c;
                    ++cs;
                } else {
                    aborted = true;
                }
            }
            if (kPingPong && !kTurnLate && (j == 1 || nseq > 0)) named_bar_sync(j == 0 ? kTurn0 : kTurn1, 2 * BM);
            if (mine && !chunked) {
                tc_fence_after();
                tmem_ld64f_nowait(s_tmem, s);
                tmem_ld64f_nowait(s_tmem + 64, s + 64);
                tmem_wait_ld_dep(s);
                reg_dep64(s + 64);
                if (kPSmem) {  // the scores are in registers: the tile's next S may overwrite them
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(C::B_SC + j));
                }
                // ---- mask (partial tiles only).  Positions increase with the local key
                // index, so the keys this row may see form a prefix of the tile.
                if (seq.partial(j)) {
                    int cnt, beg;
                    mask_bounds(seq, cnt, beg);
#pragma unroll
                    for (int cc = 0; cc < BN; ++cc)
                        if (cc >= cnt || (DOC && cc < beg)) s[cc] = -INFINITY;
                }
                // ---- row max: four chains of 3-input max
                float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
                for (int cc = 4; cc < BN - 4; cc += 8) {
                    mx0 = fmax3(mx0, s[cc], s[cc + 1]);
                    mx1 = fmax3(mx1, s[cc + 2], s[cc + 3]);
                    mx2 = fmax3(mx2, s[cc + 4], s[cc + 5]);
                    mx3 = fmax3(mx3, s[cc + 6], s[cc + 7]);
                }
                mx0 = fmax3(mx0, s[BN - 4], s[BN - 3]);
                mx1 = fmax3(mx1, s[BN - 2], s[BN - 1]);
                const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
                // Raise the exponent's max only when it grew by more than the threshold;
                // then l is rescaled here and O below, before the first half of P is
                // handed to the MMA warp.
                if (c == 0) {
                    m = mx;
                } else {
                    const bool need_rescale = mx > m + kRescaleThreshold;
                    rescale = __any_sync(0xffffffffu, need_rescale);
                    if (rescale) {
                        const float m_new = fmaxf(m, mx);
                        f_rescale = (m_new == m) ? 1.f : ex2_approx(m - m_new);
                        m = m_new;
                        l *= f_rescale;
                    }
                }
                mu = (m == -INFINITY) ? 0.f : m;
            }
            if (kPingPong && kTurnLate && (j == 1 || nseq > 0)) named_bar_sync(j == 0 ? kTurn0 : kTurn1, 2 * BM);
            if (mine && !chunked) {
                // ---- probabilities, row sum, bf16 P into TMEM columns [0, 64) of S_j,
                // 32 columns at a time so each chunk's scores die once packed.  The
                // scale-subtract and the row sum run as packed fp32x2 instructions.
                // With kSplitP, P is handed to the MMA warp in two halves (keys [0, 64),
                // then [64, 128)); a rescale of O happens before the first half, since
                // PV adds into O.
                bool okr = true;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t nmux2 = f2_pack(-mu, -mu);
                uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
                const bool emu = kEmuMod > 0 && !seq.partial(j);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float e0, e1;
                        f2_unpack(f2_fma(f2_pack(s[32 * q4 + 2 * i], s[32 * q4 + 2 * i + 1]), sl2x2, nmux2), e0, e1);
                        if (kEmuMod > 0 && (i % (kEmuMod > 0 ? kEmuMod : 1)) == kEmuMod - 1 && emu) {
                            exp2_fma2(e0, e1);
                        } else {
                            e0 = ex2_approx(e0);
                            e1 = ex2_approx(e1);
                        }
                        const uint64_t e01 = f2_pack(e0, e1);
                        if (i & 1) acc1 = f2_add(acc1, e01); else acc0 = f2_add(acc0, e01);
                        pk[i] = pack_bf16x2(e0, e1);
                    }
                    if (kPSmem) {
                        // the buffer is free once the tile's previous PV is done
                        if (q4 == 0 && cs > 0) {
                            const bool okw = mbar_wait(bar(C::B_PV + 2 * j), (cs - 1) & 1, w);
                            okr = !__any_sync(0xffffffffu, !okw);
                        }
                        if (okr) {
                            // row r_in, keys [32 q4, 32 q4 + 32): 16-byte chunks c = 4 q4 + i
                            // of the 128-byte-swizzled K-major layout (64-key blocks)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int cc = 4 * q4 + i;
                                st_shared_v4(p_row + (uint32_t)((cc >> 3) * C::SUB + (((cc & 7) ^ (r_in & 7)) << 4)),
                                             pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                            }
                        }
                    } else {
                        tmem_st16(s_tmem + 16 * q4, pk);
                    }
                    if (q4 == (kSplitP ? 1 : 3) && rescale) {
                        // O must hold every earlier tile's P V before it is rescaled
                        const bool okw = mbar_wait(bar(C::B_PV + 2 * j), (cs - 1) & 1, w);
                        okr = okr && !__any_sync(0xffffffffu, !okw);
                        if (okr) {
                            tc_fence_after();
#pragma unroll
                            for (int c0 = 0; c0 < D; c0 += 32) {
                                uint32_t r[32];
                                tmem_ld32(o_tmem + c0, r);
#pragma unroll
                                for (int cc = 0; cc < 32; ++cc)
                                    r[cc] = __float_as_uint(__uint_as_float(r[cc]) * f_rescale);
                                tmem_st32(o_tmem + c0, r);
                            }
                        }
                    }
                    if (q4 == 3 && kPingPong) named_bar_arrive(j == 0 ? kTurn1 : kTurn0, 2 * BM);
                    if ((kSplitP && q4 == 1) || q4 == 3) {
                        if (kPSmem) fence_async_smem();  // P stores visible to the tensor core
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0 && okr) mbar_arrive(bar((kSplitP && q4 == 1) ? C::B_PF + j : C::B_PH + 2 * j));
                        if (q4 == 3 && stagger && j == 0 && lane == 0) mbar_arrive(bar(C::B_STAG));
                    }
                }
                float a0, a1, a2, a3;
                f2_unpack(acc0, a0, a1);
                f2_unpack(acc1, a2, a3);
                l += (a0 + a1) + (a2 + a3);
                if (okr) {
                    ++c;
                    ++cs;
                } else {
                    aborted = true;
                }
            } else if (kPingPong) {
                named_bar_arrive(j == 0 ? kTurn1 : kTurn0, 2 * BM);
            }
            ++nseq;
        }
        } else {
        while (seq.next(p)) {
            bool mine = seq.need(j) && !aborted;
            if (kPingPong && !kTurnLate && (j == 1 || nseq > 0)) named_bar_sync(j == 0 ? kTurn0 : kTurn1, 2 * BM);
            // the tile's S parts (one, or two halves of 64 keys), each: scores out of
            // TMEM, mask, row max, probabilities and row sum, bf16 P back into TMEM
#pragma unroll
            for (int hp = 0; hp < NH; ++hp) {
            if (mine) {
                const bool okw = mbar_wait(bar(C::B_SF + 2 * j + hp), cs & 1, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; mine = false; }
            }
            float s[HW];
            float f_rescale = 1.f, mu = 0.f;
            bool rescale = false;
            const uint32_t sp_tmem = s_tmem + (uint32_t)(hp * HW);  // this part's S / P columns
            if (mine) {
                tc_fence_after();
                tmem_ld64f_nowait(sp_tmem, s);
                if (HW == 128) tmem_ld64f_nowait(sp_tmem + 64, s + (HW == 128 ? 64 : 0));
                tmem_wait_ld_dep(s);
                if (HW == 128) reg_dep64(s + (HW == 128 ? 64 : 0));
                // ---- mask (partial tiles only).  Positions increase with the local key
                // index, so the keys this row may see form a prefix of the tile.
                if (seq.partial(j)) {
                    const int k0 = seq.kt * BN + hp * HW;
                    int cnt = p.kv_len - k0;
                    if (cnt > HW) cnt = HW;
                    if (cnt < 0) cnt = 0;
                    if (p.causal) {
                        int lo = 0, hi = cnt;
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (range_pos(seq.kr, k0 + mid) <= pos_q) lo = mid + 1; else hi = mid;
                        }
                        cnt = lo;
                    }
                    int beg = 0;  // keys before this row's document start are invisible
                    if (DOC) {
                        int lo = 0, hi = cnt;
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (range_pos(seq.kr, k0 + mid) < ds_row) lo = mid + 1; else hi = mid;
                        }
                        beg = lo;
                    }
#pragma unroll
                    for (int cc = 0; cc < HW; ++cc)
                        if (cc >= cnt || (DOC && cc < beg)) s[cc] = -INFINITY;
                }
                // ---- row max: four chains of 3-input max
                float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
                for (int cc = 4; cc < HW - 4; cc += 8) {
                    mx0 = fmax3(mx0, s[cc], s[cc + 1]);
                    mx1 = fmax3(mx1, s[cc + 2], s[cc + 3]);
                    mx2 = fmax3(mx2, s[cc + 4], s[cc + 5]);
                    mx3 = fmax3(mx3, s[cc + 6], s[cc + 7]);
                }
                mx0 = fmax3(mx0, s[HW - 4], s[HW - 3]);
                mx1 = fmax3(mx1, s[HW - 2], s[HW - 1]);
                const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sl2;
                // Raise the exponent's max only when it grew by more than the threshold;
                // then l is rescaled here and O below, before the part's P is handed to
                // the MMA warp.
                if (c == 0 && hp == 0) {
                    m = mx;
                } else {
                    const bool need_rescale = mx > m + kRescaleThreshold;
                    rescale = __any_sync(0xffffffffu, need_rescale);
                    if (rescale) {
                        const float m_new = fmaxf(m, mx);
                        f_rescale = (m_new == m) ? 1.f : ex2_approx(m - m_new);
                        m = m_new;
                        l *= f_rescale;
                    }
                }
                mu = (m == -INFINITY) ? 0.f : m;
            }
            if (kPingPong && kTurnLate && (j == 1 || nseq > 0)) named_bar_sync(j == 0 ? kTurn0 : kTurn1, 2 * BM);
            if (mine) {
                // ---- probabilities, row sum, bf16 P into the part's first HW / 2 TMEM
                // columns, 32 scores at a time so each chunk's scores die once packed.
                // The scale-subtract and the row sum run as packed fp32x2 instructions.
                // With kSplitP (whole S), P is handed to the MMA warp in two halves
                // (keys [0, 64), then [64, 128)); a rescale of O happens before the
                // first P of the part is handed over, since PV adds into O.
                bool okr = true;
                const uint64_t sl2x2 = f2_pack(sl2, sl2);
                const uint64_t nmux2 = f2_pack(-mu, -mu);
                uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = f2_pack(0.f, 0.f);
                const bool emu = kEmuMod > 0 && !seq.partial(j);
                constexpr int NC = HW / 32;  // chunks of 32 scores
#pragma unroll
                for (int q4 = 0; q4 < NC; ++q4) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float e0, e1;
                        f2_unpack(f2_fma(f2_pack(s[32 * q4 + 2 * i], s[32 * q4 + 2 * i + 1]), sl2x2, nmux2), e0, e1);
                        if (kEmuMod > 0 && (i % (kEmuMod > 0 ? kEmuMod : 1)) == kEmuMod - 1 && emu) {
                            exp2_fma2(e0, e1);
                        } else {
                            e0 = ex2_approx(e0);
                            e1 = ex2_approx(e1);
                        }
                        const uint64_t e01 = f2_pack(e0, e1);
                        if (i & 1) acc1 = f2_add(acc1, e01); else acc0 = f2_add(acc0, e01);
                        pk[i] = pack_bf16x2(e0, e1);
                    }
                    tmem_st16(sp_tmem + 16 * q4, pk);
                    if (q4 == (kSplitP ? 1 : NC - 1) && rescale) {
                        // O must hold every earlier part's P V before it is rescaled
                        // every earlier part's PV: this tile's part 0 (hp = 1), or the
                        // previous tile's last part (hp = 0; its part 0 finished before this
                        // tile's S part 0 did)
                        const bool okw = hp == 1 ? mbar_wait(bar(C::B_PV + 2 * j), cs & 1, w)
                                                : mbar_wait(bar(C::B_PV + 2 * j + NH - 1), (cs - 1) & 1, w);
                        okr = !__any_sync(0xffffffffu, !okw);
                        if (okr) {
                            tc_fence_after();
#pragma unroll
                            for (int c0 = 0; c0 < D; c0 += 32) {
                                uint32_t r[32];
                                tmem_ld32(o_tmem + c0, r);
#pragma unroll
                                for (int cc = 0; cc < 32; ++cc)
                                    r[cc] = __float_as_uint(__uint_as_float(r[cc]) * f_rescale);
                                tmem_st32(o_tmem + c0, r);
                            }
                        }
                    }
                    if (q4 == NC - 1 && kPingPong) named_bar_arrive(j == 0 ? kTurn1 : kTurn0, 2 * BM);
                    if ((kSplitP && q4 == 1) || q4 == NC - 1) {
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0 && okr) mbar_arrive(bar((kSplitP && q4 == 1) ? C::B_PF + j : C::B_PH + 2 * j + hp));
                    }
                }
                float a0, a1, a2, a3;
                f2_unpack(acc0, a0, a1);
                f2_unpack(acc1, a2, a3);
                l += (a0 + a1) + (a2 + a3);
                if (!okr) {
                    aborted = true;
                    mine = false;
                }
            } else if (kPingPong) {
                named_bar_arrive(j == 0 ? kTurn1 : kTurn0, 2 * BM);
            }
            }  // S parts
            if (mine) {
                ++c;
                ++cs;
            }
            ++nseq;
        }
        }
        // tile 0 takes the hand-over of tile 1's last turn
        if (kPingPong && j == 0 && nseq > 0) named_bar_sync(kTurn0, 2 * BM);
        aborted = __any_sync(0xffffffffu, aborted || (*abort_flag != 0));

        // ================================================================ epilogue
        if (!aborted && c > 0) {
            // the last tile's PV of every part (each part's barrier completes once per tile)
            bool okw = true;
            for (int hp = 0; hp < NH; ++hp) okw = okw && mbar_wait(bar(C::B_PV + 2 * j + hp), (cs - 1) & 1, w);
            aborted = __any_sync(0xffffffffu, !okw);
            if (!aborted) tc_fence_after();
        }
        // a one-item CTA's tile epilogue may meet at a named barrier (the TMA store):
        // the four warps of the tile agree on going ahead (no wait that can expire
        // comes after this point)
        if (!PERSIST) aborted = bar_any(4 + j, BM, aborted || (*abort_flag != 0));
        if (!aborted && (c > 0 || p.epi == EPI_STORE || p.o_out != nullptr)) {
            const bool empty = !(l > 0.f);
            const float lse2 = empty ? -INFINITY : m + log2f(l);
            const float inv_l = empty ? 0.f : 1.f / l;
            const int64_t orow = (int64_t)rank * p.q_row_step + row;
            const int64_t obase = (int64_t)bb * p.o_sb + orow * p.o_ss + (int64_t)h * p.o_sh;
            float *lse_ptr = p.lse + (int64_t)bb * p.lse_sb + (int64_t)h * p.lse_sh + orow * p.lse_ss;
            // a row outside the output tensors (debug builds record it and skip it)
            const bool row_ok = row_in && bounds_ok(orow >= 0 && orow < q_rows_all && h < p.hq && bb < p.b,
                                                    p.status, 103);
            // bf16 tiles that lie wholly inside the block leave through shared memory and
            // one TMA store: a thread owns a row, so direct stores would touch 32 rows
            // per warp instruction.  The staging buffer is this tile's Q buffer, free
            // since the last PV product (issued after the tile's last S) completed.
            const int rt = (threadIdx.x & (BM - 1));  // row within the tile (= r_in)
            const int tile_row0 = row - rt;           // the tile's first local row
            const bool tma_o = kTmaO && !PERSIST && o_tma && p.epi == EPI_STORE && tile_row0 + BM <= p.q_len &&
                               bounds_ok(orow - rt + BM <= q_rows_all, p.status, 105);
            if (tma_o) {
                uint8_t *stile = smem + C::OFF_Q + j * C::TILE;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    if (c > 0) tmem_ld32(o_tmem + c0, r);
                    uint32_t w16[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w16[i] = (c > 0) ? pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l)
                                         : 0u;
                    // columns [c0, c0 + 32): 64-column box c0 / 64, 16-byte chunks from
                    // (c0 % 64) / 8, 128-byte swizzle (chunk index ^ row % 8)
                    uint8_t *rowp = stile + (c0 / 64) * C::SUB + rt * 128;
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int ch = (((c0 % 64) / 8) + t) ^ (rt & 7);
                        *reinterpret_cast<uint4 *>(rowp + ch * 16) =
                            make_uint4(w16[4 * t], w16[4 * t + 1], w16[4 * t + 2], w16[4 * t + 3]);
                    }
                }
                fence_async_smem();
                named_bar_sync(4 + j, BM);
                if (rt == 0) {
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_store_4d(&tm_o, s_base + C::OFF_Q + j * C::TILE + kb * C::SUB, kb * 64, h, (int)orow, bb);
                    bulk_commit();
                    bulk_wait_read_all();  // the CTA may leave once the box is read out
                }
                if (row_ok) *lse_ptr = lse2 * kLn2;
            } else if (p.epi == EPI_STORE) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    if (c > 0) tmem_ld32(o_tmem + c0, r);
                    float v[32];
#pragma unroll
                    for (int cc = 0; cc < 32; ++cc) v[cc] = (c > 0) ? __uint_as_float(r[cc]) * inv_l : 0.f;
                    if (row_ok) store_row_chunk(p.o, p.o_dtype, obase + c0, v);
                }
                if (row_ok) *lse_ptr = lse2 * kLn2;
            } else {
                // EPI_MERGE: (o, lse) in memory are fp32 and hold a partial; LSE-merge
                // this launch's result into them.  With o_out set, the merged o goes
                // there (in o_out's dtype) instead of back into o, also for rows this
                // launch gave nothing (a copy of the partial in memory).
                const bool to_out = p.o_out != nullptr;
                const float la = row_ok ? *lse_ptr * kLog2e : -INFINITY;
                float wa = 1.f, wb = 0.f, new_lse = la;
                if (!empty) {
                    if (la == -INFINITY) {
                        wa = 0.f;
                        wb = inv_l;
                        new_lse = lse2;
                    } else {
                        const float M = fmaxf(la, lse2);
                        new_lse = M + log2f(ex2_approx(la - M) + ex2_approx(lse2 - M));
                        wa = ex2_approx(la - new_lse);
                        wb = ex2_approx(lse2 - new_lse) * inv_l;
                    }
                }
                const float *orow_ptr = reinterpret_cast<const float *>(p.o) + obase;
                const int64_t out_base =
                    to_out ? (int64_t)bb * p.oo_sb + orow * p.oo_ss + (int64_t)h * p.oo_sh : obase;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    if (c > 0) tmem_ld32(o_tmem + c0, r);
                    if (row_ok && (!empty || to_out)) {
                        float v[32];
                        const float4 *src4 = reinterpret_cast<const float4 *>(orow_ptr + c0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 a = (wa != 0.f) ? src4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                            const float b0 = empty ? 0.f : wb * __uint_as_float(r[4 * i + 0]);
                            const float b1 = empty ? 0.f : wb * __uint_as_float(r[4 * i + 1]);
                            const float b2 = empty ? 0.f : wb * __uint_as_float(r[4 * i + 2]);
                            const float b3 = empty ? 0.f : wb * __uint_as_float(r[4 * i + 3]);
                            v[4 * i + 0] = fmaf(wa, a.x, b0);
                            v[4 * i + 1] = fmaf(wa, a.y, b1);
                            v[4 * i + 2] = fmaf(wa, a.z, b2);
                            v[4 * i + 3] = fmaf(wa, a.w, b3);
                        }
                        if (to_out) store_row_chunk(p.o_out, p.o_out_dtype, out_base + c0, v);
                        else store_row_chunk(p.o, DT_FP32, obase + c0, v);
                    }
                }
                if (row_ok && !empty) *lse_ptr = new_lse * kLn2;
            }
        }
        if (PERSIST && !aborted && c > 0) {
            // O of this tile is read out: the next item's first PV may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_OF + j));
        }
        };
        if (PERSIST) {
            for (int item = blockIdx.x; item < n_items && !aborted; item += gridDim.x) run_item(item);
        } else {
            run_item(blockIdx.x);
        }
        teardown();
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [b, s, H, d] bf16 with element strides (sb, ss, sh, 1) -> 4-D map {d, H, s, b},
// box {64, 1, 128, 1}, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap *m, const void *base, int64_t b, int64_t s, int64_t H, int64_t d, int64_t sb, int64_t ss,
              int64_t sh)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)s, (cuuint64_t)b};
    cuuint64_t strides[3] = {(cuuint64_t)sh * 2, (cuuint64_t)ss * 2, (cuuint64_t)sb * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)BM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, bool DOC, bool PERSIST, int NQT>
cudaError_t launch_dd(const AttnParams &p, cudaStream_t stream, const CUtensorMap &tq, const CUtensorMap &tk,
                      const CUtensorMap &tv, const CUtensorMap &to, int o_tma)
{
    using C = Cfg<D, NQT>;
    static unsigned long long attr_done = 0;
    cudaError_t e = set_smem_per_device((const void *)attn_tc_kernel<D, DOC, PERSIST, NQT>, C::SMEM, &attr_done);
    if (e != cudaSuccess) return e;
    const int64_t items = (int64_t)p.n_ranks * p.n_qt * p.b * p.hq;
    if (items == 0) return cudaSuccess;
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    // persistent: one CTA per SM walks the items (one CTA fits an SM); otherwise one per item
    const int64_t grid = PERSIST ? std::min<int64_t>(items, sm_count()) : items;
    // one CTA per item: the item one wave later prefetches its Q
    const int next_stride = PERSIST ? 0 : sm_count() * C::CTAS_PER_SM;
    attn_tc_kernel<D, DOC, PERSIST, NQT><<<(unsigned)grid, C::NTHR, C::SMEM, stream>>>(p, tq, tk, tv, to, o_tma,
                                                                                     next_stride);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttnParams &p, cudaStream_t stream, int64_t q_rows, int64_t kv_rows)
{
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, p.q, p.b, q_rows, p.hq, D, p.q_sb, p.q_ss, p.q_sh) ||
        !make_map(&tk, p.k, p.b, kv_rows, p.hkv, D, p.k_sb, p.k_ss, p.k_sh) ||
        !make_map(&tv, p.v, p.b, kv_rows, p.hkv, D, p.v_sb, p.v_ss, p.v_sh))
        return cudaErrorInvalidValue;
    // the document mask leaves few key tiles per work item: a persistent grid keeps the
    // per-item set-up (Q load, pipeline fill, epilogue) off the critical path
    // bf16 output written by TMA stores from the epilogue (when its strides allow a map)
    CUtensorMap to = tq;
    int o_tma = 0;
    if (p.epi == EPI_STORE && p.o_dtype == DT_BF16 && make_map(&to, p.o, p.b, q_rows, p.hq, D, p.o_sb, p.o_ss, p.o_sh))
        o_tma = 1;
    else
        to = tq;
    if (p.n_docs > 0) return launch_dd<D, true, kDocPersist, kDocNQ>(p, stream, tq, tk, tv, to, o_tma);
    return launch_dd<D, false, kRingPersist, kRingNQ>(p, stream, tq, tk, tv, to, o_tma);
}

}  // namespace

// Query rows per CTA of the tensor-core kernel (the work-order table counts these).
int attn_tc_rows_per_cta(bool doc) { return (doc ? kDocNQ : kRingNQ) * BM; }

cudaError_t launch_attn_tc(const AttnParams &p, cudaStream_t stream)
{
    // tensor rows covered by the maps: whole rank-major tensors for the ring, the
    // single blocks otherwise
    const int64_t q_rows = p.q_row_step ? (int64_t)p.n_ranks * p.q_row_step : p.q_len;
    const int64_t kv_rows = p.kv_row_step ? (int64_t)p.n_ranks * p.kv_row_step : p.kv_len;
    if (p.d == 128) return launch_d<128>(p, stream, q_rows, kv_rows);
    if (p.d == 64) return launch_d<64>(p, stream, q_rows, kv_rows);
    return cudaErrorInvalidValue;
}

}  // namespace cpattn
