// attn_bwd.cu -- bf16 attention backward on sm_100a tensor cores (tcgen05 + TMEM +
// TMA), the whole ring's backward in one launch.
//
// What it computes ("上下文并行与 Ring Attention", hs-black.github.io, section
// 分块注意力, paragraph on the backward pass; section Ring Attention for the
// schedule): with the forward's GLOBAL lse and D = do . o of every query row,
//   p = e^{x - lse},  dv_j += p do,  dx = p (do . v_j - D),
//   dq += scale dx k_j,  dk_j += scale dx q.
// In the ring, K/V block j visits rank (j + r) mod N at step r; dK_j, dV_j travel
// with it and dQ stays home.  On one device the travelling accumulators become
// TMEM-resident: one CTA keeps a 128-key tile of block j (K, V in shared memory,
// dK, dV in TMEM) and walks every (query head of its group, ring step, 64-row
// query tile) that sees the tile.  dQ shares leave through bulk-tensor reductions
// (fp32 add) into an accumulator in HBM.
//
// Per query tile, in the transposed form that puts keys on TMEM lanes:
//   S^T  = K Q^T        (M 128 keys, N 64 queries, K = d)   -> TMEM
//   dP^T = V dO^T       (same shapes)                        -> TMEM
//   P^T  = exp2(S^T scale log2e - lse log2e), dS^T = P^T (dP^T - D)  (softmax warps;
//          P^T bf16 back into TMEM, dS^T bf16 to shared memory, 128-byte swizzled)
//   dV  += P^T dO       (M 128 keys, N = d, K 64 queries)    TMEM accumulator
//   dK  += dS^T Q       (same)                               TMEM accumulator
//   dQ^T = K^T dS^T     (M = d, N 64 queries, K 128 keys)    -> TMEM -> fp32 staging
//                                                              -> bulk reduce-add
// Roles (448 threads):
//   warps 0-3  / 4-7  P and dS of query columns [0, 32) / [32, 64), one key row per
//                     thread; afterwards the dK (warps 0-3) and dV (4-7) epilogue
//   warps 8-11 dQ^T out of TMEM, scaled, staged, reduced into the accumulator
//   warp 12    TMA producer (K, V once; Q, dO and row statistics per query tile)
//   warp 13    TMEM owner and single-thread MMA issuer
// TMEM columns: S^T double buffer [0, 128), dP^T [128, 192), dQ^T [192, 256),
// dV [256, 384), dK [384, 512).  The softmax warps overwrite part of their own S^T
// columns with bf16 P^T, which the dV MMA reads straight from TMEM; dS^T has two
// shared-memory buffers, so tile n + 1 is written while the MMAs of tile n still
// read tile n.  Three Q/dO stages keep the next loads in flight.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "bwd.h"
#include "ptx.cuh"

namespace cpattn {
namespace {

constexpr int BK = kBwdKeyTile;    // keys per CTA
constexpr int BQ = kBwdQueryTile;  // queries per step
constexpr int HD = 128;            // head dim
constexpr int NS = 3;              // Q / dO stages
constexpr int NTHREADS = 448;
constexpr int WARP_DQ0 = 8;
constexpr int WARP_LOAD = 12;
constexpr int WARP_MMA = 13;
constexpr float kLog2eB = 1.44269504088896340736f;

struct BCfg {
    static constexpr int KV_SUB = BK * 128;  // 128 rows x 64 bf16 (one swizzle column block)
    static constexpr int Q_SUB = BQ * 128;   // 64 rows x 64 bf16
    static constexpr int KV_TILE = 2 * KV_SUB;
    static constexpr int Q_TILE = 2 * Q_SUB;
    static constexpr int STAGE = 2 * Q_TILE;  // Q then dO
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KV_TILE;
    static constexpr int OFF_Q = OFF_V + KV_TILE;
    static constexpr int PBUF = BK * 128;              // one [128 keys][64 queries] bf16 tile
    static constexpr int OFF_DS = OFF_Q + NS * STAGE;  // dS^T, two buffers
    static constexpr int OFF_DQ = OFF_DS + 2 * PBUF;   // dQ staging [64 queries][128] fp32
    static constexpr int OFF_ST = OFF_DQ + BQ * HD * 4;  // per stage: 64 x (lse log2e, D)
    static constexpr int OFF_BAR = OFF_ST + NS * BQ * 8;
    enum {
        B_KV = 0,
        B_QF = 1,
        B_QE = B_QF + NS,
        B_SF = B_QE + NS,
        B_DPF = B_SF + 2,
        B_PR,             // per tile parity: P^T in TMEM / dS^T in shared memory ready
        B_DSR = B_PR + 2, // (8 warp arrivals); dS^T buffer free (MMA commit)
        B_DSE = B_DSR + 2,
        B_DQF = B_DSE + 2,
        B_DQE,
        B_DONE,
        NBAR
    };
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;
    static_assert(SMEM <= 232448, "shared memory per CTA exceeds 227 KB");
    static constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 192, T_DV = 256, T_DK = 384, TMEM_COLS = 512;
};

// kind::f16 instruction descriptor with both operand majors selectable:
// bit 15 A MN-major, bit 16 B MN-major (other fields as idesc_bf16_f32).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t IDESC_S = idesc_bf16(BK, BQ, false, false);   // K Q^T, V dO^T
constexpr uint32_t IDESC_KV = idesc_bf16(BK, HD, false, true);   // P^T dO, dS^T Q
constexpr uint32_t IDESC_DQ = idesc_bf16(HD, BQ, true, true);    // K^T dS^T

// ---- bulk copies and reductions (no multicast)

// Contiguous global -> shared copy, completion counted on `bar` (bytes).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Element-wise fp32 add of a shared-memory box into the global tensor of `map`.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap *map, uint32_t src, int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Query-tile sequence of one CTA: (query head of the group, ring step, query tile)
// with the tile seeing at least one key of the CTA's key tile.  Every role walks it.
// End of the document that holds position pos: the first document start > pos
// (INT32_MAX past the last document).
__device__ __forceinline__ int64_t doc_end_of(const BwdParams &p, int64_t pos)
{
    if (!bounds_ok(pos >= 0 && pos < p.seq_len, p.status, 206)) return INT32_MAX;
    return (int64_t)__ldg(p.doc_pos_end + pos);
}

// First query tile (of BQ rows, q_len rows, ranges q) whose row at offset off
// (clamped to the block) has a position >= x.
__device__ __forceinline__ int first_qtile_from(const Range32 &q, int q_len, int off, int x)
{
    const int n_qt = (q_len + BQ - 1) / BQ;
    int lo = 0, hi = n_qt;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int r = mid * BQ + off;
        if (r > q_len - 1) r = q_len - 1;
        if (range_pos(q, r) < x) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// With the head-major grid the CTAs of one key block must not all reduce into the
// same dQ rows at once.  Either the ring steps of a head start at a rotation that
// depends on the key tile (p.tile_rotation = 0: concurrent CTAs spread over every
// query rank of the group's heads), or every CTA walks the steps in order and starts
// each step's query tiles at an offset that depends on the key tile, wrapping
// around (1: concurrent CTAs spread over the tiles of one or two query ranks).  The
// host picks 1 when the group's dQ rows are too many for L2 to hold.
struct QSeq {
    const BwdParams *p;
    // positions stay below 2^30 (the ABI checks it), so the ranges are 32-bit
    int j, k_lo, h0, n_qt, nsteps, rot, qrot;
    int qb_cur, left;              // first query tile of the current step, tiles left in it
    Range32 kr;
    int hi, sc, qt, qt_full, i, h;
    int qt_stop, qt_fend;          // query tiles [qt_stop, ...) see nothing; [qt_full, qt_fend) are full
    int de_first, de_last;         // document ends of the tile's first / last key (document mask)
    Range32 qr;

    __device__ void init(const BwdParams &pp, int jj, int kt, const Range &k, int hq0)
    {
        p = &pp;
        j = jj;
        k_lo = kt * BK;
        kr = to_range32(k);
        h0 = hq0;
        n_qt = (pp.q_len + BQ - 1) / BQ;
        nsteps = pp.step_end - pp.step_begin;
        rot = (nsteps > 0 && pp.head_major && !pp.tile_rotation) ? kt % nsteps : 0;
        qrot = (pp.head_major && pp.tile_rotation) ? kt : 0;
        qb_cur = 0;
        left = 0;
        hi = 0;
        sc = -1;
        qt = n_qt - 1;
        qt_full = 0;
        qt_stop = n_qt;
        qt_fend = n_qt;
        de_first = de_last = INT32_MAX;
        if (pp.n_docs > 0 && pp.kv_len > 0) {
            const int64_t k_hi = k_lo + BK - 1 < pp.kv_len - 1 ? k_lo + BK - 1 : pp.kv_len - 1;
            de_first = (int)doc_end_of(pp, range_pos(k, (int64_t)k_lo));
            de_last = (int)doc_end_of(pp, range_pos(k, k_hi));
        }
        i = 0;
        h = hq0;
    }
    __device__ bool next()
    {
        if (nsteps <= 0) return false;
        if (!p->tile_rotation) {
            ++qt;
            while (qt >= qt_stop) {
                if (!next_step()) return false;
                qt = qb_cur;
            }
            return true;
        }
        if (left > 1) {  // the next query tile of this step, wrapping past the last
            --left;
            if (++qt >= qt_stop) qt = qb_cur;
            return true;
        }
        do {
            if (!next_step()) return false;
        } while (qb_cur >= qt_stop);
        left = qt_stop - qb_cur;
        qt = qb_cur + qrot % left;
        return true;
    }
    // Moves to the next (query head, ring step) and works out its query tiles:
    // [qb_cur, qt_stop) see the key tile (qb_cur >= qt_stop: none).
    __device__ bool next_step()
    {
        if (++sc >= nsteps) {
            sc = 0;
            if (++hi >= p->group) return false;
        }
        const int r = p->step_begin + (sc + rot) % nsteps;
        const int N = p->n_ranks;
        i = (j + r) % N;
        qr = p->use_layout ? layout_range_t<int>(p->layout, N, (int)p->seq_len, i) : to_range32(p->q_range);
        h = h0 + hi;
        if (p->n_docs > 0 && p->kv_len > 0 && p->q_len > 0 &&
            range_pos(qr, 0) >= de_last) {  // the whole rank lies after the tile's documents
            qb_cur = n_qt;
            qt_stop = n_qt;
            return true;
        }
        q_tile_bounds<int>(qr, p->q_len, BQ, kr, p->kv_len, k_lo, BK, p->causal != 0, &qb_cur, &qt_full);
        qt_stop = n_qt;
        qt_fend = n_qt;
        if (p->n_docs > 0) {
            // rows at or past the end of the last key's document see none of the
            // tile; rows must end before the first key's document ends to see all
            qt_stop = first_qtile_from(qr, p->q_len, 0, de_last);
            qt_fend = first_qtile_from(qr, p->q_len, BQ - 1, de_first);
        }
        return true;
    }
    __device__ bool partial() const { return qt < qt_full || qt >= qt_fend; }
    __device__ int q_row() const { return (int)(i * p->q_row_step) + qt * BQ; }
};

// 32 consecutive bf16 of one row (64 bytes) from fp32 values.
__device__ __forceinline__ void store_bf16x32(void *dst, const float *v)
{
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
        w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
        w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
        w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
        d4[i] = w;
    }
}

// 32 bf16 (packed in 16 words) into row `row` of a [128 rows x 64] bf16 K-major
// tile with 128-byte swizzle, columns [32 half, 32 half + 32).
__device__ __forceinline__ void st_sw128_half(uint8_t *tile, int row, int half, const uint32_t *w)
{
    uint8_t *rowp = tile + row * 128;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const int ch = (half * 4 + t) ^ (row & 7);
        *reinterpret_cast<uint4 *>(rowp + ch * 16) = make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
    attn_bwd_kernel(const __grid_constant__ BwdParams p, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_dq)
{
    using C = BCfg;
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

    // ---- work item: (key rank, key tile) from the order table, then (batch, kv head)
    // head_major: (batch, kv head) outermost, so the CTAs resident at one time share a
    // few heads' dQ rows and the accumulator they reduce into stays in L2; otherwise
    // the work order outermost (heaviest key tiles of every head first)
    const int n_items = p.order_len ? p.order_len : p.n_kv_blocks * p.n_kt;
    const int bkh = p.b * p.hkv;
    const int bh = p.head_major ? (int)(blockIdx.x / n_items) : (int)(blockIdx.x % bkh);
    const int e = p.head_major ? (int)(blockIdx.x % n_items) : (int)(blockIdx.x / bkh);
    int j, kt;
    if (p.order_len) {
        j = (int)(p.order[e] >> 16);
        kt = (int)(p.order[e] & 0xffffu);
    } else {
        j = e / p.n_kt;
        kt = e % p.n_kt;
    }
    const int hk = bh % p.hkv;
    const int bb = bh / p.hkv;
    const int k_lo = kt * BK;
    // tensor rows the maps and outputs cover (for the debug build's bounds checks)
    const int64_t q_rows_all = (int64_t)p.n_ranks * p.q_row_step;
    const int64_t kv_rows_all = p.kv_row_step ? (int64_t)p.n_ranks * p.kv_row_step : p.kv_len;
    (void)q_rows_all;
    (void)kv_rows_all;
    const Range kr = (p.use_layout && !p.kv_explicit) ? layout_range(p.layout, p.n_ranks, p.seq_len, j) : p.kv_range;

    if (tid == 0) {
        mbar_init(bar(C::B_KV), 1);
        for (int s = 0; s < NS; ++s) { mbar_init(bar(C::B_QF + s), 1); mbar_init(bar(C::B_QE + s), 1); }
        for (int b2 = 0; b2 < 2; ++b2) mbar_init(bar(C::B_SF + b2), 1);
        mbar_init(bar(C::B_DPF), 1);
        for (int b2 = 0; b2 < 2; ++b2) {
            mbar_init(bar(C::B_PR + b2), 8);
            mbar_init(bar(C::B_DSR + b2), 8);
            mbar_init(bar(C::B_DSE + b2), 1);
        }
        mbar_init(bar(C::B_DQF), 1);
        mbar_init(bar(C::B_DQE), 4);
        mbar_init(bar(C::B_DONE), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    QSeq seq;
    seq.init(p, j, kt, kr, hk * p.group);

    if (warp == WARP_LOAD) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_do);
            WaitCtx w{abort_flag, p.status, 41};
            int kv_row = (int)(j * p.kv_row_step) + k_lo;
            if (p.kv_map_h > 0) kv_row = zigzag_row<int>(kv_row, p.kv_map_h, p.n_ranks);
            mbar_expect_tx(bar(C::B_KV), 2 * C::KV_TILE);
            const bool kv_ok = bounds_ok(kv_row >= 0 && kv_row < kv_rows_all && hk < p.hkv && bb < p.b, p.status, 201);
            for (int kb = 0; kb < 2 && kv_ok; ++kb) {
                tma_load_4d(s_base + C::OFF_K + kb * C::KV_SUB, &tm_k, bar(C::B_KV), kb * 64, hk, kv_row, bb);
                tma_load_4d(s_base + C::OFF_V + kb * C::KV_SUB, &tm_v, bar(C::B_KV), kb * 64, hk, kv_row, bb);
            }
            int n = 0;
            while (seq.next()) {
                const int s = n % NS;
                if (!mbar_wait(bar(C::B_QE + s), ((n / NS) & 1) ^ 1, w)) break;
                mbar_expect_tx(bar(C::B_QF + s), C::STAGE + BQ * 8);
                const int q_row = seq.q_row();
                const uint32_t st = s_base + C::OFF_Q + s * C::STAGE;
                const bool q_ok = bounds_ok(q_row >= 0 && q_row < q_rows_all && seq.h < p.hq && bb < p.b, p.status, 202);
                for (int kb = 0; kb < 2 && q_ok; ++kb) {
                    tma_load_4d(st + kb * C::Q_SUB, &tm_q, bar(C::B_QF + s), kb * 64, seq.h, q_row, bb);
                    tma_load_4d(st + C::Q_TILE + kb * C::Q_SUB, &tm_do, bar(C::B_QF + s), kb * 64, seq.h, q_row, bb);
                }
                const float2 *src =
                    p.stats + (((int64_t)bb * p.hq + seq.h) * p.n_ranks + seq.i) * p.lpad + (int64_t)seq.qt * BQ;
                if (bounds_ok(seq.i < p.n_ranks && (int64_t)seq.qt * BQ + BQ <= p.lpad, p.status, 203))
                    bulk_g2s(s_base + C::OFF_ST + s * BQ * 8, src, BQ * 8, bar(C::B_QF + s));
                ++n;
            }
            if (*abort_flag) {
                // let the copies already issued land before the CTA leaves
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar(C::B_KV), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
                for (int i = (n > NS ? n - NS : 0); i < n; ++i) {
                    const uint64_t t1 = global_timer_ns();
                    while (!mbar_try_wait(bar(C::B_QF + i % NS), (i / NS) & 1) && global_timer_ns() - t1 < kWaitLimitNs) {}
                }
            }
        }
    } else if (warp == WARP_MMA) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            WaitCtx w{abort_flag, p.status, 43};
            const uint32_t ka = s_base + C::OFF_K, va = s_base + C::OFF_V;
            // S^T(n) = K Q(n)^T into S buffer n & 1
            auto issue_s = [&](int n) {
                const uint32_t qa = s_base + C::OFF_Q + (n % NS) * C::STAGE;
                const uint32_t d_t = tbase + C::T_S + (uint32_t)((n & 1) * BQ);
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_ss(d_t, smem_desc_sw128(ka + (k >> 2) * C::KV_SUB + (k & 3) * 32, 16, 1024),
                           smem_desc_sw128(qa + (k >> 2) * C::Q_SUB + (k & 3) * 32, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
                tc_commit(bar(C::B_SF + (n & 1)));
            };
            // dP^T(n) = V dO(n)^T
            auto issue_dp = [&](int n) {
                const uint32_t da = s_base + C::OFF_Q + (n % NS) * C::STAGE + C::Q_TILE;
#pragma unroll
                for (int k = 0; k < HD / 16; ++k)
                    mma_ss(tbase + C::T_DP, smem_desc_sw128(va + (k >> 2) * C::KV_SUB + (k & 3) * 32, 16, 1024),
                           smem_desc_sw128(da + (k >> 2) * C::Q_SUB + (k & 3) * 32, 16, 1024), IDESC_S, k > 0 ? 1u : 0u);
                tc_commit(bar(C::B_DPF));
            };
            bool have = seq.next();
            bool ok = mbar_wait(bar(C::B_KV), 0, w);
            if (have && ok) {
                ok = mbar_wait(bar(C::B_QF + 0), 0, w);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                    issue_dp(0);
                }
            }
            int n = 0;
            while (have && ok) {
                const int s = n % NS;
                const bool have_next = seq.next();
                if (have_next) {
                    const int m = n + 1;
                    // S buffer m & 1 last held S^T / P^T of tile m - 2, whose dV MMA was
                    // issued earlier by this thread (MMAs run in issue order)
                    if (!mbar_wait(bar(C::B_QF + m % NS), (m / NS) & 1, w)) break;
                    tc_fence_after();
                    issue_s(m);
                }
                const uint32_t qa = s_base + C::OFF_Q + s * C::STAGE;
                const int pb = n & 1;  // P^T / dS^T buffer of this tile
                const uint32_t dsa = s_base + C::OFF_DS + pb * C::PBUF;
                // dV += P^T dO, P^T (bf16) from TMEM: queries [0, 32) in columns [0, 16) of
                // S buffer pb, queries [32, 64) in columns [32, 48)
                if (!mbar_wait(bar(C::B_PR + pb), (n >> 1) & 1, w)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < BQ / 16; ++k)
                    mma_ts(tbase + C::T_DV, tbase + C::T_S + (uint32_t)(pb * BQ + (k >> 1) * 32 + (k & 1) * 8),
                           smem_desc_sw128(qa + C::Q_TILE + k * 2048, C::Q_SUB, 1024), IDESC_KV,
                           (n > 0 || k > 0) ? 1u : 0u);
                // dS^T ready: next dP first (the softmax waits on it), then dK and dQ^T
                if (!mbar_wait(bar(C::B_DSR + pb), (n >> 1) & 1, w)) break;
                tc_fence_after();
                if (have_next) issue_dp(n + 1);
#pragma unroll
                for (int k = 0; k < BQ / 16; ++k)
                    mma_ss(tbase + C::T_DK, smem_desc_sw128(dsa + k * 32, 16, 1024),
                           smem_desc_sw128(qa + k * 2048, C::Q_SUB, 1024), IDESC_KV, (n > 0 || k > 0) ? 1u : 0u);
                tc_commit(bar(C::B_QE + s));  // the last reader of this Q / dO stage
                if (n > 0 && !mbar_wait(bar(C::B_DQE), (n - 1) & 1, w)) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_ss(tbase + C::T_DQ, smem_desc_sw128(ka + k * 2048, C::KV_SUB, 1024),
                           smem_desc_sw128(dsa + k * 2048, C::KV_SUB, 1024), IDESC_DQ, k > 0 ? 1u : 0u);
                tc_commit(bar(C::B_DQF));
                tc_commit(bar(C::B_DSE + pb));
                ++n;
                have = have_next;
            }
            // drain: every MMA issued above has finished before the epilogue and teardown
            tc_commit(bar(C::B_DONE));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
    } else if (warp >= WARP_DQ0) {
        // ================================================================ dQ warps 8-11
        const int wq = warp - WARP_DQ0;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const bool leader = (wq == 0 && lane == 0);
        WaitCtx w{abort_flag, p.status, 45};
        float *stg = reinterpret_cast<float *>(smem + C::OFF_DQ);
        const int dcol = wq * 32 + lane;
        const float scale = p.scale;
        int n = 0;
        while (seq.next()) {
            const bool okw = mbar_wait(bar(C::B_DQF), n & 1, w);
            if (leader) bulk_wait_read_all();  // the staging buffer is free again
            if (bar_any(2, 128, !okw)) break;
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(tbase + lane_off + C::T_DQ, r0);
            tmem_ld32(tbase + lane_off + C::T_DQ + 32, r1);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DQE));
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                stg[c * HD + dcol] = __uint_as_float(r0[c]) * scale;
                stg[(32 + c) * HD + dcol] = __uint_as_float(r1[c]) * scale;
            }
            fence_async_smem();
            asm volatile("barrier.sync 2, 128;" ::: "memory");
            if (leader) {
                if (bounds_ok(seq.q_row() >= 0 && seq.q_row() < q_rows_all && seq.h < p.hq, p.status, 204))
                    tma_reduce_add_4d(&tm_dq, s_base + C::OFF_DQ, 0, seq.h, seq.q_row(), bb);
                bulk_commit();
            }
            ++n;
        }
        if (leader) bulk_wait_all();
    } else {
        // ================================================================ P / dS warps 0-7
        const int half = warp >> 2;
        const int wl = warp & 3;
        const int krow = wl * 32 + lane;  // key row of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        WaitCtx w{abort_flag, p.status, 47 + half};
        const int key = k_lo + krow;
        const bool key_ok = key < p.kv_len;
        const int64_t pk = range_pos(kr, (int64_t)(key_ok ? key : (p.kv_len > 0 ? p.kv_len - 1 : 0)));
        const int64_t de_key = p.n_docs > 0 ? doc_end_of(p, pk) : (int64_t)INT32_MAX;
        const float sl2 = p.scale_log2;
        bool aborted = false;
        int n = 0;
        while (seq.next()) {
            const int s = n % NS;
            // columns [0, c_first) of this row are masked (keys past the block end,
            // or queries that precede the key)
            int c_first = 0, c_last = BQ;
            if (seq.partial()) {
                if (!key_ok) {
                    c_first = BQ;
                } else if (p.causal) {
                    // rows past the block end are clamped to its last row: a range
                    // gives positions only for its own rows, and the search needs
                    // them non-decreasing (those rows carry no probability anyway)
                    int lo = 0, hi = BQ;
                    const int64_t row0 = (int64_t)seq.qt * BQ, last = p.q_len - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi) >> 1;
                        const int64_t row = row0 + mid < last ? row0 + mid : last;
                        if (range_pos(seq.qr, (int)row) < pk) lo = mid + 1; else hi = mid;
                    }
                    c_first = lo;
                }
                if (key_ok && p.n_docs > 0 && de_key < (int64_t)INT32_MAX) {
                    // queries at or past the end of the key's document do not see it
                    int lo = 0, hi = BQ;
                    const int64_t row0 = (int64_t)seq.qt * BQ, last = p.q_len - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi) >> 1;
                        const int64_t row = row0 + mid < last ? row0 + mid : last;
                        if (range_pos(seq.qr, (int)row) < de_key) lo = mid + 1; else hi = mid;
                    }
                    c_last = lo;
                }
            }
            c_first -= half * 32;
            c_last -= half * 32;
            {
                const bool okw = mbar_wait(bar(C::B_SF + (n & 1)), (n >> 1) & 1, w) &&
                                 mbar_wait(bar(C::B_QF + s), (n / NS) & 1, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; break; }
            }
            tc_fence_after();
            uint32_t sv[32];
            const uint32_t s_cols = tbase + lane_off + C::T_S + (uint32_t)((n & 1) * BQ + half * 32);
            tmem_ld32(s_cols, sv);
            // (lse log2 e, D) of two query columns per 16-byte load
            const float4 *stat = reinterpret_cast<const float4 *>(smem + C::OFF_ST + s * BQ * 8) + half * 16;
            float pv[32];
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            if (seq.partial()) {  // warp-uniform: the element mask only where a tile needs it
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 st = stat[c];
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), sl2x2,
                                     f2_pack(-st.x, -st.z)),
                              x0, x1);
                    pv[2 * c] = (2 * c < c_first || 2 * c >= c_last) ? 0.f : ex2_approx(x0);
                    pv[2 * c + 1] = (2 * c + 1 < c_first || 2 * c + 1 >= c_last) ? 0.f : ex2_approx(x1);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float4 st = stat[c];
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), sl2x2,
                                     f2_pack(-st.x, -st.z)),
                              x0, x1);
                    pv[2 * c] = ex2_approx(x0);
                    pv[2 * c + 1] = ex2_approx(x1);
                }
            }
            uint32_t pk16[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) pk16[c] = pack_bf16x2(pv[2 * c], pv[2 * c + 1]);
            // bf16 P^T over the first 16 of this warp's own 32 score columns (no other
            // warp reads them), the A operand of the dV MMA
            const int pb = n & 1;
            tmem_st16(s_cols, pk16);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_PR + pb));
            {
                const bool okw = mbar_wait(bar(C::B_DPF), n & 1, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; break; }
            }
            tc_fence_after();
            uint32_t dv[32];
            tmem_ld32(tbase + lane_off + C::T_DP + (uint32_t)(half * 32), dv);
            tc_fence_before();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 st = stat[c];
                const uint64_t t = f2_add(f2_pack(__uint_as_float(dv[2 * c]), __uint_as_float(dv[2 * c + 1])),
                                          f2_pack(-st.y, -st.w));
                float d0, d1;
                f2_unpack(f2_fma(f2_pack(pv[2 * c], pv[2 * c + 1]), t, f2_pack(0.f, 0.f)), d0, d1);
                pk16[c] = pack_bf16x2(d0, d1);
            }
            if (n >= 2) {
                const bool okw = mbar_wait(bar(C::B_DSE + pb), ((n >> 1) - 1) & 1, w);
                if (__any_sync(0xffffffffu, !okw)) { aborted = true; break; }
            }
            st_sw128_half(smem + C::OFF_DS + pb * C::PBUF, krow, half, pk16);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_DSR + pb));
            ++n;
        }
        aborted = __any_sync(0xffffffffu, aborted || (*abort_flag != 0));

        // ================================================================ dK / dV epilogue
        if (!aborted) {
            const bool okw = mbar_wait(bar(C::B_DONE), 0, w);
            aborted = __any_sync(0xffffffffu, !okw);
            if (!aborted) tc_fence_after();
        }
        if (!aborted) {
            const uint32_t t_acc = half == 0 ? C::T_DK : C::T_DV;
            const float f = half == 0 ? p.scale : 1.f;
            void *out = half == 0 ? p.dk : p.dv;
            const int64_t sb = half == 0 ? p.dk_sb : p.dv_sb, ss = half == 0 ? p.dk_ss : p.dv_ss,
                          sh = half == 0 ? p.dk_sh : p.dv_sh;
            // the tile's keys are consecutive rows of the key tensor (also in place)
            int64_t orow = (int64_t)j * p.kv_row_step + k_lo;
            if (p.kv_map_h > 0) orow = zigzag_row<int64_t>(orow, p.kv_map_h, p.n_ranks);
            orow += krow;
            const bool key_in = key_ok && bounds_ok(orow >= 0 && orow < kv_rows_all, p.status, 205);
            if (p.accumulate) {
                // block form: add this call's share into the caller's fp32 accumulator
                // (each key row belongs to this CTA alone)
                float *dst = reinterpret_cast<float *>(out) + (int64_t)bb * sb + orow * ss + (int64_t)hk * sh;
#pragma unroll
                for (int c0 = 0; c0 < HD; c0 += 32) {
                    uint32_t r[32];
                    if (n > 0) tmem_ld32(tbase + lane_off + t_acc + (uint32_t)c0, r);
                    if (key_in && n > 0) {
                        float4 *d4 = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float4 a = d4[i];
                            a.x = fmaf(__uint_as_float(r[4 * i + 0]), f, a.x);
                            a.y = fmaf(__uint_as_float(r[4 * i + 1]), f, a.y);
                            a.z = fmaf(__uint_as_float(r[4 * i + 2]), f, a.z);
                            a.w = fmaf(__uint_as_float(r[4 * i + 3]), f, a.w);
                            d4[i] = a;
                        }
                    }
                }
            } else {
                uint16_t *dst = reinterpret_cast<uint16_t *>(out) + (int64_t)bb * sb + orow * ss + (int64_t)hk * sh;
#pragma unroll
                for (int c0 = 0; c0 < HD; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + lane_off + t_acc + (uint32_t)c0, r);
                    float v[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) v[c] = n > 0 ? __uint_as_float(r[c]) * f : 0.f;
                    if (key_in) store_bf16x32(dst + c0, v);
                }
            }
        }
    }

    // ---- teardown: all TMEM traffic done, CTA-wide barrier, owner frees TMEM
    __syncwarp();
    tc_fence_before();
    asm volatile("barrier.sync 1, %0;" ::"n"(NTHREADS) : "memory");
    if (warp == WARP_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, C::TMEM_COLS);
    }
}

// Per query row: (lse log2 e, D = do . o) into the statistics table (padding rows
// get (+inf, 0), which makes their probabilities 0), and a zeroed dQ accumulator row.
// Sixteen threads per (batch, head, rank, padded row), each with 16-byte slices of
// o and dout (8 bf16) and 32 bytes of the accumulator, two rows in flight per thread.
constexpr int kPreRowsPerThread = 2;
__global__ void __launch_bounds__(256) attn_bwd_pre_kernel(const __grid_constant__ BwdParams p, int64_t acc_rows)
{
    constexpr int TPR = HD / 8;  // threads per row
    const int part = threadIdx.x % TPR;
    const int64_t total = (int64_t)p.b * p.hq * p.n_ranks * p.lpad;
    const int64_t row_slot = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / TPR;  // first row of this thread
    const int64_t stride = (int64_t)gridDim.x * blockDim.x / TPR;
    auto lo = [](uint32_t x) { return __uint_as_float(x << 16); };
    auto hi = [](uint32_t x) { return __uint_as_float(x & 0xffff0000u); };
    for (int64_t g0 = row_slot; g0 < total; g0 += stride * kPreRowsPerThread) {
        uint4 ov[kPreRowsPerThread], gv[kPreRowsPerThread];
        int64_t gw[kPreRowsPerThread], qrow[kPreRowsPerThread];
        int hh[kPreRowsPerThread], bq[kPreRowsPerThread];
        bool live[kPreRowsPerThread];
#pragma unroll
        for (int u = 0; u < kPreRowsPerThread; ++u) {
            gw[u] = g0 + u * stride;
            const int64_t g = gw[u] < total ? gw[u] : total - 1;
            const int t = (int)(g % p.lpad);
            int64_t rest = g / p.lpad;
            const int i = (int)(rest % p.n_ranks);
            rest /= p.n_ranks;
            hh[u] = (int)(rest % p.hq);
            bq[u] = (int)(rest / p.hq);
            live[u] = gw[u] < total && t < p.q_len;
            qrow[u] = (int64_t)i * p.q_row_step + t;
            if (live[u]) {
                ov[u] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(p.o) + bq[u] * p.o_sb +
                                                         qrow[u] * p.o_ss + hh[u] * p.o_sh + part * 8);
                gv[u] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(p.dout) + bq[u] * p.do_sb +
                                                         qrow[u] * p.do_ss + hh[u] * p.do_sh + part * 8);
            }
        }
#pragma unroll
        for (int u = 0; u < kPreRowsPerThread; ++u) {
            float acc = 0.f;
            if (live[u]) {
                acc = lo(ov[u].x) * lo(gv[u].x);
                acc = fmaf(hi(ov[u].x), hi(gv[u].x), acc);
                acc = fmaf(lo(ov[u].y), lo(gv[u].y), acc);
                acc = fmaf(hi(ov[u].y), hi(gv[u].y), acc);
                acc = fmaf(lo(ov[u].z), lo(gv[u].z), acc);
                acc = fmaf(hi(ov[u].z), hi(gv[u].z), acc);
                acc = fmaf(lo(ov[u].w), lo(gv[u].w), acc);
                acc = fmaf(hi(ov[u].w), hi(gv[u].w), acc);
            }
            // the TPR threads of a row are consecutive lanes of one warp
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off, TPR);
            if (gw[u] >= total) continue;
            float2 st = make_float2(INFINITY, 0.f);
            if (live[u]) {
                const float lse = p.lse[bq[u] * p.lse_sb + hh[u] * p.lse_sh + qrow[u] * p.lse_ss];
                st.x = (lse == -INFINITY) ? INFINITY : lse * kLog2eB;
                st.y = acc;
                if (!p.accumulate) {  // the block form adds into the caller's accumulator instead
                    float4 *dq = reinterpret_cast<float4 *>(p.dq_acc + (((int64_t)bq[u] * acc_rows + qrow[u]) * p.hq + hh[u]) * HD) +
                                 part * 2;
                    dq[0] = make_float4(0.f, 0.f, 0.f, 0.f);
                    dq[1] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (part == 0) p.stats[gw[u]] = st;
        }
    }
}

// dq = dq_acc (already scaled) in bf16; 8 values per thread.
__global__ void __launch_bounds__(256) attn_bwd_post_kernel(const __grid_constant__ BwdParams p, int64_t acc_rows)
{
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t per_row = HD / 8;
    const int64_t total = (int64_t)p.b * p.n_ranks * p.q_len * p.hq * per_row;
    if (idx >= total) return;
    const int c8 = (int)(idx % per_row);
    int64_t rest = idx / per_row;
    const int h = (int)(rest % p.hq);
    rest /= p.hq;
    const int64_t t = rest % ((int64_t)p.n_ranks * p.q_len);
    const int bb = (int)(rest / ((int64_t)p.n_ranks * p.q_len));
    const int64_t row = (t / p.q_len) * p.q_row_step + t % p.q_len;
    const float4 *src = reinterpret_cast<const float4 *>(p.dq_acc + (((int64_t)bb * acc_rows + row) * p.hq + h) * HD) +
                        c8 * 2;
    const float4 a = src[0], b = src[1];
    uint4 w;
    w.x = pack_bf16x2(a.x, a.y);
    w.y = pack_bf16x2(a.z, a.w);
    w.z = pack_bf16x2(b.x, b.y);
    w.w = pack_bf16x2(b.z, b.w);
    *reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.dq) + bb * p.dq_sb + row * p.dq_ss + h * p.dq_sh +
                               c8 * 8) = w;
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFnB)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnB encode_fn_b()
{
    static EncodeTiledFnB fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFnB>(ptr);
    }
    return fn;
}

// [b, s, H, d] tensor with element strides (sb, ss, sh, 1) -> 4-D map {d, H, s, b}.
bool make_map_b(CUtensorMap *m, CUtensorMapDataType dt, int es, const void *base, int64_t b, int64_t s, int64_t H,
                int64_t d, int64_t sb, int64_t ss, int64_t sh, uint32_t box_d, uint32_t box_s, CUtensorMapSwizzle sw)
{
    EncodeTiledFnB fn = encode_fn_b();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)s, (cuuint64_t)b};
    cuuint64_t strides[3] = {(cuuint64_t)(sh * es), (cuuint64_t)(ss * es), (cuuint64_t)(sb * es)};
    cuuint32_t box[4] = {box_d, 1, box_s, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdParams &p, cudaStream_t stream)
{
    if (p.d != HD) return cudaErrorInvalidValue;
    const int64_t q_rows = (int64_t)p.n_ranks * p.q_row_step;
    const int64_t kv_rows = p.kv_row_step ? (int64_t)p.n_ranks * p.kv_row_step : p.kv_len;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const auto SW = CU_TENSOR_MAP_SWIZZLE_128B;
    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!make_map_b(&tq, BF, 2, p.q, p.b, q_rows, p.hq, HD, p.q_sb, p.q_ss, p.q_sh, 64, BQ, SW) ||
        !make_map_b(&tdo, BF, 2, p.dout, p.b, q_rows, p.hq, HD, p.do_sb, p.do_ss, p.do_sh, 64, BQ, SW) ||
        !make_map_b(&tk, BF, 2, p.k, p.b, kv_rows, p.hkv, HD, p.k_sb, p.k_ss, p.k_sh, 64, BK, SW) ||
        !make_map_b(&tv, BF, 2, p.v, p.b, kv_rows, p.hkv, HD, p.v_sb, p.v_ss, p.v_sh, 64, BK, SW) ||
        !(p.accumulate ? make_map_b(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.dq_acc, p.b, q_rows, p.hq, HD, p.dq_sb,
                                    p.dq_ss, p.dq_sh, HD, BQ, CU_TENSOR_MAP_SWIZZLE_NONE)
                       : make_map_b(&tdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.dq_acc, p.b, q_rows, p.hq, HD,
                                    q_rows * p.hq * HD, (int64_t)p.hq * HD, HD, HD, BQ, CU_TENSOR_MAP_SWIZZLE_NONE)))
        return cudaErrorInvalidValue;
    static unsigned long long attr_done = 0;
    {
        cudaError_t e = set_smem_per_device((const void *)attn_bwd_kernel, BCfg::SMEM, &attr_done);
        if (e != cudaSuccess) return e;
    }
    const int64_t rows = (int64_t)p.b * p.hq * p.n_ranks * p.lpad;
    if (rows == 0) return cudaSuccess;
    {
        // 16 threads per row, two rows each; at most 8 resident CTAs of 256 threads per SM
        const int64_t want = (rows * (HD / 8) / kPreRowsPerThread + 255) / 256;
        const int64_t cap = (int64_t)sm_count() * 8;
        attn_bwd_pre_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, stream>>>(p, q_rows);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t items = (int64_t)(p.order_len ? p.order_len : p.n_kv_blocks * p.n_kt) * p.b * p.hkv;
    if (items > 0) {
        attn_bwd_kernel<<<(unsigned)items, NTHREADS, BCfg::SMEM, stream>>>(p, tq, tk, tv, tdo, tdq);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.accumulate) return cudaSuccess;  // dq_acc is the caller's output
    const int64_t threads = (int64_t)p.b * p.n_ranks * p.q_len * p.hq * (HD / 8);
    attn_bwd_post_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p, q_rows);
    return cudaGetLastError();
}

}  // namespace cpattn
