// attn_tc.cu -- bf16 block attention on sm_100a tensor cores (tcgen05 + TMEM + TMA),
// run either as one block (cp_block_attn_fwd) or as the whole ring schedule.
//
// What one CTA computes ("上下文并行与 Ring Attention", hs-black.github.io):
//   a 128-row query tile of one rank, one query head.  For each ring step r it
//   takes the K/V block of rank (i - r) mod N (section Ring Attention), builds the
//   block partial with the online-softmax recurrence that FlashAttention uses
//   (section 分块注意力: running max m, sum l = sum e^{x - m}, unnormalised O,
//   then o_b = O / l and lse_b = m + log l), and folds the partial into the running
//   result with the LSE merge of the same section.  Key tiles that the causal mask
//   hides completely are skipped whole (figure caption of section Ring Attention).
//
// Roles (192 threads):
//   warps 0-3  softmax / merge / epilogue; thread t owns query row t = TMEM lane t.
//   warp 4     TMA producer: Q once, then K and V tiles (2 stages each).
//   warp 5     TMEM owner (512 columns) and single-thread MMA issuer.
// TMEM columns: S0 [0,128), S1 [128,256) hold the fp32 scores of two key tiles in
// flight; the softmax overwrites columns [0,64) of a score buffer with its bf16
// probabilities P, which the PV MMA reads as its A operand.  O_b [256, 256+d)
// accumulates the current step's P V; O_acc [256+d, 256+2d) holds the merged
// result when a launch spans several ring steps.
//
// Softmax details: scores are handled in the log2 domain (scale * log2 e folded
// into one FMA), and the running max used for the exponent is only raised when a
// row's max grows by more than 8 (log2 units); O and l stay consistent with the
// max actually used, so the result is exact up to rounding while most tiles skip
// the O rescale.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace cpattn {
namespace {

constexpr int BM = 128;  // query rows per tile (TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr int NSK = 2;   // K stages
constexpr int NSV = 2;   // V stages
constexpr int NTHREADS = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

template <int D>
struct Cfg {
    static constexpr int SUB = BM * 128;          // one 64-column swizzle block (16 KB)
    static constexpr int TILE = BM * D * 2;       // a 128 x D bf16 tile
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE;
    static constexpr int OFF_V = OFF_K + NSK * TILE;
    static constexpr int OFF_BAR = OFF_V + NSV * TILE;
    enum {
        B_Q = 0,
        B_KF = 1,
        B_KE = B_KF + NSK,
        B_VF = B_KE + NSK,
        B_VE = B_VF + NSV,
        B_SF = B_VE + NSV,
        B_PF = B_SF + 2,
        B_PV = B_PF + 2,
        B_DONE = B_PV + 2,
        NBAR = B_DONE + 1
    };
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 64 + 1024;  // + alignment slack
    static constexpr int T_OB = 256;
    static constexpr int T_OACC = 256 + D;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, true);
};

// Ring-step iterator shared by the three roles so that they agree on the exact
// sequence of non-skipped key tiles.
struct TileSeq {
    const AttnParams *p;
    Range qr;
    int rank, q_lo;
    int step, kt, kt_full, kt_end;
    int src;
    Range kr;

    __device__ void init(const AttnParams &pp, const Range &q, int rk, int qlo)
    {
        p = &pp;
        qr = q;
        rank = rk;
        q_lo = qlo;
        step = pp.step_begin - 1;
        kt = 0;
        kt_end = 0;
        kt_full = 0;
    }
    // Advance to the next non-skipped tile; false at the end.
    __device__ bool next()
    {
        ++kt;
        while (kt >= kt_end) {
            ++step;
            if (step >= p->step_end) return false;
            int N = p->n_ranks;
            src = ((rank - step) % N + N) % N;
            kr = p->use_layout ? layout_range(p->layout, N, p->seq_len, src) : p->kv_range;
            kv_tile_bounds(qr, p->q_len, q_lo, BM, kr, p->kv_len, BN, p->causal != 0, &kt_full,
                           &kt_end);
            kt = 0;
        }
        return true;
    }
    __device__ bool first_in_step() const { return kt == 0; }
    __device__ bool last_in_step() const { return kt == kt_end - 1; }
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
        for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(v[4 * i + 0], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v)
{
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar0 = s_base + C::OFF_BAR;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // ---- work item
    const int bh_count = p.b * p.hq;
    const int bh = blockIdx.x % bh_count;
    const int e = blockIdx.x / bh_count;
    int rank, qt;
    if (p.order_len) {
        rank = (int)(p.order[e] >> 16);
        qt = (int)(p.order[e] & 0xffffu);
    } else {
        rank = e / p.n_qt;
        qt = e % p.n_qt;
    }
    const int h = bh % p.hq;
    const int bb = bh / p.hq;
    const int hk = h / p.group;
    const int q_lo = qt * BM;
    const Range qr = p.use_layout ? layout_range(p.layout, p.n_ranks, p.seq_len, rank) : p.q_range;

    // ---- setup: barriers, TMEM
    if (tid == 0) {
        mbar_init(bar(C::B_Q), 1);
        for (int i = 0; i < NSK; ++i) { mbar_init(bar(C::B_KF + i), 1); mbar_init(bar(C::B_KE + i), 1); }
        for (int i = 0; i < NSV; ++i) { mbar_init(bar(C::B_VF + i), 1); mbar_init(bar(C::B_VE + i), 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar(C::B_SF + i), 1);
            mbar_init(bar(C::B_PF + i), BM);
            mbar_init(bar(C::B_PV + i), 1);
        }
        mbar_init(bar(C::B_DONE), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 5) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 4) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            WaitCtx w{abort_flag, p.status, 1};
            TileSeq seq;
            seq.init(p, qr, rank, q_lo);
            int n = 0;
            const int q_row = (int)(rank * p.q_row_step) + q_lo;
            while (seq.next()) {
                if (n == 0) {
                    mbar_expect_tx(bar(C::B_Q), C::TILE);
                    for (int kb = 0; kb < D / 64; ++kb)
                        tma_load_4d(s_base + C::OFF_Q + kb * C::SUB, &tm_q, bar(C::B_Q), kb * 64, h,
                                    q_row, bb);
                }
                const int kv_row = (int)(seq.src * p.kv_row_step) + seq.kt * BN;
                const int sk = n % NSK, sv = n % NSV;
                if (!mbar_wait(bar(C::B_KE + sk), ((n / NSK) & 1) ^ 1, w)) break;
                mbar_expect_tx(bar(C::B_KF + sk), C::TILE);
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_4d(s_base + C::OFF_K + sk * C::TILE + kb * C::SUB, &tm_k, bar(C::B_KF + sk),
                                kb * 64, hk, kv_row, bb);
                if (!mbar_wait(bar(C::B_VE + sv), ((n / NSV) & 1) ^ 1, w)) break;
                mbar_expect_tx(bar(C::B_VF + sv), C::TILE);
                for (int kb = 0; kb < D / 64; ++kb)
                    tma_load_4d(s_base + C::OFF_V + sv * C::TILE + kb * C::SUB, &tm_v, bar(C::B_VF + sv),
                                kb * 64, hk, kv_row, bb);
                ++n;
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
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(bar(C::B_Q), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
            }
        }
    } else if (warp == 5) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            WaitCtx w{abort_flag, p.status, 3};
            TileSeq seq;
            seq.init(p, qr, rank, q_lo);
            bool have = seq.next();
            bool ok = true;
            auto issue_s = [&](int m) -> bool {
                const int sk = m % NSK;
                if (!mbar_wait(bar(C::B_KF + sk), (m / NSK) & 1, w)) return false;
                tc_fence_after();
                const uint32_t d_tmem = tbase + (uint32_t)((m & 1) * 128);
                const uint32_t qa = s_base + C::OFF_Q;
                const uint32_t kb_ = s_base + C::OFF_K + sk * C::TILE;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t off = (k >> 2) * C::SUB + (k & 3) * 32;
                    mma_ss(d_tmem, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(kb_ + off, 16, 1024),
                           C::IDESC_QK, k > 0 ? 1u : 0u);
                }
                tc_commit(bar(C::B_KE + sk));
                tc_commit(bar(C::B_SF + (m & 1)));
                return true;
            };
            if (have) {
                ok = mbar_wait(bar(C::B_Q), 0, w);
                if (ok) { tc_fence_after(); ok = issue_s(0); }
            }
            int n = 0;
            while (have && ok) {
                const bool first_n = seq.first_in_step();
                const bool have_next = seq.next();
                if (have_next && !issue_s(n + 1)) break;
                const int sv = n % NSV;
                if (!mbar_wait(bar(C::B_PF + (n & 1)), (n >> 1) & 1, w)) break;
                if (!mbar_wait(bar(C::B_VF + sv), (n / NSV) & 1, w)) break;
                tc_fence_after();
                const uint32_t p_tmem = tbase + (uint32_t)((n & 1) * 128);
                const uint32_t vb = s_base + C::OFF_V + sv * C::TILE;
#pragma unroll
                for (int k = 0; k < BN / 16; ++k) {
                    mma_ts(tbase + C::T_OB, p_tmem + k * 8, smem_desc_sw128(vb + k * 2048, C::SUB, 1024),
                           C::IDESC_PV, (k > 0 || !first_n) ? 1u : 0u);
                }
                tc_commit(bar(C::B_VE + sv));
                tc_commit(bar(C::B_PV + (n & 1)));
                ++n;
                have = have_next;
            }
            // drain: every MMA issued above has finished before TMEM is released
            tc_commit(bar(C::B_DONE));
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(bar(C::B_DONE), 0) && global_timer_ns() - t0 < kWaitLimitNs) {}
        }
    } else {
        // ================================================================ softmax warps 0-3
        WaitCtx w{abort_flag, p.status, 5};
        const int row = q_lo + tid;  // local query index in the rank's block
        const bool row_ok = row < p.q_len;
        const int64_t pos_q = range_pos(qr, row_ok ? row : (p.q_len > 0 ? p.q_len - 1 : 0));
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        const bool multi = (p.step_end - p.step_begin) > 1;

        float m_b = -INFINITY;   // running max of the current step (log2 units)
        float l_b = 0.f;         // running sum of the current step
        float lse_acc = -INFINITY;  // merged lse so far (log2 units)
        bool have_acc = false;
        bool any_tile = false;
        bool aborted = false;

        TileSeq seq;
        seq.init(p, qr, rank, q_lo);
        int n = 0;
        while (seq.next()) {
            any_tile = true;
            const bool first = seq.first_in_step();
            const bool last = seq.last_in_step();
            const uint32_t s_tmem = tbase + lane_off + (uint32_t)((n & 1) * 128);
            {
                const bool ok = mbar_wait(bar(C::B_SF + (n & 1)), (n >> 1) & 1, w);
                if (__any_sync(0xffffffffu, !ok)) { aborted = true; break; }
            }
            tc_fence_after();
            float s[BN];
            {
                uint32_t r[64];
                tmem_ld64(s_tmem, r);
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(r[c]);
                tmem_ld64(s_tmem + 64, r);
#pragma unroll
                for (int c = 0; c < 64; ++c) s[64 + c] = __uint_as_float(r[c]);
            }
            // ---- mask (partial tiles only).  Positions increase with the local key
            // index, so the keys this row may see form a prefix of the tile.
            if (seq.kt >= seq.kt_full) {
                const int k0 = seq.kt * BN;
                int cnt = p.kv_len - k0;
                if (cnt > BN) cnt = BN;
                if (p.causal) {
                    int lo = 0, hi = cnt;
                    while (lo < hi) {
                        const int mid = (lo + hi) >> 1;
                        if (range_pos(seq.kr, k0 + mid) <= pos_q) lo = mid + 1; else hi = mid;
                    }
                    cnt = lo;
                }
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c >= cnt) s[c] = -INFINITY;
            }
            // ---- row max
            float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
            for (int c = 4; c < BN; c += 4) {
                mx0 = fmaxf(mx0, s[c]);
                mx1 = fmaxf(mx1, s[c + 1]);
                mx2 = fmaxf(mx2, s[c + 2]);
                mx3 = fmaxf(mx3, s[c + 3]);
            }
            const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
            if (first) {
                m_b = mx;
                l_b = 0.f;
            } else {
                const bool need = mx > m_b + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    // O_b must hold every earlier tile's P V before it is rescaled
                    if (!mbar_wait(bar(C::B_PV + ((n - 1) & 1)), ((n - 1) >> 1) & 1, w)) { aborted = true; }
                    aborted = __any_sync(0xffffffffu, aborted);
                    if (aborted) break;
                    tc_fence_after();
                    const float m_new = fmaxf(m_b, mx);
                    const float f = (m_new == m_b) ? 1.f : ex2_approx(m_b - m_new);
                    m_b = m_new;
                    l_b *= f;
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t r[32];
                        tmem_ld32(tbase + lane_off + C::T_OB + c0, r);
#pragma unroll
                        for (int c = 0; c < 32; ++c) r[c] = __float_as_uint(__uint_as_float(r[c]) * f);
                        tmem_st32(tbase + lane_off + C::T_OB + c0, r);
                    }
                    tmem_wait_st();
                }
            }
            const float mu = (m_b == -INFINITY) ? 0.f : m_b;
            // ---- probabilities, row sum, bf16 P into TMEM columns [0, 64)
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                s[c] = ex2_approx(fmaf(s[c], sl2, -mu));
                s[c + 1] = ex2_approx(fmaf(s[c + 1], sl2, -mu));
                sum0 += s[c];
                sum1 += s[c + 1];
            }
            l_b += sum0 + sum1;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s[64 * half + 2 * i], s[64 * half + 2 * i + 1]);
                tmem_st32(s_tmem + 32 * half, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::B_PF + (n & 1)));

            if (last) {
                // ---- this step's partial is complete: fold it into the running result
                if (!mbar_wait(bar(C::B_PV + (n & 1)), (n >> 1) & 1, w)) aborted = true;
                aborted = __any_sync(0xffffffffu, aborted);
                if (aborted) break;
                tc_fence_after();
                const float lse_b = (l_b > 0.f) ? m_b + log2f(l_b) : -INFINITY;
                if (multi) {
                    float wa = 0.f, wb = 0.f, new_lse = lse_acc;
                    const bool take_b = lse_b != -INFINITY;
                    if (take_b) {
                        if (have_acc) {
                            const float M = fmaxf(lse_acc, lse_b);
                            new_lse = M + log2f(ex2_approx(lse_acc - M) + ex2_approx(lse_b - M));
                            wa = ex2_approx(lse_acc - new_lse);
                            wb = ex2_approx(lse_b - new_lse) / l_b;
                        } else {
                            new_lse = lse_b;
                            wb = 1.f / l_b;
                        }
                    }
                    const bool read_acc = __any_sync(0xffffffffu, have_acc);
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t rb[32], ra[32];
                        tmem_ld32(tbase + lane_off + C::T_OB + c0, rb);
                        if (read_acc) tmem_ld32(tbase + lane_off + C::T_OACC + c0, ra);
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            float ob = __uint_as_float(rb[c]);
                            float oa = read_acc ? __uint_as_float(ra[c]) : 0.f;
                            float o = have_acc ? fmaf(wa, oa, wb * ob) : wb * ob;
                            if (!take_b) o = oa;
                            rb[c] = __float_as_uint(o);
                        }
                        tmem_st32(tbase + lane_off + C::T_OACC + c0, rb);
                    }
                    tmem_wait_st();
                    if (take_b) {
                        lse_acc = new_lse;
                        have_acc = true;
                    }
                } else {
                    lse_acc = lse_b;
                    have_acc = lse_b != -INFINITY;
                }
            }
            ++n;
        }
        aborted = __any_sync(0xffffffffu, aborted || (*abort_flag != 0));

        // ================================================================ epilogue
        if (!aborted && (any_tile || p.epi == EPI_STORE)) {
            const int64_t orow = (int64_t)rank * p.q_row_step + row;
            const int64_t obase = (int64_t)bb * p.o_sb + orow * p.o_ss + (int64_t)h * p.o_sh;
            float *lse_ptr = p.lse + (int64_t)bb * p.lse_sb + (int64_t)h * p.lse_sh + orow * p.lse_ss;
            const uint32_t src_col = multi ? C::T_OACC : C::T_OB;
            const float own_scale = multi ? 1.f : (l_b > 0.f ? 1.f / l_b : 0.f);
            const bool empty = !have_acc;
            if (p.epi == EPI_STORE) {
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    if (any_tile) tmem_ld32(tbase + lane_off + src_col + c0, r);
                    float v[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) v[c] = (empty || !any_tile) ? 0.f : __uint_as_float(r[c]) * own_scale;
                    if (row_ok) store_row_chunk(p.o, p.o_dtype, obase + c0, v);
                }
                if (row_ok) *lse_ptr = empty ? -INFINITY : lse_acc * kLn2;
            } else {
                // EPI_MERGE: (o, lse) in memory are fp32 and already hold a partial
                float la = row_ok ? *lse_ptr * kLog2e : -INFINITY;
                float wa = 1.f, wb = 0.f, new_lse = la;
                if (!empty) {
                    const float M = fmaxf(la, lse_acc);
                    if (la == -INFINITY) {
                        wa = 0.f;
                        wb = own_scale;
                        new_lse = lse_acc;
                    } else {
                        new_lse = M + log2f(ex2_approx(la - M) + ex2_approx(lse_acc - M));
                        wa = ex2_approx(la - new_lse);
                        wb = ex2_approx(lse_acc - new_lse) * own_scale;
                    }
                }
                float *orow_ptr = reinterpret_cast<float *>(p.o) + obase;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + lane_off + src_col + c0, r);
                    if (row_ok && !empty) {
                        float v[32];
                        const float4 *src4 = reinterpret_cast<const float4 *>(orow_ptr + c0);
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float4 a = (wa != 0.f) ? src4[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                            v[4 * i + 0] = fmaf(wa, a.x, wb * __uint_as_float(r[4 * i + 0]));
                            v[4 * i + 1] = fmaf(wa, a.y, wb * __uint_as_float(r[4 * i + 1]));
                            v[4 * i + 2] = fmaf(wa, a.z, wb * __uint_as_float(r[4 * i + 2]));
                            v[4 * i + 3] = fmaf(wa, a.w, wb * __uint_as_float(r[4 * i + 3]));
                        }
                        store_row_chunk(p.o, DT_FP32, obase + c0, v);
                    }
                }
                if (row_ok && !empty) *lse_ptr = new_lse * kLn2;
            }
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tbase, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

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
bool make_map(CUtensorMap *m, const void *base, int64_t b, int64_t s, int64_t H, int64_t d, int64_t sb,
              int64_t ss, int64_t sh)
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

template <int D>
cudaError_t launch_d(const AttnParams &p, cudaStream_t stream, int64_t q_rows, int64_t kv_rows)
{
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, p.q, p.b, q_rows, p.hq, D, p.q_sb, p.q_ss, p.q_sh) ||
        !make_map(&tk, p.k, p.b, kv_rows, p.hkv, D, p.k_sb, p.k_ss, p.k_sh) ||
        !make_map(&tv, p.v, p.b, kv_rows, p.hkv, D, p.v_sb, p.v_ss, p.v_sh))
        return cudaErrorInvalidValue;
    static bool attr_set[2] = {false, false};
    const int slot = D == 128 ? 1 : 0;
    if (!attr_set[slot]) {
        cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg<D>::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[slot] = true;
    }
    const int64_t items = (int64_t)p.n_ranks * p.n_qt * p.b * p.hq;
    if (items == 0) return cudaSuccess;
    attn_tc_kernel<D><<<(unsigned)items, NTHREADS, Cfg<D>::SMEM, stream>>>(p, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

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
