// attn_simt_bwd.cu -- the ring backward with plain FFMA arithmetic: fp32 inputs
// (results within fp32 rounding of the definition) and head dims the tensor-core
// backward does not take (d = 64 in bf16).
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力, paragraph
// on the backward pass: with the GLOBAL lse of a query row, p_j = e^{x_j - lse} is
// exact on any key block alone, so every (query rank, key block) pair of the ring
// contributes its own share of
//   dv_j += p_j dout,   dx_j = p_j (dout . v_j - D),   D = dout . o,
//   dq += scale dx_j k_j,   dk_j += scale dx_j q      (x_j = scale q . k_j).
// Section Ring Attention for the schedule: dQ stays with the query's rank, dK and
// dV are summed over every rank that meets their block.
//
// Three launches on one stream:
//   1. per query row (lse, D) into the statistics table [b][hq][N][lpad];
//   2. dQ: CTA = 128 query rows of one rank and one query head, thread = row; for
//      every ring step the K/V block of rank (i - r) mod N streams through shared
//      memory 32 keys at a time (fully masked key tiles skipped, partial ones
//      masked key by key on original positions);
//   3. dV, then dK: CTA = 128 key rows of one rank's block and one KV head, thread =
//      key row; every query head of the group and every query rank's rows that see
//      the tile stream through shared memory 32 rows at a time.  One pass per
//      gradient keeps a single d-vector accumulator in registers.
// The All-Gather form (kv_explicit: one gathered key block in original order, met
// by every query rank) and its document mask (a query sees only keys of its own
// document; section All-Gather 式 CP) are honoured key by key.  The block form
// (use_layout = 0: one explicit query block against one explicit key block, the
// step a rank of a real ring runs) adds its shares into fp32 dq, dk, dv
// (accumulate = 1).
// Nothing waits on another CTA, so there is no bounded wait to report.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "bwd.h"

namespace cpattn {
namespace {

constexpr int SRM = 128;  // rows (query rows or key rows) per CTA
constexpr int SRN = 32;   // streamed rows per shared-memory tile

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float *p, float x) { *p = x; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

template <int D>
struct SbCfg {
    static constexpr int LD = D + 1;                 // padded resident rows (conflict-free per-thread reads)
    static constexpr int OFF_A = 0;                  // [SRM][LD] resident rows: q (dQ) or k (dK/dV)
    static constexpr int OFF_B = OFF_A + SRM * LD;   // [SRM][LD] resident rows: dout (dQ) or v (dK)
    static constexpr int OFF_X = OFF_B + SRM * LD;   // [SRN][D] streamed rows: k (dQ) or q (dK/dV)
    static constexpr int OFF_Y = OFF_X + SRN * D;    // [SRN][D] streamed rows: v (dQ) or dout (dK/dV)
    static constexpr int OFF_ST = OFF_Y + SRN * D;   // [SRN] float2 statistics of the streamed rows
    static constexpr int FLOATS = OFF_ST + 2 * SRN;
    static constexpr int SMEM = FLOATS * 4;
};

// Document of position pos: [start, end) from the sorted starts (end = seq_len for
// the last document).
__device__ __forceinline__ void doc_bounds(const BwdParams &p, int64_t pos, int64_t *start, int64_t *end)
{
    int lo = 0, hi = p.n_docs;  // first start > pos
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)p.doc_starts[mid] <= pos) lo = mid + 1; else hi = mid;
    }
    *start = lo > 0 ? (int64_t)p.doc_starts[lo - 1] : 0;
    *end = lo < p.n_docs ? (int64_t)p.doc_starts[lo] : p.seq_len;
}

__device__ __forceinline__ int64_t stat_index(const BwdParams &p, int bb, int h, int rank, int t)
{
    return ((int64_t)(bb * p.hq + h) * p.n_ranks + rank) * p.lpad + t;
}

template <typename T, int D>
__global__ void simt_bwd_stats_kernel(const __grid_constant__ BwdParams p)
{
    const int64_t rows = (int64_t)p.n_ranks * p.q_len;
    const int64_t total = (int64_t)p.b * p.hq * rows;
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int64_t row = idx % rows;
    const int h = (int)((idx / rows) % p.hq);
    const int bb = (int)(idx / rows / p.hq);
    const int rank = (int)(row / p.q_len), t = (int)(row % p.q_len);
    const int64_t grow = (int64_t)rank * p.q_row_step + t;
    const T *o = static_cast<const T *>(p.o) + bb * p.o_sb + grow * p.o_ss + (int64_t)h * p.o_sh;
    const T *g = static_cast<const T *>(p.dout) + bb * p.do_sb + grow * p.do_ss + (int64_t)h * p.do_sh;
    float dsum = 0.f;
    for (int i = 0; i < D; ++i) dsum = fmaf(ldf(o + i), ldf(g + i), dsum);
    const float lse = p.lse[bb * p.lse_sb + (int64_t)h * p.lse_sh + grow * p.lse_ss];
    p.stats[stat_index(p, bb, h, rank, t)] = make_float2(lse, dsum);
}

template <typename T, int D>
__global__ void __launch_bounds__(SRM) simt_bwd_dq_kernel(const __grid_constant__ BwdParams p)
{
    using C = SbCfg<D>;
    extern __shared__ float sm[];
    float *q_s = sm + C::OFF_A, *g_s = sm + C::OFF_B, *k_s = sm + C::OFF_X, *v_s = sm + C::OFF_Y;

    const int tid = threadIdx.x;
    const int bh_count = p.b * p.hq;
    const int bh = blockIdx.x % bh_count;
    const int e = blockIdx.x / bh_count;
    const int n_qt = (p.q_len + SRM - 1) / SRM;
    const int rank = e / n_qt, qt = e % n_qt;
    const int h = bh % p.hq, bb = bh / p.hq, hk = h / p.group;
    const int q_lo = qt * SRM;
    const int row = q_lo + tid;
    const bool row_ok = row < p.q_len;
    const Range qr = p.use_layout ? layout_range(p.layout, p.n_ranks, p.seq_len, rank) : p.q_range;
    const int64_t pos_q = range_pos(qr, (int64_t)(row_ok ? row : p.q_len - 1));
    const int64_t grow = (int64_t)rank * p.q_row_step + (row_ok ? row : 0);
    int64_t ds_q = 0, de_q = 0;
    if (p.n_docs > 0) doc_bounds(p, pos_q, &ds_q, &de_q);

    {
        const T *qs = static_cast<const T *>(p.q) + bb * p.q_sb + grow * p.q_ss + (int64_t)h * p.q_sh;
        const T *gs = static_cast<const T *>(p.dout) + bb * p.do_sb + grow * p.do_ss + (int64_t)h * p.do_sh;
        for (int i = 0; i < D; ++i) {
            q_s[tid * C::LD + i] = row_ok ? ldf(qs + i) : 0.f;
            g_s[tid * C::LD + i] = row_ok ? ldf(gs + i) : 0.f;
        }
    }
    const float2 st = row_ok ? p.stats[stat_index(p, bb, h, rank, row)] : make_float2(-INFINITY, 0.f);
    const bool live = row_ok && st.x != -INFINITY;  // a row without visible keys has no gradient
    const float scale = p.scale;
    const T *K = static_cast<const T *>(p.k);
    const T *V = static_cast<const T *>(p.v);

    float dq[D];
#pragma unroll
    for (int i = 0; i < D; ++i) dq[i] = 0.f;

    // the ring: every step's block; the All-Gather form: the one gathered block
    const int n_steps = p.kv_explicit ? 1 : p.n_ranks;
    for (int step = 0; step < n_steps; ++step) {
        const int N = p.n_ranks;
        const int src = p.kv_explicit ? 0 : ((rank - step) % N + N) % N;
        const Range kr = p.kv_explicit ? p.kv_range : layout_range(p.layout, N, p.seq_len, src);
        int kt_full, kt_end;
        kv_tile_bounds<int64_t>(qr, p.q_len, q_lo, SRM, kr, p.kv_len, SRN, p.causal != 0, &kt_full, &kt_end);
        for (int kt = 0; kt < kt_end; ++kt) {
            __syncthreads();
            const int k0 = kt * SRN;
            for (int idx = tid; idx < SRN * D; idx += SRM) {
                const int j = idx / D, c = idx % D;
                const int key = k0 + j;
                float kk = 0.f, vv = 0.f;
                if (key < p.kv_len) {
                    const int64_t krow = (int64_t)src * p.kv_row_step + key;
                    kk = ldf(K + bb * p.k_sb + krow * p.k_ss + (int64_t)hk * p.k_sh + c);
                    vv = ldf(V + bb * p.v_sb + krow * p.v_ss + (int64_t)hk * p.v_sh + c);
                }
                k_s[j * D + c] = kk;
                v_s[j * D + c] = vv;
            }
            __syncthreads();
            if (!live) continue;
            for (int j = 0; j < SRN; ++j) {
                const int key = k0 + j;
                if (key >= p.kv_len) break;
                if (p.causal && kt >= kt_full && range_pos(kr, (int64_t)key) > pos_q) continue;
                if (p.n_docs > 0 && range_pos(kr, (int64_t)key) < ds_q) continue;
                float x = 0.f, dp = 0.f;
#pragma unroll 16
                for (int i = 0; i < D; ++i) {
                    x = fmaf(q_s[tid * C::LD + i], k_s[j * D + i], x);
                    dp = fmaf(g_s[tid * C::LD + i], v_s[j * D + i], dp);
                }
                const float pr = expf(x * scale - st.x);
                const float ds = pr * (dp - st.y);
#pragma unroll
                for (int i = 0; i < D; ++i) dq[i] = fmaf(ds, k_s[j * D + i], dq[i]);
            }
        }
    }
    if (!row_ok) return;
    const int64_t off = bb * p.dq_sb + grow * p.dq_ss + (int64_t)h * p.dq_sh;
    if (p.accumulate) {
        float *out = static_cast<float *>(p.dq) + off;  // one thread owns the row: plain add
#pragma unroll
        for (int i = 0; i < D; ++i) out[i] += dq[i] * scale;
    } else {
        T *out = static_cast<T *>(p.dq) + off;
#pragma unroll
        for (int i = 0; i < D; ++i) stf(out + i, dq[i] * scale);
    }
}

template <typename T, int D, bool DK>
__global__ void __launch_bounds__(SRM) simt_bwd_dkv_kernel(const __grid_constant__ BwdParams p)
{
    using C = SbCfg<D>;
    extern __shared__ float sm[];
    float *k_s = sm + C::OFF_A, *v_s = sm + C::OFF_B, *q_s = sm + C::OFF_X, *g_s = sm + C::OFF_Y;
    float2 *st_s = reinterpret_cast<float2 *>(sm + C::OFF_ST);

    const int tid = threadIdx.x;
    const int bh_count = p.b * p.hkv;
    const int bh = blockIdx.x % bh_count;
    const int e = blockIdx.x / bh_count;
    const int n_kt = (p.kv_len + SRM - 1) / SRM;
    const int j = e / n_kt, kt = e % n_kt;   // key block (its rank) and key tile
    const int hk = bh % p.hkv, bb = bh / p.hkv;
    const int k_lo = kt * SRM;
    const int key = k_lo + tid;
    const bool key_ok = key < p.kv_len;
    const int N = p.n_ranks;
    const Range kr = p.kv_explicit ? p.kv_range : layout_range(p.layout, N, p.seq_len, j);
    const int64_t pos_k = range_pos(kr, (int64_t)(key_ok ? key : p.kv_len - 1));
    const int64_t krow = (int64_t)j * p.kv_row_step + (key_ok ? key : 0);
    int64_t ds_k = 0, de_k = INT64_MAX;  // queries at or past de_k lie in a later document
    if (p.n_docs > 0) doc_bounds(p, pos_k, &ds_k, &de_k);

    {
        const T *ks = static_cast<const T *>(p.k) + bb * p.k_sb + krow * p.k_ss + (int64_t)hk * p.k_sh;
        const T *vs = static_cast<const T *>(p.v) + bb * p.v_sb + krow * p.v_ss + (int64_t)hk * p.v_sh;
        for (int i = 0; i < D; ++i) {
            k_s[tid * C::LD + i] = key_ok ? ldf(ks + i) : 0.f;
            if (DK) v_s[tid * C::LD + i] = key_ok ? ldf(vs + i) : 0.f;
        }
    }
    const float scale = p.scale;
    const T *Q = static_cast<const T *>(p.q);
    const T *G = static_cast<const T *>(p.dout);

    float acc[D];
#pragma unroll
    for (int i = 0; i < D; ++i) acc[i] = 0.f;

    const int n_qt = (p.q_len + SRN - 1) / SRN;
    for (int hh = 0; hh < p.group; ++hh) {
        const int h = hk * p.group + hh;
        for (int r = 0; r < N; ++r) {
            const int qrank = (j + r) % N;  // the rank that holds block j at ring step r
            const Range qr = p.use_layout ? layout_range(p.layout, N, p.seq_len, qrank) : p.q_range;
            int qt_begin, qt_full;
            q_tile_bounds<int64_t>(qr, p.q_len, SRN, kr, p.kv_len, k_lo, SRM, p.causal != 0, &qt_begin, &qt_full);
            for (int qt = qt_begin; qt < n_qt; ++qt) {
                __syncthreads();
                const int q0 = qt * SRN;
                for (int idx = tid; idx < SRN * D; idx += SRM) {
                    const int i = idx / D, c = idx % D;
                    const int row = q0 + i;
                    float qq = 0.f, gg = 0.f;
                    if (row < p.q_len) {
                        const int64_t grow = (int64_t)qrank * p.q_row_step + row;
                        qq = ldf(Q + bb * p.q_sb + grow * p.q_ss + (int64_t)h * p.q_sh + c);
                        gg = ldf(G + bb * p.do_sb + grow * p.do_ss + (int64_t)h * p.do_sh + c);
                    }
                    q_s[i * D + c] = qq;
                    g_s[i * D + c] = gg;
                }
                if (tid < SRN) {
                    const int row = q0 + tid;
                    st_s[tid] = row < p.q_len ? p.stats[stat_index(p, bb, h, qrank, row)] : make_float2(-INFINITY, 0.f);
                }
                __syncthreads();
                if (!key_ok) continue;
                for (int i = 0; i < SRN; ++i) {
                    const int row = q0 + i;
                    if (row >= p.q_len) break;
                    const float2 st = st_s[i];
                    if (st.x == -INFINITY) continue;
                    if (p.causal && qt < qt_full && pos_k > range_pos(qr, (int64_t)row)) continue;
                    if (p.n_docs > 0 && range_pos(qr, (int64_t)row) >= de_k) continue;
                    float x = 0.f, dp = 0.f;
#pragma unroll 16
                    for (int c = 0; c < D; ++c) {
                        x = fmaf(k_s[tid * C::LD + c], q_s[i * D + c], x);
                        if (DK) dp = fmaf(v_s[tid * C::LD + c], g_s[i * D + c], dp);
                    }
                    const float pr = expf(x * scale - st.x);
                    if (DK) {
                        const float ds = pr * (dp - st.y);
#pragma unroll
                        for (int c = 0; c < D; ++c) acc[c] = fmaf(ds, q_s[i * D + c], acc[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < D; ++c) acc[c] = fmaf(pr, g_s[i * D + c], acc[c]);
                    }
                }
            }
        }
    }
    if (!key_ok) return;
    const int64_t off = DK ? bb * p.dk_sb + krow * p.dk_ss + (int64_t)hk * p.dk_sh
                           : bb * p.dv_sb + krow * p.dv_ss + (int64_t)hk * p.dv_sh;
    void *base = DK ? p.dk : p.dv;
    if (p.accumulate) {
        float *out = static_cast<float *>(base) + off;  // one thread owns the row: plain add
#pragma unroll
        for (int c = 0; c < D; ++c) out[c] += DK ? acc[c] * scale : acc[c];
    } else {
        T *out = static_cast<T *>(base) + off;
#pragma unroll
        for (int c = 0; c < D; ++c) stf(out + c, DK ? acc[c] * scale : acc[c]);
    }
}


template <typename T, int D>
cudaError_t launch_simt_bwd_t(const BwdParams &p, cudaStream_t st)
{
    using C = SbCfg<D>;
    static unsigned long long done_dq = 0, done_dv = 0, done_dk = 0;
    cudaError_t e;
    if ((e = set_smem_per_device((const void *)simt_bwd_dq_kernel<T, D>, C::SMEM, &done_dq)) != cudaSuccess) return e;
    if ((e = set_smem_per_device((const void *)simt_bwd_dkv_kernel<T, D, false>, C::SMEM, &done_dv)) != cudaSuccess)
        return e;
    if ((e = set_smem_per_device((const void *)simt_bwd_dkv_kernel<T, D, true>, C::SMEM, &done_dk)) != cudaSuccess)
        return e;
    const int64_t rows = (int64_t)p.b * p.hq * p.n_ranks * p.q_len;
    if (rows == 0) return cudaSuccess;
    simt_bwd_stats_kernel<T, D><<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(p);
    const int64_t n_qt = (p.q_len + SRM - 1) / SRM, n_kt = (p.kv_len + SRM - 1) / SRM;
    simt_bwd_dq_kernel<T, D><<<(unsigned)(p.n_ranks * n_qt * p.b * p.hq), SRM, C::SMEM, st>>>(p);
    const unsigned kv_items = (unsigned)(p.n_kv_blocks * n_kt * p.b * p.hkv);
    simt_bwd_dkv_kernel<T, D, false><<<kv_items, SRM, C::SMEM, st>>>(p);
    simt_bwd_dkv_kernel<T, D, true><<<kv_items, SRM, C::SMEM, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_simt(const BwdParams &p, bool fp32, cudaStream_t stream)
{
    if (fp32) {
        if (p.d == 64) return launch_simt_bwd_t<float, 64>(p, stream);
        if (p.d == 128) return launch_simt_bwd_t<float, 128>(p, stream);
    } else {
        if (p.d == 64) return launch_simt_bwd_t<__nv_bfloat16, 64>(p, stream);
        if (p.d == 128) return launch_simt_bwd_t<__nv_bfloat16, 128>(p, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace cpattn
