// attn_simt.cu -- fp32 block attention with plain FFMA arithmetic, for callers
// who need fp32 inputs and results (tf32 tensor cores keep only 10 mantissa bits).
//
// Same work decomposition and ring walk as the tensor-core kernel
// ("上下文并行与 Ring Attention", hs-black.github.io, sections 分块注意力 and
// Ring Attention): a CTA owns 128 query rows of one rank and one query head, one
// thread per row; for each ring step it runs the online-softmax recurrence over
// the step's visible keys (K/V staged in shared memory 32 keys at a time), turns
// the running (m, l, O) into the step partial o_b = O / l, lse_b = m + log l, and
// merges it into the running result with the LSE merge.  Fully masked key tiles
// are skipped; partial tiles are masked key by key on original positions.
// The All-Gather form (kv_explicit: one gathered key block in original order) and
// its document mask (section All-Gather 式 CP: a query sees only keys of its own
// document) are honoured key by key.
#include <cuda_runtime.h>
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace cpattn {
namespace {

constexpr int RM = 128;  // query rows per CTA
constexpr int RN = 32;   // keys per shared-memory tile

// Document start of position pos: the last of the sorted starts that is <= pos.
__device__ __forceinline__ int64_t simt_doc_start(const int *starts, int n, int64_t pos)
{
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((int64_t)starts[mid] <= pos) lo = mid + 1; else hi = mid;
    }
    return lo > 0 ? (int64_t)starts[lo - 1] : 0;
}

template <int D>
struct SimtCfg {
    static constexpr int LD = D + 1;                       // padded row (conflict-free)
    static constexpr int OFF_Q = 0;                        // [RM][LD] queries
    static constexpr int OFF_ACC = OFF_Q + RM * LD;        // [RM][LD] merged output
    static constexpr int OFF_K = OFF_ACC + RM * LD;        // [RN][D]
    static constexpr int OFF_V = OFF_K + RN * D;           // [RN][D]
    static constexpr int FLOATS = OFF_V + RN * D;
    static constexpr int SMEM = FLOATS * 4;
};

template <int D>
__global__ void __launch_bounds__(RM) attn_simt_kernel(const __grid_constant__ AttnParams p)
{
    using C = SimtCfg<D>;
    extern __shared__ float sm[];
    float *q_s = sm + C::OFF_Q;
    float *acc_s = sm + C::OFF_ACC;
    float *k_s = sm + C::OFF_K;
    float *v_s = sm + C::OFF_V;

    const int tid = threadIdx.x;
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
    const int h = bh % p.hq, bb = bh / p.hq, hk = h / p.group;
    const int q_lo = qt * RM;
    const int row = q_lo + tid;
    const bool row_ok = row < p.q_len;
    const Range qr = p.use_layout ? layout_range(p.layout, p.n_ranks, p.seq_len, rank) : p.q_range;
    const int64_t pos_q = range_pos(qr, row_ok ? row : p.q_len - 1);
    const int64_t ds_q = p.n_docs > 0 ? simt_doc_start(p.doc_starts, p.n_docs, pos_q) : 0;

    const float *Q = reinterpret_cast<const float *>(p.q);
    const float *K = reinterpret_cast<const float *>(p.k);
    const float *V = reinterpret_cast<const float *>(p.v);

    // this thread's query row
    {
        const int64_t qrow = (int64_t)rank * p.q_row_step + (row_ok ? row : 0);
        const float *src = Q + (int64_t)bb * p.q_sb + qrow * p.q_ss + (int64_t)h * p.q_sh;
        for (int i = 0; i < D; ++i) q_s[tid * C::LD + i] = row_ok ? src[i] : 0.f;
    }

    const float scale = p.scale;
    float lse_acc = -INFINITY;  // natural log
    bool have_acc = false;
    bool any_key_tile = false;

    for (int step = p.step_begin; step < p.step_end; ++step) {
        const int N = p.n_ranks;
        const int src = ((rank - step) % N + N) % N;
        const Range kr = (p.use_layout && !p.kv_explicit) ? layout_range(p.layout, N, p.seq_len, src) : p.kv_range;
        int kt_full, kt_end;
        kv_tile_bounds<int64_t>(qr, p.q_len, q_lo, RM, kr, p.kv_len, RN, p.causal != 0, &kt_full, &kt_end);
        if (kt_end == 0) continue;
        any_key_tile = true;
        float m = -INFINITY, l = 0.f;
        float ob[D];
#pragma unroll
        for (int i = 0; i < D; ++i) ob[i] = 0.f;
        for (int kt = 0; kt < kt_end; ++kt) {
            __syncthreads();
            const int k0 = kt * RN;
            for (int idx = tid; idx < RN * D; idx += RM) {
                const int j = idx / D, c = idx % D;
                const int key = k0 + j;
                float kvk = 0.f, kvv = 0.f;
                if (key < p.kv_len) {
                    const int64_t krow = (int64_t)src * p.kv_row_step + key;
                    kvk = K[(int64_t)bb * p.k_sb + krow * p.k_ss + (int64_t)hk * p.k_sh + c];
                    kvv = V[(int64_t)bb * p.v_sb + krow * p.v_ss + (int64_t)hk * p.v_sh + c];
                }
                k_s[j * D + c] = kvk;
                v_s[j * D + c] = kvv;
            }
            __syncthreads();
            for (int j = 0; j < RN; ++j) {
                const int key = k0 + j;
                if (key >= p.kv_len) break;
                if (p.causal && kt >= kt_full && range_pos(kr, key) > pos_q) continue;
                if (p.n_docs > 0 && range_pos(kr, key) < ds_q) continue;
                float x = 0.f;
#pragma unroll 16
                for (int i = 0; i < D; ++i) x = fmaf(q_s[tid * C::LD + i], k_s[j * D + i], x);
                x *= scale;
                const float m_new = fmaxf(m, x);
                const float a = expf(m - m_new);  // m = -inf on the first key gives 0
                const float w = expf(x - m_new);
                l = l * a + w;
#pragma unroll
                for (int i = 0; i < D; ++i) ob[i] = fmaf(ob[i], a, w * v_s[j * D + i]);
                m = m_new;
            }
        }
        // step partial (o_b = ob / l, lse_b = m + log l), merged into acc_s / lse_acc
        if (l > 0.f) {
            const float lse_b = m + logf(l);
            float wa = 0.f, wb = 1.f / l, new_lse = lse_b;
            if (have_acc) {
                const float M = fmaxf(lse_acc, lse_b);
                new_lse = M + logf(expf(lse_acc - M) + expf(lse_b - M));
                wa = expf(lse_acc - new_lse);
                wb = expf(lse_b - new_lse) / l;
            }
            for (int i = 0; i < D; ++i) {
                const float prev = have_acc ? acc_s[tid * C::LD + i] : 0.f;
                acc_s[tid * C::LD + i] = have_acc ? fmaf(wa, prev, wb * ob[i]) : wb * ob[i];
            }
            lse_acc = new_lse;
            have_acc = true;
        }
    }

    if (!row_ok) return;
    if (!any_key_tile && p.epi == EPI_MERGE) return;
    const int64_t orow = (int64_t)rank * p.q_row_step + row;
    const int64_t obase = (int64_t)bb * p.o_sb + orow * p.o_ss + (int64_t)h * p.o_sh;
    float *lse_ptr = p.lse + (int64_t)bb * p.lse_sb + (int64_t)h * p.lse_sh + orow * p.lse_ss;
    if (p.epi == EPI_STORE) {
        float *o = reinterpret_cast<float *>(p.o) + obase;
        for (int i = 0; i < D; ++i) o[i] = have_acc ? acc_s[tid * C::LD + i] : 0.f;
        *lse_ptr = have_acc ? lse_acc : -INFINITY;
    } else if (have_acc) {
        float *o = reinterpret_cast<float *>(p.o) + obase;
        const float la = *lse_ptr;
        float wa = 0.f, wb = 1.f, new_lse = lse_acc;
        if (la != -INFINITY) {
            const float M = fmaxf(la, lse_acc);
            new_lse = M + logf(expf(la - M) + expf(lse_acc - M));
            wa = expf(la - new_lse);
            wb = expf(lse_acc - new_lse);
        }
        for (int i = 0; i < D; ++i)
            o[i] = (la != -INFINITY) ? fmaf(wa, o[i], wb * acc_s[tid * C::LD + i]) : acc_s[tid * C::LD + i];
        *lse_ptr = new_lse;
    }
}

template <int D>
cudaError_t launch_simt_d(const AttnParams &p, cudaStream_t stream)
{
    static unsigned long long attr_done = 0;
    {
        cudaError_t e = set_smem_per_device((const void *)attn_simt_kernel<D>, SimtCfg<D>::SMEM, &attr_done);
        if (e != cudaSuccess) return e;
    }
    const int64_t items = (int64_t)p.n_ranks * p.n_qt * p.b * p.hq;
    if (items == 0) return cudaSuccess;
    attn_simt_kernel<D><<<(unsigned)items, RM, SimtCfg<D>::SMEM, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

// The SIMT kernel tiles queries by 128 like the tensor-core kernel, so one
// work-order table serves both.
cudaError_t launch_attn_simt(const AttnParams &p, cudaStream_t stream)
{
    if (p.d == 64) return launch_simt_d<64>(p, stream);
    if (p.d == 128) return launch_simt_d<128>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace cpattn
