// bwd.h -- internal launch interface of the backward pass (attn_bwd.cu), shared
// with the C ABI (abi.cu).
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力, paragraph
// on the backward pass: with the GLOBAL lse of a query row, p_j = e^{x_j - lse}
// is exact on any key block alone, so each ring step's block yields its own share
//   dv_j += p_j do,   dx_j = p_j (do . v_j - D),   D = do . o,
//   dq += scale dx_j k_j,   dk_j += scale dx_j q   (x_j = scale q . k_j);
// dQ accumulates on the query's rank while dK, dV travel with their K/V block.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "layout.h"

namespace cpattn {

// Key rows one backward CTA owns (TMEM lanes) and query rows per inner step.
constexpr int kBwdKeyTile = 128;
constexpr int kBwdQueryTile = 64;

// For key tile [k_lo, k_lo + tile_k) of a key block (ranges k, kv_len rows) against
// a query block of q_len rows (ranges q) in tiles of tile_q, with positions that
// increase with the local index: query tiles [0, *qt_begin) see none of the keys,
// [*qt_begin, *qt_full) need the per-element mask, [*qt_full, n_qt) see every key.
// A key tile that runs past kv_len is masked in every query tile it meets.
template <typename I>
CP_HD void q_tile_bounds(const RangeT<I> &q, I q_len, int tile_q, const RangeT<I> &k, I kv_len, I k_lo, int tile_k,
                         bool causal, int *qt_begin, int *qt_full)
{
    const int n_qt = (int)((q_len + tile_q - 1) / tile_q);
    const bool ragged_k = k_lo + tile_k > kv_len;
    if (!causal) {
        *qt_begin = 0;
        *qt_full = ragged_k ? n_qt : 0;
        return;
    }
    I k_hi = k_lo + tile_k - 1;
    if (k_hi > kv_len - 1) k_hi = kv_len - 1;
    const I pk_first = range_pos(k, k_lo), pk_last = range_pos(k, k_hi);
    int lo = 0, hi = n_qt;  // first tile whose last row sees the first key
    while (lo < hi) {
        const int mid = (lo + hi) / 2;
        I last = (I)mid * tile_q + tile_q - 1;
        if (last > q_len - 1) last = q_len - 1;
        if (range_pos(q, last) < pk_first) lo = mid + 1; else hi = mid;
    }
    *qt_begin = lo;
    hi = n_qt;  // first tile whose first row sees the last key
    while (lo < hi) {
        const int mid = (lo + hi) / 2;
        if (range_pos(q, (I)mid * tile_q) < pk_last) lo = mid + 1; else hi = mid;
    }
    *qt_full = ragged_k ? n_qt : lo;
}

// One backward launch.  Work item = (key rank j, key tile, batch, kv head); it walks
// the query heads of its group, ring steps r in [step_begin, step_end) (query rank
// (j + r) mod n_ranks, the rank that holds block j at step r) and the query tiles
// that see the key tile, accumulating dK, dV on chip and adding dQ shares into the
// fp32 dq_acc with bulk reductions.
struct BwdParams {
    int b, hq, hkv, group, d;
    int q_len, kv_len;          // rows of one rank's query / key block
    int n_ranks, step_begin, step_end;
    int causal, use_layout, layout;
    int64_t seq_len;
    Range q_range, kv_range;    // explicit ranges (use_layout == 0)
    int64_t q_row_step, kv_row_step;
    float scale, scale_log2;
    // inputs
    const void *q, *k, *v, *o, *dout;
    int64_t q_sb, q_ss, q_sh, k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    int64_t o_sb, o_ss, o_sh, do_sb, do_ss, do_sh;
    const float *lse;
    int64_t lse_sb, lse_sh, lse_ss;
    // workspace: per-row statistics (lse * log2 e, D) [b][hq][n_ranks][lpad] and the
    // fp32 dQ accumulator [b, n_ranks * q_row_step, hq, d] (dense)
    float2 *stats;
    int lpad;
    float *dq_acc;
    // outputs
    void *dq, *dk, *dv;
    int64_t dq_sb, dq_ss, dq_sh, dk_sb, dk_ss, dk_sh, dv_sb, dv_ss, dv_sh;
    int *status;
    // All-Gather form: kv_explicit = 1 takes kv_range as the one key block (the
    // gathered sequence, kv_row_step = 0); n_kv_blocks counts the key blocks (the
    // ring: n_ranks; the gathered form: 1).  Document mask: doc_starts [n_docs]
    // device array, sorted, first 0 (n_docs = 0: none); a query sees a key only
    // inside its own document.
    int kv_explicit, n_kv_blocks;
    const int *doc_starts;
    int n_docs;
    // tensor-core path: doc_pos_end[pos] = first position past the document holding
    // position pos (INT32_MAX for the last document), from launch_doc_tables
    const int *doc_pos_end;
    // as AttnParams::kv_map_h: the key block read (K, V) and written (dK, dV) in place
    // in zig-zag rank-major order, chunks of kv_map_h positions (0: rows = positions)
    int kv_map_h;
    // accumulate = 1 (the block form): dq, dk, dv are fp32 and this call's shares are
    // added to them (the tensor-core kernel reduces dQ straight into dq_acc = dq and
    // adds dK, dV in its epilogue; no dq conversion); 0: they are written in the
    // input dtype
    int accumulate;
    // work order: entry e -> (key block, key tile) = (order[e] >> 16, order[e] & 0xffff);
    // head_major puts (batch, kv head) outside the order in the grid
    int head_major;
    // with head_major: 1 = each CTA starts every ring step's query tiles at an offset
    // set by its key tile (wrapping around); 0 = it starts its ring steps at such an
    // offset (see QSeq in attn_bwd.cu)
    int tile_rotation;
    int n_kt;
    int order_len;
    uint32_t order[kMaxOrder];
};

// Statistics + dq_acc zeroing, the main tcgen05 kernel, then dq_acc -> dq.
cudaError_t launch_attn_bwd(const BwdParams &p, cudaStream_t stream);

// The FFMA backward (attn_simt_bwd.cu) for fp32 inputs or bf16 with d = 64, and for
// the block form: the ring layout (use_layout = 1), the gathered block (kv_explicit)
// with documents, or one explicit query block against one key block (use_layout =
// 0, kv_explicit = 1, n_ranks = 1); uses p.stats as its (lse, D) table and leaves
// dq_acc untouched.
cudaError_t launch_attn_bwd_simt(const BwdParams &p, bool fp32, cudaStream_t stream);

}  // namespace cpattn
