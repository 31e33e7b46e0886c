// kernels.h -- internal launch interface between the C ABI (abi.cu) and the
// CUDA kernels of libcpattn.  Not installed; the public ABI is include/cpattn.h.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/cpattn.h"
#include "layout.h"

namespace cpattn {

enum { DT_BF16 = 0, DT_FP32 = 1 };
enum { EPI_STORE = 0, EPI_MERGE = 1 };

// Largest number of (rank, query tile) entries the work-order table in the kernel
// parameters can hold; longer problems fall back to the natural order.
constexpr int kMaxOrder = 2048;

// One attention launch: for every (rank, query tile, batch, query head) work item,
// walk ring steps [step_begin, step_end) (source rank (rank - step) mod n_ranks),
// build each step's partial (o_b, lse_b) over the non-skipped key tiles, merge the
// partials with the LSE formula, and finish with the epilogue:
//   EPI_STORE: write (o, lse) of the merged result (o in o_dtype, lse fp32);
//   EPI_MERGE: LSE-merge the result into the fp32 (o, lse) already in memory.
// A block call is n_ranks = 1, one step, explicit ranges.
struct AttnParams {
    // sizes
    int b, hq, hkv, group, d;
    int q_len, kv_len;         // rows of one rank's query / key block
    int n_ranks, step_begin, step_end;
    int causal;
    int use_layout;            // 1: ranges from (layout, n_ranks, seq_len); 0: explicit
    int layout;
    int64_t seq_len;
    Range q_range, kv_range;   // explicit ranges (use_layout == 0)
    int64_t q_row_step, kv_row_step;  // tensor row offset of rank i's block = i * step
    float scale;               // softmax scale
    float scale_log2;          // softmax scale * log2(e)
    // inputs (fp32 SIMT kernel reads these; the tcgen05 kernel uses tensor maps)
    const void *q, *k, *v;
    int64_t q_sb, q_ss, q_sh, k_sb, k_ss, k_sh, v_sb, v_ss, v_sh;
    // outputs
    int epi;
    void *o;
    int o_dtype;
    int64_t o_sb, o_ss, o_sh;
    float *lse;
    int64_t lse_sb, lse_sh, lse_ss;
    // EPI_MERGE only (tensor-core path): when o_out is set, the merged o is written
    // there in o_out_dtype (strides oo_*) and o is left as it was; lse is updated.
    void *o_out;
    int o_out_dtype;
    int64_t oo_sb, oo_ss, oo_sh;
    int *status;
    // All-Gather form: kv_explicit = 1 takes kv_range for every rank and step (one
    // gathered key block, kv_row_step = 0).  Document mask (bf16 path): doc_starts
    // [n_docs] device array, sorted, first 0; a key in another document than the
    // query is invisible; n_docs = 0 means none.
    int kv_explicit;
    const int *doc_starts;
    int n_docs;
    // tensor-core path: doc_pos_start[pos] = first position of the document holding
    // position pos (of the seq_len positions), from launch_doc_tables
    const int *doc_pos_start;
    // kv_explicit with a zig-zag rank-major K/V (the All-Gather entry reading the
    // ranks' blocks in place): the chunk length h > 0, a multiple of the key tile, and
    // key tile rows map through zigzag_row(position, h, n_ranks); 0: rows = positions
    int kv_map_h;
    // work order: entry e -> (rank, row group) = (order[e] >> 16, order[e] & 0xffff);
    // a row group is the query rows one CTA covers (256 tensor-core, 128 SIMT)
    int n_qt;                  // row groups per rank
    int order_len;             // 0 = natural order
    uint32_t order[kMaxOrder];
};

struct TensorMaps;  // defined in attn_tc.cu

// bf16 tcgen05 path (d in {64, 128}).  q/k/v base pointers and strides in p are
// used to build TMA tensor maps.  Returns a cudaError_t.
cudaError_t launch_attn_tc(const AttnParams &p, cudaStream_t stream);

// Query rows one CTA of the tensor-core kernel covers (the unit of the work order);
// doc: the document-mask instantiation.
int attn_tc_rows_per_cta(bool doc);

// fp32 SIMT path (d in {64, 128}); one CTA covers 128 query rows.
cudaError_t launch_attn_simt(const AttnParams &p, cudaStream_t stream);

struct MergeParams {
    int64_t b, s, h, d;
    float *o_acc;  int64_t oa_sb, oa_ss, oa_sh;
    float *lse_acc; int64_t la_sb, la_sh, la_ss;
    const void *o_b; int ob_dtype; int64_t ob_sb, ob_ss, ob_sh;
    const float *lse_b; int64_t lb_sb, lb_sh, lb_ss;
    void *o_out; int out_dtype; int64_t out_sb, out_ss, out_sh;  // o_out == nullptr: in place
};
cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream);

struct PermuteParams {
    int layout, n_ranks, inverse;
    int64_t outer, seq, inner_bytes;  // contiguous [outer, seq, inner]
    const void *src;
    void *dst;
};
cudaError_t launch_permute(const PermuteParams &p, cudaStream_t stream);

// Raises the dynamic shared-memory limit of kernel `fn` to `bytes` on the current
// device, once per device (the attribute belongs to the device, not the process):
// `done` keeps one bit per device ordinal below 64; higher ordinals set it on every
// call.  From status.cu.
cudaError_t set_smem_per_device(const void *fn, int bytes, unsigned long long *done);

// Per-position document bounds (doc_tables.cu): for every position p < seq_len,
// doc_start[p] = the first position of the document holding p and doc_end[p] = the
// first position past it (INT32_MAX for the last document); starts: the n_docs
// sorted document starts in HOST memory, the first 0 (they reach the kernel as
// launch parameters, so nothing is copied from pageable memory), also written to
// starts_dev [n_docs] for the FFMA kernels.
cudaError_t launch_doc_tables(const int64_t *starts, int n_docs, int64_t seq_len, int *starts_dev, int *doc_start,
                              int *doc_end, cudaStream_t stream);

// Streaming multiprocessors of the current device (looked up once per device), from
// status.cu.
int sm_count();

// Device status word of the current device (2 ints), from status.cu.
cudaError_t status_word(int **ptr);

// Launches a one-warp kernel whose bounded mbarrier wait is made to expire after
// limit_ns (nothing arrives), raising the timeout bit of the status word.
cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream);

// Records a printf-style message for cp_last_error() and returns `status` (abi.cu).
cp_status report_error(cp_status status, const char *fmt, ...);

}  // namespace cpattn
