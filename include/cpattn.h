/*
 * cpattn.h -- C ABI of libcpattn: ring-scheduled blockwise softmax attention
 * (context parallelism with N virtual ranks) on one NVIDIA B200 (sm_100a).
 *
 * The operations follow "上下文并行与 Ring Attention" (hs-black.github.io):
 *   - section 分块注意力: block partial (o_b, lse_b) of a query set against one
 *     key/value block, with m_b = max x_j, l_b = sum e^{x_j - m_b},
 *     o_b = sum e^{x_j - m_b} v_j / l_b, lse_b = m_b + log l_b (natural log), and
 *     the merge o = e^{lse_1-lse} o_1 + e^{lse_2-lse} o_2, lse = M + log(e^{lse_1-M}
 *     + e^{lse_2-M}), M = max(lse_1, lse_2) (the boxed identity and its stable form);
 *   - section Ring Attention: at ring step r rank i attends its local Q to the K/V
 *     that rank (i - r) mod N started with, and merges the partial into its
 *     running (o, lse); Q and O never move;
 *   - sections 因果掩码带来的负载不均 / Zig-zag / Striped / 重排 token 的代价: the
 *     causal mask is judged on original token positions, and the three token
 *     layouts are permutations applied once at model entry;
 *   - section 分块注意力, paragraph on the backward pass: with the global lse any
 *     key block alone gives its exact share of dq, dk, dv;
 *   - section All-Gather 式 CP: K/V gathered once per layer, any attention mask
 *     (documents) applied in one local pass;
 *   - section DeepSpeed-Ulysses: an all-to-all switches the sharded dimension from
 *     the sequence to the heads, attention runs per head group, and back.
 *
 * Conventions shared by every entry point
 *   - Token tensors are [b, s, H, d] with d contiguous; lse tensors are
 *     [b, H, s] fp32 holding natural-log values.  Strides are in elements.
 *   - Ownership: the caller owns every buffer and the stream.  No entry point
 *     allocates device memory; no pointer is kept after return, apart from work
 *     already queued on `stream` and the mappings cp_peer_import makes (kept until
 *     cp_peer_close).
 *   - Errors: argument problems are reported synchronously through the return
 *     value (and a message from cp_last_error()).  Device-side problems (a
 *     bounded wait that ran out, a CUDA launch error) are reported by
 *     cp_stream_check() or by the next call's return value.  Nothing throws.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Thread-compatible: the global state is the per-device status word read by
 *     cp_stream_check(), the per-thread last-error message, and caches guarded by
 *     locks (work orders per shape, the peer mappings of cp_peer_import, the static
 *     scratch address per device).
 */
#ifndef CPATTN_H
#define CPATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CP_OK = 0,
    CP_ERR_INVALID_ARG = 1, /* null pointer, bad enum, bad dtype, bad stride */
    CP_ERR_UNSUPPORTED = 2, /* valid request the library does not implement (e.g. d) */
    CP_ERR_SHAPE = 3,       /* inconsistent or indivisible sizes */
    CP_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    CP_ERR_TIMEOUT = 5,     /* a device-side bounded wait expired (see cp_stream_check) */
    CP_ERR_BOUNDS = 6       /* debug build (libcpattn_debug.so) only: a kernel's bounds check
                               of a TMA coordinate or global index failed; the access was
                               skipped (see cp_stream_check) */
} cp_status;

typedef enum { CP_BF16 = 0, CP_FP32 = 1 } cp_dtype;

/* CP_MASK_CAUSAL: key t is visible to query p iff pos_k(t) <= pos_q(p), positions
 * taken from the cp_range arguments (original token positions). */
typedef enum { CP_MASK_NONE = 0, CP_MASK_CAUSAL = 1 } cp_mask_mode;

/* Token layouts over N ranks of c = S/N tokens each (section Zig-zag / Striped):
 *   CONTIGUOUS: rank i holds positions [i*c, (i+1)*c)
 *   ZIGZAG    : 2N chunks of c/2; rank i holds chunk i then chunk 2N-1-i
 *   STRIPED   : rank i holds positions i, i+N, i+2N, ... (token p on rank p mod N) */
typedef enum { CP_LAYOUT_CONTIGUOUS = 0, CP_LAYOUT_ZIGZAG = 1, CP_LAYOUT_STRIPED = 2 } cp_layout;

/* How cp_ring_attn_fwd runs the N steps (section Ring Attention):
 *   FUSED        : one launch; each CTA owns two 128-row query tiles of one rank and
 *                  walks the ring steps in order, keeping each step's partial
 *                  (o_b, lse_b) and the running (o, lse) on chip and merging them
 *                  with the LSE formula.
 *   STEPWISE     : the page's loop as written: N launches of the block kernel (all
 *                  ranks per launch) writing (o_b, lse_b) to the workspace, each
 *                  followed by a standalone merge launch; the last merge writes the
 *                  output.  Needs a workspace.
 *   STEPWISE_EPI : N launches of the block kernel, one ring step each; from step 1
 *                  on the block kernel merges its partial into the running fp32
 *                  (o, lse) in its epilogue (no o_b in memory, no merge launch); the
 *                  last step writes o in the output dtype.  Needs a workspace for a
 *                  bf16 output (the fp32 running o), none for fp32. */
typedef enum { CP_RING_FUSED = 0, CP_RING_STEPWISE = 1, CP_RING_STEPWISE_EPI = 2 } cp_ring_mode;

/* A strided 4-D view.  Token tensors: [b, s, H, d]; lse tensors: [b, H, s, 1]
 * (shape[3] = 1).  dtype is a cp_dtype.  Strides in elements; stride[3] must be 1. */
typedef struct {
    void *data;
    int32_t dtype;
    int32_t reserved;
    int64_t shape[4];
    int64_t stride[4];
} cp_tensor;

/* Original position of local token t (0 <= t < len[0] + len[1]):
 *   t <  len[0]: start[0] + t * stride
 *   t >= len[0]: start[1] + (t - len[0]) * stride      (only when nseg == 2)
 * stride >= 1.  Contiguous rank i: {1, {i*c}, {c}, 1}; zig-zag rank i:
 * {2, {i*c/2, (2N-1-i)*c/2}, {c/2, c/2}, 1}; striped rank i: {1, {i}, {c}, N}. */
typedef struct {
    int32_t nseg;
    int32_t reserved;
    int64_t start[2];
    int64_t len[2];
    int64_t stride;
} cp_range;

/* Block attention (section 分块注意力; the flash_attn call of section Ring Attention).
 *   q [b, sq, Hq, d], k/v [b, sk, Hkv, d]: same dtype (CP_BF16 or CP_FP32),
 *     Hq % Hkv == 0, query head h reads KV head h / (Hq/Hkv); d in {64, 128}.
 *   q_range / kv_range: original positions of the sq query / sk key rows
 *     (len[0] + len[1] must equal sq / sk).  Used only when mask_mode is causal.
 *   softmax_scale: multiplies q.k; 0 selects the standard 1/sqrt(d) (section
 *     分块注意力: x_j = q.k_j / sqrt(d_h)), any other value must be finite and > 0.
 *     The same holds for every entry point below that takes softmax_scale.
 *   accumulate == 0: writes o_b into o ([b, sq, Hq, d], dtype = q's dtype or
 *     CP_FP32) and lse_b into lse ([b, Hq, sq, 1] fp32).  Rows that see no key get
 *     o = 0, lse = -inf.
 *   accumulate == 1: o must be CP_FP32; (o, lse) hold a running partial and are
 *     updated in place with the LSE merge of (o_b, lse_b) (fused epilogue).
 * Fully masked key tiles are skipped whole.  Asynchronous on `stream`. */
cp_status cp_block_attn_fwd(const cp_tensor *q, const cp_tensor *k, const cp_tensor *v,
                            const cp_range *q_range, const cp_range *kv_range, int32_t mask_mode,
                            float softmax_scale, cp_tensor *o, cp_tensor *lse, int32_t accumulate,
                            void *stream);

/* Standalone LSE merge (section 分块注意力, stable form), one HBM pass:
 *   (o_acc, lse_acc) <- merge((o_acc, lse_acc), (o_b, lse_b))
 *   o_acc [b, s, H, d] CP_FP32, o_b same shape CP_BF16 or CP_FP32,
 *   lse_acc / lse_b [b, H, s, 1] CP_FP32.
 * o_out: NULL to write the merged o back into o_acc; otherwise a [b, s, H, d]
 *   tensor (CP_BF16 or CP_FP32) that receives the merged o (rounded to nearest
 *   even for bf16) while o_acc is left unchanged; lse_acc is always updated.
 * An empty side (lse = -inf) contributes nothing; two empty sides give (0, -inf).
 * Rows are 16-byte aligned: d * sizeof(element) must be a multiple of 16. */
cp_status cp_lse_merge(cp_tensor *o_acc, cp_tensor *lse_acc, const cp_tensor *o_b,
                       const cp_tensor *lse_b, cp_tensor *o_out, void *stream);

/* Ring attention forward over N virtual ranks on one GPU (section Ring Attention).
 *   q [b, S, Hq, d], k/v [b, S, Hkv, d] in RANK-MAJOR order (as produced by
 *   cp_layout_permute): rows [i*c, (i+1)*c) belong to rank i, c = S/N.
 *   causal: 1 for the causal mask on original positions, 0 for none.
 *   o [b, S, Hq, d] (q's dtype), lse [b, Hq, S, 1] fp32, both in rank-major order.
 *   mode: cp_ring_mode.  workspace / workspace_bytes: device memory of at least
 *   cp_ring_workspace_bytes(...) bytes (may be NULL/0 when that is 0); the
 *   caller keeps it alive until the work on `stream` has finished.
 * Requires S % N == 0, S % (2N) == 0 for zig-zag, Hq % Hkv == 0, d in {64, 128}. */
cp_status cp_ring_attn_fwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                           const cp_tensor *k, const cp_tensor *v, float softmax_scale,
                           cp_tensor *o, cp_tensor *lse, int32_t mode, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Workspace bytes cp_ring_attn_fwd needs for this problem (section Ring Attention:
 * the running (o, lse) the loop keeps and, in the stepwise loop, each step's
 * partial (o_b, lse_b)): 0 for CP_RING_FUSED; the fp32 running o for
 * CP_RING_STEPWISE_EPI with bf16 (0 with fp32); the fp32 running o, o_b in dtype
 * and lse_b fp32 for CP_RING_STEPWISE.  Returns 0 as well for invalid arguments
 * (cp_ring_attn_fwd then reports them). */
size_t cp_ring_workspace_bytes(int32_t layout, int32_t N, int32_t mode, int32_t dtype, int64_t b,
                               int64_t S, int64_t Hq, int64_t d);

/* All-Gather context parallelism over N virtual ranks on one GPU (section
 * All-Gather 式 CP): before attention the K/V blocks of all ranks are gathered into
 * one copy of the whole sequence, then every rank's local Q attends to it in one
 * pass, with an optional document mask (documents packed into one sequence do not
 * see each other) -- the mask the page gives as the reason to gather instead of
 * ringing.
 *   q [b, S, Hq, d], k / v [b, S, Hkv, d]: bf16 (tensor cores) or fp32 (FFMA),
 *   d = 64 or 128, rank-major (as for cp_ring_attn_fwd); k and v contiguous.
 *   o [b, S, Hq, d] in q's dtype and lse [b, Hq, S, 1] fp32 come out rank-major.
 *   doc_starts: HOST array of n_docs first positions (original order), strictly
 *   increasing, doc_starts[0] = 0, all < S; n_docs = 1 means no document mask.
 *   Key t is visible to query p iff pos_k(t) <= pos_q(p) (causal) and both lie in
 *   the same document; n_docs > 1 requires causal = 1.
 *   workspace: at least cp_allgather_workspace_bytes(...) bytes, 256-byte aligned
 *   (the gathered K and V and the document table); kept alive by the caller until
 *   the work on `stream` has finished.
 * The result equals the ring's when n_docs = 1 (same FLOPs, one step). */
cp_status cp_allgather_attn_fwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                                const cp_tensor *k, const cp_tensor *v, const int64_t *doc_starts,
                                int32_t n_docs, float softmax_scale, cp_tensor *o, cp_tensor *lse,
                                void *workspace, size_t workspace_bytes, void *stream);

/* All-Gather backward (section All-Gather 式 CP: the reduce-scatter of dK, dV in
 * the backward): K and V gathered again, every rank's queries against the whole
 * sequence with the same document mask, the summed dK, dV handed back to each
 * rank's block.  Arguments as cp_allgather_attn_fwd (o and lse its results) plus
 * dout [b, S, Hq, d]; dq [b, S, Hq, d], dk / dv [b, S, Hkv, d] outputs in q's
 * dtype, all rank-major; k, v, dk, dv contiguous.  The dtypes and head dims of
 * cp_ring_attn_bwd (bf16 d = 128 on the tensor cores, the rest on FFMA kernels).
 *   workspace: cp_allgather_bwd_workspace_bytes(...) bytes, 256-byte aligned. */
cp_status cp_allgather_attn_bwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                                const cp_tensor *k, const cp_tensor *v, const cp_tensor *o,
                                const cp_tensor *lse, const cp_tensor *dout, const int64_t *doc_starts,
                                int32_t n_docs, float softmax_scale, cp_tensor *dq, cp_tensor *dk,
                                cp_tensor *dv, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_allgather_attn_bwd needs (0 for invalid arguments). */
size_t cp_allgather_bwd_workspace_bytes(int32_t N, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                                        int64_t Hkv, int64_t d, int32_t n_docs);

/* Workspace bytes cp_allgather_attn_fwd needs (0 for invalid arguments). */
size_t cp_allgather_workspace_bytes(int32_t N, int32_t dtype, int64_t b, int64_t S, int64_t Hkv,
                                    int64_t d, int32_t n_docs);

/* DeepSpeed-Ulysses all-to-all on one GPU (section DeepSpeed-Ulysses): the
 * exchange that moves block (s_i, h_j) -- the i-th sequence shard's j-th head
 * group -- from rank i to rank j.
 *   x_seq [b, S, H, d]: sequence-sharded, rank i holds tokens [i S/P, (i+1) S/P)
 *     (the original order, contiguous split);
 *   y_head [P * b, S, H/P, d]: head-sharded, entry r * b + bb holds every token of
 *     heads [r H/P, (r+1) H/P) of batch bb.
 *   direction 0 writes y_head from x_seq, 1 writes x_seq from y_head.  Both
 *   contiguous, same dtype, not overlapping; P must divide H and S.  Bit-exact. */
cp_status cp_ulysses_all_to_all(int32_t P, int32_t direction, const cp_tensor *x_seq, cp_tensor *y_head,
                                void *stream);

/* Ulysses attention over P virtual ranks on one GPU: all-to-all of q, k, v to the
 * head-sharded layout, each rank's n_h/P heads attend over the whole sequence (one
 * launch of the tensor-core kernel, bf16, or the FFMA kernel, fp32), all-to-all of o
 * and lse back.
 *   q [b, S, Hq, d], k / v [b, S, Hkv, d], o [b, S, Hq, d] in original order (the
 *   sequence-sharded layout), contiguous; lse [b, Hq, S, 1] fp32 contiguous.
 *   P must divide Hq and Hkv (a rank owns whole KV groups; with GQA, P <= Hkv) and
 *   S; S % 4 == 0.  causal: the causal mask on positions.
 *   workspace: cp_ulysses_workspace_bytes(...) bytes, 256-byte aligned (the
 *   head-sharded q, k, v, o, lse). */
cp_status cp_ulysses_attn_fwd(int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                              const cp_tensor *v, float softmax_scale, cp_tensor *o, cp_tensor *lse,
                              void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_ulysses_attn_fwd needs (0 for invalid arguments). */
size_t cp_ulysses_workspace_bytes(int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                                  int64_t Hkv, int64_t d);

/* Ulysses backward: the exchange of q, k, v, o, dout and lse to the head-sharded
 * layout, the ring backward with N = 1 over every rank's head group (the same
 * kernels as cp_ring_attn_bwd), and the exchange of dq, dk, dv back.
 *   Tensors in original order as for cp_ulysses_attn_fwd (o and lse its results);
 *   dq [b, S, Hq, d], dk / dv [b, S, Hkv, d] outputs in q's dtype; all contiguous.
 *   The dtypes and head dims of cp_ring_attn_bwd and the conditions of
 *   cp_ulysses_attn_fwd.
 *   workspace: cp_ulysses_bwd_workspace_bytes(...) bytes, 256-byte aligned. */
cp_status cp_ulysses_attn_bwd(int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                              const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse,
                              const cp_tensor *dout, float softmax_scale, cp_tensor *dq, cp_tensor *dk,
                              cp_tensor *dv, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_ulysses_attn_bwd needs (0 for invalid arguments). */
size_t cp_ulysses_bwd_workspace_bytes(int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                                      int64_t Hkv, int64_t d);

/* USP, Ulysses inside a group and the ring across groups, on one GPU ("DeepSpeed-
 * Ulysses" page, section on USP; hs-black.github.io context-parallel post, end of
 * section DeepSpeed-Ulysses).  N ring groups of P Ulysses ranks each (N * P virtual
 * ranks): ring group g holds the layout's block g (the ring layout over N, as
 * cp_layout_permute(layout, N) orders it), and Ulysses rank u of that group holds
 * the contiguous u-th of the block's P slices, all heads.  The exchange inside every
 * group gives rank (g, u) the group's whole block for heads [u Hq/P, (u+1) Hq/P)
 * (KV heads likewise); the ring attention over the N groups runs for every head
 * group (one fused launch, the head groups as batch entries); the exchange back
 * returns o and lse to the sequence-sharded ranks.
 *   q [b, S, Hq, d], k / v [b, S, Hkv, d], o [b, S, Hq, d]: the S axis in the
 *   ring's rank-major order for (layout, N), contiguous; lse [b, Hq, S, 1] fp32
 *   contiguous, same order.  P must divide Hq and Hkv; S % (N P) == 0, and
 *   S % 2N == 0 under zig-zag; S % 4 == 0.  N = 1 is cp_ulysses_attn_fwd, P = 1
 *   the fused ring.
 *   workspace: cp_usp_workspace_bytes(...) bytes, 256-byte aligned (the head-
 *   sharded q, k, v, o, lse).  Argument errors return synchronously; device
 *   errors surface through cp_stream_check. */
cp_status cp_usp_attn_fwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q,
                          const cp_tensor *k, const cp_tensor *v, float softmax_scale, cp_tensor *o,
                          cp_tensor *lse, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_usp_attn_fwd needs (0 for invalid arguments). */
size_t cp_usp_workspace_bytes(int32_t layout, int32_t N, int32_t P, int32_t dtype, int64_t b, int64_t S,
                              int64_t Hq, int64_t Hkv, int64_t d);

/* USP backward: the exchange of q, k, v, o, dout and lse inside every group, the
 * ring backward over the N groups for every head group (the kernels of
 * cp_ring_attn_bwd; dK, dV travel with their block), the exchange of dq, dk, dv
 * back.  Tensors as for cp_usp_attn_fwd (o and lse its results); dq [b, S, Hq, d],
 * dk / dv [b, S, Hkv, d] outputs in q's dtype and the same order; all contiguous.
 * The dtypes and head dims of cp_ring_attn_bwd and the conditions of
 * cp_usp_attn_fwd.
 *   workspace: cp_usp_bwd_workspace_bytes(...) bytes, 256-byte aligned. */
cp_status cp_usp_attn_bwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q,
                          const cp_tensor *k, const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse,
                          const cp_tensor *dout, float softmax_scale, cp_tensor *dq, cp_tensor *dk,
                          cp_tensor *dv, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_usp_attn_bwd needs (0 for invalid arguments). */
size_t cp_usp_bwd_workspace_bytes(int32_t layout, int32_t N, int32_t P, int32_t dtype, int64_t b,
                                  int64_t S, int64_t Hq, int64_t Hkv, int64_t d);

/* Ring attention backward over N virtual ranks on one GPU (section 分块注意力,
 * paragraph on the backward pass; section Ring Attention for the schedule).
 * With the forward's GLOBAL o and lse of every query row and the output gradient
 * dout, computes the gradients of L with dL/do = dout:
 *   p = e^{x - lse},  dv_j = sum_q p dout,  dx = p (dout . v_j - D),  D = dout . o,
 *   dq = scale sum_j dx k_j,  dk_j = scale sum_q dx q      (x = scale q . k).
 * The K/V blocks walk the ring once more; dK, dV travel with their block and dQ
 * accumulates on its rank.  One launch covers all N steps (like CP_RING_FUSED),
 * between a statistics pass (D and zeroed accumulators) and the dq conversion.
 *   q, o, dout [b, S, Hq, d]; k, v [b, S, Hkv, d]; lse [b, Hq, S, 1] fp32; all in
 *   rank-major order, as cp_ring_attn_fwd takes and returns them (o and lse are its
 *   results for the same q, k, v, layout, N, causal and softmax_scale).
 *   dq [b, S, Hq, d], dk / dv [b, S, Hkv, d]: outputs (q's dtype, rank-major), overwritten.
 *   workspace: device memory of at least cp_ring_bwd_workspace_bytes(...) bytes,
 *   256-byte aligned (row statistics and the fp32 dQ accumulator); the caller keeps
 *   it alive until the work on `stream` has finished.
 * All tensors but lse share q's dtype.  bf16 with d = 128 runs the tensor-core
 * kernel; fp32 (d = 64 or 128) and bf16 with d = 64 run FFMA kernels (fp32
 * arithmetic, results rounded once to the dtype).  Besides that the conditions of
 * cp_ring_attn_fwd.  Rows whose lse is -inf contribute nothing.  On the tensor-core
 * path dq sums its shares with fp32 atomic reductions, so its rounding can differ
 * from run to run; dk and dv are summed in a fixed order (every output of the FFMA
 * path is). */
cp_status cp_ring_attn_bwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                           const cp_tensor *k, const cp_tensor *v, const cp_tensor *o,
                           const cp_tensor *lse, const cp_tensor *dout, float softmax_scale,
                           cp_tensor *dq, cp_tensor *dk, cp_tensor *dv, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Block backward ("上下文并行与 Ring Attention", section 分块注意力, paragraph on the
 * backward pass): one query block against one key block with the query rows' GLOBAL
 * statistics, the step one rank of a real ring runs per held K/V block.  With
 * p_j = e^{x_j - lse} (lse of the whole sequence), D = dout . o (o of the whole
 * sequence) and x_j = scale q . k_j, this call ADDS its shares
 *   dq_acc += scale sum_j p_j (dout . v_j - D) k_j,
 *   dk_acc_j += scale sum_q p_j (dout . v_j - D) q,   dv_acc_j += sum_q p_j dout
 * over the visible (query, key) pairs of the two blocks.
 *   q, o, dout [b, sq, Hq, d] and k, v [b, sk, Hkv, d]: bf16 or fp32 (one dtype),
 *   d = 64 or 128; lse [b, Hq, sq, 1] fp32: the forward's GLOBAL lse of these rows;
 *   q_range / kv_range: original positions of the rows (as cp_block_attn_fwd);
 *   mask_mode: CP_MASK_CAUSAL or CP_MASK_NONE.
 *   dq_acc [b, sq, Hq, d], dk_acc / dv_acc [b, sk, Hkv, d]: fp32 accumulators the
 *   shares are added to (the caller zeroes them once).
 *   workspace: cp_block_bwd_workspace_bytes(b, sq, Hq) bytes, 256-byte aligned (the
 *   rows' lse and D).
 * bf16 with d = 128 runs the tensor-core backward kernel (P and dS rounded to bf16
 * for the tensor cores, fp32 accumulation; dK, dV added in its epilogue, dQ added
 * with fp32 atomic reductions, so dq_acc's rounding can vary from run to run);
 * fp32 and bf16 with d = 64 run the FFMA backward kernels (fp32 arithmetic).  Rows
 * whose lse is -inf add nothing.  Argument errors return synchronously. */
cp_status cp_block_attn_bwd(const cp_tensor *q, const cp_tensor *k, const cp_tensor *v,
                            const cp_tensor *o, const cp_tensor *lse, const cp_tensor *dout,
                            const cp_range *q_range, const cp_range *kv_range, int32_t mask_mode,
                            float softmax_scale, cp_tensor *dq_acc, cp_tensor *dk_acc, cp_tensor *dv_acc,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes cp_block_attn_bwd needs (the (lse, D) table, rows padded to 64). */
size_t cp_block_bwd_workspace_bytes(int64_t b, int64_t sq, int64_t Hq);

/* Workspace bytes cp_ring_attn_bwd needs (0 for invalid arguments). */
size_t cp_ring_bwd_workspace_bytes(int32_t layout, int32_t N, int32_t dtype, int64_t b, int64_t S,
                                   int64_t Hq, int64_t d);

/* Token permutation into / out of rank-major order (section 重排 token 的代价).
 *   x and x_ranked: same shape, dtype and contiguous layout; the sequence axis is
 *   seq_axis (1 for [b, S, H, d], 2 for lse [b, H, S, 1]).
 *   inverse == 0: x_ranked[.., i*c + t, ..] = x[.., pos(i, t), ..]
 *   inverse == 1: x[.., pos(i, t), ..] = x_ranked[.., i*c + t, ..]
 *     (here x_ranked is read and x is written).
 * Bit-exact copy; x and x_ranked must not overlap. */
cp_status cp_layout_permute(int32_t layout, int32_t N, int32_t seq_axis, const cp_tensor *x,
                            cp_tensor *x_ranked, int32_t inverse, void *stream);

/* Host only: the cp_range of rank `rank` for a sequence of S tokens split over N
 * ranks in `layout` (sections 因果掩码带来的负载不均 for the contiguous split, Zig-zag
 * for 2N chunks with rank i holding chunks i and 2N-1-i, Striped for token p on rank
 * p mod N).  Requires S % N == 0 (S % 2N == 0 for zig-zag) and 0 <= rank < N. */
cp_status cp_layout_range(int32_t layout, int32_t N, int64_t S, int32_t rank, cp_range *out);

/* Host only: the tile classes the kernels use for a (query block, key block) pair
 * (caption of the ring figure in section Ring Attention: blocks the causal mask
 * hides completely are skipped whole; section Zig-zag: the steps j != i of the
 * zig-zag layout are unmasked rectangles).
 * out[qt * n_kt + kt] = 0 (skip: no visible pair), 1 (full: every pair visible),
 * 2 (partial: masked element by element), for tiles of tile_q x tile_k local
 * rows; n_qt = ceil(q_len / tile_q), n_kt = ceil(kv_len / tile_k).  Rows past
 * q_len / kv_len are not tokens (a tile holding them is partial in the key axis). */
cp_status cp_tile_classes(const cp_range *q_range, int64_t q_len, const cp_range *kv_range,
                          int64_t kv_len, int32_t mask_mode, int32_t tile_q, int32_t tile_k,
                          int8_t *out);

/* Synchronises `stream`, then reports (and clears) the device status word of the
 * current device: CP_ERR_BOUNDS if a bounds check of the debug build failed,
 * CP_ERR_TIMEOUT if a kernel's bounded wait expired since the last check,
 * CP_ERR_CUDA if the stream reported an error, else CP_OK. */
cp_status cp_stream_check(void *stream);

/* Failure-detection self-test: launches on `stream` a one-warp kernel that waits on
 * a barrier nothing ever completes, with the same bounded wait every kernel of this
 * library uses, cut to limit_ns (1 ms .. 1 s).  The wait expires, the kernel sets the
 * device status word and returns normally; the next cp_stream_check(stream) then
 * reports CP_ERR_TIMEOUT (and clears the word).  The context stays usable.
 * Returns CP_ERR_INVALID_ARG for a limit outside the range.  No counterpart on the
 * pages: it exercises this library's own fault reporting. */
cp_status cp_selftest_wait_timeout(uint64_t limit_ns, void *stream);

/* Static description of a status code. */
const char *cp_status_string(cp_status s);

/* Message of the last failing call on this host thread ("" if none). */
const char *cp_last_error(void);

/* ABI version, bumped on incompatible changes. */
int32_t cp_abi_version(void);

/* ---- Blocks of other ranks on one node (real ranks, one process per GPU) ----
 * Section Ring Attention: at ring step r rank i attends its Q to the K/V block that
 * rank (i - r) mod N started with, and the block travels from rank to rank.  Between
 * the processes of one node no rank needs to send: every rank maps the other ranks'
 * blocks into its own address space with these calls, then either pulls the block of
 * the next step into a local buffer (cp_peer_copy, copy engines, overlapped with the
 * current step's kernel) or passes the mapped addresses to the block kernels
 * directly (cp_block_attn_fwd / cp_block_attn_bwd: plain TMA tile loads, no
 * multicast, and plain stores into a peer's dK, dV accumulators).  No collective
 * sits on the data path.
 *
 * cp_peer_handle: `ipc` is the CUDA IPC handle of the device allocation holding a
 * block, `offset` the block's byte offset inside that allocation, `bytes` the bytes
 * from the block's start to the allocation's end (an upper bound on what may be read
 * through the mapping).  It is plain bytes: send it to the other processes by any
 * host channel. */
typedef struct {
    uint8_t ipc[64];
    uint64_t offset;
    uint64_t bytes;
} cp_peer_handle;

/* Describes the block at `ptr`: device memory this process allocated with cudaMalloc
 * (a caching allocator's block inside such an allocation qualifies; memory from
 * stream-ordered pools or virtual-memory mappings does not and gives CP_ERR_CUDA).
 * Host-only.  The caller keeps the memory allocated while any peer has it mapped.
 * Errors: CP_ERR_INVALID_ARG for NULL arguments or a pointer that is not device
 * memory of this process. */
cp_status cp_peer_export(const void *ptr, cp_peer_handle *out);

/* Maps the block described by `h`, exported by ANOTHER process, on the current device
 * and returns its address there in *ptr.  Mappings are counted per (device,
 * allocation), so several blocks of one allocation map it once.  When the memory
 * lives on another GPU, peer access from the current device is enabled as needed.
 * Host-only.  Errors: CP_ERR_CUDA when the driver refuses (a handle exported by this
 * same process, no peer path between the GPUs, an allocation already freed). */
cp_status cp_peer_import(const cp_peer_handle *h, void **ptr);

/* Drops one import of `h` on the current device; the allocation is unmapped when its
 * last import is closed.  The caller makes sure that no queued kernel still reads it.
 * Errors: CP_ERR_INVALID_ARG when `h` is not mapped on the current device. */
cp_status cp_peer_close(const cp_peer_handle *h);

/* Queues on `stream` a copy of `bytes` from `src` (typically a block mapped with
 * cp_peer_import) to `dst` (device memory of the current device), done by the copy
 * engines (cudaMemcpyAsync, device to device), so a block read by many CTAs crosses
 * the link between GPUs once.  Errors: CP_ERR_INVALID_ARG for NULL pointers with
 * bytes > 0; CP_ERR_CUDA when the copy cannot be queued. */
cp_status cp_peer_copy(void *dst, const void *src, size_t bytes, void *stream);

/* Bytes of device scratch the library reserves for cp_ring_attn_fwd_static_scratch. */
#define CP_STATIC_SCRATCH_BYTES ((size_t)64 << 20)

/* Stepwise ring attention that allocates nothing, for callers that cannot call
 * cudaMalloc (for example a plug-in whose host engine owns all device memory and
 * passes it only input and output pointers, or a caller that must not take the
 * synchronisation an allocation can cause).  The pages have no counterpart: this
 * is a packaging variant of cp_ring_attn_fwd(..., CP_RING_STEPWISE, ...).
 *   Arguments and results are those of cp_ring_attn_fwd; the caller still owns q,
 *   k, v, o and lse.  The workspace comes from a static device array of
 *   CP_STATIC_SCRATCH_BYTES that every GPU loading the library holds until exit.
 *   Errors: CP_ERR_UNSUPPORTED (returned before any launch) when
 *   cp_ring_workspace_bytes(layout, N, CP_RING_STEPWISE, ...) exceeds
 *   CP_STATIC_SCRATCH_BYTES; otherwise as cp_ring_attn_fwd.
 *   All calls on a device share the array and it keeps the last call's contents
 *   (the ring writes everything it reads, so nothing needs clearing); calls whose
 *   work overlaps on the GPU race on it.  The first call on each device looks up
 *   the array's device address; make that first call before any stream capture.
 *   The address is kept for the life of the process: after a reset of the device
 *   (cudaDeviceReset) the array is gone and this entry point must not be called on
 *   that device again. */
cp_status cp_ring_attn_fwd_static_scratch(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q,
                                          const cp_tensor *k, const cp_tensor *v, float softmax_scale,
                                          cp_tensor *o, cp_tensor *lse, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CPATTN_H */
