"""Ring-scheduled blockwise softmax attention on one B200: Python binding of libcpattn.

Argument marshalling only.  Every step of the path runs in the CUDA kernels of
libcpattn.so (built in-tree by context_attention_cp_b200.build); if that library
is missing the first call raises ImportError instead of computing anything.

Entry points mirror include/cpattn.h:
  block_attn_fwd(q, k, v, q_range, kv_range, causal, scale, o, lse, accumulate)
  block_attn_bwd(q, k, v, o, lse, do, q_range, kv_range, causal, scale, dq_acc, dk_acc, dv_acc)
  lse_merge(o_acc, lse_acc, o_b, lse_b, o_out=None)
  ring_attn_fwd(q, k, v, layout, N, causal, scale, o=None, lse=None, mode="fused")
  ring_attn_bwd(q, k, v, o, lse, do, layout, N, causal, scale) -> (dq, dk, dv)
  allgather_attn_fwd(q, k, v, layout, N, causal, doc_starts=None, scale=None)
  allgather_attn_bwd(q, k, v, o, lse, do, layout, N, causal, doc_starts=None) -> (dq, dk, dv)
  ulysses_attn_fwd(q, k, v, P, causal, scale=None); ulysses_all_to_all(x, P, inverse=False)
  ulysses_attn_bwd(q, k, v, o, lse, do, P, causal, scale=None) -> (dq, dk, dv)
  usp_attn_fwd(q, k, v, layout, N, P, causal, scale=None)     (Ulysses x ring)
  usp_attn_bwd(q, k, v, o, lse, do, layout, N, P, causal, scale=None) -> (dq, dk, dv)
  layout_permute(x, layout, N, seq_axis=1, inverse=False, out=None)
  layout_range(layout, N, S, rank) -> (nseg, start, len, stride)
  tile_classes(q_range, q_len, kv_range, kv_len, causal, tile_q, tile_k)
  stream_check()
The real-rank ring (one process per GPU, K/V passed with torch.distributed
point-to-point transfers, or read in place from the other ranks' memory with
PeerBlocks / ring_attn_fwd_peer) lives in context_attention_cp_b200.ring_dist;
peer_export / peer_import / peer_close map another process's device block, peer_copy
pulls one into local memory.
Tensors are torch tensors on the current CUDA device; token tensors are
[b, s, H, d] with d contiguous, lse tensors [b, H, s] fp32.
"""
from ._binding import (  # noqa: F401
    CPError, LAYOUTS, MODES, allgather_attn_bwd, allgather_attn_fwd, allgather_workspace_bytes, block_attn_bwd, block_attn_fwd, layout_permute,
    layout_range, lib, lib_path,
    lse_merge, ring_attn_bwd, ring_attn_fwd, ring_attn_fwd_static_scratch, ring_bwd_workspace_bytes,
    ring_workspace_bytes, selftest_wait_timeout, stream_check, tile_classes, ulysses_all_to_all, ulysses_attn_bwd, ulysses_attn_fwd,
    ulysses_workspace_bytes, usp_attn_bwd, usp_attn_fwd, usp_workspace_bytes, peer_close, peer_copy, peer_export, peer_import,
)
