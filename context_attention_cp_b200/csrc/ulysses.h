// ulysses.h -- the Ulysses all-to-all on one device (permute.cu), shared with the C
// ABI (abi.cu).
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section DeepSpeed-Ulysses:
// around attention the sharded dimension switches from the sequence ([s/P, n_h,
// d_h] per rank) to the heads ([s, n_h/P, d_h] per rank) and back; block (s_i, h_j)
// moves from rank i to rank j.  With every rank on one device that is a transpose
// of (rank, head group) blocks.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace cpattn {

// x [b][rows][P][chunk_bytes] <-> y [P][b][rows][chunk_bytes]; inverse = 0 writes y
// from x, inverse = 1 writes x from y.
struct ShardParams {
    int64_t P, b, rows, chunk_bytes;
    int inverse;
    const void *src;
    void *dst;
};
cudaError_t launch_shard_transpose(const ShardParams &p, cudaStream_t stream);

}  // namespace cpattn
