// permute.cu -- bit-exact gather/scatter of token rows into / out of rank-major order.
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 重排 token 的代价:
// attention is permutation-equivariant when the mask uses original positions, so
// a zig-zag or striped layout only needs the tokens reordered once at model entry
// (and the outputs put back).  Row i*c + t of the ranked tensor is the token at
// original position pos(i, t) of the layout (see layout.h).
//
// The tensor is viewed as [outer, seq, inner] bytes; each thread moves one 16-,
// 4- or 1-byte piece, consecutive threads covering consecutive bytes of a row.
//
// The same file holds the Ulysses all-to-all (section DeepSpeed-Ulysses: the
// sequence-sharded [s/P, n_h, d_h] blocks become head-sharded [s, n_h/P, d_h] ones
// and back), which on one device is a transpose of (rank, head group) blocks.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ulysses.h"

namespace cpattn {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) permute_kernel(const __grid_constant__ PermuteParams p)
{
    const int64_t per_row = p.inner_bytes / (int64_t)sizeof(T);
    const int64_t total = p.outer * p.seq * per_row;
    const int64_t c = p.seq / p.n_ranks;
    const T *src = reinterpret_cast<const T *>(p.src);
    T *dst = reinterpret_cast<T *>(p.dst);
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t piece = idx % per_row;
        const int64_t rr = (idx / per_row) % p.seq;  // ranked row
        const int64_t o = idx / (per_row * p.seq);
        const int rank = (int)(rr / c);
        const Range r = layout_range(p.layout, p.n_ranks, p.seq, rank);
        const int64_t pos = range_pos(r, rr - (int64_t)rank * c);
        const int64_t from = p.inverse ? rr : pos;
        const int64_t to = p.inverse ? pos : rr;
        dst[(o * p.seq + to) * per_row + piece] = src[(o * p.seq + from) * per_row + piece];
    }
}

// Ulysses all-to-all on one device: x [b][rows][P][chunk] <-> y [P][b][rows][chunk]
// (chunk bytes contiguous; forward y[r][bb][i] = x[bb][i][r], inverse the reverse).
template <typename T>
__global__ void __launch_bounds__(256) shard_transpose_kernel(const __grid_constant__ ShardParams p)
{
    const int64_t per = p.chunk_bytes / (int64_t)sizeof(T);
    const int64_t total = p.P * p.b * p.rows * per;
    const T *src = reinterpret_cast<const T *>(p.src);
    T *dst = reinterpret_cast<T *>(p.dst);
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t e = idx % per;
        int64_t rest = idx / per;
        const int64_t i = rest % p.rows;
        rest /= p.rows;
        const int64_t bb = rest % p.b;
        const int64_t r = rest / p.b;
        const int64_t xo = ((bb * p.rows + i) * p.P + r) * per + e;  // x[bb][i][r][e]
        const int64_t yo = ((r * p.b + bb) * p.rows + i) * per + e;  // y[r][bb][i][e]
        if (p.inverse) dst[xo] = src[yo]; else dst[yo] = src[xo];
    }
}

}  // namespace

cudaError_t launch_shard_transpose(const ShardParams &p, cudaStream_t stream)
{
    const int64_t rows = p.P * p.b * p.rows;
    if (rows == 0 || p.chunk_bytes == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.src) | reinterpret_cast<uintptr_t>(p.dst);
    int width = 1;
    if (p.chunk_bytes % 16 == 0 && al % 16 == 0) width = 16;
    else if (p.chunk_bytes % 4 == 0 && al % 4 == 0) width = 4;
    const int64_t total = rows * (p.chunk_bytes / width);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    if (width == 16) shard_transpose_kernel<uint4><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else if (width == 4) shard_transpose_kernel<uint32_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else shard_transpose_kernel<uint8_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteParams &p, cudaStream_t stream)
{
    const int64_t rows = p.outer * p.seq;
    if (rows == 0 || p.inner_bytes == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.src) | reinterpret_cast<uintptr_t>(p.dst);
    int width = 1;
    if (p.inner_bytes % 16 == 0 && al % 16 == 0) width = 16;
    else if (p.inner_bytes % 4 == 0 && al % 4 == 0) width = 4;
    const int64_t total = rows * (p.inner_bytes / width);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    if (width == 16) permute_kernel<uint4><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else if (width == 4) permute_kernel<uint32_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else permute_kernel<uint8_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace cpattn
