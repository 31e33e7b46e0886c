// permute.cu -- bit-exact gather/scatter of token rows into / out of rank-major order.
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 重排 token 的代价:
// attention is permutation-equivariant when the mask uses original positions, so
// a zig-zag or striped layout only needs the tokens reordered once at model entry
// (and the outputs put back).  Row i*c + t of the ranked tensor is the token at
// original position pos(i, t) of the layout (see layout.h).
//
// The tensor is viewed as [outer, seq, inner] bytes and copied in 16-, 4- or
// 1-byte pieces.  A row of at least one piece per lane of a warp goes to one warp
// (a long row in 8 KB segments, a warp each): the row's source and destination are
// worked out once, and the lanes stream the row with several loads in flight each.  4-byte rows (the LSE) go four to a thread
// with 16-byte accesses where the positions allow; other short rows take one piece
// per thread.
//
// The same file holds the Ulysses all-to-all (section DeepSpeed-Ulysses: the
// sequence-sharded [s/P, n_h, d_h] blocks become head-sharded [s, n_h/P, d_h] ones
// and back), which on one device is a transpose of (rank, head group) blocks.
#include <cuda_runtime.h>

#include "kernels.h"
#include "ulysses.h"

// 1: rows (chunks) of at least 32 pieces go one per warp and 4-byte rows four per
// thread; 0: one piece per thread everywhere (measured against each other).
#ifndef CP_PERMUTE_ROWS
#define CP_PERMUTE_ROWS 1
#endif

namespace cpattn {
namespace {

constexpr int kRowUnroll = 4;  // loads in flight per lane in a row copy

template <typename T>
__device__ __forceinline__ void copy_row(const T *__restrict__ s, T *__restrict__ d, int64_t n, int lane)
{
    // every load of a pass is issued before its stores, a ragged last pass included
    for (int64_t e = lane; e < n; e += 32 * kRowUnroll) {
        T r[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u)
            if (e + 32 * u < n) r[u] = s[e + 32 * u];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u)
            if (e + 32 * u < n) d[e + 32 * u] = r[u];
    }
}

// Ranked row rr of a sequence in the layout -> original position.
__device__ __forceinline__ int64_t ranked_to_pos(const PermuteParams &p, int64_t c, int64_t rr)
{
    const int rank = (int)(rr / c);
    const Range r = layout_range(p.layout, p.n_ranks, p.seq, rank);
    return range_pos(r, rr - (int64_t)rank * c);
}

// A row (chunk) of more than kSegPieces pieces is cut into segments of kSegPieces, a
// warp per segment, so a few long rows still spread over the whole grid.
constexpr int64_t kSegPieces = 512;

template <typename T>
__global__ void __launch_bounds__(256) permute_rows_kernel(const __grid_constant__ PermuteParams p, int64_t n_seg)
{
    const int64_t per_row = p.inner_bytes / (int64_t)sizeof(T);
    const int64_t units = p.outer * p.seq * n_seg;
    const int64_t c = p.seq / p.n_ranks;
    const int lane = threadIdx.x & 31;
    const T *src = reinterpret_cast<const T *>(p.src);
    T *dst = reinterpret_cast<T *>(p.dst);
    const int64_t n_warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += n_warps) {
        const int64_t row = n_seg == 1 ? u : u / n_seg;
        const int64_t e0 = n_seg == 1 ? 0 : (u - row * n_seg) * kSegPieces;
        const int64_t n = per_row - e0 < kSegPieces || n_seg == 1 ? per_row - e0 : kSegPieces;
        const int64_t o = row / p.seq, rr = row - o * p.seq;
        const int64_t pos = ranked_to_pos(p, c, rr);
        const int64_t from = p.inverse ? rr : pos;
        const int64_t to = p.inverse ? pos : rr;
        copy_row(src + (o * p.seq + from) * per_row + e0, dst + (o * p.seq + to) * per_row + e0, n, lane);
    }
}

// 4-byte rows (the fp32 LSE, sequence last) in general: a thread moves groups of 4 consecutive
// ranked rows, one 16-byte access on the ranked side.  The launcher sends only
// sequences whose rank length c and zig-zag chunk length c / 2 are multiples of 4, so
// a group never straddles a rank or a chunk and its positions are pos0 + u * stride,
// worked out once per group.  On the original side that is one 16-byte access when
// stride == 1 (contiguous, zig-zag; pos0 is then a multiple of 4) and 4 word accesses
// when striped.  kWordUnroll groups, a grid-stride apart, are loaded before any of
// them is stored.
constexpr int kWordUnroll = 4;

template <typename I>
__global__ void __launch_bounds__(256) permute_words_kernel(const __grid_constant__ PermuteParams p)
{
    // I: int32_t when the group indices with the unrolled strides fit, else int64_t
    const I seq = (I)p.seq;
    const I groups_per_seq = seq / 4;
    const I groups = (I)p.outer * groups_per_seq;
    const I c = seq / p.n_ranks;
    const I threads = (I)gridDim.x * blockDim.x;
    const uint32_t *src = static_cast<const uint32_t *>(p.src);
    uint32_t *dst = static_cast<uint32_t *>(p.dst);
    for (I g0 = (I)blockIdx.x * blockDim.x + threadIdx.x; g0 < groups; g0 += threads * kWordUnroll) {
        int64_t ranked[kWordUnroll], orig[kWordUnroll];  // word offsets of the group's first row
        I stride[kWordUnroll];
        uint4 v[kWordUnroll];
#pragma unroll
        for (int u = 0; u < kWordUnroll; ++u) {
            const I g = g0 + (I)u * threads;
            stride[u] = 0;  // 0: no group here
            if (g >= groups) continue;
            const I o = g / groups_per_seq;
            const I rr = (g - o * groups_per_seq) * 4;
            const int rank = (int)(rr / c);
            const RangeT<I> r = layout_range_t<I>(p.layout, p.n_ranks, seq, rank);
            const int64_t base = (int64_t)o * seq;
            ranked[u] = base + rr;
            orig[u] = base + range_pos(r, rr - (I)rank * c);
            stride[u] = r.stride;
        }
#pragma unroll
        for (int u = 0; u < kWordUnroll; ++u) {
            if (stride[u] == 0) continue;
            if (p.inverse) {
                v[u] = *reinterpret_cast<const uint4 *>(src + ranked[u]);
            } else if (stride[u] == 1) {
                v[u] = *reinterpret_cast<const uint4 *>(src + orig[u]);
            } else {
                const int64_t s1 = stride[u];
                v[u].x = src[orig[u]];
                v[u].y = src[orig[u] + s1];
                v[u].z = src[orig[u] + 2 * s1];
                v[u].w = src[orig[u] + 3 * s1];
            }
        }
#pragma unroll
        for (int u = 0; u < kWordUnroll; ++u) {
            if (stride[u] == 0) continue;
            if (!p.inverse) {
                *reinterpret_cast<uint4 *>(dst + ranked[u]) = v[u];
            } else if (stride[u] == 1) {
                *reinterpret_cast<uint4 *>(dst + orig[u]) = v[u];
            } else {
                const int64_t s1 = stride[u];
                dst[orig[u]] = v[u].x;
                dst[orig[u] + s1] = v[u].y;
                dst[orig[u] + 2 * s1] = v[u].z;
                dst[orig[u] + 3 * s1] = v[u].w;
            }
        }
    }
}

// The same copy when every segment of every rank (c rows; c / 2 for zig-zag) is a
// multiple of kSpanRows: a CTA takes a span of kSpanRows consecutive ranked rows,
// which then lies inside one segment of one rank, so the span's first position is
// decoded once per thread and its rows sit at pos0 + x * stride; each thread moves
// kWordUnroll groups of 4 rows, all loaded before any is stored.
constexpr int kSpanRows = 256 * 4 * kWordUnroll;

template <typename I>
__global__ void __launch_bounds__(256) permute_words_span_kernel(const __grid_constant__ PermuteParams p)
{
    // I: int32_t when outer * seq fits, else int64_t
    const I seq = (I)p.seq;
    const I c = seq / p.n_ranks;
    const I spans_per_seq = seq / kSpanRows;
    const I n_spans = (I)p.outer * spans_per_seq;
    const uint32_t *src = static_cast<const uint32_t *>(p.src);
    uint32_t *dst = static_cast<uint32_t *>(p.dst);
    for (I sp = (I)blockIdx.x; sp < n_spans; sp += (I)gridDim.x) {
        const I o = sp / spans_per_seq;
        const I rr0 = (sp - o * spans_per_seq) * kSpanRows;
        const int rank = (int)(rr0 / c);
        const RangeT<I> r = layout_range_t<I>(p.layout, p.n_ranks, seq, rank);
        const int64_t base = (int64_t)o * seq;
        const int64_t ranked0 = base + rr0;
        const int64_t orig0 = base + range_pos(r, rr0 - (I)rank * c);
        const int64_t st = r.stride;
        uint4 v[kWordUnroll];
#pragma unroll
        for (int u = 0; u < kWordUnroll; ++u) {
            const int64_t x = 4 * ((int64_t)u * 256 + threadIdx.x);  // row offset inside the span
            if (p.inverse) {
                v[u] = *reinterpret_cast<const uint4 *>(src + ranked0 + x);
            } else if (st == 1) {
                v[u] = *reinterpret_cast<const uint4 *>(src + orig0 + x);
            } else {
                const int64_t a = orig0 + x * st;
                v[u].x = src[a];
                v[u].y = src[a + st];
                v[u].z = src[a + 2 * st];
                v[u].w = src[a + 3 * st];
            }
        }
#pragma unroll
        for (int u = 0; u < kWordUnroll; ++u) {
            const int64_t x = 4 * ((int64_t)u * 256 + threadIdx.x);
            if (!p.inverse) {
                *reinterpret_cast<uint4 *>(dst + ranked0 + x) = v[u];
            } else if (st == 1) {
                *reinterpret_cast<uint4 *>(dst + orig0 + x) = v[u];
            } else {
                const int64_t a = orig0 + x * st;
                dst[a] = v[u].x;
                dst[a + st] = v[u].y;
                dst[a + 2 * st] = v[u].z;
                dst[a + 3 * st] = v[u].w;
            }
        }
    }
}

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
        const int64_t pos = ranked_to_pos(p, c, rr);
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

// The same with one warp per chunk (chunks of at least 32 pieces; longer ones in
// segments of kSegPieces).
template <typename T>
__global__ void __launch_bounds__(256) shard_transpose_rows_kernel(const __grid_constant__ ShardParams p, int64_t n_seg)
{
    const int64_t per = p.chunk_bytes / (int64_t)sizeof(T);
    const int64_t units = p.P * p.b * p.rows * n_seg;
    const int lane = threadIdx.x & 31;
    const T *src = reinterpret_cast<const T *>(p.src);
    T *dst = reinterpret_cast<T *>(p.dst);
    const int64_t n_warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t u = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += n_warps) {
        const int64_t ch = n_seg == 1 ? u : u / n_seg;  // ch walks y in order: y[r][bb][i]
        const int64_t e0 = n_seg == 1 ? 0 : (u - ch * n_seg) * kSegPieces;
        const int64_t n = per - e0 < kSegPieces || n_seg == 1 ? per - e0 : kSegPieces;
        const int64_t i = ch % p.rows;
        const int64_t rest = ch / p.rows;
        const int64_t bb = rest % p.b;
        const int64_t r = rest / p.b;
        const int64_t xo = ((bb * p.rows + i) * p.P + r) * per + e0;
        const int64_t yo = ch * per + e0;
        if (p.inverse) copy_row(src + yo, dst + xo, n, lane);
        else copy_row(src + xo, dst + yo, n, lane);
    }
}

}  // namespace

cudaError_t launch_shard_transpose(const ShardParams &p, cudaStream_t stream)
{
    const int64_t rows = p.P * p.b * p.rows;
    if (rows == 0 || p.chunk_bytes == 0) return cudaSuccess;
    const int sms = sm_count();
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.src) | reinterpret_cast<uintptr_t>(p.dst);
    int width = 1;
    if (p.chunk_bytes % 16 == 0 && al % 16 == 0) width = 16;
    else if (p.chunk_bytes % 4 == 0 && al % 4 == 0) width = 4;
    const int64_t per = p.chunk_bytes / width;
    if (CP_PERMUTE_ROWS && per >= 32) {  // one warp per chunk (segment), 8 per block
        const int64_t n_seg = per > 2 * kSegPieces ? (per + kSegPieces - 1) / kSegPieces : 1;
        int64_t blocks = (rows * n_seg + 7) / 8;
        if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
        if (width == 16) shard_transpose_rows_kernel<uint4><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        else if (width == 4) shard_transpose_rows_kernel<uint32_t><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        else shard_transpose_rows_kernel<uint8_t><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        return cudaGetLastError();
    }
    const int64_t total = rows * per;
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
    const int sms = sm_count();
    const uintptr_t al = reinterpret_cast<uintptr_t>(p.src) | reinterpret_cast<uintptr_t>(p.dst);
    int width = 1;
    if (p.inner_bytes % 16 == 0 && al % 16 == 0) width = 16;
    else if (p.inner_bytes % 4 == 0 && al % 4 == 0) width = 4;
    const int64_t per = p.inner_bytes / width;
    if (CP_PERMUTE_ROWS && per >= 32) {  // one warp per row (segment), 8 per block
        const int64_t n_seg = per > 2 * kSegPieces ? (per + kSegPieces - 1) / kSegPieces : 1;
        int64_t blocks = (rows * n_seg + 7) / 8;
        if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
        if (width == 16) permute_rows_kernel<uint4><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        else if (width == 4) permute_rows_kernel<uint32_t><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        else permute_rows_kernel<uint8_t><<<(unsigned)blocks, 256, 0, stream>>>(p, n_seg);
        return cudaGetLastError();
    }
    const int64_t c_rank = p.n_ranks > 0 ? p.seq / p.n_ranks : 0;
    const bool groups_aligned = c_rank % 4 == 0 && (p.layout != LAYOUT_ZIGZAG || (c_rank / 2) % 4 == 0);
    const int64_t seg = p.layout == LAYOUT_ZIGZAG ? c_rank / 2 : c_rank;
    if (CP_PERMUTE_ROWS && p.inner_bytes == 4 && seg > 0 && seg % kSpanRows == 0 && al % 16 == 0) {
        const int64_t spans = rows / kSpanRows;
        const int64_t blocks = spans < (int64_t)sms * 16 ? spans : (int64_t)sms * 16;
        if (rows + (int64_t)sms * 16 * kSpanRows <= INT32_MAX)
            permute_words_span_kernel<int32_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
        else
            permute_words_span_kernel<int64_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
        return cudaGetLastError();
    }
    if (CP_PERMUTE_ROWS && p.inner_bytes == 4 && p.seq % 4 == 0 && groups_aligned && al % 16 == 0) {
        const int64_t groups = rows / 4;
        int64_t blocks = (groups + 256 * kWordUnroll - 1) / (256 * kWordUnroll);
        if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
        // group indices reach groups + kWordUnroll * (threads in the grid)
        if (groups + (int64_t)kWordUnroll * blocks * 256 <= INT32_MAX)
            permute_words_kernel<int32_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
        else
            permute_words_kernel<int64_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
        return cudaGetLastError();
    }
    const int64_t total = rows * per;
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    if (width == 16) permute_kernel<uint4><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else if (width == 4) permute_kernel<uint32_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    else permute_kernel<uint8_t><<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace cpattn
