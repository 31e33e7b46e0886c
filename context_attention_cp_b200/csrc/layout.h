// layout.h -- token-layout ranges and tile classification, shared by the host
// ABI code and the device kernels of libcpattn.
//
// "上下文并行与 Ring Attention" (hs-black.github.io):
//   section Ring Attention   : at step r rank i holds the K/V of rank (i - r) mod N;
//   section 因果掩码带来的负载不均 : contiguous split, causal mask pos_k <= pos_q;
//   section Zig-zag          : 2N chunks of c/2, rank i holds C_i then C_{2N-1-i};
//   section Striped          : token p lives on rank p mod N;
//   section 重排 token 的代价   : the mask is judged on original positions.
//
// All three layouts give positions that increase with the local index (for
// zig-zag, every position of C_{2N-1-i} exceeds every position of C_i), and the
// ABI requires the same of user ranges.  With increasing positions the key tiles
// of one (query tile, key block) pair split into a prefix of FULL tiles, then
// PARTIAL tiles, then SKIP tiles; kv_tile_bounds() returns the two cut points.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define CP_HD __host__ __device__ __forceinline__
#else
#define CP_HD inline
#endif

namespace cpattn {

enum { LAYOUT_CONTIGUOUS = 0, LAYOUT_ZIGZAG = 1, LAYOUT_STRIPED = 2 };
enum { TILE_SKIP = 0, TILE_FULL = 1, TILE_PARTIAL = 2 };

// Position map of one rank's (or one block's) local tokens.  The host uses 64-bit
// fields; the kernels use the 32-bit form (positions stay below 2^30, which the
// ABI checks).
template <typename I>
struct RangeT {
    I start0, start1;  // first position of segment 0 / 1
    I len0, len1;      // tokens in segment 0 / 1 (len1 = 0 for one segment)
    I stride;          // position step between neighbouring local tokens
};
using Range = RangeT<int64_t>;
using Range32 = RangeT<int32_t>;

template <typename I>
CP_HD I range_pos(const RangeT<I> &r, I t)
{
    return t < r.len0 ? r.start0 + t * r.stride : r.start1 + (t - r.len0) * r.stride;
}

CP_HD int64_t range_pos(const Range &r, int64_t t)
{
    return t < r.len0 ? r.start0 + t * r.stride : r.start1 + (t - r.len0) * r.stride;
}

CP_HD Range32 to_range32(const Range &r)
{
    return Range32{(int32_t)r.start0, (int32_t)r.start1, (int32_t)r.len0, (int32_t)r.len1, (int32_t)r.stride};
}

CP_HD int64_t range_len(const Range &r) { return r.len0 + r.len1; }

// True if positions strictly increase with the local index.
CP_HD bool range_increasing(const Range &r)
{
    if (r.stride < 1 || r.len0 < 0 || r.len1 < 0) return false;
    if (r.len1 == 0 || r.len0 == 0) return true;
    return r.start1 > r.start0 + (r.len0 - 1) * r.stride;
}

// Range of rank `rank` in a sequence of S tokens split over N ranks.
template <typename I>
CP_HD RangeT<I> layout_range_t(int layout, int N, I S, int rank)
{
    RangeT<I> r;
    I c = S / N;
    r.start1 = 0;
    r.len1 = 0;
    r.stride = 1;
    if (layout == LAYOUT_ZIGZAG) {
        I h = c / 2;
        r.start0 = rank * h;
        r.len0 = h;
        r.start1 = (I)(2 * N - 1 - rank) * h;
        r.len1 = h;
    } else if (layout == LAYOUT_STRIPED) {
        r.start0 = rank;
        r.len0 = c;
        r.stride = N;
    } else {
        r.start0 = rank * c;
        r.len0 = c;
    }
    return r;
}

CP_HD Range layout_range(int layout, int N, int64_t S, int rank) { return layout_range_t<int64_t>(layout, N, S, rank); }

// Row of original position pos in a zig-zag rank-major sequence (chunks of h
// positions, N ranks of 2h rows): rank i holds chunk i, then chunk 2N - 1 - i.
template <typename I>
CP_HD I zigzag_row(I pos, I h, int N)
{
    const I ch = pos / h;
    return ch < (I)N ? ch * 2 * h + (pos - ch * h) : ((I)(2 * N - 1) - ch) * 2 * h + h + (pos - ch * h);
}

// For query tile [q_lo, q_lo + tile_q) of a block of q_len rows (ranges q) against a
// key block of kv_len rows (ranges k) cut into tiles of tile_k: key tiles
// [0, *kt_full) are FULL, [*kt_full, *kt_end) PARTIAL, [*kt_end, n_kt) SKIP.
template <typename I>
CP_HD void kv_tile_bounds(const RangeT<I> &q, I q_len, I q_lo, int tile_q, const RangeT<I> &k, I kv_len, int tile_k,
                          bool causal, int *kt_full, int *kt_end)
{
    int n_kt = (int)((kv_len + tile_k - 1) / tile_k);
    bool ragged = (kv_len % tile_k) != 0;
    if (!causal) {
        *kt_end = n_kt;
        *kt_full = ragged ? n_kt - 1 : n_kt;
        return;
    }
    I q_hi = q_lo + tile_q - 1;
    if (q_hi > q_len - 1) q_hi = q_len - 1;
    const I qmin = range_pos(q, q_lo), qmax = range_pos(q, q_hi);
    // kt_end: number of tiles whose first key is visible to the last query row.
    int lo = 0, hi = n_kt;  // answer in [lo, hi]
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (range_pos(k, (I)mid * tile_k) <= qmax) lo = mid + 1; else hi = mid;
    }
    *kt_end = lo;
    // kt_full: number of leading tiles that are whole (inside kv_len) and whose last
    // key is visible to the first query row.
    lo = 0;
    hi = ragged ? n_kt - 1 : n_kt;
    if (hi > *kt_end) hi = *kt_end;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (range_pos(k, (I)mid * tile_k + tile_k - 1) <= qmin) lo = mid + 1; else hi = mid;
    }
    *kt_full = lo;
}

}  // namespace cpattn
