// doc_tables.cu -- per-position document bounds for the document mask.
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section All-Gather 式 CP: with
// several documents packed into one sequence, a query sees only the keys of its own
// document.  The attention kernels need, for a position p, the first position of
// the document that holds p (the forward: keys before it are hidden from the
// query at p) and the first position past that document (the backward: queries
// from there on do not see the key at p).  One parallel pass turns the sorted
// document starts into these two tables, so every lookup in the kernels is one
// load instead of a binary search of dependent global loads.
//
// The starts travel as kernel parameters, up to kDocChunk per launch, so the call
// never copies from pageable host memory (such a copy waits for the stream to
// drain and stalls the caller).  A launch covers the positions of its own chunk's
// documents, [starts[i0], start of the next chunk), and also writes its starts
// into the device array that the FFMA kernels search.
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace cpattn {
namespace {

constexpr int kDocChunk = 2048;

struct DocChunk {
    int count;        // starts in this chunk
    int i0;           // index of the first one among all starts
    int next_start;   // the start after the chunk (INT32_MAX past the last document)
    int pos_lo, pos_hi;  // positions covered: [starts[0], next start or seq_len)
    int starts[kDocChunk];
};

__global__ void __launch_bounds__(256) doc_tables_kernel(const __grid_constant__ DocChunk c, int *starts_dev,
                                                          int *doc_start, int *doc_end)
{
    __shared__ int s[kDocChunk];
    for (int i = threadIdx.x; i < c.count; i += blockDim.x) {
        s[i] = c.starts[i];
        if (blockIdx.x == 0) starts_dev[c.i0 + i] = c.starts[i];
    }
    __syncthreads();
    const int64_t span = (int64_t)c.pos_hi - c.pos_lo;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < span; t += (int64_t)gridDim.x * blockDim.x) {
        const int pos = c.pos_lo + (int)t;
        int lo = 1, hi = c.count;  // first start of the chunk > pos (s[0] <= pos always)
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (s[mid] <= pos) lo = mid + 1; else hi = mid;
        }
        doc_start[pos] = s[lo - 1];
        doc_end[pos] = lo < c.count ? s[lo] : c.next_start;
    }
}

}  // namespace

cudaError_t launch_doc_tables(const int64_t *starts, int n_docs, int64_t seq_len, int *starts_dev, int *doc_start,
                              int *doc_end, cudaStream_t stream)
{
    if (seq_len <= 0 || n_docs < 1) return cudaSuccess;
    if (seq_len > INT32_MAX) return cudaErrorInvalidValue;
    thread_local DocChunk c;
    for (int i0 = 0; i0 < n_docs; i0 += kDocChunk) {
        const int count = n_docs - i0 < kDocChunk ? n_docs - i0 : kDocChunk;
        c.count = count;
        c.i0 = i0;
        for (int i = 0; i < count; ++i) c.starts[i] = (int)starts[i0 + i];
        c.next_start = i0 + count < n_docs ? (int)starts[i0 + count] : INT32_MAX;
        c.pos_lo = c.starts[0];
        c.pos_hi = i0 + count < n_docs ? c.next_start : (int)seq_len;
        int64_t blocks = ((int64_t)c.pos_hi - c.pos_lo + 255) / 256;
        if (blocks < 1) blocks = 1;
        if (blocks > 2048) blocks = 2048;
        doc_tables_kernel<<<(unsigned)blocks, 256, 0, stream>>>(c, starts_dev, doc_start, doc_end);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace cpattn
