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
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace cpattn {
namespace {

__global__ void __launch_bounds__(256) doc_tables_kernel(const int *starts, int n_docs, int64_t seq_len,
                                                          int *doc_start, int *doc_end)
{
    for (int64_t pos = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; pos < seq_len;
         pos += (int64_t)gridDim.x * blockDim.x) {
        int lo = 0, hi = n_docs;  // first start > pos
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if ((int64_t)__ldg(starts + mid) <= pos) lo = mid + 1; else hi = mid;
        }
        doc_start[pos] = lo > 0 ? __ldg(starts + lo - 1) : 0;
        doc_end[pos] = lo < n_docs ? __ldg(starts + lo) : INT32_MAX;
    }
}

}  // namespace

cudaError_t launch_doc_tables(const int *starts, int n_docs, int64_t seq_len, int *doc_start, int *doc_end,
                              cudaStream_t stream)
{
    if (seq_len <= 0) return cudaSuccess;
    int64_t blocks = (seq_len + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    doc_tables_kernel<<<(unsigned)blocks, 256, 0, stream>>>(starts, n_docs, seq_len, doc_start, doc_end);
    return cudaGetLastError();
}

}  // namespace cpattn
