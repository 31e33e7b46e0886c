// merge.cu -- standalone LSE merge, one coalesced HBM pass.
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力: two partials
// (o_1, lse_1), (o_2, lse_2) over disjoint key sets combine into
//   lse = M + log(e^{lse_1 - M} + e^{lse_2 - M}),  M = max(lse_1, lse_2),
//   o   = e^{lse_1 - lse} o_1 + e^{lse_2 - lse} o_2   (the weights sum to 1).
// A side with lse = -inf is empty and contributes nothing; two empty sides give
// (0, -inf).
//
// Work split: a group of d/8 threads owns one (batch, token, head) row; each thread
// moves 8 elements with 16-byte accesses (two float4 of the fp32 accumulator, one
// 16-byte load of bf16 partials or two float4 of fp32 partials).  Rows are visited
// in memory order of the [b, s, H, d] tensors, so consecutive groups touch
// consecutive addresses.  Bytes per row: (8 + sizeof(o_b)) * d + 12.
#include <cuda_runtime.h>
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace cpattn {
namespace {

__device__ __forceinline__ void load8(const void *base, int dtype, int64_t off, float *v)
{
    if (dtype == DT_BF16) {
        const uint4 w = __ldcs(reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(base) + off));
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(u[i] << 16);
            v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(base) + off);
        const float4 a = __ldcs(p), b = __ldcs(p + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

__device__ __forceinline__ void store8(void *base, int dtype, int64_t off, const float *v)
{
    if (dtype == DT_BF16) {
        uint4 w;
        w.x = pack_bf16x2(v[0], v[1]);
        w.y = pack_bf16x2(v[2], v[3]);
        w.z = pack_bf16x2(v[4], v[5]);
        w.w = pack_bf16x2(v[6], v[7]);
        __stcs(reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(base) + off), w);
    } else {
        float4 *p = reinterpret_cast<float4 *>(reinterpret_cast<float *>(base) + off);
        __stcs(p, make_float4(v[0], v[1], v[2], v[3]));
        __stcs(p + 1, make_float4(v[4], v[5], v[6], v[7]));
    }
}

__global__ void __launch_bounds__(256) lse_merge_kernel(const __grid_constant__ MergeParams p)
{
    const int gpr = (int)(p.d / 8);  // threads per row; divides 32, so a row never spans warps
    const int64_t rows = p.b * p.s * p.h;
    const int64_t total = rows * gpr;
    const int lane = threadIdx.x & 31;
    const int64_t warp_id = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    // the loop bound is uniform per warp, so __syncwarp() below sees every lane
    for (int64_t base = warp_id * 32; base < total; base += n_warps * 32) {
        const int64_t idx = base + lane;
        const bool active = idx < total;
        const int64_t r = active ? idx / gpr : 0;
        const int part = (int)(idx - r * gpr);
        const int64_t hh = r % p.h;
        const int64_t ss = (r / p.h) % p.s;
        const int64_t bb = r / (p.h * p.s);
        float *la_ptr = p.lse_acc + bb * p.la_sb + hh * p.la_sh + ss * p.la_ss;
        float lse = -INFINITY;
        if (active) {
            const float la = *la_ptr;
            const float lb = p.lse_b[bb * p.lb_sb + hh * p.lb_sh + ss * p.lb_ss];
            const float M = fmaxf(la, lb);
            float wa = 0.f, wb = 0.f;
            if (M != -INFINITY) {
                lse = M + logf(__expf(la - M) + __expf(lb - M));
                wa = __expf(la - lse);
                wb = __expf(lb - lse);
            }
            const int64_t oa_off = bb * p.oa_sb + ss * p.oa_ss + hh * p.oa_sh + part * 8;
            const int64_t ob_off = bb * p.ob_sb + ss * p.ob_ss + hh * p.ob_sh + part * 8;
            float a[8], b[8], o[8];
            load8(p.o_acc, DT_FP32, oa_off, a);
            load8(p.o_b, p.ob_dtype, ob_off, b);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                // an empty side may hold anything; select instead of multiplying by 0
                const float ta = (la == -INFINITY) ? 0.f : wa * a[i];
                const float tb = (lb == -INFINITY) ? 0.f : wb * b[i];
                o[i] = ta + tb;
            }
            if (p.o_out)
                store8(p.o_out, p.out_dtype, bb * p.out_sb + ss * p.out_ss + hh * p.out_sh + part * 8, o);
            else
                store8(p.o_acc, DT_FP32, oa_off, o);
        }
        __syncwarp();  // every lane of the row has read lse_acc before it is replaced
        if (active && part == 0) *la_ptr = lse;
    }
}

}  // namespace

cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream)
{
    const int64_t total = p.b * p.s * p.h * (p.d / 8);
    if (total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = (int64_t)sms * 8;  // 8 resident 256-thread blocks per SM
    if (blocks > cap) blocks = cap;
    lse_merge_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace cpattn
