// merge.cu -- standalone LSE merge, one coalesced HBM pass.
//
// "上下文并行与 Ring Attention" (hs-black.github.io), section 分块注意力: two partials
// (o_1, lse_1), (o_2, lse_2) over disjoint key sets combine into
//   lse = M + log(e^{lse_1 - M} + e^{lse_2 - M}),  M = max(lse_1, lse_2),
//   o   = e^{lse_1 - lse} o_1 + e^{lse_2 - lse} o_2   (the weights sum to 1).
// A side with lse = -inf is empty and contributes nothing; two empty sides give
// (0, -inf).
//
// Work split: one CTA per (batch, 8 consecutive positions); the LSE weights of
// its (head, position) pairs are computed once into shared memory, then d/8
// threads per (position, head) row move 8 elements each with 16-byte streaming
// accesses (two float4 of the fp32 accumulator, one 16-byte load of bf16 partials
// or two float4 of fp32 partials), consecutive threads on consecutive addresses.
// Bytes per row: (8 + sizeof(o_b)) * d + 12.
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

#ifndef CP_MERGE_THREADS
#define CP_MERGE_THREADS 256
#endif
constexpr int MT = CP_MERGE_THREADS;  // threads per CTA
#ifndef CP_MERGE_TS
#define CP_MERGE_TS 8
#endif
#ifndef CP_MERGE_U
#define CP_MERGE_U 2
#endif
#ifndef CP_MERGE_CTAS_PER_SM
#define CP_MERGE_CTAS_PER_SM 4
#endif
constexpr int TS = CP_MERGE_TS;  // sequence positions per work item

// One CTA merges TS consecutive positions of one batch row, all heads.
//   Phase 1: the LSE weights w_acc = e^{lse_acc - lse}, w_b = e^{lse_b - lse} and the
//   new lse of every (head, position) go to shared memory (lse reads are coalesced
//   along the sequence).  Phase 2: the o rows stream through with 16-byte accesses,
//   thread t owning elements [8 (t % (D/8)), +8) of head h0 + t / (D/8).
template <int D>
__global__ void __launch_bounds__(MT, CP_MERGE_CTAS_PER_SM) lse_merge_kernel(const __grid_constant__ MergeParams p)
{
    extern __shared__ float wsm[];  // [2][H][TS]
    const int H = (int)p.h;
    float *wa_s = wsm;
    float *wb_s = wsm + H * TS;
    const int tid = threadIdx.x;
    const int64_t tiles_per_b = (p.s + TS - 1) / TS;
    const int64_t n_work = tiles_per_b * p.b;
    // persistent: the grid strides over (batch, position tile) work items
    for (int64_t wk = blockIdx.x; wk < n_work; wk += gridDim.x) {
    const int64_t bb = wk / tiles_per_b;
    const int64_t s0 = (wk - bb * tiles_per_b) * TS;
    const int ns = (int)min((int64_t)TS, p.s - s0);

    for (int i = tid; i < H * TS; i += MT) {
        const int hh = i / TS, t = i % TS;
        if (t >= ns) continue;
        float *la_ptr = p.lse_acc + bb * p.la_sb + hh * p.la_sh + (s0 + t) * p.la_ss;
        const float la = *la_ptr;
        const float lb = p.lse_b[bb * p.lb_sb + hh * p.lb_sh + (s0 + t) * p.lb_ss];
        const float M = fmaxf(la, lb);
        float wa = 0.f, wb = 0.f, lse = -INFINITY;
        if (M != -INFINITY) {
            lse = M + logf(__expf(la - M) + __expf(lb - M));
            // an empty side may hold anything in o: its weight is exactly 0
            wa = (la == -INFINITY) ? 0.f : __expf(la - lse);
            wb = (lb == -INFINITY) ? 0.f : __expf(lb - lse);
        }
        wa_s[i] = wa;
        wb_s[i] = wb;
        *la_ptr = lse;
    }
    __syncthreads();

    constexpr int TPR = D / 8;     // threads per (position, head) row
    constexpr int HPB = MT / TPR;  // heads per pass
    constexpr int U = CP_MERGE_U;  // rows in flight per thread
    const int part = tid % TPR;
    const int hl = tid / TPR;
    const int passes = (H + HPB - 1) / HPB;
    const int items = ns * passes;  // (position, head pass) pairs
    for (int it0 = 0; it0 < items; it0 += U) {
        float a[U][8], bv[U][8];
        float wa[U], wb[U];
        int64_t oa_off[U], out_off[U];
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int it = it0 + u;
            const int t = it / passes;
            const int hh = (it - t * passes) * HPB + hl;
            ok[u] = it < items && hh < H;
            const int64_t ss = s0 + t;
            wa[u] = ok[u] ? wa_s[hh * TS + t] : 0.f;
            wb[u] = ok[u] ? wb_s[hh * TS + t] : 0.f;
            oa_off[u] = bb * p.oa_sb + ss * p.oa_ss + (int64_t)hh * p.oa_sh + part * 8;
            out_off[u] = p.o_out ? bb * p.out_sb + ss * p.out_ss + (int64_t)hh * p.out_sh + part * 8 : oa_off[u];
            if (ok[u]) {
                load8(p.o_b, p.ob_dtype, bb * p.ob_sb + ss * p.ob_ss + (int64_t)hh * p.ob_sh + part * 8, bv[u]);
                if (wa[u] != 0.f) load8(p.o_acc, DT_FP32, oa_off[u], a[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (!ok[u]) continue;
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float ta = (wa[u] != 0.f) ? wa[u] * a[u][i] : 0.f;
                const float tb = (wb[u] != 0.f) ? wb[u] * bv[u][i] : 0.f;
                o[i] = ta + tb;
            }
            if (p.o_out) store8(p.o_out, p.out_dtype, out_off[u], o);
            else store8(p.o_acc, DT_FP32, out_off[u], o);
        }
    }
    __syncthreads();  // the weights of this item are consumed before the next item's
    }
}

}  // namespace

cudaError_t launch_lse_merge(const MergeParams &p, cudaStream_t stream)
{
    if (p.b * p.s * p.h == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n_work = (p.s + TS - 1) / TS * p.b;
    const int64_t cap = (int64_t)sms * CP_MERGE_CTAS_PER_SM;
    const unsigned grid = (unsigned)(n_work < cap ? n_work : cap);
    const size_t smem = 2 * (size_t)p.h * TS * sizeof(float);
    if (smem > 48 * 1024) return cudaErrorInvalidValue;
    switch (p.d) {
    case 8: lse_merge_kernel<8><<<grid, MT, smem, stream>>>(p); break;
    case 16: lse_merge_kernel<16><<<grid, MT, smem, stream>>>(p); break;
    case 32: lse_merge_kernel<32><<<grid, MT, smem, stream>>>(p); break;
    case 64: lse_merge_kernel<64><<<grid, MT, smem, stream>>>(p); break;
    case 128: lse_merge_kernel<128><<<grid, MT, smem, stream>>>(p); break;
    case 256: lse_merge_kernel<256><<<grid, MT, smem, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace cpattn
