// mma_rate.cu -- rate of the tensor pipe on the forward kernel's product shapes.
//
// A standalone diagnostic program (not part of libcpattn).  One CTA per SM, operands
// zero-filled in shared memory (128-byte-swizzled K-major tiles, the layout the
// attention kernels' TMA loads produce), 512 TMEM columns; one thread issues R
// products back to back and commits, and clock64 around the issue and the commit's
// completion gives cycles per product.  Modes: SS products at N = 128, 256 and 64;
// a TS product (A from TMEM, the PV form); the forward kernel's mix (S0, S1 SS, PV0,
// PV1 TS); the mix with other warps storing to shared memory at ~32 B per clock; S
// and PV with two warpgroups loading and storing TMEM (paced, and flat out); the mix
// with PV as an SS product; and that with ~64 B per clock of shared-memory stores.
// Every wait is bounded.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o mma_rate \
//        context_attention_cp_b200/csrc/probes/mma_rate.cu -lcuda && ./mma_rate
#include <cstdio>
#include <vector>
#include <algorithm>
#include <cuda_runtime.h>
#include "../ptx.cuh"
using namespace cpattn;

constexpr int SMEM = 192 * 1024 + 1024;

__global__ void __launch_bounds__(384) probe(int mode, int R, long long *out, int *err)
{
    extern __shared__ __align__(1024) unsigned char raw[];
    const uint32_t base0 = smem_u32(raw);
    const uint32_t base = (base0 + 1023u) & ~1023u;
    unsigned char *sp = raw + (base - base0);
    __shared__ uint64_t barmem;
    __shared__ uint32_t tslot;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < 192 * 1024 / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sp)[i] = make_uint4(0, 0, 0, 0);
    const uint32_t bar = smem_u32(&barmem);
    if (threadIdx.x == 0) { mbar_init(bar, 1); mbar_fence_init(); }
    if (warp == 0) tmem_alloc(smem_u32(&tslot), 512);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tslot;
    const uint32_t A0 = base, A1 = base + 32768, B = base + 65536, V = base + 131072;
    long long t0 = 0, t1 = 0;
    if (warp == 0 && lane == 0) {
        const uint32_t i128 = idesc_bf16_f32(128, 128, false), i256 = idesc_bf16_f32(128, 256, false),
                       i64 = idesc_bf16_f32(128, 64, false), ipv = idesc_bf16_f32(128, 128, true);
        auto ss = [&](uint32_t d, uint32_t a, uint32_t b, int nrows, uint32_t id) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t oa = (k >> 2) * 16384 + (k & 3) * 32, ob = (k >> 2) * (nrows * 128) + (k & 3) * 32;
                mma_ss(d, smem_desc_sw128(a + oa, 16, 1024), smem_desc_sw128(b + ob, 16, 1024), id, k > 0);
            }
        };
        auto ts = [&](uint32_t d, uint32_t a_t) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_ts(d, a_t + k * 8, smem_desc_sw128(V + k * 2048, 16384, 1024), ipv, 1u);
        };
        auto ssv = [&](uint32_t d, uint32_t a) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t oa = (k >> 2) * 16384 + (k & 3) * 32;
                mma_ss(d, smem_desc_sw128(a + oa, 16, 1024), smem_desc_sw128(V + k * 2048, 16384, 1024), ipv, 1u);
            }
        };
        t0 = clock64();
        for (int r = 0; r < R; ++r) {
            if (mode == 0) ss(tb, A0, B, 128, i128);
            else if (mode == 1) ss(tb, A0, B, 256, i256);
            else if (mode == 2) ts(tb + 256, tb);
            else if (mode == 3) ss(tb, A0, B, 64, i64);
            else if (mode >= 8) {  // S0, S1 (SS), PV0, PV1 as SS (P from shared memory)
                ss(tb, A0, B, 128, i128);
                ss(tb + 128, A1, B, 128, i128);
                ssv(tb + 256, A0);
                ssv(tb + 384, A1);
            }
            else if (mode >= 6) {  // S (SS) into [0,128), PV (TS, P from [256,320)) into [128,256)
                ss(tb, A0, B, 128, i128);
                ts(tb + 128, tb + 256);
                ss(tb, A1, B, 128, i128);
                ts(tb + 128, tb + 256);
            }
            else {  // the forward's mix: S0, S1 (SS), PV0, PV1 (TS)
                ss(tb, A0, B, 128, i128);
                ss(tb + 128, A1, B, 128, i128);
                ts(tb + 256, tb);
                ts(tb + 384, tb + 128);
            }
        }
        tc_commit(bar);
        long long spins = 0;
        while (!mbar_try_wait(bar, 0)) {
            if (++spins > (1ll << 26)) { atomicOr(err, 1); break; }
        }
        t1 = clock64();
        out[blockIdx.x] = t1 - t0;
    } else if (mode == 5 && warp >= 1 && warp <= 3) {
        // shared-memory writes beside the products at ~32 B/clk (the K/V tile loads' rate)
        const int iters = R * 43;
        uint4 *scr = reinterpret_cast<uint4 *>(sp + 160 * 1024);
        for (int it = 0; it < iters; ++it) {
            scr[((it * 96) + threadIdx.x - 32) & 2047] = make_uint4(it, it, it, it);
            const long long c0 = clock64();
            while (clock64() - c0 < 40) {}
        }
    }
    else if (mode == 9 && warp >= 1) {
        // 11 warps write 64 KB per 32 products (P tiles and K/V tiles: ~32 + 32 B/clk)
        const int iters = R * 22;
        uint4 *scr = reinterpret_cast<uint4 *>(sp + 160 * 1024);
        for (int it = 0; it < iters; ++it) {
            scr[((it * 352) + threadIdx.x - 32) & 2047] = make_uint4(it, it, it, it);
            const long long c0 = clock64();
            while (clock64() - c0 < 70) {}
        }
    }
    else if (mode >= 6 && mode < 8 && warp >= 4) {
        // two "softmax" warpgroups: load 128 score columns ([320, 448)), store 64 P
        // columns ([448, 512)), then idle (mode 6: ~1500 cycles, mode 7: none)
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const int iters = mode == 6 ? R / 2 : R * 2;
        float acc = 0.f;
        for (int it = 0; it < iters; ++it) {
            float v[128];
            tmem_ld64f(tb + lane_base + 320, v);
            tmem_ld64f(tb + lane_base + 384, v + 64);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = __float_as_uint(v[i] + v[i + 64] + v[i + 32] + v[i + 96]);
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_st16(tb + lane_base + 448 + 16 * q, pk);
            tmem_wait_st();
            acc += v[7];
            if (mode == 6) {
                const long long c0 = clock64();
                while (clock64() - c0 < 1500) {}
            }
        }
        if (acc == 12345.f) out[0] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) { tmem_relinquish(); tmem_dealloc(tb, 512); }
}

int main()
{
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    long long *out; int *err;
    cudaMalloc(&out, sms * sizeof(long long));
    cudaMalloc(&err, sizeof(int));
    cudaMemset(err, 0, sizeof(int));
    const char *names[] = {"SS M128 N128 K16", "SS M128 N256 K16", "TS M128 N128 K16 (PV)", "SS M128 N64 K16",
                           "mix S0 S1 PV0 PV1", "mix + smem writes 32B/clk",
                           "S/PV + tmem ld/st (throttled)", "S/PV + tmem ld/st (flat out)",
                           "S0 S1 PV0 PV1 all SS", "all SS + smem writes 64B/clk"};
    const int per[] = {8, 8, 8, 8, 32, 32, 32, 32, 32, 32};
    for (int mode = 0; mode < 10; ++mode) {
        const int R = mode >= 4 ? 64 : 256;
        for (int rep = 0; rep < 2; ++rep) {
            probe<<<sms, 384, SMEM>>>(mode, R, out, err);
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
        }
        std::vector<long long> h(sms);
        cudaMemcpy(h.data(), out, sms * sizeof(long long), cudaMemcpyDeviceToHost);
        std::sort(h.begin(), h.end());
        const double n = (double)R * per[mode];
        printf("%-28s cycles per mma: median %.1f  min %.1f  max %.1f\n", names[mode], h[sms / 2] / n, h[0] / n,
               h[sms - 1] / n);
    }
    int he = 0;
    cudaMemcpy(&he, err, sizeof(int), cudaMemcpyDeviceToHost);
    printf("err %d\n", he);
    return 0;
}
