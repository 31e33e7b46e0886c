// abi.cu -- the C ABI of libcpattn (include/cpattn.h): argument checks, the ring
// scheduler (work order and step launches) and dispatch to the kernels.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/cpattn.h"
#include "bwd.h"
#include "kernels.h"
#include "ulysses.h"

using namespace cpattn;

// The backward's grid is head-major (the CTAs resident at one time share a few heads'
// Q, dO and dQ rows in L2) once one head's work items fill a wave of the device;
// CP_BWD_HEAD_MAJOR=1 makes it always head-major, -1 never.
#ifndef CP_BWD_HEAD_MAJOR
#define CP_BWD_HEAD_MAJOR 0
#endif
constexpr bool kBwdHeadMajor = CP_BWD_HEAD_MAJOR > 0;
constexpr bool kBwdNeverHeadMajor = CP_BWD_HEAD_MAJOR < 0;

// Head-major backward: the resident CTAs of one kv head reduce into its group's dQ
// rows.  When those rows (group x rows x d fp32) fit in L2, the CTAs start their ring
// steps at rotated offsets (spread over every query rank); otherwise every CTA walks
// the steps in order from a rotated query tile, which keeps one or two query ranks'
// rows in L2 at a time.  CP_BWD_TILE_ROTATION: -1 decides by that rule, 0 (the
// default: the rule's choice measured no faster on the 70B 128K workload) always
// rotates the ring steps, 1 always rotates the query tiles.
#ifndef CP_BWD_TILE_ROTATION
#define CP_BWD_TILE_ROTATION 0
#endif
static bool bwd_tile_rotation(int64_t group, int64_t rows, int64_t d, int dev)
{
    if (CP_BWD_TILE_ROTATION >= 0) return CP_BWD_TILE_ROTATION != 0;
    int l2 = 0;
    if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0) l2 = 126 << 20;
    return group * rows * d * 4 > (int64_t)l2;
}

namespace {

// NVTX range for profilers (a no-op unless a tool is attached): the entry points and,
// in the stepwise ring modes, every ring step.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    NvtxRange(const char *fmt, int a, int b)
    {
        char buf[64];
        snprintf(buf, sizeof buf, fmt, a, b);
        nvtxRangePushA(buf);
    }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

thread_local char g_last_error[512] = "";

cp_status fail(cp_status s, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

cp_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(CP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int64_t elem_size(int32_t dt) { return dt == CP_BF16 ? 2 : (dt == CP_FP32 ? 4 : 0); }

cp_status check_tensor(const cp_tensor *t, const char *name, bool need_data = true)
{
    if (!t) return fail(CP_ERR_INVALID_ARG, "%s is NULL", name);
    if (need_data && !t->data) return fail(CP_ERR_INVALID_ARG, "%s->data is NULL", name);
    if (t->dtype != CP_BF16 && t->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "%s has an unknown dtype", name);
    for (int i = 0; i < 4; ++i)
        if (t->shape[i] < 0 || t->stride[i] < 0) return fail(CP_ERR_INVALID_ARG, "%s has a negative size or stride", name);
    if (t->stride[3] != 1 && t->shape[3] > 1) return fail(CP_ERR_INVALID_ARG, "%s: innermost stride must be 1", name);
    return CP_OK;
}

// A token tensor [b, s, H, d] whose rows start on 16-byte boundaries.
cp_status check_rows16(const cp_tensor *t, const char *name)
{
    const int64_t es = elem_size(t->dtype);
    const int64_t per16 = 16 / es;
    if (reinterpret_cast<uintptr_t>(t->data) % 16)
        return fail(CP_ERR_INVALID_ARG, "%s->data must be 16-byte aligned", name);
    for (int i = 0; i < 3; ++i)
        if (t->shape[i] > 1 && t->stride[i] % per16)
            return fail(CP_ERR_INVALID_ARG, "%s: stride[%d] must be a multiple of 16 bytes", name, i);
    if ((t->shape[3] * es) % 16) return fail(CP_ERR_INVALID_ARG, "%s: rows must be a multiple of 16 bytes", name);
    return CP_OK;
}

bool same_shape(const cp_tensor *a, const cp_tensor *b)
{
    for (int i = 0; i < 4; ++i)
        if (a->shape[i] != b->shape[i]) return false;
    return true;
}

Range to_range(const cp_range &r)
{
    Range x;
    x.start0 = r.start[0];
    x.len0 = r.len[0];
    x.start1 = r.nseg == 2 ? r.start[1] : 0;
    x.len1 = r.nseg == 2 ? r.len[1] : 0;
    x.stride = r.stride;
    return x;
}

cp_status check_range(const cp_range *r, int64_t len, const char *name)
{
    if (!r) return fail(CP_ERR_INVALID_ARG, "%s is NULL", name);
    if (r->nseg != 1 && r->nseg != 2) return fail(CP_ERR_INVALID_ARG, "%s: nseg must be 1 or 2", name);
    Range x = to_range(*r);
    if (range_len(x) != len) return fail(CP_ERR_SHAPE, "%s covers %lld tokens, the tensor has %lld", name,
                                         (long long)range_len(x), (long long)len);
    if (!range_increasing(x) || x.start0 < 0)
        return fail(CP_ERR_INVALID_ARG, "%s: positions must be >= 0 and increase with the local index", name);
    const int64_t last = len > 0 ? range_pos(x, len - 1) : 0;
    if (last >= ((int64_t)1 << 30))
        return fail(CP_ERR_UNSUPPORTED, "%s: positions must stay below 2^30", name);
    return CP_OK;
}

// The softmax scale: 0 asks for the standard 1 / sqrt(d) ("上下文并行与 Ring
// Attention", section 分块注意力: x_j = q . k_j / sqrt(d_h)); any other value must be
// finite and > 0 and is taken as given.
cp_status resolve_scale(float *scale, int64_t d)
{
    if (*scale == 0.f) {
        if (d <= 0) return fail(CP_ERR_SHAPE, "head dim must be > 0");
        *scale = (float)(1.0 / std::sqrt((double)d));
        return CP_OK;
    }
    if (!(*scale > 0.f) || !std::isfinite(*scale))
        return fail(CP_ERR_INVALID_ARG, "softmax_scale must be 0 (1/sqrt(d)) or finite and > 0");
    return CP_OK;
}

void set_status_ptr(AttnParams &p)
{
    int *s = nullptr;
    status_word(&s);
    p.status = s;
}

void fill_inputs(AttnParams &p, const cp_tensor *q, const cp_tensor *k, const cp_tensor *v)
{
    p.q = q->data; p.k = k->data; p.v = v->data;
    p.q_sb = q->stride[0]; p.q_ss = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = k->stride[0]; p.k_ss = k->stride[1]; p.k_sh = k->stride[2];
    p.v_sb = v->stride[0]; p.v_ss = v->stride[1]; p.v_sh = v->stride[2];
}

void fill_outputs(AttnParams &p, int epi, const cp_tensor *o, const cp_tensor *lse)
{
    p.epi = epi;
    p.o = o->data;
    p.o_dtype = o->dtype;
    p.o_sb = o->stride[0]; p.o_ss = o->stride[1]; p.o_sh = o->stride[2];
    p.lse = static_cast<float *>(lse->data);
    p.lse_sb = lse->stride[0]; p.lse_sh = lse->stride[1]; p.lse_ss = lse->stride[2];
}

cp_status launch_attn(const AttnParams &p, int32_t dtype, cudaStream_t stream)
{
    cudaError_t e = dtype == CP_BF16 ? launch_attn_tc(p, stream) : launch_attn_simt(p, stream);
    if (e != cudaSuccess) return cuda_fail(e, "attention launch");
    return CP_OK;
}

// ---------------------------------------------------------------- ring scheduler

// Work order for the ring: (rank, row group) entries sorted by the number of key
// tiles their 128-row query tiles visit over all steps, heaviest first, so the long
// causal rows start early and the tail of the launch is made of short ones.
struct OrderKey {
    int layout, n, causal, rows;
    int64_t seq;
    bool operator<(const OrderKey &o) const
    {
        return std::tie(layout, n, causal, rows, seq) < std::tie(o.layout, o.n, o.causal, o.rows, o.seq);
    }
};
std::mutex g_order_mu;
std::map<OrderKey, std::vector<uint32_t>> g_order_cache;

// The caches keep at most this many shapes each; a new shape beyond that empties
// the cache first (orders are copied out under the lock, so nothing refers into it).
constexpr size_t kOrderCacheMax = 64;

const std::vector<uint32_t> &ring_order_locked(int layout, int N, int64_t S, int causal, int rows_per_cta)
{
    OrderKey key{layout, N, causal, rows_per_cta, S};
    auto it = g_order_cache.find(key);
    if (it != g_order_cache.end()) return it->second;
    if (g_order_cache.size() >= kOrderCacheMax) g_order_cache.clear();
    const int64_t c = S / N;
    const int n_groups = (int)((c + rows_per_cta - 1) / rows_per_cta);
    std::vector<std::pair<int64_t, uint32_t>> work;
    work.reserve((size_t)N * n_groups);
    for (int i = 0; i < N; ++i) {
        Range qr = layout_range(layout, N, S, i);
        for (int g = 0; g < n_groups; ++g) {
            int64_t tiles = 0;
            for (int64_t q_lo = (int64_t)g * rows_per_cta; q_lo < std::min<int64_t>(c, (int64_t)(g + 1) * rows_per_cta);
                 q_lo += 128) {
                for (int r = 0; r < N; ++r) {
                    Range kr = layout_range(layout, N, S, ((i - r) % N + N) % N);
                    int kf, ke;
                    kv_tile_bounds(qr, c, q_lo, 128, kr, c, 128, causal != 0, &kf, &ke);
                    tiles += ke;
                }
            }
            work.push_back({tiles, ((uint32_t)i << 16) | (uint32_t)g});
        }
    }
    std::stable_sort(work.begin(), work.end(),
                     [](const std::pair<int64_t, uint32_t> &a, const std::pair<int64_t, uint32_t> &b) {
                         return a.first > b.first;
                     });
    std::vector<uint32_t> out;
    for (auto &w : work) out.push_back(w.second);
    return g_order_cache.emplace(key, std::move(out)).first->second;
}

int rows_per_cta(int32_t dtype, bool doc = false) { return dtype == CP_BF16 ? attn_tc_rows_per_cta(doc) : 128; }

// Work order of the backward: (key rank, key tile) entries sorted by the number of
// query tiles that see the key tile over all steps, heaviest first.
std::map<std::tuple<int, int, int, int64_t>, std::vector<uint32_t>> g_bwd_order_cache;

const std::vector<uint32_t> &bwd_order_locked(int layout, int N, int64_t S, int causal)
{
    const auto key = std::make_tuple(layout, N, causal, S);
    auto it = g_bwd_order_cache.find(key);
    if (it != g_bwd_order_cache.end()) return it->second;
    if (g_bwd_order_cache.size() >= kOrderCacheMax) g_bwd_order_cache.clear();
    const int64_t c = S / N;
    const int n_kt = (int)((c + kBwdKeyTile - 1) / kBwdKeyTile);
    const int n_qt = (int)((c + kBwdQueryTile - 1) / kBwdQueryTile);
    std::vector<std::pair<int64_t, uint32_t>> work;
    work.reserve((size_t)N * n_kt);
    for (int jr = 0; jr < N; ++jr) {
        Range kr = layout_range(layout, N, S, jr);
        for (int kt = 0; kt < n_kt; ++kt) {
            int64_t tiles = 0;
            for (int r = 0; r < N; ++r) {
                Range qr = layout_range(layout, N, S, (jr + r) % N);
                int qb, qf;
                q_tile_bounds<int64_t>(qr, c, kBwdQueryTile, kr, c, (int64_t)kt * kBwdKeyTile, kBwdKeyTile,
                                       causal != 0, &qb, &qf);
                tiles += n_qt - qb;
            }
            work.push_back({tiles, ((uint32_t)jr << 16) | (uint32_t)kt});
        }
    }
    std::stable_sort(work.begin(), work.end(),
                     [](const std::pair<int64_t, uint32_t> &a, const std::pair<int64_t, uint32_t> &b) {
                         return a.first > b.first;
                     });
    std::vector<uint32_t> out;
    for (auto &w : work) out.push_back(w.second);
    return g_bwd_order_cache.emplace(key, std::move(out)).first->second;
}

// Copies the work order into p.order (natural order, order_len = 0, when it does
// not fit the table), holding the cache lock throughout.
void set_ring_order(AttnParams &p, int layout, int N, int64_t S, int causal, int rows_per_cta)
{
    std::lock_guard<std::mutex> lk(g_order_mu);
    const std::vector<uint32_t> &ord = ring_order_locked(layout, N, S, causal, rows_per_cta);
    p.order_len = 0;
    if ((int64_t)ord.size() <= kMaxOrder) {
        p.order_len = (int)ord.size();
        std::copy(ord.begin(), ord.end(), p.order);
    }
}

template <typename P>
void set_bwd_order(P &p, int layout, int N, int64_t S, int causal)
{
    std::lock_guard<std::mutex> lk(g_order_mu);
    const std::vector<uint32_t> &ord = bwd_order_locked(layout, N, S, causal);
    p.order_len = 0;
    if ((int64_t)ord.size() <= kMaxOrder) {
        p.order_len = (int)ord.size();
        std::copy(ord.begin(), ord.end(), p.order);
    }
}

// Workspace regions of the backward: statistics [b][Hq][N][lpad] float2, then the
// fp32 dQ accumulator [b, S, Hq, d]; each 256-byte aligned.
struct BwdWorkspace {
    int64_t lpad, stats_bytes, acc_bytes;
};
BwdWorkspace bwd_workspace(int32_t N, int64_t b, int64_t S, int64_t Hq, int64_t d)
{
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    BwdWorkspace w;
    const int64_t c = S / N;
    w.lpad = (c + kBwdQueryTile - 1) / kBwdQueryTile * kBwdQueryTile;
    w.stats_bytes = up(b * Hq * N * w.lpad * 8);
    w.acc_bytes = up(b * S * Hq * d * 4);
    return w;
}

cp_status check_attn_dtypes(const cp_tensor *q, const cp_tensor *k, const cp_tensor *v)
{
    if (k->dtype != q->dtype || v->dtype != q->dtype)
        return fail(CP_ERR_INVALID_ARG, "q, k and v must share one dtype");
    const int64_t d = q->shape[3];
    if (d != 64 && d != 128) return fail(CP_ERR_UNSUPPORTED, "head dim %lld is not supported (64 or 128)", (long long)d);
    if (k->shape[3] != d || v->shape[3] != d) return fail(CP_ERR_SHAPE, "q, k, v head dims differ");
    if (q->shape[0] != k->shape[0] || !same_shape(k, v)) return fail(CP_ERR_SHAPE, "q/k/v batch or k/v shapes differ");
    if (q->shape[2] <= 0 || k->shape[2] <= 0 || q->shape[2] % k->shape[2])
        return fail(CP_ERR_SHAPE, "query heads (%lld) must be a multiple of kv heads (%lld)", (long long)q->shape[2],
                    (long long)k->shape[2]);
    if (q->dtype == CP_BF16) {
        cp_status s;
        if ((s = check_rows16(q, "q")) != CP_OK || (s = check_rows16(k, "k")) != CP_OK ||
            (s = check_rows16(v, "v")) != CP_OK)
            return s;
    }
    return CP_OK;
}

cp_status check_out(const cp_tensor *o, const cp_tensor *lse, const cp_tensor *q, int64_t rows, bool need_fp32)
{
    cp_status s;
    if ((s = check_tensor(o, "o")) != CP_OK || (s = check_tensor(lse, "lse")) != CP_OK) return s;
    if (o->shape[0] != q->shape[0] || o->shape[1] != rows || o->shape[2] != q->shape[2] || o->shape[3] != q->shape[3])
        return fail(CP_ERR_SHAPE, "o must be [b, s, Hq, d] like q");
    if (need_fp32 && o->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "o must be fp32 when accumulating");
    if (o->dtype != q->dtype && o->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype or fp32");
    if (q->dtype == CP_FP32 && o->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "fp32 inputs give fp32 outputs");
    if ((s = check_rows16(o, "o")) != CP_OK) return s;
    if (lse->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "lse must be fp32");
    if (lse->shape[0] != q->shape[0] || lse->shape[1] != q->shape[2] || lse->shape[2] != rows || lse->shape[3] != 1)
        return fail(CP_ERR_SHAPE, "lse must be [b, Hq, s, 1]");
    return CP_OK;
}

}  // namespace

cp_status cpattn::report_error(cp_status status, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

extern "C" {

const char *cp_status_string(cp_status s)
{
    switch (s) {
    case CP_OK: return "ok";
    case CP_ERR_INVALID_ARG: return "invalid argument";
    case CP_ERR_UNSUPPORTED: return "unsupported";
    case CP_ERR_SHAPE: return "shape mismatch";
    case CP_ERR_CUDA: return "CUDA error";
    case CP_ERR_TIMEOUT: return "device wait timed out";
    case CP_ERR_BOUNDS: return "bounds check failed (debug build)";
    }
    return "unknown status";
}

const char *cp_last_error(void) { return g_last_error; }

int32_t cp_abi_version(void) { return 1; }

cp_status cp_layout_range(int32_t layout, int32_t N, int64_t S, int32_t rank, cp_range *out)
{
    g_last_error[0] = 0;
    if (!out) return fail(CP_ERR_INVALID_ARG, "out is NULL");
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (N < 1 || N > 65535 || S < 0 || S > INT32_MAX) return fail(CP_ERR_INVALID_ARG, "bad N or S");
    if (S % N) return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N = %d", (long long)S, N);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if (rank < 0 || rank >= N) return fail(CP_ERR_INVALID_ARG, "rank out of range");
    Range r = layout_range(layout, N, S, rank);
    out->nseg = r.len1 > 0 ? 2 : 1;
    out->reserved = 0;
    out->start[0] = r.start0;
    out->start[1] = r.start1;
    out->len[0] = r.len0;
    out->len[1] = r.len1;
    out->stride = r.stride;
    return CP_OK;
}

cp_status cp_tile_classes(const cp_range *q_range, int64_t q_len, const cp_range *kv_range, int64_t kv_len,
                          int32_t mask_mode, int32_t tile_q, int32_t tile_k, int8_t *out)
{
    g_last_error[0] = 0;
    cp_status s;
    if (!out) return fail(CP_ERR_INVALID_ARG, "out is NULL");
    if (tile_q < 1 || tile_k < 1) return fail(CP_ERR_INVALID_ARG, "tile sizes must be positive");
    if ((s = check_range(q_range, q_len, "q_range")) != CP_OK) return s;
    if ((s = check_range(kv_range, kv_len, "kv_range")) != CP_OK) return s;
    const Range qr = to_range(*q_range), kr = to_range(*kv_range);
    const int64_t n_qt = (q_len + tile_q - 1) / tile_q, n_kt = (kv_len + tile_k - 1) / tile_k;
    for (int64_t qt = 0; qt < n_qt; ++qt) {
        int kf, ke;
        kv_tile_bounds(qr, q_len, qt * tile_q, tile_q, kr, kv_len, tile_k, mask_mode == CP_MASK_CAUSAL, &kf, &ke);
        for (int64_t kt = 0; kt < n_kt; ++kt)
            out[qt * n_kt + kt] = (int8_t)(kt < kf ? TILE_FULL : (kt < ke ? TILE_PARTIAL : TILE_SKIP));
    }
    return CP_OK;
}

cp_status cp_block_attn_fwd(const cp_tensor *q, const cp_tensor *k, const cp_tensor *v, const cp_range *q_range,
                            const cp_range *kv_range, int32_t mask_mode, float softmax_scale, cp_tensor *o,
                            cp_tensor *lse, int32_t accumulate, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if (mask_mode != CP_MASK_NONE && mask_mode != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask mode");
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    if (accumulate != 0 && accumulate != 1) return fail(CP_ERR_INVALID_ARG, "accumulate must be 0 or 1");
    const int64_t sq = q->shape[1], sk = k->shape[1];
    if (sq > INT32_MAX / 2 || sk > INT32_MAX / 2) return fail(CP_ERR_SHAPE, "sequence too long");
    if ((s = check_out(o, lse, q, sq, accumulate == 1)) != CP_OK) return s;
    if ((s = check_range(q_range, sq, "q_range")) != CP_OK) return s;
    if ((s = check_range(kv_range, sk, "kv_range")) != CP_OK) return s;
    if (q->shape[0] == 0 || sq == 0) return CP_OK;

    thread_local AttnParams p;  // large (work-order table); built fresh below
    std::memset(&p, 0, sizeof p);
    p.b = (int)q->shape[0];
    p.hq = (int)q->shape[2];
    p.hkv = (int)k->shape[2];
    p.group = p.hq / p.hkv;
    p.d = (int)q->shape[3];
    p.q_len = (int)sq;
    p.kv_len = (int)sk;
    p.n_ranks = 1;
    p.step_begin = 0;
    p.step_end = 1;
    p.causal = mask_mode == CP_MASK_CAUSAL;
    p.use_layout = 0;
    p.q_range = to_range(*q_range);
    p.kv_range = to_range(*kv_range);
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.n_qt = (int)((sq + rows_per_cta(q->dtype) - 1) / rows_per_cta(q->dtype));
    if (p.n_qt > 65535) return fail(CP_ERR_SHAPE, "too many query tiles");
    fill_inputs(p, q, k, v);
    fill_outputs(p, accumulate ? EPI_MERGE : EPI_STORE, o, lse);
    set_status_ptr(p);
    return launch_attn(p, q->dtype, static_cast<cudaStream_t>(stream));
}

cp_status cp_lse_merge(cp_tensor *o_acc, cp_tensor *lse_acc, const cp_tensor *o_b, const cp_tensor *lse_b,
                       cp_tensor *o_out, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if ((s = check_tensor(o_acc, "o_acc")) != CP_OK || (s = check_tensor(lse_acc, "lse_acc")) != CP_OK ||
        (s = check_tensor(o_b, "o_b")) != CP_OK || (s = check_tensor(lse_b, "lse_b")) != CP_OK)
        return s;
    if (o_acc->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "o_acc must be fp32");
    if (lse_acc->dtype != CP_FP32 || lse_b->dtype != CP_FP32) return fail(CP_ERR_INVALID_ARG, "lse must be fp32");
    if (!same_shape(o_acc, o_b)) return fail(CP_ERR_SHAPE, "o_acc and o_b differ in shape");
    const int64_t b = o_acc->shape[0], S = o_acc->shape[1], H = o_acc->shape[2], d = o_acc->shape[3];
    if (!same_shape(lse_acc, lse_b) || lse_acc->shape[0] != b || lse_acc->shape[1] != H || lse_acc->shape[2] != S ||
        lse_acc->shape[3] != 1)
        return fail(CP_ERR_SHAPE, "lse tensors must be [b, H, s, 1]");
    if (d % 8 || d > 256 || 32 % (d / 8))
        return fail(CP_ERR_UNSUPPORTED, "d must be 8, 16, 32, 64, 128 or 256");
    if ((s = check_rows16(o_acc, "o_acc")) != CP_OK || (s = check_rows16(o_b, "o_b")) != CP_OK) return s;
    if (o_out) {
        if ((s = check_tensor(o_out, "o_out")) != CP_OK) return s;
        if (!same_shape(o_out, o_acc)) return fail(CP_ERR_SHAPE, "o_out differs in shape");
        if ((s = check_rows16(o_out, "o_out")) != CP_OK) return s;
    }
    MergeParams p;
    p.b = b; p.s = S; p.h = H; p.d = d;
    p.o_acc = static_cast<float *>(o_acc->data);
    p.oa_sb = o_acc->stride[0]; p.oa_ss = o_acc->stride[1]; p.oa_sh = o_acc->stride[2];
    p.lse_acc = static_cast<float *>(lse_acc->data);
    p.la_sb = lse_acc->stride[0]; p.la_sh = lse_acc->stride[1]; p.la_ss = lse_acc->stride[2];
    p.o_b = o_b->data; p.ob_dtype = o_b->dtype;
    p.ob_sb = o_b->stride[0]; p.ob_ss = o_b->stride[1]; p.ob_sh = o_b->stride[2];
    p.lse_b = static_cast<const float *>(lse_b->data);
    p.lb_sb = lse_b->stride[0]; p.lb_sh = lse_b->stride[1]; p.lb_ss = lse_b->stride[2];
    p.o_out = o_out ? o_out->data : nullptr;
    p.out_dtype = o_out ? o_out->dtype : CP_FP32;
    p.out_sb = o_out ? o_out->stride[0] : 0; p.out_ss = o_out ? o_out->stride[1] : 0;
    p.out_sh = o_out ? o_out->stride[2] : 0;
    cudaError_t e = launch_lse_merge(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    return CP_OK;
}

size_t cp_ring_workspace_bytes(int32_t layout, int32_t N, int32_t mode, int32_t dtype, int64_t b, int64_t S,
                               int64_t Hq, int64_t d)
{
    if (mode != CP_RING_STEPWISE && mode != CP_RING_STEPWISE_EPI) return 0;
    if (layout < 0 || layout > 2 || N < 1 || b < 0 || S < 0 || Hq < 0 || d < 0) return 0;
    if (N == 1) return 0;
    const int64_t es = elem_size(dtype);
    if (!es) return 0;
    const int64_t rows = b * S * Hq;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    // STEPWISE_EPI: the fp32 running o (an fp32 output is its own accumulator)
    if (mode == CP_RING_STEPWISE_EPI) return dtype == CP_FP32 ? 0 : (size_t)up(rows * d * 4);
    // STEPWISE: o_acc fp32, o_b in the input dtype, lse_b fp32; each region 256-byte aligned
    return (size_t)(up(rows * d * 4) + up(rows * d * es) + up(rows * 4));
}

cp_status cp_ring_attn_fwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                           const cp_tensor *v, float softmax_scale, cp_tensor *o, cp_tensor *lse, int32_t mode,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (mode != CP_RING_FUSED && mode != CP_RING_STEPWISE && mode != CP_RING_STEPWISE_EPI)
        return fail(CP_ERR_INVALID_ARG, "unknown ring mode");
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t S = q->shape[1];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if (S % N) return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N = %d", (long long)S, N);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    if (o->dtype != q->dtype) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype");
    const int64_t c = S / N;
    if (q->shape[0] == 0 || S == 0) return CP_OK;
    const int rows = rows_per_cta(q->dtype);
    const int n_qt = (int)((c + rows - 1) / rows);
    if (n_qt > 65535) return fail(CP_ERR_SHAPE, "too many query tiles per rank");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    NvtxRange call_range(mode == CP_RING_FUSED ? "cp_ring_attn_fwd fused" : "cp_ring_attn_fwd stepwise");

    thread_local AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.b = (int)q->shape[0];
    p.hq = (int)q->shape[2];
    p.hkv = (int)k->shape[2];
    p.group = p.hq / p.hkv;
    p.d = (int)q->shape[3];
    p.q_len = (int)c;
    p.kv_len = (int)c;
    p.n_ranks = N;
    p.causal = causal;
    p.use_layout = 1;
    p.layout = layout;
    p.seq_len = S;
    p.q_row_step = c;
    p.kv_row_step = c;
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.n_qt = n_qt;
    set_ring_order(p, layout, N, S, causal, rows);
    fill_inputs(p, q, k, v);
    set_status_ptr(p);

    if (mode == CP_RING_FUSED || N == 1) {
        p.step_begin = 0;
        p.step_end = N;
        fill_outputs(p, EPI_STORE, o, lse);
        return launch_attn(p, q->dtype, st);
    }

    const size_t need = cp_ring_workspace_bytes(layout, N, mode, q->dtype, q->shape[0], S, q->shape[2], q->shape[3]);
    if (need && (!workspace || workspace_bytes < need))
        return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const int64_t b = q->shape[0], Hq = q->shape[2], d = q->shape[3], nrows = b * S * Hq;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    char *ws = static_cast<char *>(workspace);
    cp_tensor o_acc{ws, CP_FP32, 0, {b, S, Hq, d}, {S * Hq * d, Hq * d, d, 1}};

    if (mode == CP_RING_STEPWISE_EPI) {
        // N launches, one ring step each; step 0 stores the running (o, lse) in fp32,
        // every later step LSE-merges its partial into them in the block epilogue,
        // and the last one writes the merged o in the output dtype.  An fp32 output
        // is the running o itself.
        const cp_tensor *acc = q->dtype == CP_FP32 ? o : &o_acc;
        for (int r = 0; r < N; ++r) {
            NvtxRange step_range("cp ring step %d of %d", r, N);
            p.step_begin = r;
            p.step_end = r + 1;
            fill_outputs(p, r == 0 ? EPI_STORE : EPI_MERGE, acc, lse);
            if (r == N - 1 && acc != o) {
                p.o_out = o->data;
                p.o_out_dtype = o->dtype;
                p.oo_sb = o->stride[0]; p.oo_ss = o->stride[1]; p.oo_sh = o->stride[2];
            }
            if ((s = launch_attn(p, q->dtype, st)) != CP_OK) return s;
        }
        return CP_OK;
    }

    // STEPWISE: the ring as N block launches plus N-1 standalone merges
    cp_tensor o_b{ws + up(nrows * d * 4), q->dtype, 0, {b, S, Hq, d}, {S * Hq * d, Hq * d, d, 1}};
    cp_tensor lse_b{ws + up(nrows * d * 4) + up(nrows * d * elem_size(q->dtype)), CP_FP32, 0, {b, Hq, S, 1},
                    {Hq * S, S, 1, 1}};
    for (int r = 0; r < N; ++r) {
        NvtxRange step_range("cp ring step %d of %d", r, N);
        p.step_begin = r;
        p.step_end = r + 1;
        if (r == 0) fill_outputs(p, EPI_STORE, &o_acc, lse);  // first partial initialises the running result
        else fill_outputs(p, EPI_STORE, &o_b, &lse_b);
        if ((s = launch_attn(p, q->dtype, st)) != CP_OK) return s;
        if (r > 0 && (s = cp_lse_merge(&o_acc, lse, &o_b, &lse_b, r == N - 1 ? o : nullptr, stream)) != CP_OK)
            return s;
    }
    return CP_OK;
}

cp_status cp_ulysses_all_to_all(int32_t P, int32_t direction, const cp_tensor *x_seq, cp_tensor *y_head, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if ((s = check_tensor(x_seq, "x_seq")) != CP_OK || (s = check_tensor(y_head, "y_head")) != CP_OK) return s;
    if (direction != 0 && direction != 1) return fail(CP_ERR_INVALID_ARG, "direction must be 0 or 1");
    if (P < 1) return fail(CP_ERR_INVALID_ARG, "P must be >= 1");
    if (x_seq->dtype != y_head->dtype) return fail(CP_ERR_INVALID_ARG, "x_seq and y_head differ in dtype");
    const int64_t b = x_seq->shape[0], S = x_seq->shape[1], H = x_seq->shape[2], d = x_seq->shape[3];
    if (H % P || S % P) return fail(CP_ERR_SHAPE, "P must divide the heads (%lld) and the sequence (%lld)",
                                    (long long)H, (long long)S);
    if (y_head->shape[0] != P * b || y_head->shape[1] != S || y_head->shape[2] != H / P || y_head->shape[3] != d)
        return fail(CP_ERR_SHAPE, "y_head must be [P*b, S, H/P, d]");
    for (const cp_tensor *t : {x_seq, static_cast<const cp_tensor *>(y_head)}) {
        int64_t expect = 1;
        for (int i = 3; i >= 0; --i) {
            if (t->shape[i] > 1 && t->stride[i] != expect) return fail(CP_ERR_INVALID_ARG, "tensors must be contiguous");
            expect *= t->shape[i];
        }
    }
    const int64_t bytes = b * S * H * d * elem_size(x_seq->dtype);
    const char *a = static_cast<const char *>(x_seq->data), *bp = static_cast<const char *>(y_head->data);
    if (bytes && a < bp + bytes && bp < a + bytes) return fail(CP_ERR_INVALID_ARG, "x_seq and y_head overlap");
    ShardParams sp{P, b, S, (H / P) * d * elem_size(x_seq->dtype), direction, direction ? y_head->data : x_seq->data,
                   direction ? const_cast<void *>(x_seq->data) : y_head->data};
    cudaError_t e = launch_shard_transpose(sp, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "all-to-all launch");
    return CP_OK;
}

size_t cp_ulysses_workspace_bytes(int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq, int64_t Hkv, int64_t d)
{
    if (P < 1 || b < 0 || S < 0 || Hq < 0 || Hkv < 0 || d < 0 || !elem_size(dtype)) return 0;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t es = elem_size(dtype);
    // head-sharded q, k, v, o and lse
    return (size_t)(2 * up(b * S * Hq * d * es) + 2 * up(b * S * Hkv * d * es) + up(b * Hq * S * 4));
}

// Ulysses exchange around a ring: the head-sharded tensors [P*b, S, H/P, d] keep
// the sequence axis as it came in, so with N = 1 this is plain Ulysses and with a
// rank-major sequence of N ring groups it is the Ulysses x ring hybrid (every
// ring group's exchange moves tokens only inside the group's block).
static cp_status uly_ring_fwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q,
                              const cp_tensor *k, const cp_tensor *v, float softmax_scale, cp_tensor *o, cp_tensor *lse,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t b = q->shape[0], S = q->shape[1], Hq = q->shape[2], Hkv = k->shape[2], d = q->shape[3];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (P < 1) return fail(CP_ERR_INVALID_ARG, "P must be >= 1");
    if (Hq % P || Hkv % P)
        return fail(CP_ERR_SHAPE, "P must divide the query heads (%lld) and the kv heads (%lld)", (long long)Hq,
                    (long long)Hkv);
    if (S % ((int64_t)N * P))
        return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N * P = %d * %d", (long long)S, N, P);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if (S % 4) return fail(CP_ERR_SHAPE, "S must be a multiple of 4");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    if (o->dtype != q->dtype) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype");
    for (const cp_tensor *t : {q, k, v, static_cast<const cp_tensor *>(o)}) {
        int64_t expect = 1;
        for (int i = 3; i >= 0; --i) {
            if (t->shape[i] > 1 && t->stride[i] != expect) return fail(CP_ERR_INVALID_ARG, "tensors must be contiguous");
            expect *= t->shape[i];
        }
    }
    if (!(lse->stride[2] == 1 && lse->stride[1] == S && (b <= 1 || lse->stride[0] == Hq * S)))
        return fail(CP_ERR_INVALID_ARG, "lse must be contiguous");
    const size_t need = cp_ulysses_workspace_bytes(P, q->dtype, b, S, Hq, Hkv, d);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (b == 0 || S == 0) return CP_OK;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t es = elem_size(q->dtype), hp = Hq / P, hkp = Hkv / P;
    char *ws = static_cast<char *>(workspace);
    const int64_t qb = up(b * S * Hq * d * es), kb = up(b * S * Hkv * d * es);
    cp_tensor qh{ws, q->dtype, 0, {P * b, S, hp, d}, {S * hp * d, hp * d, d, 1}};
    cp_tensor kh{ws + qb, q->dtype, 0, {P * b, S, hkp, d}, {S * hkp * d, hkp * d, d, 1}};
    cp_tensor vh{ws + qb + kb, q->dtype, 0, {P * b, S, hkp, d}, {S * hkp * d, hkp * d, d, 1}};
    cp_tensor oh{ws + qb + 2 * kb, q->dtype, 0, {P * b, S, hp, d}, {S * hp * d, hp * d, d, 1}};
    cp_tensor lh{ws + 2 * qb + 2 * kb, CP_FP32, 0, {P * b, hp, S, 1}, {hp * S, S, 1, 1}};
    // all-to-all: sequence-sharded -> head-sharded
    if ((s = cp_ulysses_all_to_all(P, 0, q, &qh, stream)) != CP_OK) return s;
    if ((s = cp_ulysses_all_to_all(P, 0, k, &kh, stream)) != CP_OK) return s;
    if ((s = cp_ulysses_all_to_all(P, 0, v, &vh, stream)) != CP_OK) return s;
    // every rank's heads over the whole sequence (with N > 1: the ring over the
    // groups' blocks): one launch, the head groups as batch entries
    if ((s = cp_ring_attn_fwd(layout, N, causal, &qh, &kh, &vh, softmax_scale, &oh, &lh, CP_RING_FUSED, nullptr, 0,
                              stream)) != CP_OK)
        return s;
    // and back: o [P*b, S, hp, d] -> [b, S, Hq, d]; lse [P][b][hp * S] -> [b][P][hp * S]
    if ((s = cp_ulysses_all_to_all(P, 1, o, &oh, stream)) != CP_OK) return s;
    ShardParams sp{P, b, 1, hp * S * 4, 1, lh.data, lse->data};
    cudaError_t e = launch_shard_transpose(sp, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "all-to-all launch");
    return CP_OK;
}

cp_status cp_ulysses_attn_fwd(int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k, const cp_tensor *v,
                              float softmax_scale, cp_tensor *o, cp_tensor *lse, void *workspace,
                              size_t workspace_bytes, void *stream)
{
    return uly_ring_fwd(CP_LAYOUT_CONTIGUOUS, 1, P, causal, q, k, v, softmax_scale, o, lse, workspace, workspace_bytes,
                        stream);
}

size_t cp_usp_workspace_bytes(int32_t layout, int32_t N, int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                              int64_t Hkv, int64_t d)
{
    if (layout < 0 || layout > 2 || N < 1) return 0;
    return cp_ulysses_workspace_bytes(P, dtype, b, S, Hq, Hkv, d);
}

cp_status cp_usp_attn_fwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                          const cp_tensor *v, float softmax_scale, cp_tensor *o, cp_tensor *lse, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    return uly_ring_fwd(layout, N, P, causal, q, k, v, softmax_scale, o, lse, workspace, workspace_bytes, stream);
}

size_t cp_allgather_bwd_workspace_bytes(int32_t N, int32_t dtype, int64_t b, int64_t S, int64_t Hq, int64_t Hkv,
                                        int64_t d, int32_t n_docs)
{
    if (N < 1 || b < 0 || S < 0 || Hq < 0 || Hkv < 0 || d < 0 || n_docs < 1 || !elem_size(dtype) || S % N) return 0;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t kb = up(b * S * Hkv * d * elem_size(dtype));
    // gathered K, V, dK, dV; the document starts and the per-position document
    // bounds; the statistics and the dQ accumulator
    return (size_t)(4 * kb + up((int64_t)n_docs * 4) + 2 * up(S * 4)) +
           cp_ring_bwd_workspace_bytes(CP_LAYOUT_CONTIGUOUS, N, dtype, b, S, Hq, d);
}

cp_status cp_allgather_attn_bwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                                const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse, const cp_tensor *dout,
                                const int64_t *doc_starts, int32_t n_docs, float softmax_scale, cp_tensor *dq,
                                cp_tensor *dk, cp_tensor *dv, void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK || (s = check_tensor(dout, "dout")) != CP_OK ||
        (s = check_tensor(dq, "dq")) != CP_OK || (s = check_tensor(dk, "dk")) != CP_OK ||
        (s = check_tensor(dv, "dv")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    // bf16 with d = 128 on the tensor cores, fp32 and bf16 d = 64 on the FFMA kernels
    const int32_t dt = q->dtype;
    const bool tc_path = dt == CP_BF16 && q->shape[3] == 128;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t S = q->shape[1];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if (S % N) return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N = %d", (long long)S, N);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    if (o->dtype != dt) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype");
    const cp_tensor *like_q[2] = {dout, dq};
    for (const cp_tensor *t : like_q) {
        if (!same_shape(t, q) || t->dtype != dt) return fail(CP_ERR_SHAPE, "dout and dq must be shaped like q, same dtype");
        if ((s = check_rows16(t, t == dq ? "dq" : "dout")) != CP_OK) return s;
    }
    const cp_tensor *like_k[4] = {k, v, dk, dv};
    for (const cp_tensor *t : like_k) {
        if (!same_shape(t, k) || t->dtype != dt) return fail(CP_ERR_SHAPE, "dk and dv must be shaped like k, same dtype");
        int64_t expect = 1;
        for (int i = 3; i >= 0; --i) {
            if (t->shape[i] > 1 && t->stride[i] != expect)
                return fail(CP_ERR_INVALID_ARG, "k, v, dk and dv must be contiguous");
            expect *= t->shape[i];
        }
    }
    if (n_docs < 1 || !doc_starts) return fail(CP_ERR_INVALID_ARG, "doc_starts must hold at least one start");
    if (doc_starts[0] != 0) return fail(CP_ERR_INVALID_ARG, "the first document must start at 0");
    for (int32_t i = 1; i < n_docs; ++i)
        if (doc_starts[i] <= doc_starts[i - 1] || doc_starts[i] >= S)
            return fail(CP_ERR_INVALID_ARG, "document starts must increase and stay below S");
    if (n_docs > 1 && !causal) return fail(CP_ERR_UNSUPPORTED, "the document mask is defined with the causal mask");
    const int64_t b = q->shape[0], Hq = q->shape[2], Hkv = k->shape[2], d = q->shape[3];
    const int64_t c = S / N;
    const int64_t n_kt = (S + kBwdKeyTile - 1) / kBwdKeyTile;
    if (n_kt > 65535) return fail(CP_ERR_SHAPE, "too many key tiles");
    const size_t need = cp_allgather_bwd_workspace_bytes(N, q->dtype, b, S, Hq, Hkv, d, n_docs);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (b == 0 || S == 0) return CP_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    NvtxRange call_range("cp_allgather_attn_bwd");
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    char *ws = static_cast<char *>(workspace);
    const int64_t kb = up(b * S * Hkv * d * elem_size(dt));
    auto kv_t = [&](int i) {
        return cp_tensor{ws + i * kb, dt, 0, {b, S, Hkv, d}, {S * Hkv * d, Hkv * d, d, 1}};
    };
    cp_tensor kg = kv_t(0), vg = kv_t(1), dkg = kv_t(2), dvg = kv_t(3);
    int *docs_dev = reinterpret_cast<int *>(ws + 4 * kb);
    int *doc_pos_start = reinterpret_cast<int *>(ws + 4 * kb + up((int64_t)n_docs * 4));
    int *doc_pos_end = reinterpret_cast<int *>(ws + 4 * kb + up((int64_t)n_docs * 4) + up(S * 4));
    char *ws_q = ws + 4 * kb + up((int64_t)n_docs * 4) + 2 * up(S * 4);
    // the gather of K and V into original order (as in the forward), unless the
    // tensor-core kernel reads K, V and writes dK, dV in place (same rule as the forward)
    const int64_t kv_map_h = (tc_path && layout == CP_LAYOUT_ZIGZAG && (c / 2) % kBwdKeyTile == 0) ? c / 2 : 0;
    const bool kv_in_place = tc_path && (layout == CP_LAYOUT_CONTIGUOUS || kv_map_h > 0);
    if (!kv_in_place) {
        if ((s = cp_layout_permute(layout, N, 1, &kg, const_cast<cp_tensor *>(k), 1, stream)) != CP_OK) return s;
        if ((s = cp_layout_permute(layout, N, 1, &vg, const_cast<cp_tensor *>(v), 1, stream)) != CP_OK) return s;
    }
    const cp_tensor &kx = kv_in_place ? *k : kg, &vx = kv_in_place ? *v : vg;
    const cp_tensor &dkx = kv_in_place ? *dk : dkg, &dvx = kv_in_place ? *dv : dvg;
    cudaError_t e = cudaSuccess;
    if (n_docs > 1) {  // device starts for the FFMA kernels, per-position bounds for the tensor-core one
        e = launch_doc_tables(doc_starts, n_docs, S, docs_dev, doc_pos_start, doc_pos_end, st);
        if (e != cudaSuccess) return cuda_fail(e, "document bounds launch");
    }

    thread_local BwdParams p;
    std::memset(&p, 0, sizeof p);
    p.b = (int)b;
    p.hq = (int)Hq;
    p.hkv = (int)Hkv;
    p.group = p.hq / p.hkv;
    p.d = (int)d;
    p.q_len = (int)c;
    p.kv_len = (int)S;
    p.n_ranks = N;
    p.step_begin = 0;
    p.step_end = N;  // key block 0 meets query rank r at step r
    p.causal = causal;
    p.use_layout = 1;
    p.layout = layout;
    p.seq_len = S;
    p.kv_explicit = 1;
    p.kv_range = Range{0, 0, S, 0, 1};
    p.n_kv_blocks = 1;
    p.q_row_step = c;
    p.kv_row_step = 0;
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.q = q->data; p.k = kx.data; p.v = vx.data; p.o = o->data; p.dout = dout->data;
    p.q_sb = q->stride[0]; p.q_ss = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = kx.stride[0]; p.k_ss = kx.stride[1]; p.k_sh = kx.stride[2];
    p.v_sb = vx.stride[0]; p.v_ss = vx.stride[1]; p.v_sh = vx.stride[2];
    p.o_sb = o->stride[0]; p.o_ss = o->stride[1]; p.o_sh = o->stride[2];
    p.do_sb = dout->stride[0]; p.do_ss = dout->stride[1]; p.do_sh = dout->stride[2];
    p.lse = static_cast<const float *>(lse->data);
    p.lse_sb = lse->stride[0]; p.lse_sh = lse->stride[1]; p.lse_ss = lse->stride[2];
    const BwdWorkspace w = bwd_workspace(N, b, S, Hq, d);
    p.stats = reinterpret_cast<float2 *>(ws_q);
    p.lpad = (int)w.lpad;
    p.dq_acc = reinterpret_cast<float *>(ws_q + w.stats_bytes);
    p.dq = dq->data; p.dk = dkx.data; p.dv = dvx.data;
    p.dq_sb = dq->stride[0]; p.dq_ss = dq->stride[1]; p.dq_sh = dq->stride[2];
    p.dk_sb = dkx.stride[0]; p.dk_ss = dkx.stride[1]; p.dk_sh = dkx.stride[2];
    p.dv_sb = dvx.stride[0]; p.dv_ss = dvx.stride[1]; p.dv_sh = dvx.stride[2];
    p.kv_map_h = (int)kv_map_h;
    p.doc_starts = n_docs > 1 ? docs_dev : nullptr;
    p.n_docs = n_docs > 1 ? n_docs : 0;
    p.doc_pos_end = doc_pos_end;
    int *word = nullptr;
    status_word(&word);
    p.status = word;
    p.n_kt = (int)n_kt;
    if (!tc_path) {
        e = launch_attn_bwd_simt(p, dt == CP_FP32, st);
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
        if ((s = cp_layout_permute(layout, N, 1, &dkg, dk, 0, stream)) != CP_OK) return s;
        if ((s = cp_layout_permute(layout, N, 1, &dvg, dv, 0, stream)) != CP_OK) return s;
        return CP_OK;
    }
    // work order, heaviest first: a key tile of the gathered block costs the query
    // tiles of every rank it meets, from the first that sees its first key (causal)
    // to the last that starts before the end of its last key's document
    if (n_kt <= kMaxOrder) {
        const int n_qt = (int)((c + kBwdQueryTile - 1) / kBwdQueryTile);
        std::vector<std::pair<int64_t, uint32_t>> work;
        work.reserve((size_t)n_kt);
        const Range kr{0, 0, S, 0, 1};
        for (int kt = 0; kt < (int)n_kt; ++kt) {
            const int64_t k_hi = std::min<int64_t>((int64_t)kt * kBwdKeyTile + kBwdKeyTile - 1, S - 1);
            const int64_t *next_doc = std::upper_bound(doc_starts, doc_starts + n_docs, k_hi);
            const int64_t de = next_doc == doc_starts + n_docs ? S : *next_doc;  // end of the last key's document
            int64_t tiles = 0;
            for (int r = 0; r < N; ++r) {
                const Range qr = layout_range(layout, N, S, r);
                int qb, qf;
                q_tile_bounds<int64_t>(qr, c, kBwdQueryTile, kr, S, (int64_t)kt * kBwdKeyTile, kBwdKeyTile,
                                       causal != 0, &qb, &qf);
                int lo = qb, hi = n_qt;  // first tile whose first row lies at or past de
                while (lo < hi) {
                    const int mid = (lo + hi) / 2;
                    if (range_pos(qr, (int64_t)mid * kBwdQueryTile) < de) lo = mid + 1; else hi = mid;
                }
                tiles += lo - qb;
            }
            work.push_back({tiles, (uint32_t)kt});
        }
        std::stable_sort(work.begin(), work.end(),
                         [](const std::pair<int64_t, uint32_t> &x, const std::pair<int64_t, uint32_t> &y) {
                             return x.first > y.first;
                         });
        p.order_len = (int)n_kt;
        for (int64_t i = 0; i < n_kt; ++i) p.order[i] = work[(size_t)i].second;
    }
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    p.head_major = !kBwdNeverHeadMajor && (kBwdHeadMajor || n_kt >= (int64_t)sms);
    p.tile_rotation = p.head_major && bwd_tile_rotation(p.group, S, p.d, dev);
    e = launch_attn_bwd(p, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    if (kv_in_place) return CP_OK;  // dK, dV were written to the ranks' blocks directly
    // the reduce-scatter: the summed dK, dV of the gathered block back to each rank
    if ((s = cp_layout_permute(layout, N, 1, &dkg, dk, 0, stream)) != CP_OK) return s;
    if ((s = cp_layout_permute(layout, N, 1, &dvg, dv, 0, stream)) != CP_OK) return s;
    return CP_OK;
}

static size_t uly_ring_bwd_ws(int32_t layout, int32_t N, int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                              int64_t Hkv, int64_t d)
{
    if (layout < 0 || layout > 2 || N < 1 || P < 1 || b < 0 || S < 0 || Hq < 0 || Hkv < 0 || d < 0 ||
        !elem_size(dtype) || Hq % P || S % N)
        return 0;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t es = elem_size(dtype);
    const int64_t qb = up(b * S * Hq * d * es), kb = up(b * S * Hkv * d * es), lb = up(b * Hq * S * 4);
    // head-sharded q, o, dout, dq; k, v, dk, dv; lse; then the ring backward's own
    return (size_t)(4 * qb + 4 * kb + lb) + cp_ring_bwd_workspace_bytes(layout, N, dtype, P * b, S, Hq / P, d);
}

size_t cp_ulysses_bwd_workspace_bytes(int32_t P, int32_t dtype, int64_t b, int64_t S, int64_t Hq, int64_t Hkv,
                                      int64_t d)
{
    return uly_ring_bwd_ws(CP_LAYOUT_CONTIGUOUS, 1, P, dtype, b, S, Hq, Hkv, d);
}

size_t cp_usp_bwd_workspace_bytes(int32_t layout, int32_t N, int32_t P, int32_t dtype, int64_t b, int64_t S,
                                  int64_t Hq, int64_t Hkv, int64_t d)
{
    return uly_ring_bwd_ws(layout, N, P, dtype, b, S, Hq, Hkv, d);
}

static cp_status uly_ring_bwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q,
                              const cp_tensor *k, const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse,
                              const cp_tensor *dout, float softmax_scale, cp_tensor *dq, cp_tensor *dk, cp_tensor *dv,
                              void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK || (s = check_tensor(dout, "dout")) != CP_OK ||
        (s = check_tensor(dq, "dq")) != CP_OK || (s = check_tensor(dk, "dk")) != CP_OK ||
        (s = check_tensor(dv, "dv")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t b = q->shape[0], S = q->shape[1], Hq = q->shape[2], Hkv = k->shape[2], d = q->shape[3];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (P < 1) return fail(CP_ERR_INVALID_ARG, "P must be >= 1");
    if (Hq % P || Hkv % P)
        return fail(CP_ERR_SHAPE, "P must divide the query heads (%lld) and the kv heads (%lld)", (long long)Hq,
                    (long long)Hkv);
    if (S % ((int64_t)N * P))
        return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N * P = %d * %d", (long long)S, N, P);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if (S % 4) return fail(CP_ERR_SHAPE, "S must be a multiple of 4");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    const int32_t dt = q->dtype;
    const cp_tensor *like_q[3] = {o, dout, dq};
    for (const cp_tensor *t : like_q)
        if (!same_shape(t, q) || t->dtype != dt) return fail(CP_ERR_SHAPE, "o, dout and dq must be shaped like q, same dtype");
    const cp_tensor *like_k[2] = {dk, dv};
    for (const cp_tensor *t : like_k)
        if (!same_shape(t, k) || t->dtype != dt) return fail(CP_ERR_SHAPE, "dk and dv must be shaped like k, same dtype");
    if (!(lse->stride[2] == 1 && lse->stride[1] == S && (b <= 1 || lse->stride[0] == Hq * S)))
        return fail(CP_ERR_INVALID_ARG, "lse must be contiguous");
    const size_t need = uly_ring_bwd_ws(layout, N, P, q->dtype, b, S, Hq, Hkv, d);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (b == 0 || S == 0) return CP_OK;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    const int64_t hp = Hq / P, hkp = Hkv / P;
    const int64_t es = elem_size(dt);
    const int64_t qb = up(b * S * Hq * d * es), kb = up(b * S * Hkv * d * es), lb = up(b * Hq * S * 4);
    char *ws = static_cast<char *>(workspace);
    auto qt = [&](int i) {
        return cp_tensor{ws + i * qb, dt, 0, {P * b, S, hp, d}, {S * hp * d, hp * d, d, 1}};
    };
    auto kt = [&](int i) {
        return cp_tensor{ws + 4 * qb + i * kb, dt, 0, {P * b, S, hkp, d}, {S * hkp * d, hkp * d, d, 1}};
    };
    cp_tensor qh = qt(0), oh = qt(1), doh = qt(2), dqh = qt(3);
    cp_tensor kh = kt(0), vh = kt(1), dkh = kt(2), dvh = kt(3);
    cp_tensor lh{ws + 4 * qb + 4 * kb, CP_FP32, 0, {P * b, hp, S, 1}, {hp * S, S, 1, 1}};
    char *ws_ring = ws + 4 * qb + 4 * kb + lb;
    const size_t ring_need = cp_ring_bwd_workspace_bytes(layout, N, dt, P * b, S, hp, d);
    // exchange in: q, k, v, o, dout and lse to the head-sharded layout
    const cp_tensor *ins[5] = {q, k, v, o, dout};
    cp_tensor *outs[5] = {&qh, &kh, &vh, &oh, &doh};
    for (int i = 0; i < 5; ++i)
        if ((s = cp_ulysses_all_to_all(P, 0, ins[i], outs[i], stream)) != CP_OK) return s;
    ShardParams sp{P, b, 1, hp * S * 4, 0, lse->data, lh.data};
    cudaError_t e = launch_shard_transpose(sp, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "all-to-all launch");
    // each rank's head group over the whole sequence (with N > 1: the ring backward
    // over the groups' blocks, dK and dV travelling with their block)
    if ((s = cp_ring_attn_bwd(layout, N, causal, &qh, &kh, &vh, &oh, &lh, &doh, softmax_scale, &dqh, &dkh, &dvh,
                              ws_ring, ring_need, stream)) != CP_OK)
        return s;
    // exchange out: the gradients back to the sequence-sharded layout
    if ((s = cp_ulysses_all_to_all(P, 1, dq, &dqh, stream)) != CP_OK) return s;
    if ((s = cp_ulysses_all_to_all(P, 1, dk, &dkh, stream)) != CP_OK) return s;
    if ((s = cp_ulysses_all_to_all(P, 1, dv, &dvh, stream)) != CP_OK) return s;
    return CP_OK;
}

cp_status cp_ulysses_attn_bwd(int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k, const cp_tensor *v,
                              const cp_tensor *o, const cp_tensor *lse, const cp_tensor *dout, float softmax_scale,
                              cp_tensor *dq, cp_tensor *dk, cp_tensor *dv, void *workspace, size_t workspace_bytes,
                              void *stream)
{
    return uly_ring_bwd(CP_LAYOUT_CONTIGUOUS, 1, P, causal, q, k, v, o, lse, dout, softmax_scale, dq, dk, dv, workspace,
                        workspace_bytes, stream);
}

cp_status cp_usp_attn_bwd(int32_t layout, int32_t N, int32_t P, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                          const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse, const cp_tensor *dout,
                          float softmax_scale, cp_tensor *dq, cp_tensor *dk, cp_tensor *dv, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    return uly_ring_bwd(layout, N, P, causal, q, k, v, o, lse, dout, softmax_scale, dq, dk, dv, workspace,
                        workspace_bytes, stream);
}

size_t cp_allgather_workspace_bytes(int32_t N, int32_t dtype, int64_t b, int64_t S, int64_t Hkv, int64_t d,
                                    int32_t n_docs)
{
    if (N < 1 || b < 0 || S < 0 || Hkv < 0 || d < 0 || n_docs < 1 || !elem_size(dtype)) return 0;
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    // gathered K and V in original token order, then the document starts (int32) and
    // the per-position document bounds (two int32 tables of S entries)
    return (size_t)(2 * up(b * S * Hkv * d * elem_size(dtype)) + up((int64_t)n_docs * 4) + 2 * up(S * 4));
}

cp_status cp_allgather_attn_fwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                                const cp_tensor *v, const int64_t *doc_starts, int32_t n_docs, float softmax_scale,
                                cp_tensor *o, cp_tensor *lse, void *workspace, size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t S = q->shape[1];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if (S % N) return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N = %d", (long long)S, N);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    if (o->dtype != q->dtype) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype");
    if (n_docs < 1 || !doc_starts) return fail(CP_ERR_INVALID_ARG, "doc_starts must hold at least one start");
    if (doc_starts[0] != 0) return fail(CP_ERR_INVALID_ARG, "the first document must start at 0");
    for (int32_t i = 1; i < n_docs; ++i)
        if (doc_starts[i] <= doc_starts[i - 1] || doc_starts[i] >= S)
            return fail(CP_ERR_INVALID_ARG, "document starts must increase and stay below S");
    if (n_docs > 1 && !causal) return fail(CP_ERR_UNSUPPORTED, "the document mask is defined with the causal mask");
    for (const cp_tensor *t : {k, v}) {
        int64_t expect = 1;
        for (int i = 3; i >= 0; --i) {
            if (t->shape[i] > 1 && t->stride[i] != expect)
                return fail(CP_ERR_INVALID_ARG, "k and v must be contiguous for the gather");
            expect *= t->shape[i];
        }
    }
    const int64_t b = q->shape[0], Hkv = k->shape[2], d = q->shape[3];
    const size_t need = cp_allgather_workspace_bytes(N, q->dtype, b, S, Hkv, d, n_docs);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const int64_t c = S / N;
    if (b == 0 || S == 0) return CP_OK;
    const int rows = rows_per_cta(q->dtype, n_docs > 1);  // the document instantiation's CTA
    const int n_qt = (int)((c + rows - 1) / rows);
    if (n_qt > 65535) return fail(CP_ERR_SHAPE, "too many query tiles per rank");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    NvtxRange call_range("cp_allgather_attn_fwd");

    // the all-gather: every rank's K/V block back into one original-order copy.  The
    // tensor-core kernel reads the ranks' blocks in place instead when every key tile
    // of the original order is a run of consecutive rank-major rows: the contiguous
    // layout (rank-major order is the original order), or zig-zag chunks that are a
    // whole number of key tiles (rows through zigzag_row)
    auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
    char *ws = static_cast<char *>(workspace);
    const int64_t kv_bytes = up(b * S * Hkv * d * elem_size(q->dtype));
    cp_tensor kg{ws, q->dtype, 0, {b, S, Hkv, d}, {S * Hkv * d, Hkv * d, d, 1}};
    cp_tensor vg{ws + kv_bytes, q->dtype, 0, {b, S, Hkv, d}, {S * Hkv * d, Hkv * d, d, 1}};
    int *docs_dev = reinterpret_cast<int *>(ws + 2 * kv_bytes);
    const bool tc_fwd = q->dtype == CP_BF16;
    const int64_t kv_map_h = (tc_fwd && layout == CP_LAYOUT_ZIGZAG && (c / 2) % 128 == 0) ? c / 2 : 0;
    const bool kv_in_place = tc_fwd && (layout == CP_LAYOUT_CONTIGUOUS || kv_map_h > 0);
    if (!kv_in_place) {
        if ((s = cp_layout_permute(layout, N, 1, &kg, const_cast<cp_tensor *>(k), 1, stream)) != CP_OK) return s;
        if ((s = cp_layout_permute(layout, N, 1, &vg, const_cast<cp_tensor *>(v), 1, stream)) != CP_OK) return s;
    }
    int *doc_pos_start = reinterpret_cast<int *>(ws + 2 * kv_bytes + up((int64_t)n_docs * 4));
    int *doc_pos_end = doc_pos_start + up(S * 4) / 4;
    if (n_docs > 1) {  // device starts for the FFMA kernel, per-position bounds for the tensor-core one
        const cudaError_t e = launch_doc_tables(doc_starts, n_docs, S, docs_dev, doc_pos_start, doc_pos_end, st);
        if (e != cudaSuccess) return cuda_fail(e, "document bounds launch");
    }

    thread_local AttnParams p;
    std::memset(&p, 0, sizeof p);
    p.b = (int)b;
    p.hq = (int)q->shape[2];
    p.hkv = (int)Hkv;
    p.group = p.hq / p.hkv;
    p.d = (int)d;
    p.q_len = (int)c;
    p.kv_len = (int)S;
    p.n_ranks = N;
    p.step_begin = 0;
    p.step_end = 1;
    p.causal = causal;
    p.use_layout = 1;
    p.layout = layout;
    p.seq_len = S;
    p.kv_explicit = 1;
    p.kv_range = Range{0, 0, S, 0, 1};
    p.q_row_step = c;
    p.kv_row_step = 0;
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.n_qt = n_qt;
    p.doc_starts = n_docs > 1 ? docs_dev : nullptr;
    p.n_docs = n_docs > 1 ? n_docs : 0;
    p.doc_pos_start = doc_pos_start;
    // work order, heaviest (rank, row group) first: the key tiles each 128-row query
    // tile of the group walks, from the document start of its first row to its last
    // row (the document mask's bounds on the gathered block)
    {
        std::vector<std::pair<int64_t, uint32_t>> work;
        const int n_groups = (int)((c + rows - 1) / rows);
        auto doc_start = [&](int64_t pos) {  // the last start <= pos
            return *(std::upper_bound(doc_starts, doc_starts + n_docs, pos) - 1);
        };
        for (int i2 = 0; i2 < N; ++i2) {
            const Range qr = layout_range(layout, N, S, i2);
            for (int g = 0; g < n_groups; ++g) {
                int64_t tiles = 0;
                for (int64_t q_lo = (int64_t)g * rows; q_lo < std::min<int64_t>(c, (int64_t)(g + 1) * rows); q_lo += 128) {
                    const int64_t q_hi = std::min<int64_t>(q_lo + 127, c - 1);
                    const int64_t first = range_pos(qr, q_lo), last = range_pos(qr, q_hi);
                    const int64_t lo = causal ? doc_start(first) : 0, hi = causal ? last : S - 1;
                    tiles += hi / 128 - lo / 128 + 1;
                }
                work.push_back({tiles, ((uint32_t)i2 << 16) | (uint32_t)g});
            }
        }
        std::stable_sort(work.begin(), work.end(),
                         [](const std::pair<int64_t, uint32_t> &x, const std::pair<int64_t, uint32_t> &y) {
                             return x.first > y.first;
                         });
        if ((int64_t)work.size() <= kMaxOrder) {
            p.order_len = (int)work.size();
            for (size_t e2 = 0; e2 < work.size(); ++e2) p.order[e2] = work[e2].second;
        }
    }
    p.kv_map_h = (int)kv_map_h;
    fill_inputs(p, q, kv_in_place ? k : &kg, kv_in_place ? v : &vg);
    fill_outputs(p, EPI_STORE, o, lse);
    set_status_ptr(p);
    return launch_attn(p, q->dtype, st);
}

size_t cp_block_bwd_workspace_bytes(int64_t b, int64_t sq, int64_t Hq)
{
    if (b < 0 || sq < 0 || Hq < 0) return 0;
    // (lse, D) per query row, rows padded to the tensor-core kernel's query tile
    const int64_t lpad = (sq + kBwdQueryTile - 1) / kBwdQueryTile * kBwdQueryTile;
    return (size_t)((b * Hq * lpad * 8 + 255) / 256 * 256);
}

cp_status cp_block_attn_bwd(const cp_tensor *q, const cp_tensor *k, const cp_tensor *v, const cp_tensor *o,
                            const cp_tensor *lse, const cp_tensor *dout, const cp_range *q_range,
                            const cp_range *kv_range, int32_t mask_mode, float softmax_scale, cp_tensor *dq_acc,
                            cp_tensor *dk_acc, cp_tensor *dv_acc, void *workspace, size_t workspace_bytes,
                            void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK || (s = check_tensor(o, "o")) != CP_OK ||
        (s = check_tensor(dout, "dout")) != CP_OK || (s = check_tensor(dq_acc, "dq_acc")) != CP_OK ||
        (s = check_tensor(dk_acc, "dk_acc")) != CP_OK || (s = check_tensor(dv_acc, "dv_acc")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    if (mask_mode != CP_MASK_NONE && mask_mode != CP_MASK_CAUSAL) return fail(CP_ERR_INVALID_ARG, "unknown mask mode");
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t b = q->shape[0], sq = q->shape[1], sk = k->shape[1], Hq = q->shape[2];
    if (sq > INT32_MAX / 2 || sk > INT32_MAX / 2) return fail(CP_ERR_SHAPE, "sequence too long");
    if ((s = check_out(o, lse, q, sq, false)) != CP_OK) return s;
    if (o->dtype != q->dtype || dout->dtype != q->dtype || !same_shape(o, q) || !same_shape(dout, q))
        return fail(CP_ERR_SHAPE, "o and dout must be shaped like q, same dtype");
    if (!same_shape(dq_acc, q) || dq_acc->dtype != CP_FP32) return fail(CP_ERR_SHAPE, "dq_acc must be fp32 shaped like q");
    if (!same_shape(dk_acc, k) || dk_acc->dtype != CP_FP32 || !same_shape(dv_acc, k) || dv_acc->dtype != CP_FP32)
        return fail(CP_ERR_SHAPE, "dk_acc and dv_acc must be fp32 shaped like k");
    if ((s = check_range(q_range, sq, "q_range")) != CP_OK) return s;
    if ((s = check_range(kv_range, sk, "kv_range")) != CP_OK) return s;
    const size_t need = cp_block_bwd_workspace_bytes(b, sq, Hq);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (b == 0 || sq == 0 || sk == 0) return CP_OK;

    thread_local BwdParams p;
    std::memset(&p, 0, sizeof p);
    p.b = (int)b;
    p.hq = (int)Hq;
    p.hkv = (int)k->shape[2];
    p.group = p.hq / p.hkv;
    p.d = (int)q->shape[3];
    p.q_len = (int)sq;
    p.kv_len = (int)sk;
    p.n_ranks = 1;
    p.step_begin = 0;
    p.step_end = 1;
    p.causal = mask_mode == CP_MASK_CAUSAL;
    p.use_layout = 0;
    p.seq_len = 0;
    p.q_range = to_range(*q_range);
    p.kv_range = to_range(*kv_range);
    p.kv_explicit = 1;
    p.n_kv_blocks = 1;
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.q = q->data; p.k = k->data; p.v = v->data; p.o = o->data; p.dout = dout->data;
    p.q_sb = q->stride[0]; p.q_ss = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = k->stride[0]; p.k_ss = k->stride[1]; p.k_sh = k->stride[2];
    p.v_sb = v->stride[0]; p.v_ss = v->stride[1]; p.v_sh = v->stride[2];
    p.o_sb = o->stride[0]; p.o_ss = o->stride[1]; p.o_sh = o->stride[2];
    p.do_sb = dout->stride[0]; p.do_ss = dout->stride[1]; p.do_sh = dout->stride[2];
    p.lse = static_cast<const float *>(lse->data);
    p.lse_sb = lse->stride[0]; p.lse_sh = lse->stride[1]; p.lse_ss = lse->stride[2];
    p.stats = static_cast<float2 *>(workspace);
    p.lpad = (int)sq;
    p.dq = dq_acc->data; p.dk = dk_acc->data; p.dv = dv_acc->data;
    p.dq_sb = dq_acc->stride[0]; p.dq_ss = dq_acc->stride[1]; p.dq_sh = dq_acc->stride[2];
    p.dk_sb = dk_acc->stride[0]; p.dk_ss = dk_acc->stride[1]; p.dk_sh = dk_acc->stride[2];
    p.dv_sb = dv_acc->stride[0]; p.dv_ss = dv_acc->stride[1]; p.dv_sh = dv_acc->stride[2];
    p.accumulate = 1;
    cudaError_t e;
    if (q->dtype == CP_BF16 && q->shape[3] == 128) {
        // tensor cores: one launch over the key tiles, dQ reduced into dq_acc
        if ((s = check_rows16(dq_acc, "dq_acc")) != CP_OK || (s = check_rows16(dk_acc, "dk_acc")) != CP_OK ||
            (s = check_rows16(dv_acc, "dv_acc")) != CP_OK)
            return s;
        if ((s = check_rows16(o, "o")) != CP_OK || (s = check_rows16(dout, "dout")) != CP_OK) return s;
        const int64_t n_kt = (sk + kBwdKeyTile - 1) / kBwdKeyTile;
        if (n_kt > 65535) return fail(CP_ERR_SHAPE, "too many key tiles");
        p.lpad = (int)((sq + kBwdQueryTile - 1) / kBwdQueryTile * kBwdQueryTile);
        p.q_row_step = sq;
        p.kv_row_step = 0;
        p.dq_acc = static_cast<float *>(dq_acc->data);
        p.n_kt = (int)n_kt;
        p.order_len = 0;
        int *word = nullptr;
        if ((e = status_word(&word)) != cudaSuccess) return cuda_fail(e, "status word");
        p.status = word;
        e = launch_attn_bwd(p, static_cast<cudaStream_t>(stream));
    } else {
        e = launch_attn_bwd_simt(p, q->dtype == CP_FP32, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return CP_OK;
}

size_t cp_ring_bwd_workspace_bytes(int32_t layout, int32_t N, int32_t dtype, int64_t b, int64_t S, int64_t Hq,
                                   int64_t d)
{
    if (layout < 0 || layout > 2 || N < 1 || b < 0 || S < 0 || Hq < 0 || d < 0 || !elem_size(dtype)) return 0;
    if (S % N) return 0;
    const BwdWorkspace w = bwd_workspace(N, b, S, Hq, d);
    return (size_t)(w.stats_bytes + w.acc_bytes);
}

cp_status cp_ring_attn_bwd(int32_t layout, int32_t N, int32_t causal, const cp_tensor *q, const cp_tensor *k,
                           const cp_tensor *v, const cp_tensor *o, const cp_tensor *lse, const cp_tensor *dout,
                           float softmax_scale, cp_tensor *dq, cp_tensor *dk, cp_tensor *dv, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (causal != 0 && causal != 1) return fail(CP_ERR_INVALID_ARG, "causal must be 0 or 1");
    if ((s = check_tensor(q, "q")) != CP_OK || (s = check_tensor(k, "k")) != CP_OK ||
        (s = check_tensor(v, "v")) != CP_OK || (s = check_tensor(dout, "dout")) != CP_OK ||
        (s = check_tensor(dq, "dq")) != CP_OK || (s = check_tensor(dk, "dk")) != CP_OK ||
        (s = check_tensor(dv, "dv")) != CP_OK)
        return s;
    if ((s = check_attn_dtypes(q, k, v)) != CP_OK) return s;
    // bf16 with d = 128 runs on the tensor cores; fp32 (d 64 or 128) and bf16 with
    // d = 64 on the FFMA backward
    const cp_dtype dt = static_cast<cp_dtype>(q->dtype);
    const bool tc_path = dt == CP_BF16 && q->shape[3] == 128;
    if ((s = resolve_scale(&softmax_scale, q->shape[3])) != CP_OK) return s;
    const int64_t S = q->shape[1];
    if (k->shape[1] != S) return fail(CP_ERR_SHAPE, "q and k/v sequence lengths differ");
    if (N < 1 || N > 4096) return fail(CP_ERR_INVALID_ARG, "N must be in [1, 4096]");
    if (S >= ((int64_t)1 << 30)) return fail(CP_ERR_SHAPE, "sequence too long (S must be below 2^30)");
    if (S % N) return fail(CP_ERR_SHAPE, "S = %lld is not a multiple of N = %d", (long long)S, N);
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    NvtxRange call_range("cp_ring_attn_bwd");
    if ((s = check_out(o, lse, q, S, false)) != CP_OK) return s;
    if (o->dtype != dt) return fail(CP_ERR_INVALID_ARG, "o must have q's dtype");
    const cp_tensor *like_q[2] = {dout, dq};
    for (const cp_tensor *t : like_q) {
        if (!same_shape(t, q) || t->dtype != dt) return fail(CP_ERR_SHAPE, "dout and dq must be shaped like q, same dtype");
        if ((s = check_rows16(t, t == dq ? "dq" : "dout")) != CP_OK) return s;
    }
    const cp_tensor *like_k[2] = {dk, dv};
    for (const cp_tensor *t : like_k) {
        if (!same_shape(t, k) || t->dtype != dt) return fail(CP_ERR_SHAPE, "dk and dv must be shaped like k, same dtype");
        if ((s = check_rows16(t, t == dk ? "dk" : "dv")) != CP_OK) return s;
    }
    const int64_t c = S / N;
    const int64_t b = q->shape[0], Hq = q->shape[2], d = q->shape[3];
    const int64_t n_kt = (c + kBwdKeyTile - 1) / kBwdKeyTile;
    if (n_kt > 65535) return fail(CP_ERR_SHAPE, "too many key tiles per rank");
    const size_t need = cp_ring_bwd_workspace_bytes(layout, N, q->dtype, b, S, Hq, d);
    if (!workspace || workspace_bytes < need) return fail(CP_ERR_INVALID_ARG, "workspace of %zu bytes needed", need);
    if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CP_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (b == 0 || S == 0) return CP_OK;

    thread_local BwdParams p;
    std::memset(&p, 0, sizeof p);
    p.b = (int)b;
    p.hq = (int)Hq;
    p.hkv = (int)k->shape[2];
    p.group = p.hq / p.hkv;
    p.d = (int)d;
    p.q_len = (int)c;
    p.kv_len = (int)c;
    p.n_ranks = N;
    p.step_begin = 0;
    p.step_end = N;
    p.causal = causal;
    p.use_layout = 1;
    p.layout = layout;
    p.seq_len = S;
    p.q_row_step = c;
    p.kv_row_step = c;
    p.scale = softmax_scale;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.q = q->data; p.k = k->data; p.v = v->data; p.o = o->data; p.dout = dout->data;
    p.q_sb = q->stride[0]; p.q_ss = q->stride[1]; p.q_sh = q->stride[2];
    p.k_sb = k->stride[0]; p.k_ss = k->stride[1]; p.k_sh = k->stride[2];
    p.v_sb = v->stride[0]; p.v_ss = v->stride[1]; p.v_sh = v->stride[2];
    p.o_sb = o->stride[0]; p.o_ss = o->stride[1]; p.o_sh = o->stride[2];
    p.do_sb = dout->stride[0]; p.do_ss = dout->stride[1]; p.do_sh = dout->stride[2];
    p.lse = static_cast<const float *>(lse->data);
    p.lse_sb = lse->stride[0]; p.lse_sh = lse->stride[1]; p.lse_ss = lse->stride[2];
    const BwdWorkspace w = bwd_workspace(N, b, S, Hq, d);
    p.stats = static_cast<float2 *>(workspace);
    p.lpad = (int)w.lpad;
    p.dq_acc = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.stats_bytes);
    p.dq = dq->data; p.dk = dk->data; p.dv = dv->data;
    p.dq_sb = dq->stride[0]; p.dq_ss = dq->stride[1]; p.dq_sh = dq->stride[2];
    p.dk_sb = dk->stride[0]; p.dk_ss = dk->stride[1]; p.dk_sh = dk->stride[2];
    p.dv_sb = dv->stride[0]; p.dv_ss = dv->stride[1]; p.dv_sh = dv->stride[2];
    int *word = nullptr;
    status_word(&word);
    p.status = word;
    p.n_kt = (int)n_kt;
    p.n_kv_blocks = N;
    if (!tc_path) {
        cudaError_t e = launch_attn_bwd_simt(p, dt == CP_FP32, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
        return CP_OK;
    }
    set_bwd_order(p, layout, N, S, causal);
    // head-major grid once one head's work items fill a wave of the device
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    p.head_major = !kBwdNeverHeadMajor && (kBwdHeadMajor || (int64_t)N * n_kt >= (int64_t)sms);
    p.tile_rotation = p.head_major && bwd_tile_rotation(p.group, S, p.d, dev);
    e = launch_attn_bwd(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return CP_OK;
}

cp_status cp_layout_permute(int32_t layout, int32_t N, int32_t seq_axis, const cp_tensor *x, cp_tensor *x_ranked,
                            int32_t inverse, void *stream)
{
    g_last_error[0] = 0;
    cp_status s;
    if ((s = check_tensor(x, "x")) != CP_OK || (s = check_tensor(x_ranked, "x_ranked")) != CP_OK) return s;
    if (layout < 0 || layout > 2) return fail(CP_ERR_INVALID_ARG, "unknown layout %d", layout);
    if (seq_axis < 0 || seq_axis > 3) return fail(CP_ERR_INVALID_ARG, "seq_axis must be 0..3");
    if (inverse != 0 && inverse != 1) return fail(CP_ERR_INVALID_ARG, "inverse must be 0 or 1");
    if (x->dtype != x_ranked->dtype || !same_shape(x, x_ranked)) return fail(CP_ERR_SHAPE, "x and x_ranked differ");
    // both must be densely packed (row-major, no gaps)
    const cp_tensor *pair[2] = {x, x_ranked};
    for (const cp_tensor *t : pair) {
        int64_t expect = 1;
        for (int i = 3; i >= 0; --i) {
            if (t->shape[i] > 1 && t->stride[i] != expect) return fail(CP_ERR_INVALID_ARG, "tensors must be contiguous");
            expect *= t->shape[i];
        }
    }
    const int64_t S = x->shape[seq_axis];
    if (N < 1 || S % N) return fail(CP_ERR_SHAPE, "sequence axis length must be a multiple of N");
    if (layout == CP_LAYOUT_ZIGZAG && S % (2 * N)) return fail(CP_ERR_SHAPE, "zig-zag needs S to be a multiple of 2N");
    PermuteParams p;
    p.layout = layout;
    p.n_ranks = N;
    p.inverse = inverse;
    p.outer = 1;
    for (int i = 0; i < seq_axis; ++i) p.outer *= x->shape[i];
    p.seq = S;
    p.inner_bytes = elem_size(x->dtype);
    for (int i = seq_axis + 1; i < 4; ++i) p.inner_bytes *= x->shape[i];
    p.src = inverse ? x_ranked->data : x->data;
    p.dst = inverse ? x->data : x_ranked->data;
    if (p.outer * p.seq * p.inner_bytes == 0) return CP_OK;
    const char *a = static_cast<const char *>(p.src), *bptr = static_cast<const char *>(p.dst);
    const int64_t bytes = p.outer * p.seq * p.inner_bytes;
    if (a < bptr + bytes && bptr < a + bytes) return fail(CP_ERR_INVALID_ARG, "x and x_ranked overlap");
    cudaError_t e = launch_permute(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "permute launch");
    return CP_OK;
}

cp_status cp_selftest_wait_timeout(uint64_t limit_ns, void *stream)
{
    g_last_error[0] = 0;
    if (limit_ns < 1000000ull || limit_ns > 1000000000ull)
        return fail(CP_ERR_INVALID_ARG, "limit_ns must be in [1 ms, 1 s]");
    cudaError_t e = launch_wait_timeout_selftest(limit_ns, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
    return CP_OK;
}

cp_status cp_stream_check(void *stream)
{
    g_last_error[0] = 0;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int *word = nullptr;
    if ((e = status_word(&word)) != cudaSuccess) return cuda_fail(e, "status word");
    int h[2] = {0, 0};
    if ((e = cudaMemcpy(h, word, sizeof h, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e, "status read");
    if (h[0]) {
        const int zero[2] = {0, 0};
        cudaMemcpy(word, zero, sizeof zero, cudaMemcpyHostToDevice);
        if (h[0] & 2)
            return fail(CP_ERR_BOUNDS, "a bounds check of the debug build failed (status %d, first at check %d)", h[0],
                        h[1]);
        return fail(CP_ERR_TIMEOUT, "a device wait expired (status %d, first at wait tag %d)", h[0], h[1]);
    }
    return CP_OK;
}

}  // extern "C"
