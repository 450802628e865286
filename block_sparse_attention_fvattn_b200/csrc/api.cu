// api.cu -- the extern "C" boundary declared in include/fvattn.h.
//
// Validation mirrors the FastVideo VSA backend's acceptance rules (zskr.cn
// guide, section 5: bf16 tensors, equal Q/K/V head counts, no mask,
// non-causal equal-length self-attention, a block product of 256 -- or 64 on
// the (4,4,4) route; this library also takes 128 --, grid product == sequence
// length; section 3: top-k
// above num_blocks is rejected, top-k == num_blocks accepted). Where that
// backend falls back to SDPA, this library returns a status instead: it has
// no fallback path.
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "fvattn.h"
#include "internal.h"

namespace fvattn {

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(const Geo &g)
{
    WsLayout L;
    size_t off = align256(sizeof(WsHeader));
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    // with tc_scores both hold two planes (the TF32 head and rest of each mean)
    const size_t planes = g.tc_scores ? 2 : 1;
    L.qbar = take(planes * g.BH * g.nb * g.D * sizeof(float));
    L.kbarT = take(planes * g.BH * g.D * g.nbp * sizeof(float));
    L.scores = take(g.tc_scores ? (size_t)g.BH * g.nb * g.nbp * sizeof(float) : 0);
    L.unit_cost = take((size_t)g.BH * (g.nb + g.npair) * sizeof(int32_t));
    L.head_sorted = take((size_t)g.BH * (g.nb + 2) * sizeof(int32_t));
    L.head_len = take((size_t)g.BH * sizeof(int32_t));
    L.head_cost = take((size_t)g.BH * sizeof(int64_t));
    L.pair_cnt = take(g.paired ? (size_t)g.BH * g.npair * sizeof(int32_t) : 0);
    L.pair_list = take(g.paired ? (size_t)g.BH * g.npair * g.nb * sizeof(int32_t) : 0);
    L.aug_state = take(augment_state_bytes());
    L.aug_row_tie = take((size_t)g.BH * g.nb * sizeof(long long));
    L.total = off;
    return L;
}

// Resolve and check a problem. Returns FVATTN_OK with *g filled in.
static fvattn_status resolve(const fvattn_problem *p, Geo *g)
{
    if (!p) return FVATTN_ERR_INVALID_ARG;
    if (p->B < 0 || p->H < 0 || p->N < 1 || p->D < 1) return FVATTN_ERR_INVALID_ARG;
    if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1) return FVATTN_ERR_INVALID_ARG;
    if (p->blk_t < 1 || p->blk_h < 1 || p->blk_w < 1) return FVATTN_ERR_INVALID_ARG;
    if ((long long)p->grid_t * p->grid_h * p->grid_w != (long long)p->N) return FVATTN_ERR_INVALID_ARG;
    if (isnan(p->softmax_scale) || isinf(p->softmax_scale)) return FVATTN_ERR_INVALID_ARG;
    if (p->D != 64 && p->D != 128) return FVATTN_ERR_UNSUPPORTED;
    if (p->dtype != FVATTN_DTYPE_BF16 && p->dtype != FVATTN_DTYPE_F16) return FVATTN_ERR_UNSUPPORTED;
    const long long bp = (long long)p->blk_t * p->blk_h * p->blk_w;
    if (!(bp == 256 && p->blk_t % 2 == 0) && bp != 128 && bp != 64) return FVATTN_ERR_UNSUPPORTED;
    if (p->blk_w > 256 || p->blk_h > 256 || p->blk_t > 256) return FVATTN_ERR_UNSUPPORTED;
    // the attention kernel keeps one column mask per extent along each block axis
    if (p->blk_w + p->blk_h + (bp == 256 ? p->blk_t / 2 : p->blk_t) > 40) return FVATTN_ERR_UNSUPPORTED;
    Geo G;
    G.B = p->B;
    G.H = p->H;
    G.N = p->N;
    G.D = p->D;
    G.f16 = p->dtype == FVATTN_DTYPE_F16 ? 1 : 0;
    G.T = p->grid_t;
    G.Hg = p->grid_h;
    G.W = p->grid_w;
    G.bt = p->blk_t;
    G.bh = p->blk_h;
    G.bw = p->blk_w;
    G.nbt = ceil_div(G.T, G.bt);
    G.nbh = ceil_div(G.Hg, G.bh);
    G.nbw = ceil_div(G.W, G.bw);
    const long long nb = (long long)G.nbt * G.nbh * G.nbw;
    if (nb > kMaxBlocks) return FVATTN_ERR_UNSUPPORTED;
    G.nb = (int)nb;
    const long long bh = (long long)G.B * G.H;
    if (bh > 65535) return FVATTN_ERR_UNSUPPORTED;
    G.BH = (int)bh;
    G.nbp = (G.nb + 3) & ~3;
    if (bp == 256) {
        // two 128-row sub-tiles per block, the halves along t
        G.subt = G.bt / 2;
        G.nsub = 2;
        G.rows = 128;
    } else if (bp == 128) {
        // one 128-row sub-tile per block: one query tile per unit
        G.subt = G.bt;
        G.nsub = 1;
        G.rows = 128;
    } else {
        // 64-token blocks: two query blocks share a 128-row tile (paired)
        G.subt = G.bt;
        G.nsub = 1;
        G.rows = 64;
    }
    G.tc_scores = G.nb >= kTcScoresMinBlocks ? 1 : 0;
    G.paired = G.rows == 64;
    G.npair = G.paired ? ceil_div(G.nb, 2) : 0;
    G.upb = G.paired ? ceil_div(G.nb, 4) : G.nb;
    G.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf((float)G.D);
    G.fd_nbw = make_fastdiv((uint32_t)G.nbw);
    G.fd_hw = make_fastdiv((uint32_t)(G.nbh * G.nbw));
    *g = G;
    return FVATTN_OK;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
static bool aligned4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

static int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
}

static fvattn_status check_ws(const Geo &g, const void *ws, size_t ws_bytes)
{
    if (!ws || !aligned16(ws)) return FVATTN_ERR_WORKSPACE;
    if (ws_bytes < ws_layout(g).total) return FVATTN_ERR_WORKSPACE;
    return FVATTN_OK;
}

}  // namespace fvattn

using namespace fvattn;

extern "C" {

int32_t fvattn_num_blocks(const fvattn_problem *prob)
{
    Geo g;
    if (resolve(prob, &g) != FVATTN_OK) return -1;
    return g.nb;
}

int32_t fvattn_default_num_ctas(void) { return num_sms(); }

size_t fvattn_workspace_size(const fvattn_problem *prob, int32_t num_ctas)
{
    (void)num_ctas;
    Geo g;
    if (resolve(prob, &g) != FVATTN_OK) return 0;
    return ws_layout(g).total;
}

fvattn_status fvattn_workspace_init(void *ws, size_t ws_bytes, fvattn_stream_t stream)
{
    if (!ws || ws_bytes < sizeof(WsHeader) || !aligned16(ws)) return FVATTN_ERR_WORKSPACE;
    if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream) != cudaSuccess) return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_route(const fvattn_problem *prob, const void *q, const void *k, float p, int32_t k_min,
                           int32_t *kv_cnt, int32_t *kv_idx, float *block_probs, void *ws, size_t ws_bytes,
                           fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (!(p > 0.f && p <= 1.f)) return FVATTN_ERR_INVALID_ARG;  // also rejects NaN
    if (k_min < 1 || k_min > g.nb) return FVATTN_ERR_INVALID_ARG;
    if (!q || !k || !aligned16(q) || !aligned16(k)) return FVATTN_ERR_INVALID_ARG;
    if (!kv_cnt || !kv_idx || !aligned4(kv_cnt) || !aligned4(kv_idx)) return FVATTN_ERR_INVALID_ARG;
    if (block_probs && !aligned4(block_probs)) return FVATTN_ERR_INVALID_ARG;
    st = check_ws(g, ws, ws_bytes);
    if (st != FVATTN_OK) return st;
    if (g.BH == 0) return FVATTN_OK;
    const WsLayout L = ws_layout(g);
    uint8_t *w = static_cast<uint8_t *>(ws);
    float *qbar = reinterpret_cast<float *>(w + L.qbar);
    float *kbarT = reinterpret_cast<float *>(w + L.kbarT);
    uint32_t *status = reinterpret_cast<uint32_t *>(w);
    cudaStream_t s = (cudaStream_t)stream;
    float *scores = g.tc_scores ? reinterpret_cast<float *>(w + L.scores) : nullptr;
    if (launch_pool(g, q, k, qbar, kbarT, s) != cudaSuccess) return FVATTN_ERR_CUDA;
    // the TF32 planes of each head: hi at the head's start, lo one plane later
    if (scores && launch_score_gemm(g, qbar, qbar + (size_t)g.nb * g.D, kbarT, kbarT + (size_t)g.nbp * g.D, scores,
                                    status, s) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    if (launch_score_select(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, block_probs, status, s) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_schedule(const fvattn_problem *prob, const int32_t *kv_cnt, const int32_t *kv_idx,
                              int32_t dense, int32_t num_ctas, int32_t *work, int32_t *cta_range,
                              int64_t *cta_cost, void *ws, size_t ws_bytes, fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (num_ctas < 0 || num_ctas > kMaxCtas) return FVATTN_ERR_INVALID_ARG;
    if (!dense && (!kv_cnt || !kv_idx)) return FVATTN_ERR_INVALID_ARG;
    if (!work || !cta_range) return FVATTN_ERR_INVALID_ARG;
    st = check_ws(g, ws, ws_bytes);
    if (st != FVATTN_OK) return st;
    if (num_ctas == 0) {
        num_ctas = num_sms();
        if (num_ctas <= 0) return FVATTN_ERR_CUDA;
    }
    cudaStream_t s = (cudaStream_t)stream;
    if (g.BH == 0) {
        if (cudaMemsetAsync(cta_range, 0, sizeof(int32_t) * (size_t)(num_ctas + 1), s) != cudaSuccess)
            return FVATTN_ERR_CUDA;
        if (cta_cost && cudaMemsetAsync(cta_cost, 0, sizeof(int64_t) * (size_t)num_ctas, s) != cudaSuccess)
            return FVATTN_ERR_CUDA;
        return FVATTN_OK;
    }
    const WsLayout L = ws_layout(g);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *pair_cnt = reinterpret_cast<int32_t *>(w + L.pair_cnt);
    // paired mode: the unions of the pairs' lists are the attention's work
    // lists; build them here (the costs need their sizes) for fvattn_sparse_attn
    if (g.paired && !dense &&
        launch_pair_lists(g, kv_cnt, kv_idx, pair_cnt, reinterpret_cast<int32_t *>(w + L.pair_list), s) !=
            cudaSuccess)
        return FVATTN_ERR_CUDA;
    if (launch_schedule(g, kv_cnt, kv_idx, dense ? 1 : 0, num_ctas, work, cta_range, cta_cost,
                        reinterpret_cast<int32_t *>(w + L.unit_cost), reinterpret_cast<int32_t *>(w + L.head_sorted),
                        reinterpret_cast<int32_t *>(w + L.head_len), reinterpret_cast<int64_t *>(w + L.head_cost),
                        pair_cnt, s) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_sparse_attn(const fvattn_problem *prob, const void *q, const void *k, const void *v,
                                 const int32_t *kv_cnt, const int32_t *kv_idx, const int32_t *work,
                                 const int32_t *cta_range, int32_t num_ctas, int32_t dense, void *out,
                                 int64_t *cta_ns, void *ws, size_t ws_bytes, fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (!q || !k || !v || !out) return FVATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FVATTN_ERR_INVALID_ARG;
    if (!dense && (!kv_cnt || !kv_idx)) return FVATTN_ERR_INVALID_ARG;
    if ((work == nullptr) != (cta_range == nullptr)) return FVATTN_ERR_INVALID_ARG;
    if (num_ctas < 0 || num_ctas > kMaxCtas) return FVATTN_ERR_INVALID_ARG;
    st = check_ws(g, ws, ws_bytes);
    if (st != FVATTN_OK) return st;
    if (num_ctas == 0) {
        num_ctas = num_sms();
        if (num_ctas <= 0) return FVATTN_ERR_CUDA;
    }
    if (g.BH == 0) return FVATTN_OK;
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    const WsLayout L = ws_layout(g);
    uint8_t *w = static_cast<uint8_t *>(ws);
    int32_t *pair_cnt = reinterpret_cast<int32_t *>(w + L.pair_cnt);
    int32_t *pair_list = reinterpret_cast<int32_t *>(w + L.pair_list);
    cudaStream_t s = (cudaStream_t)stream;
    // paired mode without work lists: no fvattn_schedule built the pair lists
    if (g.paired && !dense && !work && launch_pair_lists(g, kv_cnt, kv_idx, pair_cnt, pair_list, s) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    int kind = 0;
    if (launch_attn(g, q, k, v, kv_cnt, kv_idx, pair_cnt, pair_list, work, cta_range, num_ctas, dense ? 1 : 0, out,
                    cta_ns, status, s, &kind) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_head_cost(const fvattn_problem *prob, const int32_t *kv_cnt, const int32_t *kv_idx,
                               int32_t dense, int64_t *head_cost, fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (!head_cost || (!dense && (!kv_cnt || !kv_idx))) return FVATTN_ERR_INVALID_ARG;
    if (!aligned4(kv_cnt) || !aligned4(kv_idx) || ((uintptr_t)head_cost & 7u)) return FVATTN_ERR_INVALID_ARG;
    if (g.BH == 0) return FVATTN_OK;
    if (launch_head_cost(g, kv_cnt, kv_idx, dense ? 1 : 0, head_cost, (cudaStream_t)stream) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_augment(const fvattn_problem *prob, const float *block_probs, int64_t budget, int32_t *kv_cnt,
                             int32_t *kv_idx, int64_t *added_pairs, double *added_mass, void *ws, size_t ws_bytes,
                             fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (budget < 0 || !block_probs || !kv_cnt || !kv_idx) return FVATTN_ERR_INVALID_ARG;
    if (!aligned4(block_probs) || !aligned4(kv_cnt) || !aligned4(kv_idx)) return FVATTN_ERR_INVALID_ARG;
    if (((uintptr_t)added_pairs & 7u) || ((uintptr_t)added_mass & 7u)) return FVATTN_ERR_INVALID_ARG;
    st = check_ws(g, ws, ws_bytes);
    if (st != FVATTN_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (g.BH == 0) {
        if (added_pairs && cudaMemsetAsync(added_pairs, 0, sizeof(int64_t), s) != cudaSuccess) return FVATTN_ERR_CUDA;
        if (added_mass && cudaMemsetAsync(added_mass, 0, sizeof(double), s) != cudaSuccess) return FVATTN_ERR_CUDA;
        return FVATTN_OK;
    }
    const WsLayout L = ws_layout(g);
    uint8_t *w = static_cast<uint8_t *>(ws);
    if (launch_augment(g, block_probs, (long long)budget, kv_cnt, kv_idx, w + L.aug_state,
                       reinterpret_cast<long long *>(w + L.aug_row_tie),
                       reinterpret_cast<unsigned long long *>(added_pairs), added_mass, s) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_set_wait_limit(void *ws, size_t ws_bytes, uint64_t limit_ns, fvattn_stream_t stream)
{
    if (!ws || ws_bytes < sizeof(WsHeader) || !aligned16(ws)) return FVATTN_ERR_WORKSPACE;
    if (launch_header_write(static_cast<uint32_t *>(ws), kHdrWaitLimit, limit_ns, (cudaStream_t)stream) !=
        cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_test_withhold_unit(void *ws, size_t ws_bytes, int32_t rank, fvattn_stream_t stream)
{
    if (!ws || ws_bytes < sizeof(WsHeader) || !aligned16(ws)) return FVATTN_ERR_WORKSPACE;
    if (rank < -1) return FVATTN_ERR_INVALID_ARG;
    if (launch_header_write(static_cast<uint32_t *>(ws), -kHdrWithhold, (uint64_t)(uint32_t)(rank + 1),
                            (cudaStream_t)stream) != cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}

fvattn_status fvattn_read_device_status(void *ws, fvattn_stream_t stream, uint32_t *flags)
{
    if (!ws || !flags) return FVATTN_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t host = 0;
    if (cudaMemcpyAsync(&host, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FVATTN_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return FVATTN_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return FVATTN_ERR_CUDA;
    *flags = host;
    return FVATTN_OK;
}

const char *fvattn_status_string(fvattn_status s)
{
    switch (s) {
    case FVATTN_OK: return "ok";
    case FVATTN_ERR_INVALID_ARG: return "invalid argument";
    case FVATTN_ERR_UNSUPPORTED: return "unsupported problem shape";
    case FVATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case FVATTN_ERR_CUDA: return "CUDA call failed";
    case FVATTN_STATUS_NONFINITE: return "non-finite block scores were repaired";
    case FVATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    }
    return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Routing without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc at the point where they route: a
// runtime that hands a plug-in only its input and output tensors, code that
// runs under a memory-pool reservation that must not grow, or a process that
// fixes its device footprint at start-up. For them the routing scratch -- the
// status word and the pooled block means of Q and K -- lives in one array
// compiled into this library, sized kNoAllocScratchBytes. Every GPU that
// loads the library holds that array until the process exits. The scores are
// always computed on the CUDA cores in fp32 here (the fixed array has no room
// for a score matrix), so from kTcScoresMinBlocks blocks on the lists can
// differ from fvattn_route's (which then uses the TF32 tensor-core split)
// where two blocks' scores lie within fp32 rounding of each other.
#include <mutex>

namespace fvattn {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device
static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

namespace {
// The array's name in host code is only a stand-in for the device symbol;
// kernels must get its device address, which cudaGetSymbolAddress returns for
// the context current on the calling thread. Each context (a device's primary
// context, or a context the caller made current itself) has its own copy, so
// the address is cached per context, keyed on the context's process-unique id
// (cuCtxGetId): a context created later -- for example after cudaDeviceReset
// -- gets a new id and a fresh lookup, never a stale address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct ScratchEntry {
    unsigned long long ctx_id;
    void *addr;
};
constexpr int kMaxContexts = 64;
std::mutex g_scratch_mu;
ScratchEntry g_scratch_cache[kMaxContexts];
int g_scratch_cached = 0;

template <class Fn>
Fn driver_fn(const char *name)
{
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<Fn>(p);
}

cudaError_t route_scratch_address(void **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    unsigned long long id = 0;
    bool have_id = false;
    CUcontext ctx = nullptr;
    if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx && get_id(ctx, &id) == CUDA_SUCCESS)
        have_id = true;
    if (have_id) {
        for (int i = 0; i < g_scratch_cached; ++i) {
            if (g_scratch_cache[i].ctx_id == id) {
                *out = g_scratch_cache[i].addr;
                return cudaSuccess;
            }
        }
    }
    // first call in this context (with its device current): look the array up;
    // with lazy module loading this also loads the library's device code and
    // maps the array
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    if (!have_id && get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
        get_id(ctx, &id) == CUDA_SUCCESS)
        have_id = true;  // the lookup above made the primary context current
    if (have_id && g_scratch_cached < kMaxContexts) g_scratch_cache[g_scratch_cached++] = ScratchEntry{id, p};
    *out = p;
    return cudaSuccess;
}
}  // namespace

}  // namespace fvattn

extern "C" fvattn_status fvattn_route_noalloc(const fvattn_problem *prob, const void *q, const void *k, float p,
                                              int32_t k_min, int32_t *kv_cnt, int32_t *kv_idx, float *block_probs,
                                              fvattn_stream_t stream)
{
    Geo g;
    fvattn_status st = resolve(prob, &g);
    if (st != FVATTN_OK) return st;
    if (!(p > 0.f && p <= 1.f)) return FVATTN_ERR_INVALID_ARG;
    if (k_min < 1 || k_min > g.nb) return FVATTN_ERR_INVALID_ARG;
    if (!q || !k || !aligned16(q) || !aligned16(k)) return FVATTN_ERR_INVALID_ARG;
    if (!kv_cnt || !kv_idx || !aligned4(kv_cnt) || !aligned4(kv_idx)) return FVATTN_ERR_INVALID_ARG;
    if (block_probs && !aligned4(block_probs)) return FVATTN_ERR_INVALID_ARG;
    g.tc_scores = 0;  // the fixed scratch holds no score matrix: scores on the CUDA cores
    const WsLayout L = ws_layout(g);
    const size_t needed = L.kbarT + (size_t)g.BH * g.D * g.nbp * sizeof(float);
    if (needed > kNoAllocScratchBytes) return FVATTN_ERR_WORKSPACE;
    if (g.BH == 0) return FVATTN_OK;
    void *scratch = nullptr;
    if (route_scratch_address(&scratch) != cudaSuccess) return FVATTN_ERR_CUDA;
    uint8_t *w = static_cast<uint8_t *>(scratch);
    // Pooled means are written in full before they are read, so nothing needs
    // clearing; the status word only collects flags nobody reads back here.
    cudaStream_t s = (cudaStream_t)stream;
    if (launch_pool(g, q, k, reinterpret_cast<float *>(w + L.qbar), reinterpret_cast<float *>(w + L.kbarT), s) !=
        cudaSuccess)
        return FVATTN_ERR_CUDA;
    if (launch_score_select(g, reinterpret_cast<float *>(w + L.qbar), reinterpret_cast<float *>(w + L.kbarT),
                            nullptr, p, k_min, kv_cnt, kv_idx, block_probs, reinterpret_cast<uint32_t *>(w), s) !=
        cudaSuccess)
        return FVATTN_ERR_CUDA;
    return FVATTN_OK;
}
