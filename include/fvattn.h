/*
 * fvattn.h -- C ABI of the B200 (sm_100a) adaptive block-sparse attention path.
 *
 * The method (FVAttn, "Adaptive Sparse Attention with Runtime Load Balancing
 * for Video Generation"; ai-feeds.com summary and hotpaper.ai abstract) routes
 * each query block of a video DiT's self-attention to a Top-p set of key/value
 * blocks with a Top-k safety floor over video-aware spatio-temporal blocks,
 * repairs the mask, balances the resulting uneven per-head work, and runs
 * attention only over the kept blocks. This library implements the
 * single-GPU data path of that method in three calls:
 *
 *   fvattn_route        block pooling, block scores, softmax, Top-p + Top-k
 *                       floor, mask repair, compact per-(head, query block)
 *                       key/value block lists
 *   fvattn_schedule     longest-first, balanced work lists for persistent CTAs
 *   fvattn_sparse_attn  FlashAttention-style online-softmax attention over the
 *                       kept blocks only (or every block: dense mode)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors.  Q, K, V and O are bf16 or fp16 (fvattn_problem.dtype), contiguous,
 *   [B, H, N, D] (row-major, D innermost). Attention runs the products on the
 *   tensor cores in that type with fp32 accumulation; P is rounded to it too. Token n of a head sits at latent position (t, y, x) with
 *   n = (t * grid_h + y) * grid_w + x (raster order, T slowest), as in the
 *   FastVideo VSA backend's (T, H, W) post-patch latent grid (zskr.cn guide,
 *   section 1). Q and KV have the same length (non-causal self-attention,
 *   zskr.cn guide, section 1) and the same head count (no GQA/MQA, section 5).
 * Blocks.  The grid is cut into (blk_t, blk_h, blk_w) blocks; the block count
 *   is nb = ceil(T/bt) * ceil(H/bh) * ceil(W/bw) (zskr.cn guide, section 3:
 *   (31,22,40) with (4,8,8) gives 8*3*5 = 120). Block j = (jt*nbh + jy)*nbw + jx.
 *   Edge blocks hold fewer valid tokens; padded positions never act as keys
 *   and never produce output (section 6, packed [real, pad] contract).
 *   Supported: blk_t*blk_h*blk_w == 256 with blk_t even (the 256-token route,
 *   e.g. (4,8,8)), == 64 (the 64-token (4,4,4) route, section 1), or == 128
 *   (e.g. (2,8,8): one 128-row query tile per block, which leaves one of the
 *   attention kernel's two softmax warpgroups idle -- correct, about half the
 *   throughput of the other routes); blk_w + blk_h + (blk_t, or blk_t/2 for
 *   256-token blocks) <= 40; D in {64, 128}; nb <= 2048; B*H <= 65535.
 * Pointers.  Device pointers unless stated; 16-byte aligned. The caller owns
 *   every buffer. The library allocates no device memory; the only state it
 *   keeps is per-device function attributes and a cached driver entry point.
 * Streams.  Every call is asynchronous on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream). Argument errors are returned synchronously,
 *   before anything is enqueued. No call synchronises with the host except
 *   fvattn_read_device_status.
 * Workspace.  One caller-owned device buffer of fvattn_workspace_size() bytes
 *   serves all three calls of one problem; fvattn_workspace_init must run on
 *   it once before first use. It holds the sticky device status word, the
 *   pooled block means and the scheduler's scratch. Calls that share a
 *   workspace must be ordered on one stream.
 * Device-detected conditions (non-finite block scores, a bounded wait that
 *   ran out) never trap: kernels OR a flag into the workspace status word,
 *   which fvattn_read_device_status returns.
 */
#ifndef FVATTN_H
#define FVATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FVATTN_API __attribute__((visibility("default")))
#else
#define FVATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA header. */
typedef struct CUstream_st *fvattn_stream_t;

typedef enum fvattn_status {
    FVATTN_OK = 0,
    FVATTN_ERR_INVALID_ARG = 1,   /* a size, pointer, p or k_min out of range */
    FVATTN_ERR_UNSUPPORTED = 2,   /* valid problem outside the supported shapes */
    FVATTN_ERR_WORKSPACE = 3,     /* workspace NULL or smaller than required */
    FVATTN_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    FVATTN_STATUS_NONFINITE = 5,  /* device flag: a score row was not finite and was repaired */
    FVATTN_ERR_TIMEOUT = 6        /* device flag: a bounded wait inside a kernel gave up */
} fvattn_status;

/* Device status word bits (as returned, combined, by fvattn_read_device_status). */
#define FVATTN_FLAG_NONFINITE 0x1u
#define FVATTN_FLAG_TIMEOUT 0x2u
/* a schedule entry, unit id or list size was out of range (work lists not
 * made by fvattn_schedule for this problem, or corrupted): the attention
 * kernel stopped taking units and part of `out` is not written */
#define FVATTN_FLAG_BAD_WORK 0x4u

/* Element type of Q, K, V and O (the FastVideo VSA backend accepts both,
 * zskr.cn guide, section 5). */
#define FVATTN_DTYPE_BF16 0
#define FVATTN_DTYPE_F16 1

typedef struct fvattn_problem {
    int32_t B, H, N, D;               /* batch, heads, tokens (= T*Hg*W), head dim */
    int32_t grid_t, grid_h, grid_w;   /* latent grid (T, H, W) */
    int32_t blk_t, blk_h, blk_w;      /* block shape */
    float softmax_scale;              /* <= 0 selects 1/sqrt(D); used for routing and attention */
    int32_t dtype;                    /* FVATTN_DTYPE_BF16 or FVATTN_DTYPE_F16; other values: UNSUPPORTED */
} fvattn_problem;

/* nb = ceil(T/bt)*ceil(H/bh)*ceil(W/bw), or -1 if the problem is invalid. */
FVATTN_API int32_t fvattn_num_blocks(const fvattn_problem *prob);

/* Number of SMs of the current device (the default persistent-CTA count), or -1. */
FVATTN_API int32_t fvattn_default_num_ctas(void);

/* Bytes of workspace the three calls need for `prob` with `num_ctas` persistent
 * CTAs (0 = fvattn_default_num_ctas()). Returns 0 if the problem is invalid. */
FVATTN_API size_t fvattn_workspace_size(const fvattn_problem *prob, int32_t num_ctas);

/* Zero the workspace header: the status word and the work counters the
 * kernels use (the kernels leave the counters at zero when they finish).
 * Asynchronous. */
FVATTN_API fvattn_status fvattn_workspace_init(void *ws, size_t ws_bytes, fvattn_stream_t stream);

/*
 * fvattn_route -- the sparse-routing frontend (ai-feeds.com FVAttn summary,
 * "Key modules" 1: Top-p routing with a Top-k safety floor over video-aware
 * blocks, runtime mask repair; hotpaper.ai abstract; zskr.cn guide, section 1:
 * block-level scores select key/value blocks per query block).
 *
 * For every (b, h, query block i):
 *   Qbar_i, Kbar_j = means of Q, K over the valid tokens of the block;
 *   s[j] = scale * dot(Qbar_i, Kbar_j);  P = softmax(s);
 *   rank blocks by P descending (= s descending), equal scores by lower j;
 *   m_p = smallest m whose inclusive cumulative P reaches p (p >= 1: nb);
 *   m = min(nb, max(m_p, k_min)); S_i = first m ranked blocks plus block i;
 *   a row with a non-finite score keeps every block and sets FLAG_NONFINITE.
 *
 *   q, k          [B,H,N,D] in the problem's element type (bf16 or fp16)
 *   p             Top-p threshold, 0 < p <= 1
 *   k_min         Top-k floor, 1 <= k_min <= nb (k_min > nb is INVALID_ARG,
 *                 k_min == nb keeps every block, like VSA's topk rules,
 *                 zskr.cn guide, section 3)
 *   kv_cnt        out int32 [B,H,nb]      |S_i|
 *   kv_idx        out int32 [B,H,nb,nb]   S_i ascending in the first kv_cnt
 *                 entries of each row; the rest of the row is left untouched
 *   block_probs   out fp32 [B,H,nb,nb] P in block order, or NULL
 *   ws, ws_bytes  workspace
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE (synchronous); CUDA on a failed
 * launch.
 */
FVATTN_API fvattn_status fvattn_route(const fvattn_problem *prob, const void *q, const void *k,
                           float p, int32_t k_min, int32_t *kv_cnt, int32_t *kv_idx,
                           float *block_probs, void *ws, size_t ws_bytes, fvattn_stream_t stream);

/*
 * fvattn_schedule -- longest-first balanced work lists for the persistent
 * attention CTAs: the single-GPU analogue of the method's per-head load
 * problem (ai-feeds.com summary: per-head workload heterogeneity makes the
 * heaviest rank the critical path; Runtime Load Balancing moves heavy heads
 * to shorten it; load imbalance = max/mean, ideal 1.0).
 *
 * A work unit is one (b, h, query block i). Its cost is the number of
 * (128-row query tile, key/value sub-tile) pairs the attention kernel runs for
 * it. With 64-token blocks the attention runs query blocks (2p, 2p+1) as one
 * 128-row tile over the union of their two kept lists, two key blocks per
 * step; a unit is then four query blocks 4q .. 4q+3 (two such tiles), its id
 * u = (b*H + h)*ceil(nb/4) + q, and its cost the two tiles' steps. A unit of
 * at least 64 steps is split (not in dense mode): it becomes one unit per
 * pair p, id B*H*ceil(nb/4) + (b*H + h)*ceil(nb/2) + p, which both halves of
 * the attention kernel run over the two halves of the pair's union, so the
 * longest units are half as long. The number of units is cta_range[num_ctas].
 * For that case this call also writes the unions into the workspace, where
 * fvattn_sparse_attn reads them: give both calls the same workspace.
 * Units are ordered heads by total cost descending, then units within a
 * head by cost descending (ties: lower index); rank r goes to CTA
 * zigzag(r) = r mod 2C < C ? r mod C : 2C-1 - r mod C, so each round of C
 * consecutive ranks (one head's units run together, which keeps its key/value
 * blocks in L2) gives every CTA one unit, alternating the largest end.
 * cta_cost is the cost of that static deal; fvattn_sparse_attn runs the same
 * ranked order dynamically (see there), which evens out what the cost model
 * misses.
 *
 *   kv_cnt, kv_idx  the lists from fvattn_route (ignored if dense != 0)
 *   dense           nonzero: schedule the all-blocks problem
 *   num_ctas        persistent CTAs (0 = SM count)
 *   work            out int32 [B*H*nb]    unit ids u = (b*H + h)*nb + i, grouped by CTA
 *                                         (64-token blocks: the ids above; the first
 *                                         cta_range[num_ctas] entries are written)
 *   cta_range       out int32 [num_ctas+1] CTA c runs work[cta_range[c] .. cta_range[c+1])
 *   cta_cost        out int64 [num_ctas]  predicted cost per CTA, or NULL
 */
FVATTN_API fvattn_status fvattn_schedule(const fvattn_problem *prob, const int32_t *kv_cnt,
                              const int32_t *kv_idx, int32_t dense, int32_t num_ctas,
                              int32_t *work, int32_t *cta_range, int64_t *cta_cost,
                              void *ws, size_t ws_bytes, fvattn_stream_t stream);

/*
 * fvattn_sparse_attn -- block-sparse attention over the kept blocks (the
 * source of the method's 4.41x attention speedup over FlashAttention,
 * ai-feeds.com summary "Key findings"; zskr.cn guide, section 1: attention is
 * computed only for the selected key/value blocks of each query block).
 *
 * For every valid query token r of block i: o_r = sum over the valid tokens k
 * of the blocks in S_i of softmax_k(scale * q_r . k_k) * v_k, computed with an
 * online softmax over 128-token key/value tiles (64-token blocks: two key
 * blocks per tile, shared by two query blocks, each of which masks the key
 * blocks it did not keep).
 * dense != 0 uses every block (the VSA_ALL_BLOCKS route, section 3/5), giving
 * the in-library dense comparison.
 *
 *   q, k, v        [B,H,N,D] in the problem's element type (bf16 or fp16)
 *   kv_cnt, kv_idx lists from fvattn_route (ignored if dense)
 *   work, cta_range from fvattn_schedule with the same num_ctas, dense flag
 *                  and workspace (both NULL: units in index order; with
 *                  64-token blocks the call then builds the pair unions in the
 *                  workspace itself, one extra kernel). The CTAs take ranks
 *                  0, 1, 2, ... of the scheduler's longest-first order from a
 *                  counter shared through the workspace (rank r is entry
 *                  r / num_ctas of list zigzag(r)), so a CTA that finishes early
 *                  takes the next unit; the last CTA resets the counter.
 *   num_ctas       grid size (0 = SM count); must match fvattn_schedule's
 *   out            [B,H,N,D] in the same element type; every valid token is
 *                  written (TMA tile stores of whole 128-byte lines), nothing
 *                  else is touched. It must not overlap q, k or v: other CTAs
 *                  still read those while a tile of out is stored (not checked).
 *   cta_ns         out int64 [num_ctas] busy time of each CTA in ns, or NULL
 */
FVATTN_API fvattn_status fvattn_sparse_attn(const fvattn_problem *prob, const void *q, const void *k,
                                 const void *v, const int32_t *kv_cnt, const int32_t *kv_idx,
                                 const int32_t *work, const int32_t *cta_range, int32_t num_ctas,
                                 int32_t dense, void *out, int64_t *cta_ns,
                                 void *ws, size_t ws_bytes, fvattn_stream_t stream);

/*
 * fvattn_route_noalloc -- fvattn_route for callers that cannot allocate device
 * memory. The paper has no counterpart; it is a deployment convenience.
 *
 * Some callers cannot call cudaMalloc where they route: a runtime that hands
 * a plug-in only its input and output tensors, code running under a memory
 * pool reservation that must not grow, or a process whose device footprint
 * is fixed at start-up. This entry point computes the same routing as
 * fvattn_route, with the same arguments except the workspace, with one
 * difference: its block scores are always fp32 dot products on the CUDA
 * cores, where fvattn_route scores rows of 320 or more blocks with a TF32
 * split on the tensor cores; on such rows a block whose score lies within
 * fp32 rounding of the boundary block's can land on the other side. Its
 * scratch (the pooled block means of Q and K) lives in a fixed 16 MiB array
 * inside this library, which every GPU that loads the library holds until
 * the process exits. The call allocates nothing (no cudaMalloc/cudaFree, no
 * allocating library routine).
 *   Limit: 4*(B*H*nb*D + B*H*D*round_up(nb,4)) plus 256 bytes must fit in
 *   16 MiB (e.g. 24 heads x 120 blocks at D=128, or 40 x 360); larger problems
 *   return FVATTN_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: the first call in each CUDA context (normally once per device)
 *   looks up the array's device address with that device current and caches
 *   it per context (keyed on the context's unique id, so a context made after
 *   cudaDeviceReset gets a fresh lookup). With lazy module loading, the CUDA
 *   default, that first call also loads this library's device code and maps
 *   the 16 MiB array: a caller whose device footprint must not grow later
 *   should make one call at start-up, and before any stream capture.
 *   Sharing: every call on a device uses the same array, so calls that can
 *   overlap on the GPU (different streams, no ordering between them) race and
 *   may produce wrong lists; order them on one stream. Non-finite score rows
 *   are repaired as in fvattn_route (kv_cnt == nb, NaN block_probs) but no
 *   flag is reported.
 */
FVATTN_API fvattn_status fvattn_route_noalloc(const fvattn_problem *prob, const void *q, const void *k,
                                              float p, int32_t k_min, int32_t *kv_cnt, int32_t *kv_idx,
                                              float *block_probs, fvattn_stream_t stream);

/*
 * fvattn_head_cost -- the actual work of every head under its kept lists, the
 * quantity the method's Runtime Load Balancing profiles per head before it
 * moves heavy heads off the critical rank (ai-feeds.com FVAttn summary, "Key
 * modules" 2; hotpaper.ai summary, RLB bullet: heads are rebalanced by their
 * real per-head workload).
 *
 *   head_cost[b*H + h] = sum over query blocks i of |i| * sum_{j in S_i} |j|
 * with |j| the valid tokens of block j: the (query, key) token pairs the
 * attention evaluates, proportional to its FLOPs (4*D per pair). Exact int64.
 *   kv_cnt, kv_idx  lists from fvattn_route (ignored if dense != 0: every
 *                   block kept, cost N*N per head)
 *   head_cost       out int64 [B*H], 8-byte aligned
 * Asynchronous on `stream`; needs no workspace.
 */
FVATTN_API fvattn_status fvattn_head_cost(const fvattn_problem *prob, const int32_t *kv_cnt, const int32_t *kv_idx,
                                          int32_t dense, int64_t *head_cost, fvattn_stream_t stream);

/*
 * fvattn_rlb_plan -- head migration plan of Runtime Load Balancing (host
 * code; no GPU). Heads start on their owner ranks; the most loaded rank moves
 * one of its own heads to the least loaded rank that can still receive,
 * choosing the head that leaves the larger of the two loads smallest (ties:
 * the heavier head, then the lower index), as long as the move shortens the
 * critical rank; every rank sends at most max_moves heads and receives at
 * most max_moves (the pages' setting: 1, ai-feeds.com summary "Key modules"
 * 2: a few heavy heads move over P2P; hotpaper.ai summary: each rank sends
 * and receives at most one head).
 *   head_cost   host int64 [n_heads] (e.g. from fvattn_head_cost), >= 0
 *   world       ranks (>= 1)
 *   owner_in    host int32 [n_heads] initial owner of each head, or NULL for
 *               the static shards: rank r holds heads [r*n/world, (r+1)*n/world)
 *   owner_out   out host int32 [n_heads] owner after the moves
 *   rank_load   out host int64 [world] load per rank after the moves, or NULL
 * Deterministic: every rank computes the same plan from the same costs.
 */
FVATTN_API fvattn_status fvattn_rlb_plan(const int64_t *head_cost, int32_t n_heads, int32_t world,
                                         const int32_t *owner_in, int32_t max_moves, int32_t *owner_out,
                                         int64_t *rank_load);

/*
 * fvattn_lpt_assign -- heads to ranks from scratch by longest processing time
 * first (host code): heads by cost descending (ties: lower index), each to the
 * least loaded rank (ties: lower rank). For callers whose sequence-parallel
 * all-to-all can place any head on any rank at no extra cost, so no
 * migration limit applies; its largest load is at most (4/3 - 1/(3*world))
 * times the best possible (Graham's bound for this rule).
 *   head_cost  host int64 [n_heads], >= 0
 *   owner_out  out host int32 [n_heads]
 *   rank_load  out host int64 [world], or NULL
 */
FVATTN_API fvattn_status fvattn_lpt_assign(const int64_t *head_cost, int32_t n_heads, int32_t world,
                                           int32_t *owner_out, int64_t *rank_load);

/*
 * fvattn_augment -- Slack-Aware Sparse Augmentation: spend a budget of spare
 * work on extra high-value blocks (ai-feeds.com FVAttn summary, "Key modules"
 * 3: ranks below the critical path insert additional attention blocks chosen
 * by attention score without lengthening that path; hotpaper.ai summary,
 * SASA bullet).
 *
 * The candidates are every (row, block j) pair of the problem whose block j
 * the row's list does not keep; a candidate's value is its block probability
 * P (block_probs from fvattn_route) and its cost |i| * |j| token pairs.
 * Candidates are ordered by P descending, then row (b*H + h)*nb + i
 * ascending, then j ascending; the longest prefix of that order whose total
 * cost is at most `budget` is added to the lists, which stay ascending
 * (kv_cnt grows accordingly). budget 0 changes nothing; a budget at least the
 * cost of every candidate keeps every block.
 *   block_probs    fp32 [B,H,nb,nb] from fvattn_route (required)
 *   budget         token pairs, >= 0 (the rank's slack: the critical rank's
 *                  head_cost total minus its own)
 *   kv_cnt, kv_idx in/out, the lists of fvattn_route
 *   added_pairs    out int64 [1] token pairs added, or NULL
 *   added_mass     out double [1] sum of the added blocks' P, or NULL (its
 *                  summation order is not fixed: last bits may vary)
 *   ws, ws_bytes   the problem's workspace
 * Asynchronous; about 11 small kernels. Run fvattn_schedule afterwards.
 */
FVATTN_API fvattn_status fvattn_augment(const fvattn_problem *prob, const float *block_probs, int64_t budget,
                                        int32_t *kv_cnt, int32_t *kv_idx, int64_t *added_pairs, double *added_mass,
                                        void *ws, size_t ws_bytes, fvattn_stream_t stream);

/*
 * fvattn_set_wait_limit -- the time limit of every wait inside the kernels of
 * later calls on this workspace, in ns (0: the default, 2 s). A wait that runs
 * out raises FVATTN_FLAG_TIMEOUT; the kernel then lets its copies and products
 * in flight finish (each with its own bound), frees its tensor memory and
 * returns, so the context stays usable. fvattn_workspace_init restores the
 * default. Asynchronous (a one-thread kernel on `stream`).
 */
FVATTN_API fvattn_status fvattn_set_wait_limit(void *ws, size_t ws_bytes, uint64_t limit_ns, fvattn_stream_t stream);

/*
 * fvattn_test_withhold_unit -- a test of the failure path (zskr.cn guide,
 * section 6: kernel failures surface instead of being masked): the next
 * fvattn_sparse_attn on this workspace takes rank `rank` of its unit order
 * but never hands it to its roles, whose waits then run out (see
 * fvattn_set_wait_limit); that unit's output is not written. -1 turns it off;
 * fvattn_workspace_init clears it too. Asynchronous.
 */
FVATTN_API fvattn_status fvattn_test_withhold_unit(void *ws, size_t ws_bytes, int32_t rank, fvattn_stream_t stream);

/* Synchronise `stream`, return the device status word's flags (FVATTN_FLAG_*)
 * in *flags, and clear them. Returns CUDA on a failed copy. */
FVATTN_API fvattn_status fvattn_read_device_status(void *ws, fvattn_stream_t stream, uint32_t *flags);

/* Static description of a status code. */
FVATTN_API const char *fvattn_status_string(fvattn_status s);

#ifdef __cplusplus
}
#endif

#endif /* FVATTN_H */
