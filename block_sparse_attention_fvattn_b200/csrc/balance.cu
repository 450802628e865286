// balance.cu -- per-head work, head migration plans and slack augmentation.
//
// The method's load balancer works at the level of attention heads: Top-p
// routing leaves heads with very different kept work, so the rank holding the
// heaviest heads sets the critical path. Runtime Load Balancing (RLB)
// measures each head's actual work and moves a few heavy heads from the most
// loaded rank to lightly loaded ones, each rank sending and receiving at most
// one head; Slack-Aware Sparse Augmentation (SASA) then lets every rank below
// the critical path spend its slack on extra high-value blocks, chosen by
// attention probability, without lengthening that path (ai-feeds.com FVAttn
// summary, "Key modules" 2 and 3; hotpaper.ai summary, RLB and SASA bullets).
//
//   K6 head_cost_kernel   work of every head: valid (query, key) token pairs
//                         sum_i |i| * sum_{j in S_i} |j| (int64, exact)
//   K7 augmentation       the highest-probability blocks that no list keeps,
//                         across every row of the problem, in the order
//                         (P descending, row ascending, block ascending),
//                         as long a prefix of that order as fits the budget
//                         of token pairs; found by a cost-weighted radix
//                         select over the fp32 bits of P (4 passes of 8 bits),
//                         then merged into the lists in ascending order
//   fvattn_rlb_plan       the migration plan (host code)
#include <string.h>

#include "common.cuh"
#include "fvattn.h"
#include "internal.h"

namespace fvattn {

// Valid tokens of block j: the block's extent clipped to the grid on each axis.
__device__ __forceinline__ int block_valid(const Geo &g, int j)
{
    int jt, jy, jx;
    block_coords(g, j, jt, jy, jx);
    return min(g.bt, g.T - jt * g.bt) * min(g.bh, g.Hg - jy * g.bh) * min(g.bw, g.W - jx * g.bw);
}

__device__ __forceinline__ long long warp_sum_ll(long long v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// ---------------------------------------------------------------------------
// K6: one CTA per head, one warp per query-block row at a time.
constexpr int kCostWarps = 8;

__global__ void __launch_bounds__(32 * kCostWarps) head_cost_kernel(Geo g, const int32_t *__restrict__ kv_cnt,
                                                                    const int32_t *__restrict__ kv_idx, int dense,
                                                                    int64_t *__restrict__ head_cost)
{
    __shared__ long long part[kCostWarps];
    const int bh = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    long long acc = 0;
    for (int i = warp; i < g.nb; i += kCostWarps) {
        long long rs = 0;
        if (dense) {
            for (int j = lane; j < g.nb; j += 32) rs += block_valid(g, j);
        } else {
            const size_t row = (size_t)bh * g.nb + i;
            const int c = min(max(__ldg(kv_cnt + row), 0), g.nb);
            const int32_t *lst = kv_idx + row * (size_t)g.nb;
            for (int e = lane; e < c; e += 32) rs += block_valid(g, __ldg(lst + e));
        }
        acc += warp_sum_ll(rs) * block_valid(g, i);
    }
    if (lane == 0) part[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long t = 0;
        for (int w = 0; w < kCostWarps; ++w) t += part[w];
        head_cost[bh] = t;
    }
}

// ---------------------------------------------------------------------------
// K7: augmentation. A candidate is a (row, block j) pair with j not in the
// row's list; its key is the bit pattern of P (non-negative fp32, so integer
// order is value order) and its cost |i| * |j|. The state lives in the
// workspace (AugState), zeroed at the start of every call.
constexpr int kAugWarps = 8;

struct AugState {
    unsigned long long hist[256];  // cost per key digit of the current pass
    unsigned int prefix;           // key bits fixed so far
    int all_fit;                   // every candidate fits the budget
    long long remaining;           // budget left for candidates whose key starts with `prefix`
    long long total;               // total cost of all candidates (pass 0)
};

// The rows' lists as bitmaps in shared memory, one per warp.
__device__ __forceinline__ void load_row_bitmap(uint32_t *bm, int nb, const int32_t *lst, int cnt, int lane)
{
    for (int w = lane; w < (nb + 31) / 32; w += 32) bm[w] = 0u;
    __syncwarp();
    for (int e = lane; e < cnt; e += 32) {
        const int j = __ldg(lst + e);
        if (j >= 0 && j < nb) atomicOr(bm + (j >> 5), 1u << (j & 31));
    }
    __syncwarp();
}

// Pass `pass` (0..3): histogram of candidate cost by key bits [24-8*pass, 32-8*pass)
// among candidates whose higher key bits equal the prefix chosen so far.
__global__ void __launch_bounds__(32 * kAugWarps) aug_hist_kernel(Geo g, const int32_t *__restrict__ kv_cnt,
                                                                  const int32_t *__restrict__ kv_idx,
                                                                  const float *__restrict__ probs,
                                                                  AugState *__restrict__ st, int pass)
{
    __shared__ unsigned long long hist[256];
    __shared__ uint32_t bms[kAugWarps][kMaxBlocks / 32];
    __shared__ int vsz[kMaxBlocks];
    if (st->all_fit) return;  // uniform: decided by the previous pick
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0ull;
    for (int j = threadIdx.x; j < g.nb; j += blockDim.x) vsz[j] = block_valid(g, j);
    __syncthreads();
    const int shift = 24 - 8 * pass;
    const unsigned int want = pass == 0 ? 0u : (st->prefix >> (shift + 8));
    const long long rows = (long long)g.BH * g.nb;
    uint32_t *bm = bms[warp];
    for (long long row = (long long)blockIdx.x * kAugWarps + warp; row < rows; row += (long long)gridDim.x * kAugWarps) {
        const int i = (int)(row % g.nb);
        const int c = min(max(__ldg(kv_cnt + row), 0), g.nb);
        load_row_bitmap(bm, g.nb, kv_idx + row * g.nb, c, lane);
        const long long vi = vsz[i];
        const float *pr = probs + row * g.nb;
        for (int j = lane; j < g.nb; j += 32) {
            if ((bm[j >> 5] >> (j & 31)) & 1u) continue;
            const unsigned int key = __float_as_uint(fmaxf(__ldg(pr + j), 0.f));
            if (pass > 0 && (key >> (shift + 8)) != want) continue;
            atomicAdd(hist + ((key >> shift) & 255u), (unsigned long long)(vi * vsz[j]));
        }
        __syncwarp();
    }
    __syncthreads();
    for (int b = threadIdx.x; b < 256; b += blockDim.x)
        if (hist[b]) atomicAdd(st->hist + b, hist[b]);
}

// One thread: choose the digit of this pass -- the bin where the cumulative
// cost, from the largest keys down, first exceeds the budget left.
__global__ void aug_pick_kernel(AugState *__restrict__ st, long long budget, int pass)
{
    if (threadIdx.x != 0 || st->all_fit) return;
    const int shift = 24 - 8 * pass;
    if (pass == 0) {
        unsigned long long total = 0;
        for (int b = 0; b < 256; ++b) total += st->hist[b];
        st->total = (long long)total;
        st->remaining = budget;
        st->prefix = 0u;
        if ((long long)total <= budget) {
            st->all_fit = 1;
            return;
        }
    }
    long long cum = 0;
    int pick = 0;
    for (int b = 255; b >= 0; --b) {
        const long long h = (long long)st->hist[b];
        if (cum + h > st->remaining) {
            pick = b;
            break;
        }
        cum += h;
    }
    st->remaining -= cum;
    st->prefix |= (unsigned int)pick << shift;
    for (int b = 0; b < 256; ++b) st->hist[b] = 0ull;
}

// Cost of each row's candidates whose key equals the boundary key.
__global__ void __launch_bounds__(32 * kAugWarps) aug_tie_kernel(Geo g, const int32_t *__restrict__ kv_cnt,
                                                                 const int32_t *__restrict__ kv_idx,
                                                                 const float *__restrict__ probs,
                                                                 const AugState *__restrict__ st,
                                                                 long long *__restrict__ row_tie)
{
    __shared__ uint32_t bms[kAugWarps][kMaxBlocks / 32];
    if (st->all_fit) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned int t = st->prefix;
    const long long rows = (long long)g.BH * g.nb;
    uint32_t *bm = bms[warp];
    for (long long row = (long long)blockIdx.x * kAugWarps + warp; row < rows; row += (long long)gridDim.x * kAugWarps) {
        const int i = (int)(row % g.nb);
        const int c = min(max(__ldg(kv_cnt + row), 0), g.nb);
        load_row_bitmap(bm, g.nb, kv_idx + row * g.nb, c, lane);
        const float *pr = probs + row * g.nb;
        long long s = 0;
        for (int j = lane; j < g.nb; j += 32) {
            if ((bm[j >> 5] >> (j & 31)) & 1u) continue;
            if (__float_as_uint(fmaxf(__ldg(pr + j), 0.f)) == t) s += (long long)block_valid(g, j);
        }
        s = warp_sum_ll(s);
        if (lane == 0) row_tie[row] = s * block_valid(g, i);
    }
}

// One CTA: exclusive prefix sum of the rows' tie costs, in row order, in place.
__global__ void __launch_bounds__(1024) aug_scan_kernel(long long rows, const AugState *__restrict__ st,
                                                        long long *__restrict__ row_tie)
{
    __shared__ long long part[1024];
    __shared__ long long carry;
    if (st->all_fit) return;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (long long base = 0; base < rows; base += 1024) {
        const long long r = base + threadIdx.x;
        const long long v = r < rows ? row_tie[r] : 0;
        part[threadIdx.x] = v;
        __syncthreads();
        for (int o = 1; o < 1024; o <<= 1) {
            const long long add = threadIdx.x >= o ? part[threadIdx.x - o] : 0;
            __syncthreads();
            part[threadIdx.x] += add;
            __syncthreads();
        }
        if (r < rows) row_tie[r] = carry + part[threadIdx.x] - v;
        __syncthreads();
        if (threadIdx.x == 1023) carry += part[1023];
        __syncthreads();
    }
}

// Merge the chosen candidates into each row's list, ascending, and count
// what was added.
__global__ void __launch_bounds__(32 * kAugWarps) aug_insert_kernel(Geo g, int32_t *__restrict__ kv_cnt,
                                                                    int32_t *__restrict__ kv_idx,
                                                                    const float *__restrict__ probs,
                                                                    const AugState *__restrict__ st,
                                                                    const long long *__restrict__ row_tie,
                                                                    unsigned long long *__restrict__ added_cost,
                                                                    double *__restrict__ added_mass)
{
    __shared__ uint32_t bms[kAugWarps][kMaxBlocks / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const bool all = st->all_fit != 0;
    const unsigned int t = st->prefix;
    const long long rem = st->remaining;
    const long long rows = (long long)g.BH * g.nb;
    uint32_t *bm = bms[warp];
    for (long long row = (long long)blockIdx.x * kAugWarps + warp; row < rows; row += (long long)gridDim.x * kAugWarps) {
        const int i = (int)(row % g.nb);
        const int c = min(max(kv_cnt[row], 0), g.nb);
        int32_t *lst = kv_idx + row * g.nb;
        load_row_bitmap(bm, g.nb, lst, c, lane);
        const long long vi = block_valid(g, i);
        long long tie_before = all ? 0 : row_tie[row];  // tie cost of earlier rows
        const float *pr = probs + row * g.nb;
        int base = 0;
        long long my_cost = 0;
        double my_mass = 0.0;
        for (int j0 = 0; j0 < g.nb; j0 += 32) {
            const int j = j0 + lane;
            const bool valid = j < g.nb;
            const bool kept = valid && ((bm[j >> 5] >> (j & 31)) & 1u);
            const float pj = valid ? fmaxf(__ldg(pr + j), 0.f) : 0.f;
            const unsigned int key = __float_as_uint(pj);
            const long long cj = valid ? vi * block_valid(g, j) : 0;
            bool add = false;
            if (valid && !kept) {
                if (all || key > t) add = true;
            }
            if (!all) {
                // candidates at the boundary key, in (row, block) order: taken
                // while the running cost stays within the budget left for them
                const bool tie = valid && !kept && key == t;
                long long tc = tie ? cj : 0, incl = tc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const long long x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += x;
                }
                if (tie && tie_before + incl <= rem) add = true;
                tie_before += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (add) {
                my_cost += cj;
                my_mass += (double)pj;
            }
            const bool sel = kept || add;
            const uint32_t sm = __ballot_sync(0xFFFFFFFFu, sel);
            if (sel) lst[base + __popc(sm & lt_mask)] = j;
            base += __popc(sm);
        }
        if (lane == 0) kv_cnt[row] = base;
        my_cost = warp_sum_ll(my_cost);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) my_mass += __shfl_xor_sync(0xFFFFFFFFu, my_mass, o);
        if (lane == 0 && my_cost > 0) {
            if (added_cost) atomicAdd(added_cost, (unsigned long long)my_cost);
            if (added_mass) atomicAdd(added_mass, my_mass);
        }
    }
}

cudaError_t launch_head_cost(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int dense, int64_t *head_cost,
                             cudaStream_t stream)
{
    head_cost_kernel<<<(unsigned)g.BH, 32 * kCostWarps, 0, stream>>>(g, kv_cnt, kv_idx, dense, head_cost);
    return cudaGetLastError();
}

cudaError_t launch_augment(const Geo &g, const float *probs, long long budget, int32_t *kv_cnt, int32_t *kv_idx,
                           void *state, long long *row_tie, unsigned long long *added_cost, double *added_mass,
                           cudaStream_t stream)
{
    AugState *st = static_cast<AugState *>(state);
    cudaError_t e = cudaMemsetAsync(st, 0, sizeof(AugState), stream);
    if (e != cudaSuccess) return e;
    if (added_cost && (e = cudaMemsetAsync(added_cost, 0, sizeof(unsigned long long), stream)) != cudaSuccess) return e;
    if (added_mass && (e = cudaMemsetAsync(added_mass, 0, sizeof(double), stream)) != cudaSuccess) return e;
    const long long rows = (long long)g.BH * g.nb;
    const long long want = (rows + kAugWarps - 1) / kAugWarps;
    const unsigned grid = (unsigned)(want < 148 * 8 ? want : 148 * 8);
    for (int pass = 0; pass < 4; ++pass) {
        aug_hist_kernel<<<grid, 32 * kAugWarps, 0, stream>>>(g, kv_cnt, kv_idx, probs, st, pass);
        aug_pick_kernel<<<1, 32, 0, stream>>>(st, budget, pass);
    }
    aug_tie_kernel<<<grid, 32 * kAugWarps, 0, stream>>>(g, kv_cnt, kv_idx, probs, st, row_tie);
    aug_scan_kernel<<<1, 1024, 0, stream>>>(rows, st, row_tie);
    aug_insert_kernel<<<grid, 32 * kAugWarps, 0, stream>>>(g, kv_cnt, kv_idx, probs, st, row_tie, added_cost,
                                                           added_mass);
    return cudaGetLastError();
}

size_t augment_state_bytes() { return sizeof(AugState); }

__global__ void header_write_kernel(uint32_t *header, int word, uint64_t value)
{
    if (word >= 0) *reinterpret_cast<uint64_t *>(header + word) = value;
    else header[-word] = (uint32_t)value;
}

cudaError_t launch_header_write(uint32_t *header, int word, uint64_t value, cudaStream_t stream)
{
    header_write_kernel<<<1, 1, 0, stream>>>(header, word, value);
    return cudaGetLastError();
}

}  // namespace fvattn

// ---------------------------------------------------------------------------
// Host: the migration plan.
extern "C" fvattn_status fvattn_rlb_plan(const int64_t *head_cost, int32_t n_heads, int32_t world,
                                         const int32_t *owner_in, int32_t max_moves, int32_t *owner_out,
                                         int64_t *rank_load)
{
    if (!head_cost || !owner_out || n_heads < 0 || world < 1 || max_moves < 0) return FVATTN_ERR_INVALID_ARG;
    if (world > 65536) return FVATTN_ERR_UNSUPPORTED;
    for (int h = 0; h < n_heads; ++h) {
        if (head_cost[h] < 0) return FVATTN_ERR_INVALID_ARG;
        if (owner_in && (owner_in[h] < 0 || owner_in[h] >= world)) return FVATTN_ERR_INVALID_ARG;
    }
    int32_t *own = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_heads > 0 ? n_heads : 1));
    int64_t *load = (int64_t *)calloc((size_t)world, sizeof(int64_t));
    int32_t *sent = (int32_t *)calloc((size_t)world, sizeof(int32_t));
    int32_t *recv = (int32_t *)calloc((size_t)world, sizeof(int32_t));
    if (!own || !load || !sent || !recv) {
        free(own);
        free(load);
        free(sent);
        free(recv);
        return FVATTN_ERR_INVALID_ARG;
    }
    // without owner_in, the static shards: rank r holds heads [r*H/world, (r+1)*H/world)
    for (int r = 0; r < world; ++r) {
        const long long h0 = (long long)r * n_heads / world, h1 = (long long)(r + 1) * n_heads / world;
        for (long long h = h0; h < h1; ++h) own[h] = r;
    }
    for (int h = 0; h < n_heads; ++h) {
        if (owner_in) own[h] = owner_in[h];
        owner_out[h] = own[h];
        load[own[h]] += head_cost[h];
    }
    for (;;) {
        // the critical rank (ties: lowest index) must be able to send ...
        int c = 0;
        for (int r = 1; r < world; ++r)
            if (load[r] > load[c]) c = r;
        if (sent[c] >= max_moves) break;
        // ... to the lightest rank that can still receive (ties: lowest index)
        int l = -1;
        for (int r = 0; r < world; ++r)
            if (r != c && recv[r] < max_moves && (l < 0 || load[r] < load[l])) l = r;
        if (l < 0) break;
        // the head of c's own shard whose move leaves the pair's larger load
        // smallest (ties: the heavier head, then the lower index); only a
        // move that shortens the critical rank is made
        int best = -1;
        int64_t best_m = load[c];
        for (int h = 0; h < n_heads; ++h) {
            if (own[h] != c || owner_out[h] != c) continue;
            const int64_t a = load[c] - head_cost[h], b = load[l] + head_cost[h];
            const int64_t m = a > b ? a : b;
            if (m < best_m || (best >= 0 && m == best_m && head_cost[h] > head_cost[best])) {
                best = h;
                best_m = m;
            }
        }
        if (best < 0) break;
        owner_out[best] = l;
        load[c] -= head_cost[best];
        load[l] += head_cost[best];
        ++sent[c];
        ++recv[l];
    }
    if (rank_load) memcpy(rank_load, load, sizeof(int64_t) * (size_t)world);
    free(own);
    free(load);
    free(sent);
    free(recv);
    return FVATTN_OK;
}

// Host: longest-processing-time assignment of heads to ranks from scratch.
extern "C" fvattn_status fvattn_lpt_assign(const int64_t *head_cost, int32_t n_heads, int32_t world,
                                           int32_t *owner_out, int64_t *rank_load)
{
    if (!head_cost || !owner_out || n_heads < 0 || world < 1) return FVATTN_ERR_INVALID_ARG;
    if (world > 65536) return FVATTN_ERR_UNSUPPORTED;
    for (int h = 0; h < n_heads; ++h)
        if (head_cost[h] < 0) return FVATTN_ERR_INVALID_ARG;
    int32_t *order = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_heads > 0 ? n_heads : 1));
    int64_t *load = (int64_t *)calloc((size_t)world, sizeof(int64_t));
    if (!order || !load) {
        free(order);
        free(load);
        return FVATTN_ERR_INVALID_ARG;
    }
    // heads by cost descending (ties: lower index), by insertion: n_heads is small
    for (int h = 0; h < n_heads; ++h) {
        int p = h;
        while (p > 0 && head_cost[order[p - 1]] < head_cost[h]) {
            order[p] = order[p - 1];
            --p;
        }
        order[p] = h;
    }
    // each to the least loaded rank (ties: lowest index)
    for (int x = 0; x < n_heads; ++x) {
        const int h = order[x];
        int r = 0;
        for (int q = 1; q < world; ++q)
            if (load[q] < load[r]) r = q;
        owner_out[h] = r;
        load[r] += head_cost[h];
    }
    if (rank_load) memcpy(rank_load, load, sizeof(int64_t) * (size_t)world);
    free(order);
    free(load);
    return FVATTN_OK;
}
