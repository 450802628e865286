// schedule.cu -- longest-first balanced work lists for the persistent attention CTAs.
//
// The method observes that Top-p routing leaves heads with very different
// amounts of kept work, so whoever holds the heaviest heads sets the critical
// path (ai-feeds.com FVAttn summary, "Existing limitations" and "Key modules"
// 2; load imbalance = max/mean, ideal 1.0). Its remedy moves heavy heads
// between GPUs. On one GPU the same imbalance appears between persistent CTAs,
// and the remedy here is an ordering + assignment:
//   K3a sched_head_kernel  one CTA per head: cost of every (head, query block)
//       unit = active 128-row query tiles x kept key/value sub-tiles (what the
//       attention kernel executes), sorted by cost descending (ties: lower
//       block index), plus the head's total. With 64-token blocks a unit is
//       four query blocks (two pairs, one 128-row tile each) and its cost the
//       tiles of the two pairs' unions (pair_lists_kernel builds them first).
//   K3b sched_assign_kernel one CTA: heads sorted by total cost descending
//       (ties: lower head), concatenated into one ranked list; rank r goes to
//       CTA zigzag(r) (round r/C, direction alternating per round), so every
//       round of C consecutive ranks -- mostly one head, which keeps its key
//       and value blocks in L2 -- hands each CTA one unit.
#include "common.cuh"
#include "internal.h"

namespace fvattn {

__device__ void bitonic_sort_u64(unsigned long long *keys, int n)
{
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = threadIdx.x; t < n; t += blockDim.x) {
                const int ixj = t ^ j;
                if (ixj > t) {
                    const bool up = (t & k) == 0;
                    const unsigned long long a = keys[t], b = keys[ixj];
                    if ((a > b) == up) {
                        keys[t] = b;
                        keys[ixj] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Kept key/value sub-tiles of a unit: every kept block has nsub sub-tiles,
// except blocks in the last row of t-blocks when its second sub-tile lies
// wholly outside the grid. Kept lists are ascending, so those blocks are the
// list's tail, found by binary search.
__device__ __forceinline__ int unit_tiles(const Geo &g, const int32_t *lst, int cnt, int dense)
{
    const bool last_short = (g.nsub == 2) && ((g.nbt - 1) * g.bt + g.subt >= g.T);
    if (!last_short) return cnt * g.nsub;
    const int j0 = (g.nbt - 1) * g.nbh * g.nbw;
    int nlast;
    if (dense) {
        nlast = g.nb - j0;
    } else {
        int lo = 0, hi = cnt;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(lst + mid) >= j0) hi = mid;
            else lo = mid + 1;
        }
        nlast = cnt - lo;
    }
    return cnt * g.nsub - nlast;
}

// Paired mode (64-token blocks): pair p = query blocks (2p, 2p+1) of a head.
// One warp merges the two kept lists into their union, ascending, each entry
// flagged with the query blocks that keep it (kPairInA / kPairInB). The
// attention kernel runs a pair as one 128-row query tile over the union.
constexpr int kPairWarps = 8;

__global__ void __launch_bounds__(32 * kPairWarps) pair_lists_kernel(Geo g, const int32_t *__restrict__ kv_cnt,
                                                                     const int32_t *__restrict__ kv_idx,
                                                                     int32_t *__restrict__ pair_cnt,
                                                                     int32_t *__restrict__ pair_list)
{
    __shared__ uint32_t bm[kPairWarps][2][kMaxBlocks / 32];
    pdl_release();
    pdl_wait();  // the kept lists come from the routing kernels
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long pid = (long long)blockIdx.x * kPairWarps + warp;
    if (pid >= (long long)g.BH * g.npair) return;
    const int bh = (int)(pid / g.npair), pp = (int)(pid - (long long)bh * g.npair);
    const int nw = (g.nb + 31) >> 5;
    uint32_t *ma = bm[warp][0], *mb = bm[warp][1];
    for (int w = lane; w < nw; w += 32) ma[w] = mb[w] = 0u;
    __syncwarp();
    for (int s = 0; s < 2; ++s) {
        const int i = 2 * pp + s;
        if (i >= g.nb) break;
        const size_t u = (size_t)bh * g.nb + i;
        const int c = min(max(__ldg(kv_cnt + u), 0), g.nb);
        uint32_t *m = s ? mb : ma;
        for (int e = lane; e < c; e += 32) {
            const int j = __ldg(kv_idx + u * g.nb + e);
            if ((unsigned)j < (unsigned)g.nb) atomicOr(&m[j >> 5], 1u << (j & 31));
        }
    }
    __syncwarp();
    // lane l writes the union's entries of bitmap word w0 + l, after those of
    // the lower words (prefix sum of the words' counts)
    int32_t *out = pair_list + (size_t)pid * g.nb;
    int base = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        const uint32_t a = w < nw ? ma[w] : 0u, b = w < nw ? mb[w] : 0u, un = a | b;
        const int c = __popc(un);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += t;
        }
        int pos = base + incl - c;
        uint32_t rest = un;
        while (rest) {
            const int bit = __ffs(rest) - 1;
            rest &= rest - 1u;
            out[pos++] = (w * 32 + bit) | (((a >> bit) & 1u) ? kPairInA : 0) | (((b >> bit) & 1u) ? kPairInB : 0);
        }
        base += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    if (lane == 0) pair_cnt[pid] = base;
}

cudaError_t launch_pair_lists(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int32_t *pair_cnt,
                              int32_t *pair_list, cudaStream_t stream)
{
    const long long pairs = (long long)g.BH * g.npair;
    if (pairs == 0) return cudaSuccess;
    return launch_dependent(pair_lists_kernel, dim3((unsigned)((pairs + kPairWarps - 1) / kPairWarps)),
                            dim3(32 * kPairWarps), 0, stream, g, kv_cnt, kv_idx, pair_cnt, pair_list);
}

// Tiles of pair pp of head bh in paired mode: ceil(|union| / 2) steps of two
// 64-token key/value blocks (0 if the pair holds no query block).
__device__ __forceinline__ int pair_tiles(const Geo &g, int bh, int pp, const int32_t *pair_cnt, int dense)
{
    if (pp >= g.npair) return 0;
    const int c = dense ? g.nb : __ldg(pair_cnt + (size_t)bh * g.npair + pp);
    return (c + 1) >> 1;
}

// Paired mode: a unit of at least kSplitMinTiles key/value tiles runs split,
// one unit per pair (both softmax warpgroups on the same 128 query rows, each
// over half of the pair's key list), so the longest units are half as long
// and the dynamic order can even out the end of the layer; shorter units keep
// two pairs (one per warpgroup).
constexpr int kSplitMinTiles = 64;

__global__ void __launch_bounds__(1024) sched_head_kernel(Geo g, const int32_t *__restrict__ kv_cnt,
                                                          const int32_t *__restrict__ kv_idx, int dense,
                                                          const int32_t *__restrict__ pair_cnt,
                                                          int32_t *__restrict__ unit_cost,
                                                          int32_t *__restrict__ head_sorted,
                                                          int32_t *__restrict__ head_len,
                                                          int64_t *__restrict__ head_cost, int npow2)
{
    extern __shared__ unsigned long long keys[];
    __shared__ long long part[32];
    __shared__ int part_n[32];
    pdl_release();
    pdl_wait();  // kept lists or pair unions from the kernel before
    const int bh = blockIdx.x;
    const int hw = g.nbh * g.nbw;
    // candidate entries of this head: unpaired, entry i = unit i; paired,
    // entries 2q and 2q+1 = unit q, or its two pairs as split units
    const int nent = g.paired ? 2 * g.upb : g.upb;
    long long local = 0;
    int nvalid = 0;
    for (int e = threadIdx.x; e < npow2; e += blockDim.x) {
        unsigned long long key = ~0ull;
        if (e < nent) {
            int cost = -1, uid = -1;
            if (g.paired) {
                const int q = e >> 1, half = e & 1;
                const int t0 = pair_tiles(g, bh, 2 * q, pair_cnt, dense);
                const int t1 = pair_tiles(g, bh, 2 * q + 1, pair_cnt, dense);
                if (!dense && t0 + t1 >= kSplitMinTiles) {
                    const int pp = 2 * q + half;
                    if (pp < g.npair) {
                        cost = half ? t1 : t0;
                        uid = g.BH * g.upb + bh * g.npair + pp;
                    }
                } else if (half == 0) {
                    // unit q = pairs 2q (first query tile) and 2q+1 (second)
                    cost = t0 + t1;
                    uid = bh * g.upb + q;
                }
            } else {
                const size_t u = (size_t)bh * g.upb + e;
                const int it = e / hw;
                const int nh = (g.nsub == 2 && it * g.bt + g.subt < g.T) ? 2 : 1;
                const int cnt = dense ? g.nb : __ldg(kv_cnt + u);
                cost = nh * unit_tiles(g, dense ? nullptr : kv_idx + u * g.nb, cnt, dense);
                uid = (int)u;
            }
            if (uid >= 0) {
                unit_cost[uid] = cost;
                local += cost;
                ++nvalid;
                key = ((unsigned long long)(0xFFFFFFFFu - (uint32_t)cost) << 32) | (uint32_t)uid;
            }
        }
        keys[e] = key;
    }
    for (int o = 16; o > 0; o >>= 1) {
        local += __shfl_xor_sync(0xFFFFFFFFu, local, o);
        nvalid += __shfl_xor_sync(0xFFFFFFFFu, nvalid, o);
    }
    if ((threadIdx.x & 31) == 0) {
        part[threadIdx.x >> 5] = local;
        part_n[threadIdx.x >> 5] = nvalid;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        long long s = 0;
        int n = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            s += part[w];
            n += part_n[w];
        }
        head_cost[bh] = s;
        head_len[bh] = n;
    }
    bitonic_sort_u64(keys, npow2);
    for (int r = threadIdx.x; r < nent; r += blockDim.x)
        head_sorted[(size_t)bh * nent + r] = keys[r] == ~0ull ? -1 : (int32_t)(keys[r] & 0xFFFFFFFFull);
}

// First index of CTA c's list when U ranks are dealt in zigzag rounds of C.
__host__ __device__ __forceinline__ long long zigzag_start(long long c, long long U, long long C)
{
    const long long full = U / C, R = U % C;
    long long extra = 0;
    if (R) extra = (full & 1) ? ((c > C - R) ? c - (C - R) : 0) : (c < R ? c : R);
    return c * full + extra;
}

__global__ void __launch_bounds__(1024) sched_assign_kernel(Geo g, int C, const int32_t *__restrict__ unit_cost,
                                                            const int32_t *__restrict__ head_sorted,
                                                            const int32_t *__restrict__ head_len,
                                                            const int64_t *__restrict__ head_cost,
                                                            int32_t *__restrict__ work, int32_t *__restrict__ cta_range,
                                                            int64_t *__restrict__ cta_cost, int hpow2)
{
    extern __shared__ unsigned long long sa_smem[];
    __shared__ int chunk_sum[1024];
    pdl_release();
    pdl_wait();  // unit costs from sched_head_kernel
    unsigned long long *hkeys = sa_smem;          // [hpow2]
    unsigned long long *ccost = sa_smem + hpow2;  // [C]
    int *off = reinterpret_cast<int *>(ccost + C); // [hpow2 + 1]: first rank of each head in head order
    for (int h = threadIdx.x; h < hpow2; h += blockDim.x) {
        if (h < g.BH) {
            const unsigned long long c = (unsigned long long)head_cost[h];
            hkeys[h] = ((0xFFFFFFFFull - (c & 0xFFFFFFFFull)) << 32) | (uint32_t)h;
        } else {
            hkeys[h] = ~0ull;
        }
    }
    for (int c = threadIdx.x; c < C; c += blockDim.x) ccost[c] = 0ull;
    __syncthreads();
    bitonic_sort_u64(hkeys, hpow2);
    // ranks of each head in head order: an exclusive prefix of the head lengths
    const int per = (g.BH + (int)blockDim.x - 1) / (int)blockDim.x;
    const int h0 = (int)threadIdx.x * per;
    int s = 0;
    for (int x = h0; x < min(h0 + per, g.BH); ++x) s += __ldg(head_len + (int)(hkeys[x] & 0xFFFFFFFFull));
    chunk_sum[threadIdx.x] = s;
    __syncthreads();
    for (int o = 1; o < (int)blockDim.x; o <<= 1) {
        const int add = (int)threadIdx.x >= o ? chunk_sum[threadIdx.x - o] : 0;
        __syncthreads();
        chunk_sum[threadIdx.x] += add;
        __syncthreads();
    }
    int run = chunk_sum[threadIdx.x] - s;
    for (int x = h0; x < min(h0 + per, g.BH); ++x) {
        off[x] = run;
        run += __ldg(head_len + (int)(hkeys[x] & 0xFFFFFFFFull));
    }
    if (threadIdx.x == blockDim.x - 1) off[g.BH] = chunk_sum[blockDim.x - 1];
    __syncthreads();
    const long long U = off[g.BH];
    const int stride = g.paired ? 2 * g.upb : g.upb;
    for (int c = threadIdx.x; c <= C; c += blockDim.x) cta_range[c] = (int32_t)zigzag_start(c, U, C);
    for (long long r = threadIdx.x; r < U; r += blockDim.x) {
        // the head whose ranks hold r: the last x with off[x] <= r
        int lo = 0, hi = g.BH - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= r) lo = mid;
            else hi = mid - 1;
        }
        const int head = (int)(hkeys[lo] & 0xFFFFFFFFull);
        const int u = head_sorted[(size_t)head * stride + (r - off[lo])];
        const long long round = r / C, pos = r - round * C;
        const long long c = (round & 1) ? (C - 1 - pos) : pos;
        work[zigzag_start(c, U, C) + round] = (int32_t)u;
        atomicAdd(&ccost[c], (unsigned long long)unit_cost[u]);
    }
    __syncthreads();
    if (cta_cost)
        for (int c = threadIdx.x; c < C; c += blockDim.x) cta_cost[c] = (int64_t)ccost[c];
}

static int next_pow2(int n)
{
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

cudaError_t launch_schedule(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int dense, int num_ctas,
                            int32_t *work, int32_t *cta_range, int64_t *cta_cost, int32_t *unit_cost,
                            int32_t *head_sorted, int32_t *head_len, int64_t *head_cost, const int32_t *pair_cnt,
                            cudaStream_t stream)
{
    const int npow2 = next_pow2(g.paired ? 2 * g.upb : g.upb);
    const size_t smem_a = (size_t)npow2 * sizeof(unsigned long long);
    cudaError_t err = cudaFuncSetAttribute(sched_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
    if (err != cudaSuccess) return err;
    err = launch_dependent(sched_head_kernel, dim3(g.BH), dim3(1024), smem_a, stream, g, kv_cnt, kv_idx, dense,
                           pair_cnt, unit_cost, head_sorted, head_len, head_cost, npow2);
    if (err != cudaSuccess) return err;
    const int hpow2 = next_pow2(g.BH);
    const size_t smem_b = ((size_t)hpow2 + num_ctas) * sizeof(unsigned long long) + ((size_t)hpow2 + 1) * sizeof(int);
    err = cudaFuncSetAttribute(sched_assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b);
    if (err != cudaSuccess) return err;
    return launch_dependent(sched_assign_kernel, dim3(1), dim3(1024), smem_b, stream, g, num_ctas,
                            (const int32_t *)unit_cost, (const int32_t *)head_sorted, (const int32_t *)head_len,
                            (const int64_t *)head_cost, work, cta_range, cta_cost, hpow2);
}

}  // namespace fvattn
