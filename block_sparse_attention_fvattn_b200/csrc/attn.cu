// attn.cu -- K4: persistent block-sparse attention on sm_100a (TMA + tcgen05/TMEM).
//
// Attention runs only over the key/value blocks kept by the router (the
// source of the method's attention speedup over FlashAttention: ai-feeds.com
// FVAttn summary, "Key findings"; zskr.cn FastVideo VSA guide, section 1:
// each query block attends to its selected key/value blocks). Dense mode
// runs every block through the same code (the guide's VSA_ALL_BLOCKS route).
//
// Work unit = one (b, h, query block i). A 256-token block is two 128-row
// query tiles (its two halves along t), and key/value blocks are consumed in
// sub-tiles of 128 tokens, so one 256-token key block is two sub-tiles; a
// sub-tile that lies wholly outside the grid is skipped, partial ones mask
// their padded columns.
// 64-token blocks run paired: query blocks (2p, 2p+1) share one 128-row tile
// (rows 0-63 and 64-127) and walk the union of their two kept lists two key
// blocks (128 tokens) at a time; each row masks the key blocks its own query
// block did not keep. A unit is then four query blocks, i.e. two such tiles
// with separate key/value streams, interleaved tile by tile.
//
// Tiles come straight from the raster [B,H,N,D] layout: each tensor is seen
// by TMA as 5-D (D, W, H, T, B*H) and one sub-tile is one box of
// (64, bw, bh, sub_t, 1) elements per 64-column slab, 128-byte swizzled.
// Out-of-grid elements are filled with zeros by TMA; no token-level mask or
// re-packed copy of the sequence is ever built (the bjdmk.com.cn Sol-Attn
// article, section 5.1, on n x n masks at ~400k tokens).
//
// Roles (384 threads = 3 warpgroups, one CTA per SM):
//   warp 0      TMA producer of Q halves and K sub-tiles
//   warp 1      QK issuer (one thread) and owner of the TMEM allocation:
//               S = Q_h K^T (A and B from shared memory)
//   warp 2      PV issuer (one thread): O_h += P_h V (A = P_h from TMEM,
//               B = V from shared memory, MN-major). Two issuing threads keep
//               the tensor core fed while either one waits on a barrier.
//   warp 3      TMA producer of V sub-tiles; its lane 1 takes the units from
//               the shared counter once warp 0 has issued the current unit
//   warps 4-7   softmax + epilogue for query half 0
//   warps 8-11  softmax + epilogue for query half 1
// A warp reaches TMEM lanes 32*(warp % 4) .. +31, so each softmax warpgroup
// covers the 128 rows of its half (row = 32*(warp%4) + lane) and holds a
// whole 128-column score row in registers.
//
// TMEM (512 columns x 128 lanes): one S buffer [0,128) shared by both halves,
// P_0 [128,192) and P_1 [192,256) (bf16 pairs), O_0 [256,256+D), O_1 after it.
// S is free again as soon as the softmax warpgroup has copied it into
// registers, so the next QK never waits for a PV to finish, and one half's
// softmax overlaps the other half's products. The online softmax rescales O
// lazily, only when a row maximum grows by more than 2^8.
//
// Epilogue: O / l is staged in the half's Q tile (whose products are all done
// by then), in that tile's swizzled layout, and written by TMA tile stores
// with the same 5-D boxes as the loads, so rows outside the grid are skipped
// and every store is a whole 128-byte line. The next unit's Q tile is loaded
// there once the stores have read it.
// Units: lane 1 of warp 3 claims them from the counter shared by all CTAs,
// each once warp 0 has issued the previous unit's loads. A slot of the unit ring carries the unit id and, in
// paired mode, the two union sizes and the first entries of each union, so no
// role starts a unit with a chain of global loads.
#include "common.cuh"
#include "internal.h"

namespace fvattn {

constexpr int kUnitSlots = 4;  // ring of units handed from the producer to the other roles
// words of a unit slot: the unit id, then (paired mode) the two union sizes and
// the first two entries of each union, so no role reads them from global
// memory at the start of a unit
constexpr int kUnitWords = 8;
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Register split between warpgroups (setmaxnreg). The kernel is launched with
// kLaunchRegs per thread (checked on the host before every launch); the
// producer/MMA warpgroup gives registers back and the two softmax
// warpgroups take them: 128*low + 256*high <= 384*kLaunchRegs.
constexpr int kLaunchRegs = 168;
template <int D, int BKV>
struct RegSplit {
    static constexpr int kLow = 80;
    static constexpr int kHigh = 208;
    static_assert(128 * kLow + 256 * kHigh <= kThreads * kLaunchRegs, "register split exceeds the launch budget");
};

template <int D, int BKV, bool PAIRED = false>
struct AttnLayout {
    // Ring stages: a V tile waits for a softmax before its product, so V gets
    // the deeper ring (measured on B200; paired mode with 3 K / 2 V stages
    // ran 8% slower)
    static constexpr int kNK = 2;  // K ring stages
    static constexpr int kNV = 3;  // V ring stages
    static constexpr int kDH = D / 64;              // 128-byte column slabs per row
    static constexpr int kQSlab = 128 * 128;        // bytes of one 128-row slab
    static constexpr int kKVSlab = BKV * 128;
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + 2 * kDH * kQSlab;
    static constexpr int kV = kK + kNK * kDH * kKVSlab;
    static constexpr int kMask = kV + kNV * kDH * kKVSlab;
    // column masks cover one key block of the tile: all BKV columns, or one
    // 64-token block in paired mode
    static constexpr int kMaskWords = (PAIRED ? 64 : BKV) / 32;
    // per-axis column masks: entry v-1 of each axis keeps the columns whose
    // coordinate along that axis is < v; blk_w + blk_h + sub_t <= kMaskEntries
    static constexpr int kMaskEntries = 40;
    static constexpr int kUnit = kMask + kMaskEntries * kMaskWords * 4;  // int32 unit slots
    static constexpr int kBar = kUnit + kUnitSlots * kUnitWords * 4;
    // barrier indices
    static constexpr int bQFull = 0, bQEmpty = 2, bKFull = 4, bKEmpty = bKFull + kNK, bVFull = bKEmpty + kNK,
                         bVEmpty = bVFull + kNV, bSFull = bVEmpty + kNV, bSFree = bSFull + 2, bPFull = bSFree + 1,
                         bPFree = bPFull + 2, bOFull = bPFree + 2, bOEmpty = bOFull + 2, bDrain = bOEmpty + 2,
                         bUFull = bDrain + 2, bUEmpty = bUFull + kUnitSlots, bOStaged = bUEmpty + kUnitSlots,
                         bTaken = bOStaged + 2, bComb = bTaken + 1, kNumBars = bComb + 1;
    // arrivals that free a unit slot: the two producers, the QK and PV issuers
    // and the 8 softmax warps
    static constexpr int kUnitConsumers = 12;
    static constexpr int kMisc = kBar + kNumBars * 8;
    // split units (paired): the second half's row maximum and sum, per row
    static constexpr int kComb = kMisc + 64;
    static constexpr int kBytes = kComb + (PAIRED ? 128 * 8 : 0);
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
    static_assert(kAlloc <= 227 * 1024, "shared memory per CTA");
    // TMEM columns
    static constexpr uint32_t kTmS = 0, kTmP = 128, kTmO = 256;
    static uint32_t __device__ __forceinline__ tm_p(int h) { return kTmP + 64u * (uint32_t)h; }
    static uint32_t __device__ __forceinline__ tm_o(int h) { return kTmO + (uint32_t)(D * h); }
};

struct Unit {
    int bh, i, it, iy, ix, nh, cnt, nkv;
    const int32_t *list;
};

__device__ __forceinline__ Unit load_unit(const Geo &g, int u, const int32_t *kv_cnt, const int32_t *kv_idx,
                                          int dense)
{
    Unit U;
    U.bh = u / g.nb;
    U.i = u - U.bh * g.nb;
    const int hw = g.nbh * g.nbw;
    U.it = U.i / hw;
    U.iy = (U.i / g.nbw) % g.nbh;
    U.ix = U.i % g.nbw;
    U.nh = (g.nsub == 2 && U.it * g.bt + g.subt < g.T) ? 2 : 1;
    U.cnt = dense ? g.nb : __ldg(kv_cnt + u);
    U.list = dense ? nullptr : kv_idx + (size_t)u * g.nb;
    const bool last_short = (g.nsub == 2) && ((g.nbt - 1) * g.bt + g.subt >= g.T);
    int nlast = 0;
    if (last_short) {
        const int j0 = (g.nbt - 1) * hw;
        if (dense) {
            nlast = g.nb - j0;
        } else {
            int lo = 0, hi = U.cnt;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (__ldg(U.list + mid) >= j0) hi = mid;
                else lo = mid + 1;
            }
            nlast = U.cnt - lo;
        }
    }
    U.nkv = U.cnt * g.nsub - nlast;
    return U;
}

// Walks the kept sub-tiles of a unit in list order.
struct TileCursor {
    int e = 0, s = 0;
    __device__ __forceinline__ int block(const Unit &U) const { return U.list ? __ldg(U.list + e) : e; }
    __device__ __forceinline__ void advance(const Geo &g, const Unit &U)
    {
        if (g.nsub == 2 && s == 0) {
            const int jt = (int)fdiv((uint32_t)block(U), g.fd_hw);
            if (jt * g.bt + g.subt < g.T) {
                s = 1;
                return;
            }
        }
        s = 0;
        ++e;
    }
};

// Paired mode: unit u = query blocks 4q .. 4q+3 of head bh; tile half h runs
// pair 2q+h, i.e. query blocks 4q+2h (rows 0-63) and 4q+2h+1 (rows 64-127).
// A split unit (id BH*upb + bh*npair + p, from the scheduler) runs one pair p
// on both halves: the same query rows, half 0 over the first ceil(tiles/2)
// tiles of the pair's union and half 1 over the rest; half 0 combines the two
// partial results and stores the tile.
struct PairUnit {
    int bh, q;
    int p0, p1;                  // pair of each half
    int split;                   // 1: one pair over both halves
    int c0, c1;                  // union entries of each half (0: nothing)
    const int32_t *l0, *l1;      // the entries; nullptr in dense mode (entry e = block e, kept by both)
    // per-half accessors (selects, so that the struct stays in registers)
    __device__ __forceinline__ int cnt(int h) const { return h ? c1 : c0; }
    __device__ __forceinline__ int tiles(int h) const { return (cnt(h) + 1) >> 1; }
    __device__ __forceinline__ const int32_t *list(int h) const { return h ? l1 : l0; }
    __device__ __forceinline__ int pair(int h) const { return h ? p1 : p0; }
};

// Entries of a split pair's union that half 0 takes: its first ceil(tiles/2) tiles.
__device__ __forceinline__ int split_first(int c)
{
    const int tiles = (c + 1) >> 1;
    return min(c, 2 * ((tiles + 1) >> 1));
}

__device__ __forceinline__ PairUnit load_pair_unit(const Geo &g, int u, const int32_t *pair_cnt,
                                                   const int32_t *pair_list, int dense)
{
    PairUnit P;
    const int n_plain = g.BH * g.upb;
    if (u >= n_plain) {
        const int idx = u - n_plain;
        P.bh = idx / g.npair;
        P.p0 = P.p1 = idx - P.bh * g.npair;
        P.q = P.p0 >> 1;
        P.split = 1;
        const int c = __ldg(pair_cnt + idx);
        P.c0 = split_first(c);
        P.c1 = c - P.c0;
        P.l0 = pair_list + (size_t)idx * g.nb;
        P.l1 = P.c1 > 0 ? P.l0 + P.c0 : nullptr;
        return P;
    }
    P.bh = u / g.upb;
    P.q = u - P.bh * g.upb;
    P.p0 = 2 * P.q;
    P.p1 = 2 * P.q + 1;
    P.split = 0;
    P.c0 = P.c1 = 0;
    P.l0 = P.l1 = nullptr;
    for (int h = 0; h < 2; ++h) {
        const int pp = 2 * P.q + h;
        int c = 0;
        const int32_t *lst = nullptr;
        if (pp < g.npair) {
            if (dense) {
                c = g.nb;
            } else {
                const size_t pid = (size_t)P.bh * g.npair + pp;
                c = __ldg(pair_cnt + pid);
                lst = pair_list + pid * g.nb;
            }
        }
        if (h) {
            P.c1 = c;
            P.l1 = lst;
        } else {
            P.c0 = c;
            P.l0 = lst;
        }
    }
    return P;
}

// The same from the entry counts published in the unit ring (no loads).
__device__ __forceinline__ PairUnit pair_unit_from(const Geo &g, int u, int c0, int c1, const int32_t *pair_list,
                                                   int dense)
{
    PairUnit P;
    const int n_plain = g.BH * g.upb;
    P.c0 = c0;
    P.c1 = c1;
    if (u >= n_plain) {
        const int idx = u - n_plain;
        P.bh = idx / g.npair;
        P.p0 = P.p1 = idx - P.bh * g.npair;
        P.q = P.p0 >> 1;
        P.split = 1;
        P.l0 = pair_list + (size_t)idx * g.nb;
        P.l1 = c1 > 0 ? P.l0 + c0 : nullptr;
        return P;
    }
    P.bh = u / g.upb;
    P.q = u - P.bh * g.upb;
    P.p0 = 2 * P.q;
    P.p1 = 2 * P.q + 1;
    P.split = 0;
    const size_t pid = (size_t)P.bh * g.npair + 2 * P.q;
    P.l0 = (dense || c0 == 0) ? nullptr : pair_list + pid * g.nb;
    P.l1 = (dense || c1 == 0) ? nullptr : pair_list + (pid + 1) * g.nb;
    return P;
}

// Entry e of a union of c entries. Past the end (the second block of an odd
// last tile) it repeats the last block with no keeper, so that block's
// columns are masked out for every row.
__device__ __forceinline__ int pair_entry(const int32_t *lst, int c, int e)
{
    if (c <= 0) return 0;  // empty half: never used
    const bool past = e >= c;
    const int ee = past ? c - 1 : e;
    const int v = lst ? __ldg(lst + ee) : (ee | kPairInA | kPairInB);
    return past ? (v & kPairBlockMask) : v;
}

// Rank r of the longest-first order -> unit id. The scheduler deals ranks to
// C = gridDim.x lists in zigzag rounds (rank r sits at position r / C of list
// zigzag(r)); without a schedule the rank is the unit id itself.
__device__ __forceinline__ int rank_to_unit(long long r, const int32_t *work, const int32_t *cta_range)
{
    if (!work) return (int)r;
    const long long C = gridDim.x;
    const long long pos = r / C, p = r - pos * C;
    const long long c = (pos & 1) ? C - 1 - p : p;
    return __ldg(work + __ldg(cta_range + c) + pos);
}

// Consumer side of the unit ring: wait for the n-th slot and read its unit id
// (-1 ends the sequence); meta() reads the slot's other words. The caller
// frees the slot once it has read what it needs.
struct UnitFeed {
    uint32_t full0;
    const volatile int32_t *slots;
    int n;
    __device__ __forceinline__ int next(volatile int *abort_flag, bool &ok, int &slot)
    {
        slot = n % kUnitSlots;
        if (!mbar_wait(full0 + 8u * (uint32_t)slot, (uint32_t)(n / kUnitSlots) & 1u, abort_flag)) {
            ok = false;
            return -1;
        }
        ++n;
        return slots[slot * kUnitWords];
    }
    __device__ __forceinline__ int meta(int slot, int i) const { return slots[slot * kUnitWords + i]; }
};

template <int D, int BKV, bool PAIRED, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, Geo g,
                const int32_t *__restrict__ kv_cnt, const int32_t *__restrict__ kv_idx,
                const int32_t *__restrict__ pair_cnt, const int32_t *__restrict__ pair_list,
                const int32_t *__restrict__ work, const int32_t *__restrict__ cta_range, int dense,
                int64_t *__restrict__ cta_ns, uint32_t *__restrict__ status)
{
    static_assert(!PAIRED || BKV == 128, "paired mode runs 128-token key/value tiles");
    using L = AttnLayout<D, BKV, PAIRED>;
    extern __shared__ uint8_t attn_smem_raw[];
    const uint32_t raw = smem_u32(attn_smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = attn_smem_raw + (sbase - raw);
    const uint32_t *mask_w = reinterpret_cast<const uint32_t *>(gbase + L::kMask);
    const uint32_t *mask_h = mask_w + g.bw * L::kMaskWords;
    const uint32_t *mask_t = mask_h + g.bh * L::kMaskWords;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + L::kMisc);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + L::kMisc + 16);
    auto bar = [&](int idx) -> uint32_t { return sbase + L::kBar + 8u * (uint32_t)idx; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- set-up: per-axis column masks, barriers, TMEM
    {
        uint32_t *tab = reinterpret_cast<uint32_t *>(gbase + L::kMask);
        const int n_ent = g.bw + g.bh + g.subt;
        for (int ent = threadIdx.x; ent < n_ent; ent += blockDim.x) {
            const int axis = ent < g.bw ? 0 : (ent < g.bw + g.bh ? 1 : 2);
            const int v = 1 + (axis == 0 ? ent : (axis == 1 ? ent - g.bw : ent - g.bw - g.bh));
            for (int w = 0; w < L::kMaskWords; ++w) {
                uint32_t word = 0;
                for (int b = 0; b < 32; ++b) {
                    const int c = w * 32 + b;
                    const int coord = axis == 0 ? c % g.bw : (axis == 1 ? (c / g.bw) % g.bh : c / (g.bh * g.bw));
                    if (coord < v) word |= 1u << b;
                }
                tab[ent * L::kMaskWords + w] = word;
            }
        }
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int b = 0; b < L::kNumBars; ++b) {
            uint32_t cnt = 1;
            if (b == L::bSFree || b == L::bPFull || b == L::bPFull + 1 || b == L::bOEmpty || b == L::bOEmpty + 1 ||
                b == L::bOStaged || b == L::bOStaged + 1 || b == L::bComb)
                cnt = 128;  // arrived on by all 128 threads of a softmax warpgroup
            if (b >= L::bUEmpty && b < L::bUEmpty + kUnitSlots) cnt = L::kUnitConsumers;
            mbar_init(bar(b), cnt);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // launched as a programmatic dependent of the scheduler: everything above
    // overlaps its tail; lists, work and counters are read only after this
    pdl_wait();
    // the wait limit of this call (workspace header, written on the stream before)
    if (threadIdx.x == 0) wait_limit_setup(abort_flag, status);
    __syncthreads();
    const uint64_t t_start = globaltimer_ns();

    // Units are taken dynamically, longest first, from a counter shared by all
    // CTAs (workspace header word 1); the producer thread takes them and hands
    // them to the other roles through the unit ring.
    // ranks to take: the scheduler's unit count (paired layers split long
    // units), or every unit in index order without a schedule; a count beyond
    // what any schedule can hold is refused
    const long long n_max = (long long)g.BH * (g.upb + (PAIRED ? g.npair : 0));
    long long n_units = work ? (long long)__ldg(cta_range + gridDim.x) : (long long)g.BH * g.upb;
    if (n_units < 0 || n_units > n_max) {
        if (threadIdx.x == 0) atomicOr(status, kFlagBadWork);
        n_units = 0;
    }
    uint32_t *unit_cursor = status + 1, *ctas_done = status + 2;
    volatile int32_t *unit_slots = reinterpret_cast<volatile int32_t *>(gbase + L::kUnit);
    UnitFeed feed{bar(L::bUFull), unit_slots, 0};

    constexpr uint32_t kTileBytes = (uint32_t)L::kDH * BKV * 128u;
    constexpr uint32_t kHalfRows = 64u * 128u;  // bytes of 64 rows of a slab (paired mode: second block's offset)
    const uint32_t q_bytes = (uint32_t)L::kDH * (uint32_t)g.rows * 128u;

    if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<D, BKV>::kLow));
    if (warp == 3 && lane == 1) {
        // ================= unit claimer =================
        // Slot n of the unit ring: the unit id and, paired, its union sizes and
        // first entries. Unit n is claimed once warp 0 has issued every load of
        // unit n-1: the claim's chain of loads then overlaps the end of that
        // unit, and a CTA commits to its next unit only as late as the dynamic
        // longest-first order needs.
        bool ok = true;
        // test word of the workspace header: withhold rank (word - 1), so this
        // CTA's roles wait for a unit that never comes
        const long long withhold = (long long)*reinterpret_cast<volatile uint32_t *>(status + kHdrWithhold) - 1;
        for (int n = 0; ok; ++n) {
            const int slot = n % kUnitSlots;
            if (n > 0 && !mbar_wait(bar(L::bTaken), (uint32_t)(n - 1) & 1u, abort_flag)) break;
            if (n >= kUnitSlots &&
                !mbar_wait(bar(L::bUEmpty + slot), (uint32_t)((n / kUnitSlots) - 1) & 1u, abort_flag))
                break;
            const long long r = (long long)atomicAdd(unit_cursor, 1u);
            if (r == withhold) break;  // nothing is published for this rank
            int u = r < n_units ? rank_to_unit(r, work, cta_range) : -1;
            // a unit id out of range, or a CTA busy far beyond any real layer
            // (20 s), ends this CTA's units with a flag instead of running on
            if (u >= n_max || u < -1 || globaltimer_ns() - t_start > 20000000000ull) {
                atomicOr(status, kFlagBadWork);
                u = -1;
            }
            int m[kUnitWords];
            m[0] = u;
#pragma unroll
            for (int i = 1; i < kUnitWords; ++i) m[i] = 0;
            if (PAIRED && u >= 0) {
                PairUnit P = load_pair_unit(g, u, pair_cnt, pair_list, dense);
                if (P.c0 < 0 || P.c1 < 0 || P.c0 > g.nb || P.c1 > g.nb || (P.split && P.c0 + P.c1 > g.nb)) {
                    atomicOr(status, kFlagBadWork);
                    P.c0 = P.c1 = 0;
                }
                m[1] = P.c0;
                m[2] = P.c1;
                m[3] = pair_entry(P.l0, P.c0, 0);
                m[4] = pair_entry(P.l0, P.c0, 1);
                m[5] = pair_entry(P.l1, P.c1, 0);
                m[6] = pair_entry(P.l1, P.c1, 1);
            }
#pragma unroll
            for (int i = 0; i < kUnitWords; ++i) unit_slots[slot * kUnitWords + i] = m[i];
            mbar_arrive(bar(L::bUFull + slot));  // release: the slot is visible to the waiting roles
            if (u < 0) break;
        }
    } else if (warp == 0 || warp == 3) {
        // ================= TMA producers =================
        // warp 0 loads Q and K; warp 3 loads V for the same units, so a K load
        // never waits for a V slot, which frees only after a softmax and a PV
        if (lane == 0) {
            const bool vrole = warp == 3;
            if (vrole) {
                tma_prefetch_desc(&tm_v);
            } else {
                tma_prefetch_desc(&tm_q);
                tma_prefetch_desc(&tm_k);
            }
            int kc = 0, vc = 0;
            uint32_t q_par = 0, q_used = 0;  // per half: loads issued & 1, any load issued
            bool ok = true;
            // one key/value tile: blocks j0 (rows 0..) and, paired, j1 (rows 64..)
            auto load_kv = [&](int j0, int j1, int t_off, int ubh) -> bool {
                const bool pair = PAIRED;
                if (!vrole) {
                    const int ks = kc % L::kNK;
                    if (kc >= L::kNK && !mbar_wait(bar(L::bKEmpty + ks), ((kc / L::kNK) - 1) & 1, abort_flag))
                        return false;
                    mbar_arrive_expect_tx(bar(L::bKFull + ks), kTileBytes);
                    for (int s2 = 0; s2 < (pair ? 2 : 1); ++s2) {
                        int jt, jy, jx;
                        block_coords(g, s2 ? j1 : j0, jt, jy, jx);
                        for (int dh = 0; dh < L::kDH; ++dh)
                            tma_load_5d(sbase + L::kK + (ks * L::kDH + dh) * L::kKVSlab + s2 * kHalfRows, &tm_k,
                                        bar(L::bKFull + ks), dh * 64, jx * g.bw, jy * g.bh, jt * g.bt + t_off, ubh);
                    }
                    ++kc;
                } else {
                    const int vs = vc % L::kNV;
                    if (vc >= L::kNV && !mbar_wait(bar(L::bVEmpty + vs), ((vc / L::kNV) - 1) & 1, abort_flag))
                        return false;
                    mbar_arrive_expect_tx(bar(L::bVFull + vs), kTileBytes);
                    for (int s2 = 0; s2 < (pair ? 2 : 1); ++s2) {
                        int jt, jy, jx;
                        block_coords(g, s2 ? j1 : j0, jt, jy, jx);
                        for (int dh = 0; dh < L::kDH; ++dh)
                            tma_load_5d(sbase + L::kV + (vs * L::kDH + dh) * L::kKVSlab + s2 * kHalfRows, &tm_v,
                                        bar(L::bVFull + vs), dh * 64, jx * g.bw, jy * g.bh, jt * g.bt + t_off, ubh);
                    }
                    ++vc;
                }
                return true;
            };
            // Q half h: rows 0.. from block i0 at frame offset t_off, paired also rows 64.. from i0+1
            auto load_q = [&](int h, int i0, int nblk, int t_off, int ubh) -> bool {
                if (((q_used >> h) & 1u) && !mbar_wait(bar(L::bQEmpty + h), ((q_par >> h) & 1u) ^ 1u, abort_flag))
                    return false;
                mbar_arrive_expect_tx(bar(L::bQFull + h), PAIRED ? (uint32_t)nblk * L::kDH * kHalfRows : q_bytes);
                for (int s2 = 0; s2 < nblk; ++s2) {
                    int jt, jy, jx;
                    block_coords(g, i0 + s2, jt, jy, jx);
                    for (int dh = 0; dh < L::kDH; ++dh)
                        tma_load_5d(sbase + L::kQ + (h * L::kDH + dh) * L::kQSlab + s2 * kHalfRows, &tm_q,
                                    bar(L::bQFull + h), dh * 64, jx * g.bw, jy * g.bh, jt * g.bt + t_off, ubh);
                }
                q_par ^= 1u << h;
                q_used |= 1u << h;
                return true;
            };
            for (int n = 0; ok; ++n) {
                int um[kUnitWords];
                {
                    int slot;
                    um[0] = feed.next(abort_flag, ok, slot);
                    if (!ok) break;
#pragma unroll
                    for (int i = 1; i < kUnitWords; ++i) um[i] = feed.meta(slot, i);
                    mbar_arrive(bar(L::bUEmpty + slot));
                }
                const int u = um[0];
                if (u < 0) break;
                if constexpr (PAIRED) {
                    // paired units load both Q tiles first: a short unit's first
                    // products need them before any key tile
                    const PairUnit P = pair_unit_from(g, u, um[1], um[2], pair_list, dense);
                    for (int h = 0; h < 2 && ok && !vrole; ++h) {
                        if (P.cnt(h) == 0) continue;
                        const int qa = 2 * P.pair(h);  // rows 0-63: block qa, rows 64-127: block qa+1
                        ok = load_q(h, qa, qa + 1 < g.nb ? 2 : 1, 0, P.bh);
                    }
                    // key/value tiles, the two halves interleaved: round r is tile r of
                    // half 0, then tile r of half 1 (each while that half has one)
                    const int rounds = max(P.tiles(0), P.tiles(1));
                    // a round's four entries are loaded one round ahead
                    int cur[4] = {um[3], um[4], um[5], um[6]};
                    for (int r = 0; r < rounds && ok; ++r) {
                        const int nxt[4] = {pair_entry(P.l0, P.c0, 2 * r + 2), pair_entry(P.l0, P.c0, 2 * r + 3),
                                            pair_entry(P.l1, P.c1, 2 * r + 2), pair_entry(P.l1, P.c1, 2 * r + 3)};
                        for (int h = 0; h < 2 && ok; ++h) {
                            if (r >= P.tiles(h)) continue;
                            ok = load_kv((h ? cur[2] : cur[0]) & kPairBlockMask, (h ? cur[3] : cur[1]) & kPairBlockMask,
                                         0, P.bh);
                        }
#pragma unroll
                        for (int x = 0; x < 4; ++x) cur[x] = nxt[x];
                    }
                    // every load of this unit is issued: the claimer may take the next one
                    if (!vrole) mbar_arrive(bar(L::bTaken));
                    continue;
                }
                if constexpr (!PAIRED) {
                    // The first kNK key tiles of a unit go to ring slots last filled
                    // by the previous unit, so they are issued before this unit's Q
                    // loads wait for the previous unit's epilogues; a later tile's
                    // slot frees only after this unit's own first products.
                    const Unit U = load_unit(g, u, kv_cnt, kv_idx, dense);
                    const int early = vrole ? 0 : min(U.nkv, L::kNK);
                    TileCursor cur;
                    int k = 0;
                    for (; k < early && ok; ++k) {
                        ok = load_kv(cur.block(U), 0, cur.s * g.subt, U.bh);
                        cur.advance(g, U);
                    }
                    for (int h = 0; h < U.nh && ok && !vrole; ++h) ok = load_q(h, U.i, 1, h * g.subt, U.bh);
                    for (; k < U.nkv && ok; ++k) {
                        ok = load_kv(cur.block(U), 0, cur.s * g.subt, U.bh);
                        cur.advance(g, U);
                    }
                    if (!vrole) mbar_arrive(bar(L::bTaken));
                }
            }
            if (!ok) {
                // wind down: let every copy already issued land before the CTA exits
                for (int s = 0; s < L::kNK; ++s) {
                    const int n = (kc > s) ? (kc - s + L::kNK - 1) / L::kNK : 0;
                    if (n > 0) mbar_wait_for(bar(L::bKFull + s), (n - 1) & 1, 50000000ull);
                }
                for (int s = 0; s < L::kNV; ++s) {
                    const int n = (vc > s) ? (vc - s + L::kNV - 1) / L::kNV : 0;
                    if (n > 0) mbar_wait_for(bar(L::bVFull + s), (n - 1) & 1, 50000000ull);
                }
                for (int h = 0; h < 2; ++h)
                    if ((q_used >> h) & 1u) mbar_wait_for(bar(L::bQFull + h), ((q_par >> h) & 1u) ^ 1u, 50000000ull);
            }
        }
    } else if (warp == 1) {
        // ================= QK issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_16(128, BKV, false, F16);
            // descriptors of the first slab of each region; every other operand
            // is a fixed byte offset from it (added to the start-address field)
            const uint64_t q_desc = sdesc_sw128(sbase + L::kQ, 16, 1024);
            const uint64_t k_desc = sdesc_sw128(sbase + L::kK, 16, 1024);
            int kc = 0, qk_count = 0;
            uint32_t ph_q = 0;
            bool ok = true;
            // S = Q_h K^T over D in K=16 steps; Q and K slabs are K-major, 128B swizzle
            auto issue_qk = [&](int h, int ks) {
                const uint64_t kb = k_desc + (uint64_t)((ks * L::kDH * L::kKVSlab) >> 4);
                const uint64_t qa = q_desc + (uint64_t)((h * L::kDH * L::kQSlab) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off_a = ((kk >> 2) * L::kQSlab + (kk & 3) * 32) >> 4;
                    const uint32_t off_b = ((kk >> 2) * L::kKVSlab + (kk & 3) * 32) >> 4;
                    umma_ss(tmem + L::kTmS, qa + off_a, kb + off_b, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            while (ok) {
                int slot;
                const int u = feed.next(abort_flag, ok, slot);
                if (!ok) break;
                const int mc0 = feed.meta(slot, 1), mc1 = feed.meta(slot, 2);
                mbar_arrive(bar(L::bUEmpty + slot));
                if (u < 0) break;
                if constexpr (PAIRED) {
                    const PairUnit P = pair_unit_from(g, u, mc0, mc1, pair_list, dense);
                    const int rounds = max(P.tiles(0), P.tiles(1));
                    for (int r = 0; r < rounds && ok; ++r) {
                        for (int h = 0; h < 2 && ok; ++h) {
                            if (r >= P.tiles(h)) continue;
                            // each half's Q tile is waited for just before its first product
                            if (r == 0) {
                                ok = mbar_wait(bar(L::bQFull + h), (ph_q >> h) & 1u, abort_flag);
                                ph_q ^= 1u << h;
                                if (!ok) break;
                            }
                            const int ks = kc % L::kNK;
                            if (!mbar_wait(bar(L::bKFull + ks), (kc / L::kNK) & 1, abort_flag)) { ok = false; break; }
                            if (qk_count > 0 && !mbar_wait(bar(L::bSFree), (qk_count - 1) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            issue_qk(h, ks);
                            umma_commit(bar(L::bSFull + h));
                            ++qk_count;
                            umma_commit(bar(L::bKEmpty + ks));
                            ++kc;
                        }
                    }
                    continue;
                }
                const Unit U = load_unit(g, u, kv_cnt, kv_idx, dense);
                for (int h = 0; h < U.nh && ok; ++h) {
                    ok = mbar_wait(bar(L::bQFull + h), (ph_q >> h) & 1u, abort_flag);
                    ph_q ^= 1u << h;
                }
                for (int k = 0; k < U.nkv && ok; ++k) {
                    const int ks = kc % L::kNK;
                    if (!mbar_wait(bar(L::bKFull + ks), (kc / L::kNK) & 1, abort_flag)) { ok = false; break; }
                    for (int h = 0; h < U.nh; ++h) {
                        // S is shared: overwrite it only once the previous S has been
                        // copied into registers by its softmax warpgroup
                        if (qk_count > 0 && !mbar_wait(bar(L::bSFree), (qk_count - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        issue_qk(h, ks);
                        umma_commit(bar(L::bSFull + h));
                        ++qk_count;
                    }
                    if (!ok) break;
                    umma_commit(bar(L::bKEmpty + ks));
                    ++kc;
                }
            }
            // every MMA issued must finish before TMEM is released
            umma_commit(bar(L::bDrain));
            mbar_wait_for(bar(L::bDrain), 0, 100000000ull);
        }
    } else if (warp == 2) {
        // ================= PV issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_pv = idesc_16(128, D, true, F16);
            const uint64_t v_desc = sdesc_sw128(sbase + L::kV, L::kKVSlab, 1024);
            int vc = 0;
            uint32_t ph_p = 0, ph_oe = 0, o_pend = 0;
            bool ok = true;
            // O_h (+)= P_h V over the sub-tile in K=16 steps; P_h from TMEM, V MN-major
            auto issue_pv = [&](int h, int vs, bool first) {
                const uint64_t vb = v_desc + (uint64_t)((vs * L::kDH * L::kKVSlab) >> 4);
                const uint32_t d_tmem = tmem + L::tm_o(h), a_tmem = tmem + L::tm_p(h);
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    umma_ts(d_tmem, a_tmem + kk * 8, vb + (uint64_t)((kk * 16 * 128) >> 4), idesc_pv,
                            (!first || kk > 0) ? 1u : 0u);
            };
            // before the first product of a unit into O_h: the previous unit's
            // epilogue must have read O_h
            auto o_free = [&](int h) {
                if ((o_pend >> h) & 1u) {
                    if (!mbar_wait(bar(L::bOEmpty + h), (ph_oe >> h) & 1u, abort_flag)) return false;
                    ph_oe ^= 1u << h;
                    o_pend &= ~(1u << h);
                }
                return true;
            };
            while (ok) {
                int slot;
                const int u = feed.next(abort_flag, ok, slot);
                if (!ok) break;
                const int mc0 = feed.meta(slot, 1), mc1 = feed.meta(slot, 2);
                mbar_arrive(bar(L::bUEmpty + slot));
                if (u < 0) break;
                if constexpr (PAIRED) {
                    const PairUnit P = pair_unit_from(g, u, mc0, mc1, pair_list, dense);
                    const int rounds = max(P.tiles(0), P.tiles(1));
                    for (int r = 0; r < rounds && ok; ++r) {
                        for (int h = 0; h < 2 && ok; ++h) {
                            if (r >= P.tiles(h)) continue;
                            const int vs = vc % L::kNV;
                            if (!mbar_wait(bar(L::bVFull + vs), (vc / L::kNV) & 1, abort_flag)) { ok = false; break; }
                            ok = mbar_wait(bar(L::bPFull + h), (ph_p >> h) & 1u, abort_flag);
                            ph_p ^= 1u << h;
                            if (ok && r == 0) ok = o_free(h);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(h, vs, r == 0);
                            umma_commit(bar(L::bPFree + h));
                            if (r == P.tiles(h) - 1) {
                                umma_commit(bar(L::bOFull + h));
                                o_pend |= 1u << h;
                            }
                            umma_commit(bar(L::bVEmpty + vs));
                            ++vc;
                        }
                    }
                    continue;
                }
                const Unit U = load_unit(g, u, kv_cnt, kv_idx, dense);
                for (int k = 0; k < U.nkv && ok; ++k) {
                    const int vs = vc % L::kNV;
                    if (!mbar_wait(bar(L::bVFull + vs), (vc / L::kNV) & 1, abort_flag)) { ok = false; break; }
                    for (int h = 0; h < U.nh; ++h) {
                        ok = mbar_wait(bar(L::bPFull + h), (ph_p >> h) & 1u, abort_flag);
                        ph_p ^= 1u << h;
                        if (ok && k == 0) ok = o_free(h);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(h, vs, k == 0);
                        umma_commit(bar(L::bPFree + h));
                        if (k == U.nkv - 1) {
                            umma_commit(bar(L::bOFull + h));
                            o_pend |= 1u << h;
                        }
                    }
                    if (!ok) break;
                    umma_commit(bar(L::bVEmpty + vs));
                    ++vc;
                }
            }
            umma_commit(bar(L::bDrain + 1));
            mbar_wait_for(bar(L::bDrain + 1), 0, 100000000ull);
        }
    } else if (warp >= 4) {
        // ================= softmax + epilogue =================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<D, BKV>::kHigh));
        const int h = (warp - 4) >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t t_lane = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + t_lane + L::kTmS;
        const uint32_t tP = tmem + t_lane + L::tm_p(h);
        const uint32_t tO = tmem + t_lane + L::tm_o(h);
        const float sl2 = g.scale * 1.4426950408889634f;
        int sf = 0, of = 0, pw = 0;  // S tiles received, O tiles received, P tiles written
        bool ok = true;
        float m = -INFINITY, l = 0.f;
        // One key/value tile of this half: S from TMEM, masks, online softmax,
        // P into TMEM (after the previous PV of this half), lazy O rescale.
        // keep: bit 0 / bit 1 = columns 0-63 / 64-127 take part (paired mode:
        // the key block there was kept by this row's query block); apply_mask
        // masks padding inside kept columns.
        auto tile = [&](bool first, uint32_t keep, auto &&apply_mask) -> bool {
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bSFull + h), sf & 1, abort_flag))) return false;
            ++sf;
            tc_fence_after();
            // all BKV columns in one batch, one wait; the register fences keep
            // every use of the loaded values after the wait
            uint32_t r[BKV];
#pragma unroll
            for (int c = 0; c < BKV / 32; ++c) tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(r + c * 32));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < BKV / 32; ++c) reg_fence32(r + c * 32);
            // S is in registers: the next QK may overwrite it
            tc_fence_before();
            mbar_arrive(bar(L::bSFree));
            float x[BKV];
#pragma unroll
            for (int c = 0; c < BKV; ++c) x[c] = __uint_as_float(r[c]);
            apply_mask(x);
            // row maximum of each 64-column half: 4 independent chains of
            // three-input max each, then trees; a half that takes no part is left out
            float m8[8];
#pragma unroll
            for (int q8 = 0; q8 < 8; ++q8) m8[q8] = -INFINITY;
#pragma unroll
            for (int c = 0; c < BKV / 2; c += 8)
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    m8[q4] = max3f(m8[q4], x[c + 2 * q4], x[c + 2 * q4 + 1]);
                    m8[4 + q4] = max3f(m8[4 + q4], x[BKV / 2 + c + 2 * q4], x[BKV / 2 + c + 2 * q4 + 1]);
                }
            const float mxa = fmaxf(max3f(m8[0], m8[1], m8[2]), m8[3]);
            const float mxb = fmaxf(max3f(m8[4], m8[5], m8[6]), m8[7]);
            const float mx = fmaxf((keep & 1u) ? mxa : -INFINITY, (keep & 2u) ? mxb : -INFINITY);
            const float mt = mx * sl2;
            float alpha = 1.0f;
            bool rescale = false;
            if (first) {
                m = mt;
            } else {
                const bool need = mt > m + kRescaleThreshold;
                rescale = __any_sync(0xFFFFFFFFu, need);
                if (need) {
                    alpha = ex2_approx(m - mt);
                    m = mt;
                    l *= alpha;
                }
            }
            // p = 2^(x*scale*log2e - m): packed fp32x2 FMA/ADD and MUFU ex2,
            // packed to bf16 pairs in registers first, so this work
            // overlaps the PV that still reads the previous P_h
            // paired mode: a row whose own query block kept no block of the
            // tiles so far has m = -inf; its p are 0 (not inf - inf)
            const float m_use = (PAIRED && m == -INFINITY) ? 0.f : m;
            // a half that takes no part gets 2^-inf = 0
            const float na = (keep & 1u) ? -m_use : -INFINITY, nb = (keep & 2u) ? -m_use : -INFINITY;
            const uint64_t sl2x2 = f2_pack(sl2, sl2), neg_a = f2_pack(na, na), neg_b = f2_pack(nb, nb);
            uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};
            uint32_t pk[BKV / 2];
#pragma unroll
            for (int q2 = 0; q2 < BKV / 2; ++q2) {
                const uint64_t a = f2_fma(f2_pack(x[2 * q2], x[2 * q2 + 1]), sl2x2, q2 < BKV / 4 ? neg_a : neg_b);
                float a0, a1;
                f2_unpack(a, a0, a1);
                const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
                s4[q2 & 3] = f2_add(s4[q2 & 3], f2_pack(p0, p1));
                pk[q2] = pack16x2<F16>(p0, p1);
            }
            float sum;
            {
                const uint64_t t = f2_add(f2_add(s4[0], s4[1]), f2_add(s4[2], s4[3]));
                float t0, t1;
                f2_unpack(t, t0, t1);
                sum = t0 + t1;
            }
            // P_h and O_h are free once the PV of this half's previous sub-tile is done
            if (pw > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bPFree + h), (pw - 1) & 1, abort_flag)))
                return false;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < BKV / 32; ++c) tmem_st16(tP + c * 16, pk + c * 16);
            if (rescale) {
                // O_h holds the sum up to the previous sub-tile (its PV is done);
                // bring it to the new row maximum
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + c * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 32; ++v) o[v] = __float_as_uint(__uint_as_float(o[v]) * alpha);
                    tmem_st32(tO + c * 32, o);
                }
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::bPFull + h));
            ++pw;
            l += sum;
            return true;
        };
        // epilogue: O / l in the element type, staged in this half's Q tile (every
        // product that reads it is done once O_h is complete) in the tile's own
        // swizzled layout, then written by TMA stores, which skip the rows
        // outside the grid; the Q tile goes back to the producer once the stores
        // have read it
        const uint32_t o_stage = sbase + L::kQ + (uint32_t)(h * L::kDH * L::kQSlab) + (uint32_t)row * 128u;
        // split units: the second half's row maximum and sum
        float2 *comb = reinterpret_cast<float2 *>(gbase + L::kComb);
        int of1 = 0, cb = 0;  // half 0: phases of O_1's completion seen so far, split units combined
        int st = 0;           // epilogues of this half that staged a tile (the storing thread's phases)
        // comb_in (half 0 of a split unit): O = (O_0 2^(m0-m) + O_1 2^(m1-m)) / (l0 2^(m0-m) + l1 2^(m1-m)),
        // m = max(m0, m1), with (m1, l1) published by half 1 and O_1 read from TMEM
        auto epilogue = [&](int ubh, int i0, int nblk, int t_off, bool comb_in, int of1_phase) -> bool {
            // every wait's outcome is agreed by the whole warp before the next
            // warp-collective TMEM access or the caller's loop exit
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bOFull + h), of & 1, abort_flag))) return false;
            ++of;
            float w0, w1 = 0.f;
            if (comb_in) {
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bOFull + 1), of1_phase & 1, abort_flag))) return false;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bComb), cb & 1, abort_flag))) return false;
                ++cb;
                const float2 c1 = comb[row];
                // every real row keeps a block in one half at least; padded rows are never stored
                const float mm = fmaxf(m, c1.x);
                const float a0 = m == -INFINITY ? 0.f : ex2_approx(m - mm);
                const float a1 = c1.x == -INFINITY ? 0.f : ex2_approx(c1.x - mm);
                const float inv = 1.0f / (l * a0 + c1.y * a1);
                w0 = a0 * inv;
                w1 = a1 * inv;
            } else {
                w0 = 1.0f / l;
            }
            tc_fence_after();
            const uint32_t tO1 = tmem + t_lane + L::tm_o(1);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + c * 32, o);
                if (comb_in) {
                    uint32_t o1[32];
                    tmem_ld32(tO1 + c * 32, o1);
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 32; ++v)
                        o[v] = __float_as_uint(__uint_as_float(o[v]) * w0 + __uint_as_float(o1[v]) * w1);
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 32; ++v) o[v] = __float_as_uint(__uint_as_float(o[v]) * w0);
                }
                if (c == D / 32 - 1) {
                    // O_h (and, combining, O_1) have been read: the next unit's
                    // first product may overwrite them
                    tc_fence_before();
                    mbar_arrive(bar(L::bOEmpty + h));
                    if (comb_in) mbar_arrive(bar(L::bOEmpty + 1));
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 w;
                    w.x = pack16x2<F16>(__uint_as_float(o[q4 * 8 + 0]), __uint_as_float(o[q4 * 8 + 1]));
                    w.y = pack16x2<F16>(__uint_as_float(o[q4 * 8 + 2]), __uint_as_float(o[q4 * 8 + 3]));
                    w.z = pack16x2<F16>(__uint_as_float(o[q4 * 8 + 4]), __uint_as_float(o[q4 * 8 + 5]));
                    w.w = pack16x2<F16>(__uint_as_float(o[q4 * 8 + 6]), __uint_as_float(o[q4 * 8 + 7]));
                    // 16-byte piece j of the row: slab j / 8, 128-byte swizzle of piece j % 8
                    const int j = c * 4 + q4;
                    st_shared_v4(o_stage + (uint32_t)((j >> 3) * L::kQSlab) + (uint32_t)(((j & 7) ^ (row & 7)) << 4),
                                 w);
                }
            }
            // the tile is written: make it visible to the TMA engine, then the
            // storing thread waits (with the usual time limit) for all 128 rows
            fence_proxy_async();
            mbar_arrive(bar(L::bOStaged + h));
            // phase of this staging: staged epilogues so far (a split unit's second
            // half completes O_1 without staging)
            const int st_phase = st++;
            bool stored = true;
            if (row == 0) {
                stored = mbar_wait(bar(L::bOStaged + h), st_phase & 1, abort_flag);
            }
            if (row == 0 && stored) {
                for (int s2 = 0; s2 < nblk; ++s2) {
                    int jt, jy, jx;
                    block_coords(g, i0 + s2, jt, jy, jx);
                    for (int dh = 0; dh < L::kDH; ++dh)
                        tma_store_5d(&tm_o, sbase + L::kQ + (h * L::kDH + dh) * L::kQSlab + s2 * kHalfRows, dh * 64,
                                     jx * g.bw, jy * g.bh, jt * g.bt + t_off, ubh);
                }
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(bar(L::bQEmpty + h));
            }
            // the storing thread's outcome, agreed by its warp
            return __all_sync(0xFFFFFFFFu, stored);
        };
        while (ok) {
            int slot;
            const int u = feed.next(abort_flag, ok, slot);
            ok = __all_sync(0xFFFFFFFFu, ok);  // the warp leaves the loop together, or not at all
            if (!ok) break;
            int mc0 = 0, mc1 = 0, me0 = 0, me1 = 0;
            if constexpr (PAIRED) {
                mc0 = feed.meta(slot, 1);
                mc1 = feed.meta(slot, 2);
                me0 = feed.meta(slot, 3 + 2 * h);
                me1 = feed.meta(slot, 4 + 2 * h);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::bUEmpty + slot));  // every lane has read the slot
            if (u < 0) break;
            if constexpr (PAIRED) {
                const PairUnit P = pair_unit_from(g, u, mc0, mc1, pair_list, dense);
                const int c_h = P.cnt(h), n_h = P.tiles(h);
                const int32_t *lst = P.list(h);
                // phases of O_1's completion: one per unit in which half 1 has tiles
                const int of1_phase = of1;
                if (P.tiles(1) > 0) ++of1;
                if (n_h == 0) continue;
                const int hb = row >> 6;                   // 0: first query block of the pair, 1: second
                const int keeper = hb ? kPairInB : kPairInA;
                m = -INFINITY;
                l = 0.f;
                int ent0 = me0, ent1 = me1;
                for (int r = 0; r < n_h; ++r) {
                    // the next tile's entries are loaded now and used next iteration
                    const int nxt0 = pair_entry(lst, c_h, 2 * r + 2), nxt1 = pair_entry(lst, c_h, 2 * r + 3);
                    // columns [64*s2, 64*s2+64) hold key block ent(s2): they take part
                    // if this row's query block kept it, with its padding masked
                    uint32_t keep = 0, mw[4];
                    bool all = true;
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2) {
                        const int ent = s2 ? ent1 : ent0;
                        int jt, jy, jx;
                        block_coords(g, ent & kPairBlockMask, jt, jy, jx);
                        const int wv = min(g.bw, g.W - jx * g.bw), hv = min(g.bh, g.Hg - jy * g.bh);
                        const int tv = min(g.bt, g.T - jt * g.bt);
                        const bool kept = (ent & keeper) != 0;
                        const bool full = wv == g.bw && hv == g.bh && tv == g.bt;
                        keep |= kept ? (1u << s2) : 0u;
#pragma unroll
                        for (int w = 0; w < L::kMaskWords; ++w) {
                            const uint32_t word = (!kept || full) ? 0xFFFFFFFFu
                                                                  : (mask_w[(wv - 1) * L::kMaskWords + w] &
                                                                     mask_h[(hv - 1) * L::kMaskWords + w] &
                                                                     mask_t[(tv - 1) * L::kMaskWords + w]);
                            mw[s2 * L::kMaskWords + w] = word;
                            all = all && word == 0xFFFFFFFFu;
                        }
                    }
                    auto mask = [&](float(&x)[BKV]) {
                        if (all) return;
#pragma unroll
                        for (int w = 0; w < 4; ++w)
#pragma unroll
                            for (int b = 0; b < 32; ++b)
                                if (!((mw[w] >> b) & 1u)) x[w * 32 + b] = -INFINITY;
                    };
                    if (!tile(r == 0, keep, mask)) { ok = false; break; }
                    ent0 = nxt0;
                    ent1 = nxt1;
                }
                if (!ok) break;
                if (P.split && h == 1) {
                    // second half of a split unit: once O_1 is complete, publish
                    // the row maximum and sum and hand Q_1 back (its products are
                    // done); half 0 reads O_1, combines and stores the tile
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(L::bOFull + 1), of & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    ++of;
                    comb[row] = make_float2(m, l);
                    mbar_arrive(bar(L::bComb));
                    if (row == 0) mbar_arrive(bar(L::bQEmpty + 1));
                    continue;
                }
                const int qa = 2 * P.pair(h);
                if (!epilogue(P.bh, qa, qa + 1 < g.nb ? 2 : 1, 0, P.split && P.tiles(1) > 0, of1_phase)) {
                    ok = false;
                    break;
                }
                continue;
            }
            const Unit U = load_unit(g, u, kv_cnt, kv_idx, dense);
            if (h >= U.nh) continue;
            m = -INFINITY;
            l = 0.f;
            int e = 0, s_sub = 0;
            int j = U.list ? __ldg(U.list) : 0;
            for (int k = 0; k < U.nkv; ++k) {
                // the list entry after this one is loaded now and used next iteration
                const int j_next = (U.list && e + 1 < U.cnt) ? __ldg(U.list + e + 1) : e + 1;
                int jt, jy, jx;
                block_coords(g, j, jt, jy, jx);
                const int wv = min(g.bw, g.W - jx * g.bw), hv = min(g.bh, g.Hg - jy * g.bh);
                const int tv = min(g.subt, g.T - (jt * g.bt + s_sub * g.subt));
                const bool full = (wv == g.bw) && (hv == g.bh) && (tv == g.subt);
                auto mask = [&](float(&x)[BKV]) {
                    if (!full) {
    #pragma unroll
                        for (int w = 0; w < L::kMaskWords; ++w) {
                            const uint32_t word = mask_w[(wv - 1) * L::kMaskWords + w] &
                                                  mask_h[(hv - 1) * L::kMaskWords + w] &
                                                  mask_t[(tv - 1) * L::kMaskWords + w];
    #pragma unroll
                            for (int b = 0; b < 32; ++b)
                                if (!((word >> b) & 1u)) x[w * 32 + b] = -INFINITY;
                        }
                    }
                };
                if (!tile(k == 0, 3u, mask)) { ok = false; break; }
                if (g.nsub == 2 && s_sub == 0 && jt * g.bt + g.subt < g.T) {
                    s_sub = 1;
                } else {
                    s_sub = 0;
                    ++e;
                    j = j_next;
                }
            }
            if (!ok) break;
            if (!epilogue(U.bh, U.i, 1, h * g.subt, false, 0)) { ok = false; break; }
        }
        // the output stores have completed before the CTA exits
        if (row == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
    if (threadIdx.x == 0) {
        if (*abort_flag) atomicOr(status, kFlagTimeout);
        if (cta_ns) cta_ns[blockIdx.x] = (int64_t)(globaltimer_ns() - t_start);
        // every CTA has taken its last rank before it gets here; the last CTA to
        // finish resets the shared counters for the next launch on this workspace
        __threadfence();
        if (atomicAdd(ctas_done, 1u) == gridDim.x - 1) {
            atomicExch(unit_cursor, 0u);
            atomicExch(ctas_done, 0u);
        }
    }
}

// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// [B*H, T, Hg, W, D] bf16 as a 5-D TMA tensor; box = one sub-tile slab.
static bool make_map(CUtensorMap *map, const Geo &g, const void *ptr)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)g.D, (cuuint64_t)g.W, (cuuint64_t)g.Hg, (cuuint64_t)g.T,
                                (cuuint64_t)g.BH};
    const cuuint64_t es = 2;
    const cuuint64_t strides[4] = {(cuuint64_t)g.D * es, (cuuint64_t)g.W * g.D * es,
                                   (cuuint64_t)g.Hg * g.W * g.D * es, (cuuint64_t)g.N * g.D * es};
    const cuuint32_t box[5] = {64u, (cuuint32_t)g.bw, (cuuint32_t)g.bh, (cuuint32_t)g.subt, 1u};
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    CUresult r = enc(map, g.f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5,
                     const_cast<void *>(ptr), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D, int BKV, bool PAIRED, bool F16>
static cudaError_t launch_attn_f(const Geo &g, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const CUtensorMap &mo, const int32_t *kv_cnt, const int32_t *kv_idx,
                                 const int32_t *pair_cnt, const int32_t *pair_list, const int32_t *work,
                                 const int32_t *cta_range, int grid, int dense, int64_t *cta_ns, uint32_t *status,
                                 cudaStream_t stream)
{
    using L = AttnLayout<D, BKV, PAIRED>;
    auto kern = attn_kernel<D, BKV, PAIRED, F16>;
    cudaFuncAttributes fa;
    cudaError_t err = cudaFuncGetAttributes(&fa, kern);
    if (err != cudaSuccess) return err;
    // the setmaxnreg split must fit in what the launch provides, or the
    // softmax warpgroups would wait for registers forever
    if (fa.numRegs * kThreads < 128 * RegSplit<D, BKV>::kLow + 256 * RegSplit<D, BKV>::kHigh)
        return cudaErrorInvalidConfiguration;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (err != cudaSuccess) return err;
    return launch_dependent(kern, dim3(grid), dim3(kThreads), L::kAlloc, stream, mq, mk, mv, mo, g, kv_cnt, kv_idx,
                            pair_cnt, pair_list, work, cta_range, dense, cta_ns, status);
}

template <int D, int BKV, bool PAIRED>
static cudaError_t launch_attn_t(const Geo &g, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                                 const CUtensorMap &mo, const int32_t *kv_cnt, const int32_t *kv_idx,
                                 const int32_t *pair_cnt, const int32_t *pair_list, const int32_t *work,
                                 const int32_t *cta_range, int grid, int dense, int64_t *cta_ns, uint32_t *status,
                                 cudaStream_t stream)
{
    if (g.f16)
        return launch_attn_f<D, BKV, PAIRED, true>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                                   cta_range, grid, dense, cta_ns, status, stream);
    return launch_attn_f<D, BKV, PAIRED, false>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                                cta_range, grid, dense, cta_ns, status, stream);
}

cudaError_t launch_attn(const Geo &g, const void *q, const void *k, const void *v, const int32_t *kv_cnt,
                        const int32_t *kv_idx, const int32_t *pair_cnt, const int32_t *pair_list,
                        const int32_t *work, const int32_t *cta_range, int num_ctas, int dense, void *out,
                        int64_t *cta_ns, uint32_t *status, cudaStream_t stream, int *launch_error_kind)
{
    *launch_error_kind = 0;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, g, q) || !make_map(&mk, g, k) || !make_map(&mv, g, v) || !make_map(&mo, g, out)) {
        *launch_error_kind = 1;
        return cudaErrorInvalidValue;
    }
    int grid = num_ctas;
    if (!work) {
        const long long U = (long long)g.BH * g.upb;
        if (U < grid) grid = (int)U;
    }
    if (g.paired) {
        if (g.D == 128)
            return launch_attn_t<128, 128, true>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                                 cta_range, grid, dense, cta_ns, status, stream);
        return launch_attn_t<64, 128, true>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                            cta_range, grid, dense, cta_ns, status, stream);
    }
    if (g.D == 128)
        return launch_attn_t<128, 128, false>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                              cta_range, grid, dense, cta_ns, status, stream);
    return launch_attn_t<64, 128, false>(g, mq, mk, mv, mo, kv_cnt, kv_idx, pair_cnt, pair_list, work,
                                         cta_range, grid, dense, cta_ns, status, stream);
}

}  // namespace fvattn
