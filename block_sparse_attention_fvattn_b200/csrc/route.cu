// route.cu -- the sparse-routing frontend of adaptive block-sparse attention.
//
// K1 pool_kernel: block means of Q and K over the valid tokens of every
//   video-aware (t,h,w) block (zskr.cn FastVideo VSA guide, section 1: the
//   post-patch latent grid is cut into spatio-temporal blocks; section 6:
//   variable-length edge blocks, padding never acts as a key). HBM-bound: one
//   pass over Q and K with 16-byte coalesced loads; a CTA pools a strip of one
//   block row, reading its (t, y) runs of contiguous tokens.
// K2 score_select_kernel: per (head, query block) row: block scores
//   s = scale * Qbar_i . Kbar_j, softmax, Top-p with a Top-k floor, diagonal
//   repair and ascending compaction (ai-feeds.com FVAttn summary, "Key
//   modules" 1; hotpaper.ai abstract). The score rows stay in shared memory
//   (computed here, or copied from the tensor-core scores of long rows). One
//   warp owns one row. Selection is exact in fp32 on order-preserving integer
//   keys of the scores: rows of up to 256 blocks sort their keys; longer rows
//   bisect the key space to the score at the Top-p boundary (by probability
//   mass) and, if the floor binds, at rank m. Ties at the boundary go to the
//   lower block index.
#include "common.cuh"
#include "internal.h"

namespace fvattn {

// ---------------------------------------------------------------------------
// K1
// A CTA pools a strip of blocks: one block row (jt, jy) and a run of block
// columns [jx0, jx1). For every (t, y) the strip's tokens x0 .. x1-1 are one
// contiguous run of (x1 - x0) * D bf16 values, so the CTA streams tv * yv
// contiguous runs. Thread tid owns the 16-byte positions tid + kPoolThreads*s
// of every run (s < NS): a fixed token column and d-chunk, so each load is a
// pointer step and the running sums stay in registers (packed fp32x2 adds).
// At the end the columns of each block are added in ascending x through
// shared memory.
constexpr int kPoolThreads = 256;

struct PoolPlan {
    int nxs;  // strips per block row
    int ns;   // positions per thread and run (1, 2, 3, 4 or 8)
};

__host__ __device__ inline PoolPlan pool_plan(int nbw, int bw, int D)
{
    const int lpt = D / 8;
    const int cap = kPoolThreads * 3 / (bw * lpt);  // block columns per strip at NS <= 3
    PoolPlan pl;
    pl.nxs = cap >= 1 ? (nbw + cap - 1) / cap : nbw;
    const int xb = (nbw + pl.nxs - 1) / pl.nxs;
    const int need = (xb * bw * lpt + kPoolThreads - 1) / kPoolThreads;
    pl.ns = need <= 4 ? need : 8;
    return pl;
}

template <int D, int NS, bool F16>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geo g, int nxs, const uint16_t *__restrict__ q,
                                                            const uint16_t *__restrict__ k,
                                                            float *__restrict__ qbar, float *__restrict__ kbarT)
{
    constexpr int LPT = D / 8;  // 16-byte chunks per token
    constexpr int RB = NS >= 8 ? 1 : 8 / NS;  // runs per batch of loads
    extern __shared__ __align__(16) float red[];  // [positions][8]

    // task -> (which, bh, jt, jy, xs); xs fastest so neighbouring CTAs read
    // neighbouring memory
    long long task = blockIdx.x;
    const int xs = (int)(task % nxs);
    task /= nxs;
    const int nbt = g.nbt, nbh = g.nbh, nbw = g.nbw;
    const int jy = (int)(task % nbh);
    task /= nbh;
    const int jt = (int)(task % nbt);
    task /= nbt;
    const long long per = g.BH;
    const int which = task >= per ? 1 : 0;
    const int bh = (int)(task - which * per);

    const int jx0 = (int)((long long)xs * nbw / nxs), jx1 = (int)((long long)(xs + 1) * nbw / nxs);
    const int x0 = jx0 * g.bw, x1 = min(jx1 * g.bw, g.W);
    const int t0 = jt * g.bt, y0 = jy * g.bh;
    const int tv = min(g.bt, g.T - t0), yv = min(g.bh, g.Hg - y0);
    const int npos = (x1 - x0) * LPT;
    const int tid = threadIdx.x;

    const uint16_t *src = which ? k : q;
    const uint4 *run = reinterpret_cast<const uint4 *>(src + (size_t)bh * g.N * D) +
                       (((size_t)t0 * g.Hg + y0) * g.W + x0) * LPT;
    const size_t run_step = (size_t)g.W * LPT;                            // next y
    const size_t t_step = ((size_t)g.Hg - (size_t)yv) * g.W * LPT;         // extra at a new t

    bool own[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) own[s] = tid + kPoolThreads * s < npos;
    uint64_t acc[NS][4];
#pragma unroll
    for (int s = 0; s < NS; ++s)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[s][c] = 0ull;

    const int nrun = tv * yv;
    int y = 0;
    for (int r = 0; r < nrun; r += RB) {
        uint4 v[RB][NS];
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            const bool ok = r + b < nrun;
#pragma unroll
            for (int s = 0; s < NS; ++s)
                if (ok && own[s]) v[b][s] = __ldg(run + tid + kPoolThreads * s);
            if (ok) {
                run += run_step;
                if (++y == yv) {
                    y = 0;
                    run += t_step;
                }
            }
        }
#pragma unroll
        for (int b = 0; b < RB; ++b) {
            if (r + b < nrun) {
#pragma unroll
                for (int s = 0; s < NS; ++s) {
                    if (own[s]) {
                        const uint32_t w[4] = {v[b][s].x, v[b][s].y, v[b][s].z, v[b][s].w};
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                        {
                            float lo, hi;
                            unpack16x2<F16>(w[c], lo, hi);
                            acc[s][c] = f2_add(acc[s][c], f2_pack(lo, hi));
                        }
                    }
                }
            }
        }
    }
    // every load of this CTA has been consumed: the selection kernel, if it
    // was launched as a programmatic dependent, may begin its launch
    pdl_release();

#pragma unroll
    for (int s = 0; s < NS; ++s) {
        if (own[s]) {
            float4 *o = reinterpret_cast<float4 *>(red + (size_t)(tid + kPoolThreads * s) * 8);
            float a[8];
#pragma unroll
            for (int c = 0; c < 4; ++c) f2_unpack(acc[s][c], a[2 * c], a[2 * c + 1]);
            o[0] = make_float4(a[0], a[1], a[2], a[3]);
            o[1] = make_float4(a[4], a[5], a[6], a[7]);
        }
    }
    __syncthreads();
    // output (block jx, channel d): the strip's token columns of that block in
    // ascending x
    const int nout = (jx1 - jx0) * D;
    for (int o = tid; o < nout; o += kPoolThreads) {
        const int jl = o / D, d = o - jl * D;
        const int xa = jl * g.bw, xb = min(xa + g.bw, x1 - x0);
        float sum = 0.f;
        for (int x = xa; x < xb; ++x) sum += red[x * D + d];
        const float mean = sum * (1.0f / (float)(tv * yv * (xb - xa)));
        const int j = (jt * nbh + jy) * nbw + jx0 + jl;
        if (g.tc_scores) {
            // for the tensor cores: [BH][2][rows, D] (rows = nb for Q, nbp for
            // K), per head the TF32 head of the mean and then the TF32 head of
            // its rest, so that any run of heads is one contiguous slice
            const float hi = tf32_round(mean), lo = tf32_round(mean - hi);
            const size_t rows = which ? (size_t)g.nbp : (size_t)g.nb;
            float *m = which ? kbarT : qbar;
            m[((size_t)bh * 2 * rows + j) * D + d] = hi;
            m[((size_t)bh * 2 * rows + rows + j) * D + d] = lo;
        } else if (!which) {
            qbar[((size_t)bh * g.nb + j) * D + d] = mean;
        } else {
            kbarT[((size_t)bh * D + d) * g.nbp + j] = mean;
        }
    }
}

// ---------------------------------------------------------------------------
// K2
// Query blocks per CTA (rows of the score tile). A CTA that computes its
// scores (TC false) reads its head's whole pooled-key matrix once, so rows
// longer than 1024 blocks take 16 rows per CTA (two per warp) to halve that
// traffic; otherwise 8 (one per warp) keep more CTAs in flight.
template <int EPL, bool TC>
constexpr int kSelRowsFor = (!TC && EPL >= 32) ? 16 : 8;
// CTAs per SM the register budget is sized for: the row's keys live in
// registers, and so does the score tile when the CTA computes it. With scores
// from the tensor-core kernel (TC) the tile is only copied, which leaves room
// for 5 CTAs per SM on rows of up to 512 blocks (48 registers), 4 up to 1024
// and 3 up to 1536, all without spills.
template <int EPL, bool TC>
constexpr int kSelMinBlocksFor =
    TC ? (EPL >= 64 ? 2 : EPL >= 48 ? 3 : EPL >= 24 ? 4 : 5) : (EPL >= 32 ? 2 : 3);
// Rows of up to 256 blocks select by a warp sort of their keys; longer rows by
// a binary search over the key space (fewer passes over the row's elements).
template <int EPL>
constexpr bool kSortedSelect = EPL == 1 || EPL == 2 || EPL == 4 || EPL == 8;

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ uint32_t warp_min_u(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}
__device__ __forceinline__ uint32_t warp_max_u(uint32_t v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 is
// folded into +0 by the caller.
__device__ __forceinline__ uint32_t order_key(float s)
{
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Inverse of order_key on the keys of finite floats.
__device__ __forceinline__ float key_float(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Unnormalised softmax weight exp(s - mx) of a score, as 2^((s - mx) log2 e)
// on the hardware exp2 (relative error ~1e-6 here, far inside the 1e-5 Top-p
// window). Every mass of a row is computed by this one expression, so a
// block's weight is bit-identical wherever it is recomputed from its key.
__device__ __forceinline__ float row_weight(float s, float mx)
{
    return ex2_approx((s - mx) * 1.4426950408889634f);
}

// Bitonic sort, descending, of the 32*EPL keys a warp holds: lane l holds
// positions l*EPL .. l*EPL+EPL-1. Exchanges between positions closer than
// EPL stay in a lane's registers; the others go through shuffles.
template <int EPL>
__device__ __forceinline__ void warp_sort_desc(uint32_t (&key)[EPL], int lane)
{
    constexpr int N = 32 * EPL;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < EPL) {
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    if (e & j) continue;
                    const int f = e | j;
                    // the pair (e, f) is kept descending where bit k of the position is 0
                    const bool desc = k < EPL ? ((e & k) == 0) : ((lane & (k / EPL)) == 0);
                    const uint32_t a = key[e], b = key[f];
                    const uint32_t hi = max(a, b), lo = min(a, b);
                    key[e] = desc ? hi : lo;
                    key[f] = desc ? lo : hi;
                }
            } else {
                const int lm = j / EPL;  // partner lane = lane ^ lm
                const bool lower = (lane & lm) == 0;
                const bool desc = (lane & (k / EPL)) == 0;
                const bool keep_max = lower == desc;
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, key[e], lm);
                    key[e] = keep_max ? max(key[e], o) : min(key[e], o);
                }
            }
        }
    }
}

// Key at sorted position r (warp-uniform) of keys sorted by warp_sort_desc.
template <int EPL>
__device__ __forceinline__ uint32_t key_at(const uint32_t (&key)[EPL], int r)
{
    const int e = r % EPL;
    uint32_t mine = key[0];
#pragma unroll
    for (int x = 1; x < EPL; ++x)
        if (e == x) mine = key[x];
    return __shfl_sync(0xFFFFFFFFu, mine, r / EPL);
}

// Boundary of the kept set of one row, found over the key space. Block j =
// lane + 32e of the row has key[e] (0 past the row) and mass pv(e).
//   MASS:  f(t) = mass(key >= t), goal p*z: the Top-p set;
//   COUNT: f(t) = count(key >= t), goal m: the m largest keys.
// On entry f(lo) >= goal > f(hi). Bisection narrows [lo, hi) until it holds
// at most 32 keys (checked every other step from step kPruneAfter on); those
// are compacted to one per lane and sorted, and the boundary is read off
// a prefix scan of their masses (MASS) or their ranks (COUNT). Every key at or
// above hi is kept. Out: kap, the smallest kept key; ntie, the number of
// kept blocks whose key equals kap; m_out, the number of kept blocks.
constexpr int kPruneAfter = 8;

// mass(key >= t) of one row: four interleaved partial sums per lane (short
// dependency chains), combined in a fixed order, then across the warp.
template <int EPL, class PV>
__device__ __forceinline__ float mass_at_least(const uint32_t (&key)[EPL], const PV &pv, uint32_t t)
{
    float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int e = 0; e < EPL; ++e)
        if (key[e] >= t) m[e & 3] += pv(e);
    return warp_sum((m[0] + m[1]) + (m[2] + m[3]));
}

template <int EPL, bool MASS, class PV>
__device__ __forceinline__ void window_boundary(const uint32_t (&key)[EPL], const PV &pv, float mx, float target,
                                                int m_goal, uint32_t lo, uint32_t hi, uint32_t *wscr, int lane,
                                                uint32_t &kap, int &ntie, int &m_out)
{
    auto reaches = [&](uint32_t t) {
        if constexpr (MASS) {
            return mass_at_least<EPL>(key, pv, t) >= target;
        } else {
            uint32_t c = 0;
#pragma unroll
            for (int e = 0; e < EPL; ++e) c += (key[e] >= t) ? 1u : 0u;
            return __reduce_add_sync(0xFFFFFFFFu, c) >= (uint32_t)m_goal;
        }
    };
    int steps = 0;
    while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (reaches(mid)) lo = mid;
        else hi = mid;
        if (++steps >= kPruneAfter && !(steps & 1)) {
            uint32_t c = 0;
#pragma unroll
            for (int e = 0; e < EPL; ++e) c += (key[e] >= lo && key[e] < hi) ? 1u : 0u;
            if (__reduce_add_sync(0xFFFFFFFFu, c) <= 32u) break;
        }
    }
    // blocks with key >= hi are all kept: f(hi) < goal (mass_hi is the value
    // the search compared when it set hi, bit for bit)
    float mass_hi = 0.f;
    uint32_t cnt_hi = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) cnt_hi += (key[e] >= hi) ? 1u : 0u;
    cnt_hi = __reduce_add_sync(0xFFFFFFFFu, cnt_hi);
    if constexpr (MASS) mass_hi = mass_at_least<EPL>(key, pv, hi);
    if (hi - lo == 1u) {
        // one key value left: tied blocks enter one at a time
        kap = lo;
        if constexpr (MASS) {
            float p_eq = 0.f;
            uint32_t n_eq = 0;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                if (key[e] == lo) {
                    ++n_eq;
                    p_eq = pv(e);
                }
            }
            n_eq = __reduce_add_sync(0xFFFFFFFFu, n_eq);
            p_eq = warp_max(p_eq);
            float accm = mass_hi;
            int n = 0;
            while (n < (int)n_eq && accm < target) {
                accm += p_eq;
                ++n;
            }
            ntie = n;
            m_out = (int)cnt_hi + n;
        } else {
            ntie = m_goal - (int)cnt_hi;
            m_out = m_goal;
        }
        return;
    }
    // at most 32 keys in [lo, hi): one per lane, sorted descending
    const uint32_t lt_mask = (1u << lane) - 1u;
    int nc = 0;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        const bool in = key[e] >= lo && key[e] < hi;
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, in);
        if (in) wscr[nc + __popc(bal & lt_mask)] = key[e];
        nc += __popc(bal);
    }
    __syncwarp();
    uint32_t ck[1] = {lane < nc ? wscr[lane] : 0u};
    __syncwarp();
    warp_sort_desc<1>(ck, lane);
    int nk;  // kept candidates: a prefix of the sorted ones
    if constexpr (MASS) {
        const float cp = ck[0] ? row_weight(key_float(ck[0]), mx) : 0.f;  // the same value as pv of that block
        float incl = cp;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += t;
        }
        float excl = __shfl_up_sync(0xFFFFFFFFu, incl, 1);
        if (lane == 0) excl = 0.f;
        nk = __popc(__ballot_sync(0xFFFFFFFFu, ck[0] != 0u && mass_hi + excl < target));
    } else {
        nk = m_goal - (int)cnt_hi;
    }
    kap = __shfl_sync(0xFFFFFFFFu, ck[0], nk - 1);
    ntie = nk - __popc(__ballot_sync(0xFFFFFFFFu, ck[0] > kap));
    m_out = (int)cnt_hi + nk;
}

// The d range of the score dot products is cut into S slices so that all
// 256 threads work on small tiles: thread w owns 4 consecutive key blocks x
// ROWS rows over one slice (the slice's loads are all in flight at once when
// it is short), accumulated as row pairs with packed fp32x2 fmas. Per element
// the slice sums are fp32 fmas in ascending d, and the slices are then added
// in ascending order.
__host__ __device__ constexpr int sel_slices(int nbp)
{
    return (nbp >> 2) >= 256 ? 1 : (nbp >> 2) >= 128 ? 2 : (nbp >> 2) >= 64 ? 4 : 8;
}

template <int D, int S, int ROWS>
__device__ __forceinline__ void score_tile(const float *kb, const float *qsT, float *sc, int nbp, float scale)
{
    constexpr int DS = D / S;
    constexpr int kUnroll = DS <= 16 ? DS : 8;
    constexpr int RP = ROWS / 2;  // row pairs: one packed fp32x2 accumulator per pair and column
    const int NQ = nbp >> 2;
    for (int w = threadIdx.x; w < NQ * S; w += blockDim.x) {
        const int sl = S == 1 ? 0 : w / NQ;
        const int c0 = (w - sl * NQ) * 4;
        uint64_t acc[RP][4];
#pragma unroll
        for (int r = 0; r < RP; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = 0ull;
        const float *kp = kb + (size_t)(sl * DS) * nbp + c0;
        const float *qp = qsT + sl * DS * ROWS;
#pragma unroll kUnroll
        for (int d = 0; d < DS; ++d) {
            const float4 kv = __ldg(reinterpret_cast<const float4 *>(kp + (size_t)d * nbp));
            const uint64_t k2[4] = {f2_pack(kv.x, kv.x), f2_pack(kv.y, kv.y), f2_pack(kv.z, kv.z),
                                    f2_pack(kv.w, kv.w)};
            const float4 *qv = reinterpret_cast<const float4 *>(qp + d * ROWS);
#pragma unroll
            for (int r4 = 0; r4 < ROWS / 4; ++r4) {
                const float4 qq = qv[r4];
                const uint64_t q01 = f2_pack(qq.x, qq.y), q23 = f2_pack(qq.z, qq.w);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * r4][c] = f2_fma(q01, k2[c], acc[2 * r4][c]);
                    acc[2 * r4 + 1][c] = f2_fma(q23, k2[c], acc[2 * r4 + 1][c]);
                }
            }
        }
        float *dst = sc + (size_t)sl * ROWS * nbp;
        const float f = S == 1 ? scale : 1.0f;
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            float lo[4], hi[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) f2_unpack(acc[r][c], lo[c], hi[c]);
            *reinterpret_cast<float4 *>(dst + (2 * r) * nbp + c0) = make_float4(f * lo[0], f * lo[1], f * lo[2], f * lo[3]);
            *reinterpret_cast<float4 *>(dst + (2 * r + 1) * nbp + c0) =
                make_float4(f * hi[0], f * hi[1], f * hi[2], f * hi[3]);
        }
    }
    if (S > 1) {
        __syncthreads();
        const int n4 = ROWS * nbp / 4;
        for (int x = threadIdx.x; x < n4; x += blockDim.x) {
            float4 t = reinterpret_cast<const float4 *>(sc)[x];
#pragma unroll
            for (int sl = 1; sl < S; ++sl) {
                const float4 u = reinterpret_cast<const float4 *>(sc + (size_t)sl * ROWS * nbp)[x];
                t.x += u.x;
                t.y += u.y;
                t.z += u.z;
                t.w += u.w;
            }
            reinterpret_cast<float4 *>(sc)[x] = make_float4(scale * t.x, scale * t.y, scale * t.z, scale * t.w);
        }
    }
}

// The CTA (8 warps) routes query blocks i0 .. i0+ROWS-1 of head bh: scores
// into shared memory (computed here, or with TC copied from the tensor-core
// kernel's output), then each warp selects and compacts whole rows. Shared
// memory: (D + S * nbp) * ROWS floats, S = sel_slices(nbp), or 1 with TC.
template <int D, int EPL, bool TC>
__device__ __forceinline__ void select_rows(const Geo &g, int bh, int i0, float *sel_smem,
                                            const float *qbar, const float *kbarT, const float *scores, float p,
                                            int k_min, int32_t *__restrict__ kv_cnt, int32_t *__restrict__ kv_idx,
                                            float *__restrict__ probs, uint32_t *__restrict__ status)
{
    constexpr int ROWS = kSelRowsFor<EPL, TC>;
    float *qsT = sel_smem;             // [D][ROWS]
    float *sc = sel_smem + D * ROWS;   // [S][ROWS][nbp]; slice 0 ends up holding the scores
    const int nrow = min(ROWS, g.nb - i0);
    const int nbp = g.nbp;

    // launched as a programmatic dependent of the pooling kernel: let the
    // scheduler launch behind this grid, then wait for the pooled means
    pdl_release();
    pdl_wait();
    if constexpr (TC) {
        // ---- block scores computed on the tensor cores: copy the rows
        const float4 *src = reinterpret_cast<const float4 *>(scores + ((size_t)bh * g.nb + i0) * nbp);
        float4 *dst = reinterpret_cast<float4 *>(sc);
        const int n4 = nrow * nbp / 4;
        for (int x = threadIdx.x; x < n4; x += blockDim.x) dst[x] = __ldcg(src + x);
    } else {
        for (int idx = threadIdx.x; idx < ROWS * D; idx += blockDim.x) {
            const int r = idx / D, d = idx - r * D;
            qsT[d * ROWS + r] = (r < nrow) ? qbar[((size_t)bh * g.nb + i0 + r) * D + d] : 0.f;
        }
        __syncthreads();

        // ---- block scores
        const float *kb = kbarT + (size_t)bh * D * nbp;
        const int S = sel_slices(nbp);
        if (S == 8) score_tile<D, 8, ROWS>(kb, qsT, sc, nbp, g.scale);
        else if (S == 4) score_tile<D, 4, ROWS>(kb, qsT, sc, nbp, g.scale);
        else if (S == 2) score_tile<D, 2, ROWS>(kb, qsT, sc, nbp, g.scale);
        else score_tile<D, 1, ROWS>(kb, qsT, sc, nbp, g.scale);
    }
    __syncthreads();

    // ---- selection: one warp per row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int nb = g.nb;
    uint32_t *wscr = reinterpret_cast<uint32_t *>(qsT) + warp * 32;  // per-warp scratch; qsT is dead now
    for (int r = warp; r < nrow; r += blockDim.x >> 5) {
        const int i = i0 + r;
        const size_t row = (size_t)bh * nb + i;
        float *srow = sc + r * nbp;
        int32_t *out = kv_idx + row * (size_t)nb;
        uint32_t key[EPL];  // order_key of the scores; 0 (below every real key) past nb
        bool bad = false;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int j = lane + 32 * e;
            key[e] = 0u;
            if (j < nb) {
                const float s = srow[j] + 0.0f;  // folds -0 into +0
                if (!isfinite(s)) bad = true;
                else mx = fmaxf(mx, s);
                key[e] = order_key(s);
            }
        }
        if (__any_sync(0xFFFFFFFFu, bad)) {
            // repair: a row with an unusable score keeps every block
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const int j = lane + 32 * e;
                if (j < nb) {
                    out[j] = j;
                    if (probs) probs[row * nb + j] = __int_as_float(0x7FC00000);
                }
            }
            if (lane == 0) {
                kv_cnt[row] = nb;
                atomicOr(status, kFlagNonfinite);
            }
            continue;
        }
        mx = warp_max(mx);

        bool all_sel = p >= 1.0f;
        uint32_t kap = 0;   // boundary key of the kept set
        int ntie = 0;       // how many blocks with key == kap are kept (lowest indices)
        float z;            // softmax denominator
        if constexpr (kSortedSelect<EPL>) {
            // Sort the keys, then C_before(r) = mass of sorted positions < r
            // by a prefix scan in rank order; position r is kept by Top-p
            // while C_before(r) < p * z.
            uint32_t sk[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e) sk[e] = key[e];
            warp_sort_desc<EPL>(sk, lane);
            float c[EPL];
            float run = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                c[e] = run;  // mass before this position, within the lane
                run += sk[e] ? row_weight(key_float(sk[e]), mx) : 0.f;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += t;
            }
            z = __shfl_sync(0xFFFFFFFFu, incl, 31);
            float excl = __shfl_up_sync(0xFFFFFFFFu, incl, 1);
            if (lane == 0) excl = 0.f;
            if (!all_sel) {
                const float target = p * z;
                int m_p = 0;
#pragma unroll
                for (int e = 0; e < EPL; ++e) m_p += __popc(__ballot_sync(0xFFFFFFFFu, excl + c[e] < target));
                const int m = max(m_p, k_min);
                if (m >= nb) {
                    all_sel = true;
                } else {
                    kap = key_at<EPL>(sk, m - 1);
                    int c_gt = 0;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) c_gt += (key[e] > kap) ? 1 : 0;
                    ntie = m - (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)c_gt);
                }
            }
        } else {
            // Search over the key space: the largest key t whose mass
            // mass(key >= t) reaches p * z is the Top-p boundary. The masses
            // replace the scores in the row's shared memory.
            uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
            float zl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const int j = lane + 32 * e;
                if (j < nb) {
                    const float pj = row_weight(key_float(key[e]), mx);
                    srow[j] = pj;
                    kmin = min(kmin, key[e]);
                    kmax = max(kmax, key[e]);
                    zl[e & 3] += pj;
                }
            }
            const float *pvr = srow;  // pv of block j at pvr[j]; read only where key[e] != 0
            // read only under a key test that fails for the padding keys (0); the
            // shared memory is padded so those reads stay inside it
            auto pv = [&](int e) { return pvr[lane + 32 * e]; };
            z = warp_sum((zl[0] + zl[1]) + (zl[2] + zl[3]));
            kmin = warp_min_u(kmin);
            kmax = warp_max_u(kmax);
            if (!all_sel) {
                const float target = p * z;
                uint32_t kap_p;
                int ntie_p, m_p;
                window_boundary<EPL, true>(key, pv, mx, target, 0, kmin, kmax + 1u, wscr, lane, kap_p, ntie_p, m_p);
                const int m = max(m_p, k_min);
                if (m >= nb) {
                    all_sel = true;
                } else if (m == m_p) {
                    kap = kap_p;
                    ntie = ntie_p;
                } else {
                    // Top-k floor binds: the key of rank m; count(>= kap_p + 1) = m_p - ntie_p < m
                    int m_c;
                    window_boundary<EPL, false>(key, pv, mx, 0.f, m, kmin, kap_p + 1u, wscr, lane, kap, ntie, m_c);
                }
            }
        }
        // ---- compaction in ascending block order (+ diagonal repair)
        int base = 0, tie_seen = 0;
        const float invz = 1.0f / z;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int j = lane + 32 * e;
            const bool valid = j < nb;
            const bool eq = valid && !all_sel && key[e] == kap;
            const uint32_t eqm = __ballot_sync(0xFFFFFFFFu, eq);
            const int tie_rank = tie_seen + __popc(eqm & lt_mask);
            tie_seen += __popc(eqm);
            const bool sel = valid && (all_sel || key[e] > kap || (eq && tie_rank < ntie) || j == i);
            const uint32_t sm = __ballot_sync(0xFFFFFFFFu, sel);
            if (sel) out[base + __popc(sm & lt_mask)] = j;
            base += __popc(sm);
            if (probs && valid) {
                float pj;
                if constexpr (kSortedSelect<EPL>) pj = row_weight(key_float(key[e]), mx);
                else pj = srow[j];
                probs[row * nb + j] = pj * invz;
            }
        }
        if (lane == 0) kv_cnt[row] = base;
    }
}

template <int D, int EPL, bool TC>
__global__ void __launch_bounds__(256, kSelMinBlocksFor<EPL, TC>) score_select_kernel(Geo g, const float *__restrict__ qbar,
                                                           const float *__restrict__ kbarT, float p, int k_min,
                                                           const float *__restrict__ scores,
                                                           int32_t *__restrict__ kv_cnt, int32_t *__restrict__ kv_idx,
                                                           float *__restrict__ probs, uint32_t *__restrict__ status)
{
    extern __shared__ __align__(16) float sel_smem[];
    select_rows<D, EPL, TC>(g, blockIdx.y, blockIdx.x * kSelRowsFor<EPL, TC>, sel_smem, qbar, kbarT, scores, p, k_min,
                            kv_cnt, kv_idx, probs, status);
}

// ---------------------------------------------------------------------------
template <int D, int NS, bool F16>
static cudaError_t launch_pool_f(const Geo &g, int nxs, const void *q, const void *k, float *qbar, float *kbarT,
                                 cudaStream_t stream)
{
    const size_t smem = (size_t)kPoolThreads * NS * 8 * sizeof(float);
    auto kern = pool_kernel<D, NS, F16>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const long long blocks = 2ll * g.BH * g.nbt * g.nbh * nxs;
    kern<<<(unsigned)blocks, kPoolThreads, smem, stream>>>(g, nxs, (const uint16_t *)q, (const uint16_t *)k, qbar,
                                                          kbarT);
    return cudaGetLastError();
}

template <int D, int NS>
static cudaError_t launch_pool_t(const Geo &g, int nxs, const void *q, const void *k, float *qbar, float *kbarT,
                                 cudaStream_t stream)
{
    if (g.f16) return launch_pool_f<D, NS, true>(g, nxs, q, k, qbar, kbarT, stream);
    return launch_pool_f<D, NS, false>(g, nxs, q, k, qbar, kbarT, stream);
}

template <int D>
static cudaError_t launch_pool_d(const Geo &g, const void *q, const void *k, float *qbar, float *kbarT,
                                 cudaStream_t stream)
{
    const PoolPlan pl = pool_plan(g.nbw, g.bw, D);
    switch (pl.ns) {
    case 1: return launch_pool_t<D, 1>(g, pl.nxs, q, k, qbar, kbarT, stream);
    case 2: return launch_pool_t<D, 2>(g, pl.nxs, q, k, qbar, kbarT, stream);
    case 3: return launch_pool_t<D, 3>(g, pl.nxs, q, k, qbar, kbarT, stream);
    case 4: return launch_pool_t<D, 4>(g, pl.nxs, q, k, qbar, kbarT, stream);
    default: return launch_pool_t<D, 8>(g, pl.nxs, q, k, qbar, kbarT, stream);
    }
}

cudaError_t launch_pool(const Geo &g, const void *q, const void *k, float *qbar, float *kbarT,
                        cudaStream_t stream)
{
    if (g.D == 128) return launch_pool_d<128>(g, q, k, qbar, kbarT, stream);
    return launch_pool_d<64>(g, q, k, qbar, kbarT, stream);
}

template <int D, int EPL, bool TC>
static cudaError_t launch_sel_tc(const Geo &g, const float *qbar, const float *kbarT, const float *scores, float p,
                                 int k_min, int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                 cudaStream_t stream, bool programmatic)
{
    constexpr int ROWS = kSelRowsFor<EPL, TC>;
    // + 32*EPL floats: a row's lanes read positions up to 32*EPL - 1
    const int S = TC ? 1 : sel_slices(g.nbp);
    const size_t smem = ((size_t)(D + S * g.nbp) * ROWS + 32 * EPL) * sizeof(float);
    auto kern = score_select_kernel<D, EPL, TC>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    // programmatic dependent launch: the CTAs may be scheduled while the
    // pooling kernel drains and wait in-kernel for its results
    const dim3 grid((unsigned)ceil_div(g.nb, ROWS), (unsigned)g.BH);
    if (programmatic)
        return launch_dependent(kern, grid, dim3(256), smem, stream, g, qbar, kbarT, p, k_min, scores, kv_cnt, kv_idx,
                                probs, status);
    kern<<<grid, 256, smem, stream>>>(g, qbar, kbarT, p, k_min, scores, kv_cnt, kv_idx, probs, status);
    return cudaGetLastError();
}

template <int D, int EPL>
static cudaError_t launch_sel_t(const Geo &g, const float *qbar, const float *kbarT, const float *scores, float p,
                                int k_min, int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream, bool programmatic)
{
    if (scores)
        return launch_sel_tc<D, EPL, true>(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, probs, status, stream,
                                           programmatic);
    return launch_sel_tc<D, EPL, false>(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, probs, status, stream,
                                        programmatic);
}

template <int D>
static cudaError_t launch_sel_d(const Geo &g, const float *qbar, const float *kbarT, const float *scores, float p,
                                int k_min, int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream, bool programmatic)
{
    const int epl = ceil_div(g.nb, 32);
#define FV_SEL(E)                                                                                                 \
    if (epl <= E)                                                                                                 \
    return launch_sel_t<D, E>(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, probs, status, stream, programmatic)
    FV_SEL(1);
    FV_SEL(2);
    FV_SEL(4);
    FV_SEL(8);
    FV_SEL(12);
    FV_SEL(16);
    FV_SEL(24);
    FV_SEL(32);
    FV_SEL(48);
    FV_SEL(64);
#undef FV_SEL
    return cudaErrorInvalidValue;
}

cudaError_t launch_score_select(const Geo &g, const float *qbar, const float *kbarT, const float *scores, float p,
                                int k_min, int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream, bool programmatic)
{
    if (g.D == 128)
        return launch_sel_d<128>(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, probs, status, stream, programmatic);
    return launch_sel_d<64>(g, qbar, kbarT, scores, p, k_min, kv_cnt, kv_idx, probs, status, stream, programmatic);
}

}  // namespace fvattn
