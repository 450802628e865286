// route.cu -- the sparse-routing frontend of adaptive block-sparse attention.
//
// K1 pool_kernel: block means of Q and K over the valid tokens of every
//   video-aware (t,h,w) block (zskr.cn FastVideo VSA guide, section 1: the
//   post-patch latent grid is cut into spatio-temporal blocks; section 6:
//   variable-length edge blocks, padding never acts as a key). HBM-bound: one
//   pass over Q and K with 16-byte coalesced loads; a warp owns one block and
//   reads its (t, y) runs of contiguous tokens.
// K2 score_select_kernel: per (head, query block) row: block scores
//   s = scale * Qbar_i . Kbar_j, softmax, Top-p with a Top-k floor, diagonal
//   repair and ascending compaction (ai-feeds.com FVAttn summary, "Key
//   modules" 1; hotpaper.ai abstract). The nb x nb score matrix never leaves
//   shared memory. One warp owns one row. Selection is exact in fp32: an
//   order-preserving integer key of each score and a 4-ary search over the key
//   space find the score at the Top-p boundary (by probability mass) and, if
//   the floor binds, at rank m; ties at the boundary go to the lower block
//   index.
#include "common.cuh"
#include "internal.h"

namespace fvattn {

// ---------------------------------------------------------------------------
// K1
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(Geo g, const __nv_bfloat16 *__restrict__ q,
                                                   const __nv_bfloat16 *__restrict__ k, float *__restrict__ qbar,
                                                   float *__restrict__ kbarT)
{
    constexpr int LPT = D / 8;  // lanes per token (one 16-byte chunk each)
    constexpr int kBatch = 8;   // loads in flight per lane
    const int lane = threadIdx.x & 31;
    const long long warp = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const long long per = (long long)g.BH * g.nb;
    if (warp >= 2 * per) return;
    const int which = warp >= per ? 1 : 0;
    const long long rem = warp - which * per;
    const int bh = (int)(rem / g.nb), j = (int)(rem - (long long)bh * g.nb);
    const int jt = j / (g.nbh * g.nbw), jy = (j / g.nbw) % g.nbh, jx = j % g.nbw;
    const int t0 = jt * g.bt, y0 = jy * g.bh, x0 = jx * g.bw;
    const int tv = min(g.bt, g.T - t0), yv = min(g.bh, g.Hg - y0), xv = min(g.bw, g.W - x0);
    const __nv_bfloat16 *src = which ? k : q;
    const uint4 *base = reinterpret_cast<const uint4 *>(src + (size_t)bh * g.N * D);
    const int cpr = xv * LPT;  // 16-byte chunks in one (t, y) run of xv tokens

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;

    // cursor over (t, y, chunk) in the order t, y, chunk; each lane starts at
    // chunk `lane` and advances by 32 chunks. Its d-chunk (lane % LPT) is fixed.
    int t = t0, y = y0, e = lane;
    while (e >= cpr && t < t0 + tv) {
        e -= cpr;
        if (++y == y0 + yv) { y = y0; ++t; }
    }
    while (t < t0 + tv) {
        uint4 v[kBatch];
        bool ok[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            ok[b] = t < t0 + tv;
            if (ok[b]) {
                const size_t tok = ((size_t)t * g.Hg + y) * g.W + x0;
                v[b] = __ldg(base + tok * LPT + e);
                e += 32;
                while (e >= cpr && t < t0 + tv) {
                    e -= cpr;
                    if (++y == y0 + yv) { y = y0; ++t; }
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (ok[b]) {
                const uint32_t w[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] += __uint_as_float(w[c] << 16);
                    acc[2 * c + 1] += __uint_as_float(w[c] & 0xFFFF0000u);
                }
            }
        }
    }
    // lanes with the same d-chunk combine in a fixed order
#pragma unroll
    for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(0xFFFFFFFFu, acc[c], off);
    }
    if (lane < LPT) {
        const float inv = 1.0f / (float)(tv * yv * xv);
        const int d0 = lane * 8;
        if (!which) {
            float4 *o = reinterpret_cast<float4 *>(qbar + ((size_t)bh * g.nb + j) * D + d0);
            o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
            o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
        } else {
            float *o = kbarT + ((size_t)bh * D + d0) * g.nbp + j;
#pragma unroll
            for (int c = 0; c < 8; ++c) o[(size_t)c * g.nbp] = acc[c] * inv;
        }
    }
}

// ---------------------------------------------------------------------------
// K2
constexpr int kSelRows = 8;  // query blocks per CTA (rows of the score tile), one per warp

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

template <int D, int EPL>
__global__ void __launch_bounds__(256) score_select_kernel(Geo g, const float *__restrict__ qbar,
                                                           const float *__restrict__ kbarT, float p, int k_min,
                                                           int32_t *__restrict__ kv_cnt, int32_t *__restrict__ kv_idx,
                                                           float *__restrict__ probs, uint32_t *__restrict__ status)
{
    extern __shared__ __align__(16) float sel_smem[];
    float *qsT = sel_smem;                 // [D][kSelRows]
    float *sc = sel_smem + D * kSelRows;   // [kSelRows][nbp]
    const int bh = blockIdx.y;
    const int i0 = blockIdx.x * kSelRows;
    const int nrow = min(kSelRows, g.nb - i0);
    const int nbp = g.nbp;

    for (int idx = threadIdx.x; idx < kSelRows * D; idx += blockDim.x) {
        const int r = idx / D, d = idx - r * D;
        qsT[d * kSelRows + r] = (r < nrow) ? qbar[((size_t)bh * g.nb + i0 + r) * D + d] : 0.f;
    }
    __syncthreads();

    // ---- block scores: each thread owns 4 consecutive key blocks x kSelRows rows
    const float *kb = kbarT + (size_t)bh * D * nbp;
    for (int c0 = threadIdx.x * 4; c0 < nbp; c0 += blockDim.x * 4) {
        float acc[kSelRows][4];
#pragma unroll
        for (int r = 0; r < kSelRows; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
            const float4 kv = __ldg(reinterpret_cast<const float4 *>(kb + (size_t)d * nbp + c0));
            const float4 *qv = reinterpret_cast<const float4 *>(qsT + d * kSelRows);
#pragma unroll
            for (int r4 = 0; r4 < kSelRows / 4; ++r4) {
                const float4 qq = qv[r4];
                const float qr[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    acc[r4 * 4 + rr][0] = fmaf(qr[rr], kv.x, acc[r4 * 4 + rr][0]);
                    acc[r4 * 4 + rr][1] = fmaf(qr[rr], kv.y, acc[r4 * 4 + rr][1]);
                    acc[r4 * 4 + rr][2] = fmaf(qr[rr], kv.z, acc[r4 * 4 + rr][2]);
                    acc[r4 * 4 + rr][3] = fmaf(qr[rr], kv.w, acc[r4 * 4 + rr][3]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kSelRows; ++r) {
            float4 o = make_float4(g.scale * acc[r][0], g.scale * acc[r][1], g.scale * acc[r][2],
                                   g.scale * acc[r][3]);
            *reinterpret_cast<float4 *>(sc + r * nbp + c0) = o;
        }
    }
    __syncthreads();

    // ---- selection: one warp per row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int nb = g.nb;
    for (int r = warp; r < nrow; r += blockDim.x >> 5) {
        const int i = i0 + r;
        const size_t row = (size_t)bh * nb + i;
        const float *srow = sc + r * nbp;
        int32_t *out = kv_idx + row * (size_t)nb;
        float sv[EPL];
        bool bad = false;
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int j = lane + 32 * e;
            float s = -INFINITY;
            if (j < nb) {
                s = srow[j] + 0.0f;  // folds -0 into +0
                if (!isfinite(s)) bad = true;
                else mx = fmaxf(mx, s);
            }
            sv[e] = s;
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
        float pv[EPL];
        uint32_t key[EPL];
        float z = 0.f;
        uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            const int j = lane + 32 * e;
            if (j < nb) {
                pv[e] = expf(sv[e] - mx);
                key[e] = order_key(sv[e]);
                kmin = min(kmin, key[e]);
                kmax = max(kmax, key[e]);
            } else {
                pv[e] = 0.f;
                key[e] = 0u;  // below every real key; never selected
            }
            z += pv[e];
        }
        z = warp_sum(z);
        kmin = warp_min_u(kmin);
        kmax = warp_max_u(kmax);

        bool all_sel = false;
        uint32_t kap = 0;   // boundary key of the kept set
        int ntie = 0;       // how many blocks with key == kap are kept (lowest indices)
        int m = nb;
        if (p >= 1.0f) {
            all_sel = true;
        } else {
            const float target = p * z;
            // largest key t with mass(key >= t) >= target: 4-ary search, three
            // independent reductions per step
            uint32_t lo = kmin, hi = kmax + 1u;
            while (hi - lo > 1u) {
                const uint32_t q4 = (hi - lo) >> 2;
                const uint32_t t1 = lo + (q4 ? q4 : 1u), t2 = lo + (q4 ? 2u * q4 : 1u),
                               t3 = lo + (q4 ? 3u * q4 : 1u);
                float m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    m1 += (key[e] >= t1) ? pv[e] : 0.f;
                    m2 += (key[e] >= t2) ? pv[e] : 0.f;
                    m3 += (key[e] >= t3) ? pv[e] : 0.f;
                }
                m1 = warp_sum(m1);
                m2 = warp_sum(m2);
                m3 = warp_sum(m3);
                if (m3 >= target) {
                    lo = t3;
                } else if (m2 >= target) {
                    lo = t2;
                    hi = t3;
                } else if (m1 >= target) {
                    lo = t1;
                    hi = t2;
                } else {
                    hi = t1;
                }
            }
            const uint32_t kp = lo;
            float mass_gt = 0.f, p_eq = 0.f;
            int cnt_gt = 0, n_eq = 0;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                mass_gt += (key[e] >= kp + 1u) ? pv[e] : 0.f;
                cnt_gt += (key[e] > kp) ? 1 : 0;
                n_eq += (key[e] == kp) ? 1 : 0;
                if (key[e] == kp) p_eq = pv[e];
            }
            mass_gt = warp_sum(mass_gt);
            cnt_gt = (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)cnt_gt);
            n_eq = (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)n_eq);
            p_eq = warp_max(p_eq);
            // blocks tied at the boundary enter one at a time, lowest index first
            float accm = mass_gt;
            int n = 0;
            while (n < n_eq && accm < target) {
                accm += p_eq;
                ++n;
            }
            const int m_p = cnt_gt + n;
            m = max(m_p, k_min);
            if (m >= nb) {
                all_sel = true;
            } else if (m == m_p) {
                kap = kp;
                ntie = n;
            } else {
                // Top-k floor binds: boundary key of rank m (4-ary search on counts)
                uint32_t lo2 = kmin, hi2 = kp + 1u;
                while (hi2 - lo2 > 1u) {
                    const uint32_t q4 = (hi2 - lo2) >> 2;
                    const uint32_t t1 = lo2 + (q4 ? q4 : 1u), t2 = lo2 + (q4 ? 2u * q4 : 1u),
                                   t3 = lo2 + (q4 ? 3u * q4 : 1u);
                    uint32_t c1 = 0, c2 = 0, c3 = 0;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        c1 += (key[e] >= t1) ? 1u : 0u;
                        c2 += (key[e] >= t2) ? 1u : 0u;
                        c3 += (key[e] >= t3) ? 1u : 0u;
                    }
                    c1 = __reduce_add_sync(0xFFFFFFFFu, c1);
                    c2 = __reduce_add_sync(0xFFFFFFFFu, c2);
                    c3 = __reduce_add_sync(0xFFFFFFFFu, c3);
                    if (c3 >= (uint32_t)m) {
                        lo2 = t3;
                    } else if (c2 >= (uint32_t)m) {
                        lo2 = t2;
                        hi2 = t3;
                    } else if (c1 >= (uint32_t)m) {
                        lo2 = t1;
                        hi2 = t2;
                    } else {
                        hi2 = t1;
                    }
                }
                kap = lo2;
                int c_gt = 0;
#pragma unroll
                for (int e = 0; e < EPL; ++e) c_gt += (key[e] > kap) ? 1 : 0;
                c_gt = (int)__reduce_add_sync(0xFFFFFFFFu, (uint32_t)c_gt);
                ntie = m - c_gt;
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
            if (probs && valid) probs[row * nb + j] = pv[e] * invz;
        }
        if (lane == 0) kv_cnt[row] = base;
    }
}

// ---------------------------------------------------------------------------
cudaError_t launch_pool(const Geo &g, const void *q, const void *k, float *qbar, float *kbarT,
                        cudaStream_t stream)
{
    const long long warps = 2ll * g.BH * g.nb;
    const int threads = 256;
    const long long blocks = (warps * 32 + threads - 1) / threads;
    if (g.D == 128)
        pool_kernel<128><<<(unsigned)blocks, threads, 0, stream>>>(g, (const __nv_bfloat16 *)q,
                                                                   (const __nv_bfloat16 *)k, qbar, kbarT);
    else
        pool_kernel<64><<<(unsigned)blocks, threads, 0, stream>>>(g, (const __nv_bfloat16 *)q,
                                                                  (const __nv_bfloat16 *)k, qbar, kbarT);
    return cudaGetLastError();
}

template <int D, int EPL>
static cudaError_t launch_sel_t(const Geo &g, const float *qbar, const float *kbarT, float p, int k_min,
                                int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream)
{
    const size_t smem = (size_t)(D * kSelRows + kSelRows * g.nbp) * sizeof(float);
    auto kern = score_select_kernel<D, EPL>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)ceil_div(g.nb, kSelRows), (unsigned)g.BH);
    kern<<<grid, 256, smem, stream>>>(g, qbar, kbarT, p, k_min, kv_cnt, kv_idx, probs, status);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_sel_d(const Geo &g, const float *qbar, const float *kbarT, float p, int k_min,
                                int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream)
{
    const int epl = ceil_div(g.nb, 32);
#define FV_SEL(E) \
    if (epl <= E) return launch_sel_t<D, E>(g, qbar, kbarT, p, k_min, kv_cnt, kv_idx, probs, status, stream)
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

cudaError_t launch_score_select(const Geo &g, const float *qbar, const float *kbarT, float p, int k_min,
                                int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream)
{
    if (g.D == 128) return launch_sel_d<128>(g, qbar, kbarT, p, k_min, kv_cnt, kv_idx, probs, status, stream);
    return launch_sel_d<64>(g, qbar, kbarT, p, k_min, kv_cnt, kv_idx, probs, status, stream);
}

}  // namespace fvattn
