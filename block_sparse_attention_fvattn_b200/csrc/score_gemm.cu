// score_gemm.cu -- block scores on the tensor cores for long rows (K2a).
//
// The routing scores s[i][j] = scale * Qbar_i . Kbar_j of one head form an
// nb x nb matrix product with a D-long inner dimension (zskr.cn FastVideo VSA
// guide, section 1: block-level scores per query block; ai-feeds.com FVAttn
// summary, "Key modules" 1). From a few hundred blocks on, computing it with
// fp32 FMAs costs more than reading Q and K; here it runs on the tensor cores
// (tcgen05.mma kind::tf32) in three TF32 products per fp32 operand pair:
// x = hi + lo with hi = tf32(x) and lo = tf32(x - hi), and
// s ~= hi_q.hi_k + hi_q.lo_k + lo_q.hi_k, which keeps about 2^-20 of relative
// accuracy per product, far inside the rank-tie window of the Top-p selection.
// The scores go to a buffer in the workspace (it stays mostly in L2); the
// selection kernel reads its rows from there.
//
// The pooling kernel stores the means already split (hi and lo of Qbar and
// Kbar, each exactly representable in TF32). One CTA computes a 128 x 256 tile
// of one head's score matrix (two CTAs share an SM):
//   warp 0      TMA producer: 32-wide K chunks of the four operands
//   warp 1      TMEM owner and MMA issuer
//   warps 2-5   read the accumulator from TMEM and store the scaled tile
#include "common.cuh"
#include "internal.h"

namespace fvattn {

namespace {

constexpr int kGemmThreads = 192;
constexpr int kTileM = 128, kTileN = 256, kChunk = 32;  // K chunk: 32 fp32 = one 128-byte swizzle row
constexpr int kStages = 1;
constexpr uint32_t kABytes = kTileM * kChunk * 4;  // 16 KB
constexpr uint32_t kBBytes = kTileN * kChunk * 4;  // 32 KB
// per stage: A hi, A lo, B hi, B lo
constexpr uint32_t kStageBytes = 2 * kABytes + 2 * kBBytes;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + 1024 /* barriers, flags */ + 1024 /* alignment */;
static_assert(2 * kSmemBytes <= 227 * 1024, "two CTAs per SM");

// Instruction descriptor of tcgen05.mma kind::tf32: fp32 accumulator (bit 4),
// A and B TF32 (format 2 in bits 7-9 and 10-12), both K-major, N>>3, M>>4.
constexpr uint32_t kIdescTf32 = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kTileN >> 3) << 17) |
                                ((uint32_t)(kTileM >> 4) << 24);

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdescTf32), "r"(accumulate)
        : "memory");
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 2)
    score_gemm_kernel(const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                      const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo, Geo g,
                      float *__restrict__ scores, uint32_t *__restrict__ status)
{
    extern __shared__ uint8_t gemm_smem_raw[];
    const uint32_t raw = smem_u32(gemm_smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t *gbase = gemm_smem_raw + (sbase - raw);
    const uint32_t bars = sbase + kStages * kStageBytes;
    // barriers: full[s] (TMA), empty[s] (MMA done), acc (all MMAs done)
    auto full = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto empty = [&](int s) { return bars + 8u * (uint32_t)(kStages + s); };
    const uint32_t acc_bar = bars + 8u * (uint32_t)(2 * kStages);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + kStages * kStageBytes + 256);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + kStages * kStageBytes + 272);
    auto stage_a = [&](int s) { return sbase + (uint32_t)s * kStageBytes; };
    auto stage_alo = [&](int s) { return stage_a(s) + kABytes; };
    auto stage_b = [&](int s) { return stage_a(s) + 2 * kABytes; };
    auto stage_blo = [&](int s) { return stage_a(s) + 2 * kABytes + kBBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * kTileN, m0 = blockIdx.y * kTileM, bh = blockIdx.z;
    const int nchunks = g.D / kChunk;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(acc_bar, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTileN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_release();
    pdl_wait();  // the pooled means come from the pooling kernel
    if (threadIdx.x == 0) wait_limit_setup(abort_flag, status);
    __syncthreads();

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_qhi);
            tma_prefetch_desc(&tm_qlo);
            tma_prefetch_desc(&tm_khi);
            tma_prefetch_desc(&tm_klo);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                if (c >= kStages && !mbar_wait(empty(s), ((c / kStages) - 1) & 1, abort_flag)) break;
                mbar_arrive_expect_tx(full(s), kStageBytes);
                tma_load_3d(stage_a(s), &tm_qhi, full(s), c * kChunk, m0, bh);
                tma_load_3d(stage_alo(s), &tm_qlo, full(s), c * kChunk, m0, bh);
                tma_load_3d(stage_b(s), &tm_khi, full(s), c * kChunk, n0, bh);
                tma_load_3d(stage_blo(s), &tm_klo, full(s), c * kChunk, n0, bh);
                ++issued;
            }
            if (*abort_flag) {
                // wind down: every copy already issued lands before the CTA exits
                for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
                    mbar_wait_for(full(c % kStages), (c / kStages) & 1, 50000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            for (int c = 0; c < nchunks; ++c) {
                const int s = c % kStages;
                if (!mbar_wait(full(s), (c / kStages) & 1, abort_flag)) break;
                tc_fence_after();
                const uint64_t a_hi = sdesc_sw128(stage_a(s), 16, 1024), a_lo = sdesc_sw128(stage_alo(s), 16, 1024);
                const uint64_t b_hi = sdesc_sw128(stage_b(s), 16, 1024), b_lo = sdesc_sw128(stage_blo(s), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < kChunk / 8; ++kk) {
                    const uint64_t off = (uint64_t)((kk * 32) >> 4);  // 8 tf32 = 32 bytes along the swizzled row
                    umma_tf32(tmem, a_hi + off, b_hi + off, (c > 0 || kk > 0) ? 1u : 0u);
                    umma_tf32(tmem, a_hi + off, b_lo + off, 1u);
                    umma_tf32(tmem, a_lo + off, b_hi + off, 1u);
                }
                umma_commit(empty(s));
            }
            umma_commit(acc_bar);
        }
    } else {
        // ---- epilogue: TMEM lane = tile row; this warp owns lanes 32*(warp%4)..
        // Each 32 x 32 chunk goes through shared memory (the operand stages
        // are free once every MMA has completed): lane l writes its row, then
        // the warp stores the chunk row by row, each store one contiguous
        // 128-byte run of a score row.
        if (mbar_wait(acc_bar, 0, abort_flag)) {
            tc_fence_after();
            const int wq = warp & 3;
            float *tile = reinterpret_cast<float *>(gbase) + wq * (32 * 33);  // padded: row stride 33 floats
            const int row0 = m0 + wq * 32;
#pragma unroll 1
            for (int cb = 0; cb < kTileN / 32; ++cb) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)(cb * 32), r);
                tmem_wait_ld();
                reg_fence32(r);
#pragma unroll
                for (int c = 0; c < 32; ++c) tile[lane * 33 + c] = g.scale * __uint_as_float(r[c]);
                __syncwarp();
                const int col = n0 + cb * 32 + lane;
#pragma unroll 4
                for (int rr = 0; rr < 32; ++rr) {
                    const int row = row0 + rr;
                    if (row < g.nb && col < g.nbp) scores[((size_t)bh * g.nb + row) * g.nbp + col] = tile[rr * 33 + lane];
                }
                __syncwarp();
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        // no MMA may still write TMEM when it is released
        if (*abort_flag) mbar_wait_for(acc_bar, 0, 100000000ull);
        tmem_dealloc(tmem, kTileN);
    }
    if (threadIdx.x == 0 && *abort_flag) atomicOr(status, kFlagTimeout);
}

// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn gemm_encode_fn()
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

// One plane of [BH][2][rows, D] fp32 as a 3-D TMA tensor (head stride: both
// planes); box = 32 x box_rows x 1, 128-byte swizzle.
static bool make_means_map(CUtensorMap *map, const Geo &g, const float *ptr, int rows, int box_rows)
{
    EncodeTiledFn enc = gemm_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)rows, (cuuint64_t)g.BH};
    const cuuint64_t strides[2] = {(cuuint64_t)g.D * 4, (cuuint64_t)rows * g.D * 4 * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kChunk, (cuuint32_t)box_rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_score_gemm(const Geo &g, const float *qhi, const float *qlo, const float *khi, const float *klo,
                              float *scores, uint32_t *status, cudaStream_t stream, bool programmatic)
{
    CUtensorMap mqh, mql, mkh, mkl;
    if (!make_means_map(&mqh, g, qhi, g.nb, kTileM) || !make_means_map(&mql, g, qlo, g.nb, kTileM) ||
        !make_means_map(&mkh, g, khi, g.nbp, kTileN) || !make_means_map(&mkl, g, klo, g.nbp, kTileN))
        return cudaErrorInvalidValue;
    cudaError_t err =
        cudaFuncSetAttribute(score_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (err != cudaSuccess) return err;
    const dim3 grid((unsigned)ceil_div(g.nbp, kTileN), (unsigned)ceil_div(g.nb, kTileM), (unsigned)g.BH);
    if (programmatic)
        return launch_dependent(score_gemm_kernel, grid, dim3(kGemmThreads), kSmemBytes, stream, mqh, mql, mkh, mkl,
                                g, scores, status);
    score_gemm_kernel<<<grid, kGemmThreads, kSmemBytes, stream>>>(mqh, mql, mkh, mkl, g, scores, status);
    return cudaGetLastError();
}

}  // namespace fvattn
