// internal.h -- launchers shared between the C-ABI shim and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"

namespace fvattn {

// Workspace carve-up (byte offsets from the workspace base; 256-byte aligned).
struct WsLayout {
    size_t qbar;         // fp32 [BH, nb, D]   pooled query means ([BH][2][nb, D] TF32 head, rest if tc_scores)
    size_t kbarT;        // fp32 [BH, D, nbp]  pooled key means, transposed ([BH][2][nbp, D] if tc_scores)
    size_t scores;       // fp32 [BH, nb, nbp] block scores (tc_scores only)
    size_t unit_cost;    // int32 [BH*(nb+npair)] scheduler: cost per unit id (paired split units after the others)
    size_t head_sorted;  // int32 [BH*(nb+2)]  scheduler: unit ids of each head by cost
    size_t head_len;     // int32 [BH]         scheduler: units of each head
    size_t head_cost;    // int64 [BH]         scheduler: total cost per head
    size_t pair_cnt;     // int32 [BH*npair]   paired mode: union size of each pair of query blocks
    size_t pair_list;    // int32 [BH*npair*nb] paired mode: the union, ascending, with membership flags
    size_t aug_state;    // augmentation: radix-select state (histogram, boundary key, budget left)
    size_t aug_row_tie;  // int64 [BH*nb]      augmentation: boundary-key cost before each row
    size_t total;
};
WsLayout ws_layout(const Geo &g);

// Largest nb the select kernel keeps in registers.
constexpr int kMaxBlocks = 2048;
// Largest persistent-CTA count.
constexpr int kMaxCtas = 4096;

cudaError_t launch_pool(const Geo &g, const void *q, const void *k, float *qbar, float *kbarT,
                        cudaStream_t stream);
// scores != nullptr: the block scores were computed by launch_score_gemm.
// programmatic: launched as a programmatic dependent of the kernel before it
// on the stream (that kernel must be the one producing its inputs).
cudaError_t launch_score_select(const Geo &g, const float *qbar, const float *kbarT, const float *scores, float p,
                                int k_min, int32_t *kv_cnt, int32_t *kv_idx, float *probs, uint32_t *status,
                                cudaStream_t stream, bool programmatic = true);
// Scores from means split as x = hi + lo (hi, lo exact in TF32), stored
// [BH][2][nb, D] for Q and [BH][2][nbp, D] for K (hi plane, then lo plane, per
// head): qhi/khi point at the first hi plane, qlo/klo at the first lo plane.
cudaError_t launch_score_gemm(const Geo &g, const float *qhi, const float *qlo, const float *khi, const float *klo,
                              float *scores, uint32_t *status, cudaStream_t stream, bool programmatic = true);
// From this many blocks on, the routing scores run on the tensor cores (at
// 256 blocks the fused CUDA-core scoring is still faster, at 360 it is slower).
constexpr int kTcScoresMinBlocks = 320;
cudaError_t launch_schedule(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int dense, int num_ctas,
                            int32_t *work, int32_t *cta_range, int64_t *cta_cost, int32_t *unit_cost,
                            int32_t *head_sorted, int32_t *head_len, int64_t *head_cost, const int32_t *pair_cnt,
                            cudaStream_t stream);
// Paired mode (64-token blocks): entry = block | kPairInA (kept by the first
// query block of the pair) | kPairInB (kept by the second).
constexpr int32_t kPairInA = 1 << 16, kPairInB = 1 << 17, kPairBlockMask = 0xFFFF;
cudaError_t launch_pair_lists(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int32_t *pair_cnt,
                              int32_t *pair_list, cudaStream_t stream);
cudaError_t launch_attn(const Geo &g, const void *q, const void *k, const void *v, const int32_t *kv_cnt,
                        const int32_t *kv_idx, const int32_t *pair_cnt, const int32_t *pair_list,
                        const int32_t *work, const int32_t *cta_range, int num_ctas, int dense, void *out,
                        int64_t *cta_ns, uint32_t *status, cudaStream_t stream, int *launch_error_kind);

// Work of every head (valid token pairs of its kept lists).
cudaError_t launch_head_cost(const Geo &g, const int32_t *kv_cnt, const int32_t *kv_idx, int dense, int64_t *head_cost,
                             cudaStream_t stream);
// Slack augmentation of the lists (in place) within `budget` token pairs.
cudaError_t launch_augment(const Geo &g, const float *probs, long long budget, int32_t *kv_cnt, int32_t *kv_idx,
                           void *state, long long *row_tie, unsigned long long *added_cost, double *added_mass,
                           cudaStream_t stream);
size_t augment_state_bytes();
// Write a workspace header field on the stream: word >= 0 takes a uint64 at
// words (word, word+1); word < 0 takes a uint32 at word -word.
cudaError_t launch_header_write(uint32_t *header, int word, uint64_t value, cudaStream_t stream);

}  // namespace fvattn
