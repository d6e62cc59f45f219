// lsa_index_score: the Neural Memory Indexer's chunk scores.
//
// Method: every tau decode steps the indexer scores each historical chunk from
// the current query state against the chunk's cached indexer key (summary page
// "FlashMemory-DeepSeek-V4 ...", 1 Introduction and 2.1 Architecture) through
// a sigmoid (review page, "1. Key Terms & Definitions") of a dot product
// (summary page, 3 Experiments, "Limitations"):
//     score_c = sum_h w_h * sigmoid(q_h . k_c / sqrt(128)),  16 heads.
//
// B200 design: the [chunks x 128] x [128 x 16 heads] product is a dense
// contraction, computed on the tensor cores with mma.sync m16n8k16 (M = 16
// chunks, N = 8 heads, two N tiles).  Key rows are fetched straight from HBM
// into the A fragments with 16-byte loads: the contraction index is permuted
// consistently in A and B so that each lane's 16 bytes (8 consecutive dims of
// one key row) feed two k-steps, and a warp instruction covers 8 rows x 64
// contiguous bytes.  The sigmoid and the weighted head sum run in fp32 on the
// accumulator fragments; a 2-step shuffle finishes each chunk's sum.
#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

namespace lsa {
namespace score {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunksPerCta = kWarps * 16;

__device__ __forceinline__ float sigmoid_from_logit2(float neg_logit_log2) {
  // sigmoid(x) = 1 / (1 + 2^(-x log2 e)); the argument is already -x log2 e.
  return 1.f / (1.f + fast_exp2(neg_logit_log2));
}

__global__ void __launch_bounds__(kThreads)
index_score_kernel(const __nv_bfloat16* __restrict__ q_idx, const float* __restrict__ w,
                   const __nv_bfloat16* __restrict__ keys, int64_t n_slots, const int32_t* __restrict__ table,
                   const int32_t* __restrict__ n_chunks, int max_chunks, float* __restrict__ scores,
                   float neg_scale_log2, unsigned* status) {
  const int b = blockIdx.y;
  const int n = __ldg(n_chunks + b);
  if (n < 0 || n > max_chunks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, LSA_DEV_ERR_BAD_COUNT);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int base = blockIdx.x * kChunksPerCta + warp * 16;
  if (base >= n) return;
  const int gl = lane >> 2, c4 = lane & 3;

  // B operand: Q^T for heads gl (tile 0) and 8+gl (tile 1); lane c4 holds dims
  // [32 s + 8 c4, 32 s + 8 c4 + 8) of k-step pair s.
  const uint4* q0 = reinterpret_cast<const uint4*>(q_idx + (static_cast<int64_t>(b) * kIndexHeads + gl) * kIndexDim);
  const uint4* q1 = q0 + 8 * kIndexDim / 8;
  uint4 qa[4], qb[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    qa[s] = __ldg(q0 + 4 * s + c4);
    qb[s] = __ldg(q1 + 4 * s + c4);
  }

  // A operand rows: chunks base+gl and base+gl+8.
  const int r0 = base + gl, r1 = base + gl + 8;
  int64_t slot0 = -1, slot1 = -1;
  if (r0 < n) slot0 = table ? __ldg(table + static_cast<int64_t>(b) * max_chunks + r0)
                            : static_cast<int64_t>(b) * max_chunks + r0;
  if (r1 < n) slot1 = table ? __ldg(table + static_cast<int64_t>(b) * max_chunks + r1)
                            : static_cast<int64_t>(b) * max_chunks + r1;
  bool bad0 = (r0 < n) && (slot0 < 0 || slot0 >= n_slots);
  bool bad1 = (r1 < n) && (slot1 < 0 || slot1 >= n_slots);
  if (bad0 || bad1) set_status(status, LSA_DEV_ERR_BAD_SLOT);
  const bool ok0 = (r0 < n) && !bad0, ok1 = (r1 < n) && !bad1;
  uint4 ka[4], kb[4];
  const uint4 z = make_uint4(0, 0, 0, 0);
  const uint4* k0 = reinterpret_cast<const uint4*>(keys + (ok0 ? slot0 : 0) * kIndexDim);
  const uint4* k1 = reinterpret_cast<const uint4*>(keys + (ok1 ? slot1 : 0) * kIndexDim);
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    ka[s] = ok0 ? __ldg(k0 + 4 * s + c4) : z;
    kb[s] = ok1 ? __ldg(k1 + 4 * s + c4) : z;
  }

  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    mma_bf16_16816(d0, ka[s].x, kb[s].x, ka[s].y, kb[s].y, qa[s].x, qa[s].y);
    mma_bf16_16816(d1, ka[s].x, kb[s].x, ka[s].y, kb[s].y, qb[s].x, qb[s].y);
    mma_bf16_16816(d0, ka[s].z, kb[s].z, ka[s].w, kb[s].w, qa[s].z, qa[s].w);
    mma_bf16_16816(d1, ka[s].z, kb[s].z, ka[s].w, kb[s].w, qb[s].z, qb[s].w);
  }
  // d0: heads 2c4, 2c4+1; d1: heads 8+2c4, 9+2c4.  [0],[1] chunk r0; [2],[3] chunk r1.
  const float w0 = __ldg(w + 2 * c4), w1 = __ldg(w + 2 * c4 + 1);
  const float w2 = __ldg(w + 8 + 2 * c4), w3 = __ldg(w + 9 + 2 * c4);
  float p0 = w0 * sigmoid_from_logit2(d0[0] * neg_scale_log2) + w1 * sigmoid_from_logit2(d0[1] * neg_scale_log2) +
             w2 * sigmoid_from_logit2(d1[0] * neg_scale_log2) + w3 * sigmoid_from_logit2(d1[1] * neg_scale_log2);
  float p1 = w0 * sigmoid_from_logit2(d0[2] * neg_scale_log2) + w1 * sigmoid_from_logit2(d0[3] * neg_scale_log2) +
             w2 * sigmoid_from_logit2(d1[2] * neg_scale_log2) + w3 * sigmoid_from_logit2(d1[3] * neg_scale_log2);
  p0 += __shfl_xor_sync(0xffffffffu, p0, 1);
  p1 += __shfl_xor_sync(0xffffffffu, p1, 1);
  p0 += __shfl_xor_sync(0xffffffffu, p0, 2);
  p1 += __shfl_xor_sync(0xffffffffu, p1, 2);
  if (c4 == 0) {
    float* row = scores + static_cast<int64_t>(b) * max_chunks;
    if (ok0) row[r0] = p0;
    if (ok1) row[r1] = p1;
  }
}

}  // namespace score
}  // namespace lsa

extern "C" int lsa_index_score(const void* q_idx, const float* w, const void* chunk_keys, int64_t n_slots,
                               const int32_t* chunk_table, const int32_t* n_chunks, int B, int max_chunks,
                               float* scores, void* stream) {
  using namespace lsa;
  if (!q_idx || !w || !chunk_keys || !n_chunks || !scores || B <= 0 || max_chunks <= 0 || n_slots <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > 65535) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(chunk_keys)) return LSA_ERR_MISALIGNED;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  const dim3 grid((max_chunks + score::kChunksPerCta - 1) / score::kChunksPerCta, B);
  const float neg_scale_log2 = -1.4426950408889634f / sqrtf(static_cast<float>(kIndexDim));
  score::index_score_kernel<<<grid, score::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(q_idx), w, static_cast<const __nv_bfloat16*>(chunk_keys), n_slots,
      chunk_table, n_chunks, max_chunks, scores, neg_scale_log2, lsa_device_status_ptr());
  return launch_status();
}
