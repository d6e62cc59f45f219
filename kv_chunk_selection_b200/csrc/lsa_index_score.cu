// lsa_index_score: the Neural Memory Indexer's chunk scores.
//
// Method: every tau decode steps the indexer scores each historical chunk from
// the current query state against the chunk's cached indexer key (summary page
// "FlashMemory-DeepSeek-V4 ...", 1 Introduction and 2.1 Architecture) through
// a sigmoid (review page, "1. Key Terms & Definitions") of a dot product
// (summary page, 3 Experiments, "Limitations"):
//     score_c = sum_h w_h * sigmoid(q_h . k_c / sqrt(128)),  16 heads.
//
// B200 design: per sequence the scores are one dense contraction
// [chunks x 128] x [128 x 16 heads].  A CTA takes a tile of 128 chunks and
// computes D[128 x 16] = K_tile Q^T on the 5th-generation tensor cores:
// tcgen05.mma kind::f16 (M = 128 chunks, N = 16 heads, K = 16 per
// instruction, 8 instructions), bf16 operands in shared memory in the
// 128-byte swizzled K-major layout, the fp32 accumulator in tensor memory
// (16 of the 32 allocated columns).  Key rows are gathered through the chunk
// table with 16-byte loads (one row per thread) and written swizzled; one
// thread issues the MMAs and commits them to an mbarrier; each warp then reads
// its 32 TMEM lanes (one chunk per thread, 16 head logits) with tcgen05.ld and
// applies the sigmoid and the weighted head sum in fp32.
//
// lsa_token_score is the second, token-level stage (summary page, 2.1
// Architecture: native token-level scoring picks a fine-grained top-k inside
// the recalled subset): the same form with the decode step's indexer query,
// over every token of the recalled chunks.  Only the row source differs: tile
// row r is token position p = 64 j + i (token i of the j-th recalled chunk),
// whose key row is 64 * slot(kept[j]) + i of the per-token key pool.
#include <mutex>

#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

namespace lsa {
namespace score {

constexpr int kThreads = 128;       // one thread per chunk row = one TMEM lane
constexpr int kTile = 128;          // chunks per CTA (MMA M)
constexpr int kKBlockBytes = 128;   // 64 bf16 per row per swizzle atom
constexpr int kABytes = kTile * 2 * kKBlockBytes;          // 32 KiB: 2 K-blocks of [128 x 128 B]
constexpr int kBBytes = kIndexHeads * 2 * kKBlockBytes;    // 4 KiB: 2 K-blocks of [16 x 128 B]
constexpr int kSmemBytes = kABytes + kBBytes + 16 + kTile * 9;   // + barrier, TMEM slot, row addresses and flags
constexpr int kHistOffset = (kSmemBytes + 15) / 16 * 16;         // score-bin counts of the tile (token selection)
constexpr int kSmemBytesHist = kHistOffset + kScoreBins * 4;
constexpr uint32_t kTmemCols = 32;  // allocation unit (>= 16 accumulator columns)
constexpr uint32_t kIdesc = umma_idesc_bf16_f32(kTile, kIndexHeads);

// Byte offset of the 16-byte piece j (0..15, 8 bf16 each) of row r in a
// K-major SW128 operand with `rows` rows per K-block.
__device__ __forceinline__ uint32_t sw128_offset(int r, int j, int rows) {
  const int kb = j >> 3, jj = j & 7;
  return kb * rows * kKBlockBytes + r * kKBlockBytes + ((jj ^ (r & 7)) << 4);
}

// Row sources.  count(b) is the number of rows of sequence b (-1 when its
// count is invalid), stride the row pitch of the score output, and key_row()
// the key row of row c (false, with an error bit, when it is out of range).
struct ChunkRows {
  const int32_t* table;
  const int32_t* n_chunks;
  int max_chunks;
  int64_t n_slots;
  __device__ int count(int b) const {
    const int n = __ldg(n_chunks + b);
    return (n < 0 || n > max_chunks) ? -1 : n;
  }
  __device__ int64_t stride() const { return max_chunks; }
  __device__ void on_count(int, int) const {}
  __device__ int32_t* hist_of(int) const { return nullptr; }
  __device__ bool key_row(int b, int c, int64_t* row, unsigned* err) const {
    const int64_t slot =
        table ? __ldg(table + static_cast<int64_t>(b) * max_chunks + c) : static_cast<int64_t>(b) * max_chunks + c;
    if (slot < 0 || slot >= n_slots) {
      *err = LSA_DEV_ERR_BAD_SLOT;
      return false;
    }
    *row = slot;
    return true;
  }
};

struct TokenRows {
  const int32_t* table;
  const int32_t* kept;
  const int32_t* n_kept;
  int max_chunks, max_kept;
  int64_t n_slots;
  int32_t* n_tokens;   // out: 64 * n_kept[b]
  int32_t* hist;       // optional [B][kScoreBinReplicas][kScoreBins]: score-bin counts, added to (lsa_select_tokens)
  __device__ int32_t* hist_of(int b) const {
    return hist ? hist + (static_cast<int64_t>(b) * kScoreBinReplicas + blockIdx.x % kScoreBinReplicas) * kScoreBins
                : nullptr;
  }
  __device__ int count(int b) const {
    const int n = ld_dep(n_kept + b);
    return (n < 0 || n > max_kept) ? -1 : n * kChunkTokens;
  }
  __device__ int64_t stride() const { return static_cast<int64_t>(max_kept) * kChunkTokens; }
  __device__ void on_count(int b, int n) const { n_tokens[b] = n < 0 ? 0 : n; }
  __device__ bool key_row(int b, int p, int64_t* row, unsigned* err) const {
    const int j = p / kChunkTokens, i = p % kChunkTokens;
    const int c = ld_dep(kept + static_cast<int64_t>(b) * max_kept + j);
    if (c < 0 || c >= max_chunks) {
      *err = LSA_DEV_ERR_BAD_CHUNK;
      return false;
    }
    const int64_t slot =
        table ? ld_dep(table + static_cast<int64_t>(b) * max_chunks + c) : static_cast<int64_t>(b) * max_chunks + c;
    if (slot < 0 || slot >= n_slots) {
      *err = LSA_DEV_ERR_BAD_SLOT;
      return false;
    }
    *row = slot * kChunkTokens + i;
    return true;
  }
};

template <class Rows>
__global__ void __launch_bounds__(kThreads)
index_score_kernel(const __nv_bfloat16* __restrict__ q_idx, const float* __restrict__ w,
                   const __nv_bfloat16* __restrict__ keys, Rows rows, float* __restrict__ scores,
                   float neg_scale_log2, unsigned* status, int keys_unchanged) {
  extern __shared__ __align__(1024) uint8_t smem[];
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  // With keys_unchanged the caller guarantees that the preceding kernel on the
  // stream wrote none of the keys, the chunk table and the kept lists (true for
  // every decode step of a window after the first), so the key rows are
  // resolved and loaded while that kernel finishes; the query, which it may
  // have written, and every output wait for it.
  if (!keys_unchanged) griddep_wait();
  const int b = blockIdx.y;
  const int n = rows.count(b);
  if (n < 0) {
    if (keys_unchanged) griddep_wait();
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      rows.on_count(b, n);
      set_status(status, LSA_DEV_ERR_BAD_COUNT);
    }
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && !keys_unchanged) rows.on_count(b, n);
  const int base = blockIdx.x * kTile;
  if (base >= n) {
    // No rows here (a sequence shorter than the longest).  The sequence's
    // first CTA still waits and writes its count, so this grid never
    // completes before the preceding one (the next kernel's wait covers
    // both); the other empty CTAs leave at once and free their SM slots for
    // CTAs with rows to load.
    if (keys_unchanged && blockIdx.x == 0) {
      griddep_wait();
      if (threadIdx.x == 0) rows.on_count(b, n);
    }
    return;
  }
  if (smem_u32(smem) & 1023u) {   // the swizzle atoms assume 1024-byte alignment
    if (keys_unchanged) griddep_wait();   // every CTA waits before it ends
    if (threadIdx.x == 0) set_status(status, LSA_DEV_ERR_INTERNAL);
    return;
  }
  uint8_t* sa = smem;
  uint8_t* sb = smem + kABytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kABytes + kBBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  int64_t* row_at = reinterpret_cast<int64_t*>(smem + kABytes + kBBytes + 16);   // [kTile] key row or -1
  bool* row_ok = reinterpret_cast<bool*>(row_at + kTile);                            // [kTile]
  const int tid = threadIdx.x, warp = tid >> 5;
  int32_t* const ghist = rows.hist_of(b);                                            // block-uniform
  int* const shist = reinterpret_cast<int*>(smem + kHistOffset);                      // [kScoreBins] when ghist

  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  if (ghist) {   // cleared here; the barrier before the MMA publishes it
#pragma unroll
    for (int i = tid; i < kScoreBins / 4; i += kThreads) reinterpret_cast<int4*>(shist)[i] = make_int4(0, 0, 0, 0);
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }

  // A: the tile's 128 key rows (chunks, or tokens of recalled chunks).  Each
  // thread first resolves one row's address (its lookup chain); then half a
  // warp loads one 256-byte row, so a warp instruction reads two whole rows
  // instead of 32 pieces of 32 different rows, all 16 loads of a thread issued
  // before any store.  A row that is out of range or fails its lookup is zero
  // and flagged, so its score is not written.
  {
    const int c = base + tid;
    bool okr = c < n;
    int64_t krow = 0;
    if (okr) {
      unsigned err = 0;
      if (!rows.key_row(b, c, &krow, &err)) {
        set_status(status, err);
        okr = false;
      }
    }
    row_ok[tid] = okr;
    row_at[tid] = okr ? krow : -1;
  }
  __syncthreads();
  {
    const int piece = tid & 15;
    uint4 v[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const int r = it * (kThreads / 16) + (tid >> 4);
      const int64_t krow = row_at[r];
      v[it] = krow >= 0 ? ld_dep(reinterpret_cast<const uint4*>(keys + krow * kIndexDim) + piece)
                        : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const int r = it * (kThreads / 16) + (tid >> 4);
      *reinterpret_cast<uint4*>(sa + sw128_offset(r, piece, kTile)) = v[it];
    }
  }
  if (keys_unchanged) {
    griddep_wait();   // the query and the outputs: after the preceding kernel
    if (blockIdx.x == 0 && threadIdx.x == 0) rows.on_count(b, n);
  }
  // B: the 16 indexer query rows of sequence b (K-major, one row per head).
  {
    const uint4* qb = reinterpret_cast<const uint4*>(q_idx + static_cast<int64_t>(b) * kIndexHeads * kIndexDim);
#pragma unroll
    for (int i = tid; i < kIndexHeads * 16; i += kThreads) {
      const int h = i >> 4, j = i & 15;
      *reinterpret_cast<uint4*>(sb + sw128_offset(h, j, kIndexHeads)) = ld_dep(qb + i);
    }
  }
  fence_proxy_async_smem();   // generic-proxy smem writes -> visible to the tensor core
  tcgen05_fence_before();
  __syncthreads();
  tcgen05_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const uint32_t a0 = smem_u32(sa), b0 = smem_u32(sb);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t ad = umma_desc_kmajor_sw128(a0 + kb * kTile * kKBlockBytes + k * 32);
        const uint64_t bd = umma_desc_kmajor_sw128(b0 + kb * kIndexHeads * kKBlockBytes + k * 32);
        umma_bf16(tmem, ad, bd, kIdesc, (kb | k) != 0);
      }
    }
    umma_commit(bar);
  }
  int never = 0;
  // warp-uniform, so the .sync.aligned TMEM load below never diverges
  const bool done = __all_sync(0xffffffffu, mbar_wait_bounded(bar, 0, &never));
  tcgen05_fence_after();
  int bin = -1;         // this row's score bin, when it is the first of the tile in that bin
  if (!done) {
    if (tid == 0) set_status(status, LSA_DEV_ERR_TIMEOUT);
  } else {
    float logit[16];
    tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(warp * 32) << 16), logit);
    float s = 0.f;
#pragma unroll
    for (int h = 0; h < kIndexHeads; ++h) s += ld_dep(w + h) * (1.f / (1.f + fast_exp2(logit[h] * neg_scale_log2)));
    if (row_ok[tid]) {
      scores[static_cast<int64_t>(b) * rows.stride() + base + tid] = s;
      if (ghist) {
        const int bi = score_bin(s, score_bin_scale(w));
        if (atomicAdd(&shist[bi], 1) == 0) bin = bi;
      }
    }
  }
  tcgen05_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
  // One global add per bin this tile touched, by the row that touched it first.
  if (bin >= 0) atomicAdd(ghist + bin, shist[bin]);
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
  const dim3 grid((max_chunks + score::kTile - 1) / score::kTile, B);
  const float neg_scale_log2 = -1.4426950408889634f / sqrtf(static_cast<float>(kIndexDim));
  const score::ChunkRows rows{chunk_table, n_chunks, max_chunks, n_slots};
  launch_pdl(false, score::index_score_kernel<score::ChunkRows>, grid, dim3(score::kThreads), score::kSmemBytes,
             static_cast<cudaStream_t>(stream), static_cast<const __nv_bfloat16*>(q_idx), w,
             static_cast<const __nv_bfloat16*>(chunk_keys), rows, scores, neg_scale_log2, lsa_device_status_ptr(), 0);
  return launch_status();
}

namespace lsa {
namespace score {
// The token scorer's launch, shared by lsa_token_score (hist == nullptr) and
// lsa_select_tokens (hist: [B][kScoreBins] counts to add to).
int launch_token_score(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                       const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B, int max_chunks,
                       int max_kept, float* scores, int32_t* n_tokens, int32_t* hist, int keys_unchanged,
                       cudaStream_t stream) {
  if (!q_idx || !w || !token_keys || !kept || !n_kept || !scores || !n_tokens || B <= 0 || max_chunks <= 0 ||
      max_kept <= 0 || n_slots <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > 65535) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(max_kept) * kChunkTokens >= (int64_t{1} << 31) ||
      n_slots >= (int64_t{1} << 62) / kChunkTokens)
    return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q_idx) || !aligned16(token_keys)) return LSA_ERR_MISALIGNED;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  const int smem = hist ? kSmemBytesHist : kSmemBytes;
  if (hist) {   // the histogram needs more than the default 48 KB of dynamic shared memory
    static std::mutex mu;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      if (cudaFuncSetAttribute(index_score_kernel<TokenRows>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemBytesHist) != cudaSuccess) {
        cudaGetLastError();
        return LSA_ERR_CUDA;
      }
      attr_set[dev] = true;
    }
  }
  const int max_tokens = max_kept * kChunkTokens;
  const dim3 grid((max_tokens + kTile - 1) / kTile, B);
  const float neg_scale_log2 = -1.4426950408889634f / sqrtf(static_cast<float>(kIndexDim));
  TokenRows rows{chunk_table, kept, n_kept, max_chunks, max_kept, n_slots, n_tokens};
  rows.hist = hist;
  launch_pdl(true, index_score_kernel<TokenRows>, grid, dim3(kThreads), smem, stream,
             static_cast<const __nv_bfloat16*>(q_idx), w, static_cast<const __nv_bfloat16*>(token_keys), rows, scores,
             neg_scale_log2, lsa_device_status_ptr(), keys_unchanged);
  return launch_status();
}
}  // namespace score
}  // namespace lsa

extern "C" int lsa_token_score(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                               const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B,
                               int max_chunks, int max_kept, float* scores, int32_t* n_tokens, void* stream) {
  return lsa::score::launch_token_score(q_idx, w, token_keys, n_slots, chunk_table, kept, n_kept, B, max_chunks,
                                        max_kept, scores, n_tokens, nullptr, 0, static_cast<cudaStream_t>(stream));
}
