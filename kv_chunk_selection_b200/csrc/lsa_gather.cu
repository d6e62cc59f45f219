// lsa_gather_chunks / lsa_fetch_from_host: build the compact resident buffer.
//
// Method: only the chunks recalled for the coming window are kept in GPU
// memory (summary page "FlashMemory-DeepSeek-V4 ...", Abstract and 2.1
// Architecture); when the full cache lives in CPU memory they are fetched from
// there every tau steps (summary page, 3 Experiments "Experimental Setup";
// handbook page "DeepSeek-V4: Architecting for Ultra-Long Contexts", "The
// Neural Memory Indexer", item 3).
//
// B200 design: a pure bandwidth copy.  The work item is one 16 KiB
// (chunk, KV head, K-or-V) tile, contiguous at both ends; a 256-thread CTA
// moves it with 16-byte loads issued four per thread before any store, and the
// grid strides over all items of the batch (the total is read on the device
// from cu_kept, so nothing is copied back to the host and the call can be
// captured in a CUDA graph).  The host-tier variant runs the same kernel on a
// small grid over the device alias of page-locked host memory: SMs pull the
// scattered chunks over the host link directly, on the caller's side stream,
// without a host loop or a device-to-host copy of the kept list.
//
// Also here: the copies of the NEXT rows. lsa_fetch_from_host_delta reuses
// chunks already resident from the previous window. lsa_append_token writes
// a decoded token into a sequence's local chunk, and lsa_reset_local empties
// the local chunks. lsa_gather_tokens packs the fine stage's selected tokens
// into dense units.
#include <atomic>
#include <vector>

#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

namespace lsa {
namespace gather {

constexpr int kThreads = 256;
constexpr int kVecPerTile = kTileBytes / 16;        // 1024 x 16 B
constexpr int kVecPerThread = kVecPerTile / kThreads;  // 4

__device__ __forceinline__ int seq_of(const int32_t* cu, int B, int i) {
  int lo = 0, hi = B - 1;  // largest b with cu[b] <= i
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Chunks kept in the previous window and still resident in its compact
// buffer (residency across windows): a kept chunk found in the previous
// window's kept list of the same sequence is copied from device memory
// instead of the host pool.
struct PrevWindow {
  const int32_t* kept;     // [B][max_kept] ascending, or nullptr (no reuse)
  const int32_t* cu;       // [B+1]
  int max_kept;
  int64_t buf_chunks;
  const uint4* k_buf;
  const uint4* v_buf;
  int32_t* reused;         // optional counter of reused chunks
};

// Index of chunk c in the ascending list a[0..n), or -1.
__device__ __forceinline__ int find_sorted(const int32_t* a, int n, int c) {
  int lo = 0, hi = n - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int v = __ldg(a + mid);
    if (v == c) return mid;
    if (v < c) lo = mid + 1; else hi = mid - 1;
  }
  return -1;
}

__global__ void __launch_bounds__(kThreads)
gather_kernel(const uint4* __restrict__ k_pool, const uint4* __restrict__ v_pool, int64_t n_slots,
              const int32_t* __restrict__ table, const int32_t* __restrict__ kept, const int32_t* __restrict__ cu,
              int B, int max_chunks, int max_kept, uint4* __restrict__ k_buf, uint4* __restrict__ v_buf,
              int64_t buf_chunks, unsigned* status, PrevWindow prev) {
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  griddep_wait();                 // the previous kernel on the stream has finished
  const int total = __ldg(cu + B);
  if (__ldg(cu) != 0 || total < 0 || static_cast<int64_t>(total) > buf_chunks) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, LSA_DEV_ERR_CAPACITY);
    return;
  }
  const int64_t items = static_cast<int64_t>(total) * 2 * kNumKVHeads;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int i = static_cast<int>(it >> 4);        // compact chunk index
    const int kv = static_cast<int>((it >> 3) & 1);  // 0 = K, 1 = V
    const int h = static_cast<int>(it & 7);
    const int b = seq_of(cu, B, i);
    const int j = i - __ldg(cu + b);
    if (j < 0 || j >= max_kept) {
      if (threadIdx.x == 0) set_status(status, LSA_DEV_ERR_CAPACITY);
      continue;
    }
    const int c = __ldg(kept + static_cast<int64_t>(b) * max_kept + j);
    if (c < 0 || c >= max_chunks) {
      if (threadIdx.x == 0) set_status(status, LSA_DEV_ERR_BAD_CHUNK);
      continue;
    }
    const int64_t slot = table ? __ldg(table + static_cast<int64_t>(b) * max_chunks + c)
                               : static_cast<int64_t>(b) * max_chunks + c;
    if (slot < 0 || slot >= n_slots) {
      if (threadIdx.x == 0) set_status(status, LSA_DEV_ERR_BAD_SLOT);
      continue;
    }
    const int64_t tile = static_cast<int64_t>(kNumKVHeads) * kVecPerTile;  // uint4 per chunk
    const uint4* src = (kv ? v_pool : k_pool) + slot * tile + h * kVecPerTile;
    if (prev.kept) {
      const int pb = __ldg(prev.cu + b), pn = __ldg(prev.cu + b + 1) - pb;
      if (pb >= 0 && pn > 0 && pn <= prev.max_kept && static_cast<int64_t>(pb) + pn <= prev.buf_chunks) {
        const int jp = find_sorted(prev.kept + static_cast<int64_t>(b) * prev.max_kept, pn, c);
        if (jp >= 0) {
          src = (kv ? prev.v_buf : prev.k_buf) + (h * prev.buf_chunks + pb + jp) * kVecPerTile;
          if (prev.reused && kv == 0 && h == 0 && threadIdx.x == 0) atomicAdd(prev.reused, 1);
        }
      }
    }
    uint4* dst = (kv ? v_buf : k_buf) + (h * buf_chunks + i) * kVecPerTile;   // head-major compact buffer
    uint4 r[kVecPerThread];
#pragma unroll
    for (int v = 0; v < kVecPerThread; ++v) r[v] = __ldcs(src + v * kThreads + threadIdx.x);
#pragma unroll
    for (int v = 0; v < kVecPerThread; ++v) dst[v * kThreads + threadIdx.x] = r[v];
  }
}

// Appends one decoded token per sequence to its local chunk: K/V of the new
// token ([B][8][128] each) go to position local_len[b] of k_local / v_local
// ([B][8][64][128]), then local_len[b] is incremented.
__global__ void __launch_bounds__(256)
append_token_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new, uint4* __restrict__ k_local,
                    uint4* __restrict__ v_local, int32_t* __restrict__ local_len, unsigned* status) {
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  griddep_wait();                 // the previous kernel on the stream has finished
  constexpr int kVecPerToken = kNumKVHeads * kHeadDim / 8;   // 128 x 16 B per token (all 8 heads)
  constexpr int kVecPerRow = kHeadDim / 8;                   // 16 x 16 B per (head, token)
  const int b = blockIdx.x;
  const int pos = local_len[b];
  if (pos < 0 || pos >= kChunkTokens) {
    if (threadIdx.x == 0) set_status(status, LSA_DEV_ERR_CAPACITY);
    return;
  }
  for (int i = threadIdx.x; i < 2 * kVecPerToken; i += blockDim.x) {
    const int kv = i / kVecPerToken, r = i % kVecPerToken;
    const int g = r / kVecPerRow, e = r % kVecPerRow;
    const uint4 v = ld_dep((kv ? v_new : k_new) + static_cast<int64_t>(b) * kVecPerToken + r);
    (kv ? v_local : k_local)[((static_cast<int64_t>(b) * kNumKVHeads + g) * kChunkTokens + pos) * kVecPerRow + e] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) local_len[b] = pos + 1;
}

// Token gather of the fine stage: the selected token positions of each
// sequence (ascending; position p is row p % 64 of compact chunk
// cu_kept[b] + p / 64) are packed into dense 64-token units in the same
// [unit][KV head][64][128] layout as the compact buffer, so that the decode
// attention runs over them unchanged.  One CTA copies one (unit, KV head):
// 64 rows of K and of V, 256 B each, sixteen 16-byte loads per thread issued
// before any store.  Counts are multiples of 64 (the budget is), so no unit is
// partial; cu_units[b] = cu_sel[b] / 64.
constexpr int kTokThreads = 128;
constexpr int kRowVecs = kHeadDim * 2 / 16;                          // 16 x 16 B per row
constexpr int kTokVecs = 2 * kChunkTokens * kRowVecs / kTokThreads;  // 16 per thread

__global__ void __launch_bounds__(kTokThreads)
gather_tokens_kernel(const uint4* __restrict__ k_buf, const uint4* __restrict__ v_buf, int64_t buf_chunks,
                     const int32_t* __restrict__ cu_kept, const int32_t* __restrict__ sel,
                     const int32_t* __restrict__ cu_sel, int max_sel, uint4* __restrict__ k_out,
                     uint4* __restrict__ v_out, int64_t out_chunks, int32_t* __restrict__ cu_units,
                     unsigned* status) {
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  griddep_wait();                 // the previous kernel on the stream has finished
  const int b = blockIdx.y;
  const int u = blockIdx.x / kNumKVHeads, g = blockIdx.x % kNumKVHeads;
  const int tid = threadIdx.x;
  const int s0 = ld_dep(cu_sel + b), s1 = ld_dep(cu_sel + b + 1);
  const int n = s1 - s0;
  const bool lead = blockIdx.x == 0 && tid == 0;
  if (s0 < 0 || n < 0 || n > max_sel || (n % kChunkTokens) != 0 || (s0 % kChunkTokens) != 0) {
    if (lead) set_status(status, LSA_DEV_ERR_BAD_COUNT);
    return;
  }
  if (lead) {
    cu_units[b + 1] = s1 / kChunkTokens;
    if (b == 0) cu_units[0] = s0 / kChunkTokens;
  }
  if (u * kChunkTokens >= n) return;
  const int64_t c0 = ld_dep(cu_kept + b), c1 = ld_dep(cu_kept + b + 1);
  const int64_t ou = s0 / kChunkTokens + u;
  if (c0 < 0 || c1 < c0 || c1 > buf_chunks || ou >= out_chunks) {
    if (tid == 0) set_status(status, ou >= out_chunks ? LSA_DEV_ERR_CAPACITY : LSA_DEV_ERR_BAD_COUNT);
    return;
  }
  const int64_t n_pos = (c1 - c0) * kChunkTokens;
  const int32_t* my_sel = sel + static_cast<int64_t>(b) * max_sel + u * kChunkTokens;
  uint4 v[kTokVecs];
  bool ok[kTokVecs];
#pragma unroll
  for (int e = 0; e < kTokVecs; ++e) {
    const int idx = tid + e * kTokThreads;
    const int kv = idx / (kChunkTokens * kRowVecs), rem = idx % (kChunkTokens * kRowVecs);
    const int r = rem / kRowVecs, x = rem % kRowVecs;
    const int p = ld_dep(my_sel + r);
    ok[e] = p >= 0 && p < n_pos;
    v[e] = make_uint4(0, 0, 0, 0);
    if (ok[e]) {
      const int64_t src = (g * buf_chunks + c0 + p / kChunkTokens) * kChunkTokens + p % kChunkTokens;
      v[e] = ld_dep((kv ? v_buf : k_buf) + src * kRowVecs + x);
    }
  }
#pragma unroll
  for (int e = 0; e < kTokVecs; ++e) {
    const int idx = tid + e * kTokThreads;
    const int kv = idx / (kChunkTokens * kRowVecs), rem = idx % (kChunkTokens * kRowVecs);
    const int r = rem / kRowVecs, x = rem % kRowVecs;
    const int64_t dst = (g * out_chunks + ou) * kChunkTokens + r;
    (kv ? v_out : k_out)[dst * kRowVecs + x] = v[e];
    if (!ok[e] && x == 0) set_status(status, LSA_DEV_ERR_BAD_CHUNK);
  }
}

int check_common(const void* k_pool, const void* v_pool, int64_t n_slots, const int32_t* kept,
                 const int32_t* cu_kept, int B, int max_chunks, int max_kept, const void* k_buf, const void* v_buf,
                 int64_t buf_chunks) {
  if (!k_pool || !v_pool || !kept || !cu_kept || !k_buf || !v_buf || B <= 0 || max_chunks <= 0 ||
      max_kept <= 0 || n_slots <= 0 || buf_chunks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(B) * max_kept >= (int64_t{1} << 31)) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(k_buf) || !aligned16(v_buf)) return LSA_ERR_MISALIGNED;
  return LSA_OK;
}

}  // namespace gather
}  // namespace lsa

extern "C" {

int lsa_gather_chunks(const void* k_pool, const void* v_pool, int64_t n_slots, const int32_t* chunk_table,
                      const int32_t* kept, const int32_t* cu_kept, int B, int max_chunks, int max_kept, void* k_buf,
                      void* v_buf, int64_t buf_chunks, void* stream) {
  using namespace lsa;
  const int st =
      gather::check_common(k_pool, v_pool, n_slots, kept, cu_kept, B, max_chunks, max_kept, k_buf, v_buf, buf_chunks);
  if (st != LSA_OK) return st;
  const int sms = device_sm_count();
  if (sms <= 0) return LSA_ERR_NO_DEVICE;
  launch_pdl(false, gather::gather_kernel, dim3(sms * 8), dim3(gather::kThreads), 0, static_cast<cudaStream_t>(stream),
             static_cast<const uint4*>(k_pool), static_cast<const uint4*>(v_pool), n_slots, chunk_table, kept,
             cu_kept, B, max_chunks, max_kept, static_cast<uint4*>(k_buf), static_cast<uint4*>(v_buf), buf_chunks,
             lsa_device_status_ptr(), gather::PrevWindow{});
  return launch_status();
}

}  // extern "C"

namespace {
// Host-side fault injection of the fetch (lsa_debug_fail_fetch): the next
// g_fetch_fail_calls fetch calls return g_fetch_fail_status after their
// argument checks, before anything touches the device.
std::atomic<int> g_fetch_fail_calls{0};
std::atomic<int> g_fetch_fail_status{LSA_ERR_CUDA};

int injected_fetch_failure() {
  int n = g_fetch_fail_calls.load();
  while (n > 0) {
    if (g_fetch_fail_calls.compare_exchange_weak(n, n - 1)) return g_fetch_fail_status.load();
  }
  return LSA_OK;
}

int fetch_impl(const void* host_k_pool, const void* host_v_pool, int64_t n_slots, const int32_t* chunk_table,
               const int32_t* kept, const int32_t* cu_kept, int B, int max_chunks, int max_kept, void* k_buf,
               void* v_buf, int64_t buf_chunks, int num_ctas, void* stream, void* done_event,
               const lsa::gather::PrevWindow& prev) {
  using namespace lsa;
  const int st = gather::check_common(host_k_pool, host_v_pool, n_slots, kept, cu_kept, B, max_chunks, max_kept,
                                      k_buf, v_buf, buf_chunks);
  if (st != LSA_OK) return st;
  if (const int inj = injected_fetch_failure()) return inj;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  // The pools must be page-locked host memory; use their device aliases.
  void* dk = nullptr;
  void* dv = nullptr;
  cudaPointerAttributes ak, av;
  if (cudaPointerGetAttributes(&ak, host_k_pool) != cudaSuccess ||
      cudaPointerGetAttributes(&av, host_v_pool) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_NOT_PINNED;
  }
  if (ak.type != cudaMemoryTypeHost || av.type != cudaMemoryTypeHost) return LSA_ERR_NOT_PINNED;
  if (cudaHostGetDevicePointer(&dk, const_cast<void*>(host_k_pool), 0) != cudaSuccess ||
      cudaHostGetDevicePointer(&dv, const_cast<void*>(host_v_pool), 0) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_NOT_PINNED;
  }
  const int grid = num_ctas > 0 ? num_ctas : 64;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gather::gather_kernel<<<grid, gather::kThreads, 0, s>>>(
      static_cast<const uint4*>(dk), static_cast<const uint4*>(dv), n_slots, chunk_table, kept, cu_kept, B,
      max_chunks, max_kept, static_cast<uint4*>(k_buf), static_cast<uint4*>(v_buf), buf_chunks,
      lsa_device_status_ptr(), prev);
  int rc = launch_status();
  if (rc == LSA_OK && done_event) {
    if (cudaEventRecord(static_cast<cudaEvent_t>(done_event), s) != cudaSuccess) {
      cudaGetLastError();
      rc = LSA_ERR_CUDA;
    }
  }
  return rc;
}
}  // namespace

extern "C" {

int lsa_fetch_from_host(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                        const int32_t* chunk_table, const int32_t* kept, const int32_t* cu_kept, int B,
                        int max_chunks, int max_kept, void* k_buf, void* v_buf, int64_t buf_chunks, int num_ctas,
                        void* stream, void* done_event) {
  return fetch_impl(host_k_pool, host_v_pool, n_slots, chunk_table, kept, cu_kept, B, max_chunks, max_kept, k_buf,
                    v_buf, buf_chunks, num_ctas, stream, done_event, lsa::gather::PrevWindow{});
}

int lsa_fetch_from_host_delta(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                              const int32_t* chunk_table, const int32_t* kept, const int32_t* cu_kept, int B,
                              int max_chunks, int max_kept, void* k_buf, void* v_buf, int64_t buf_chunks,
                              const int32_t* prev_kept, const int32_t* prev_cu_kept, int prev_max_kept,
                              const void* prev_k_buf, const void* prev_v_buf, int64_t prev_buf_chunks,
                              int32_t* reused_chunks, int num_ctas, void* stream, void* done_event) {
  using namespace lsa;
  if (!prev_kept || !prev_cu_kept || !prev_k_buf || !prev_v_buf || prev_max_kept <= 0 || prev_buf_chunks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (!aligned16(prev_k_buf) || !aligned16(prev_v_buf)) return LSA_ERR_MISALIGNED;
  if (prev_k_buf == k_buf || prev_v_buf == v_buf) return LSA_ERR_INVALID_ARG;   // must not overlap the target
  gather::PrevWindow prev{prev_kept, prev_cu_kept, prev_max_kept, prev_buf_chunks,
                          static_cast<const uint4*>(prev_k_buf), static_cast<const uint4*>(prev_v_buf),
                          reused_chunks};
  return fetch_impl(host_k_pool, host_v_pool, n_slots, chunk_table, kept, cu_kept, B, max_chunks, max_kept, k_buf,
                    v_buf, buf_chunks, num_ctas, stream, done_event, prev);
}

int lsa_append_token(const void* k_new, const void* v_new, void* k_local, void* v_local, int32_t* local_len, int B,
                     void* stream) {
  using namespace lsa;
  if (!k_new || !v_new || !k_local || !v_local || !local_len || B <= 0) return LSA_ERR_INVALID_ARG;
  if (B > 65535) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_local) || !aligned16(v_local)) return LSA_ERR_MISALIGNED;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  launch_pdl(true, gather::append_token_kernel, dim3(B), dim3(256), 0, static_cast<cudaStream_t>(stream),
             static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), static_cast<uint4*>(k_local),
             static_cast<uint4*>(v_local), local_len, lsa_device_status_ptr());
  return launch_status();
}

int lsa_gather_tokens(const void* k_buf, const void* v_buf, int64_t buf_chunks, const int32_t* cu_kept,
                      const int32_t* sel, const int32_t* cu_sel, int B, int max_sel, void* k_out, void* v_out,
                      int64_t out_chunks, int32_t* cu_units, void* stream) {
  using namespace lsa;
  if (!k_buf || !v_buf || !cu_kept || !sel || !cu_sel || !k_out || !v_out || !cu_units || B <= 0 ||
      max_sel <= 0 || buf_chunks <= 0 || out_chunks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (max_sel % kChunkTokens != 0) return LSA_ERR_INVALID_ARG;
  if (B > 65535 || static_cast<int64_t>(B) * max_sel >= (int64_t{1} << 31) ||
      static_cast<int64_t>(max_sel / kChunkTokens) * kNumKVHeads > 0x7fffffff)
    return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(k_buf) || !aligned16(v_buf) || !aligned16(k_out) || !aligned16(v_out)) return LSA_ERR_MISALIGNED;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  const dim3 grid((max_sel / kChunkTokens) * kNumKVHeads, B);
  launch_pdl(true, gather::gather_tokens_kernel, grid, dim3(gather::kTokThreads), 0, static_cast<cudaStream_t>(stream),
             static_cast<const uint4*>(k_buf), static_cast<const uint4*>(v_buf), buf_chunks, cu_kept, sel, cu_sel,
             max_sel, static_cast<uint4*>(k_out), static_cast<uint4*>(v_out), out_chunks, cu_units,
             lsa_device_status_ptr());
  return launch_status();
}

int lsa_reset_local(int32_t* local_len, int B, void* stream) {
  using namespace lsa;
  if (!local_len || B <= 0) return LSA_ERR_INVALID_ARG;
  if (B > 65535) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  if (cudaMemsetAsync(local_len, 0, sizeof(int32_t) * static_cast<size_t>(B), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// lsa_fetch_from_host_copy: the host-tier fetch through the copy engines.  The
// kept list is read on the host, and every kept chunk becomes one 2-D copy per
// K and V: 8 rows (its KV heads) of 16 KiB, from its pool slot (rows 16 KiB
// apart) to its column of the head-major compact buffer (rows buf_chunks *
// 16 KiB apart).  A run of at least 8 chunks that are adjacent both in the
// pool and in the buffer is copied per head instead (one 2-D copy of the run's
// tiles of that head), which takes fewer calls.  Nothing runs on the SMs.
// ---------------------------------------------------------------------------
namespace {
constexpr int kRunPerHead = 8;   // a run this long takes 8 per-head copies instead of 1 per chunk

cudaError_t copy_run(const uint8_t* pool, uint8_t* buf, int64_t slot0, int64_t c0, int r, int64_t buf_chunks,
                     cudaStream_t s) {
  const size_t tile = lsa::kTileBytes;                        // one (chunk, KV head) tile
  const size_t slot_bytes = tile * lsa::kNumKVHeads;
  if (r >= kRunPerHead) {
    for (int g = 0; g < lsa::kNumKVHeads; ++g) {
      const cudaError_t e = cudaMemcpy2DAsync(buf + (g * buf_chunks + c0) * tile, tile,
                                              pool + slot0 * slot_bytes + g * tile, slot_bytes, tile, r,
                                              cudaMemcpyHostToDevice, s);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  for (int i = 0; i < r; ++i) {
    const cudaError_t e = cudaMemcpy2DAsync(buf + (c0 + i) * tile, buf_chunks * tile,
                                            pool + (slot0 + i) * slot_bytes, tile, tile, lsa::kNumKVHeads,
                                            cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}
}  // namespace

extern "C" {

int lsa_debug_fail_fetch(int calls, int status) {
  if (calls < 0 || status >= 0 || status < LSA_ERR_NO_DEVICE) return LSA_ERR_INVALID_ARG;
  g_fetch_fail_status.store(status);
  g_fetch_fail_calls.store(calls);
  return LSA_OK;
}

int lsa_fetch_from_host_copy(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                             const int32_t* chunk_table_host, const int32_t* kept_host, const int32_t* cu_kept_host,
                             int B, int max_chunks, int max_kept, void* k_buf, void* v_buf, int64_t buf_chunks,
                             void* stream, void* done_event) {
  using namespace lsa;
  if (!host_k_pool || !host_v_pool || !kept_host || !cu_kept_host || !k_buf || !v_buf || B <= 0 ||
      max_chunks <= 0 || max_kept <= 0 || n_slots <= 0 || buf_chunks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(host_k_pool) || !aligned16(host_v_pool) || !aligned16(k_buf) || !aligned16(v_buf))
    return LSA_ERR_MISALIGNED;
  // The selection, read on the host: every count and slot is checked before
  // the first copy is issued.
  if (cu_kept_host[0] != 0 || cu_kept_host[B] > buf_chunks) return LSA_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    const int n = cu_kept_host[b + 1] - cu_kept_host[b];
    if (n < 0 || n > max_kept) return LSA_ERR_INVALID_ARG;
    for (int j = 0; j < n; ++j) {
      const int c = kept_host[static_cast<int64_t>(b) * max_kept + j];
      if (c < 0 || c >= max_chunks) return LSA_ERR_INVALID_ARG;
      const int64_t slot = chunk_table_host ? chunk_table_host[static_cast<int64_t>(b) * max_chunks + c]
                                            : static_cast<int64_t>(b) * max_chunks + c;
      if (slot < 0 || slot >= n_slots) return LSA_ERR_INVALID_ARG;
    }
  }
  if (const int inj = injected_fetch_failure()) return inj;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  cudaPointerAttributes ak, av;
  if (cudaPointerGetAttributes(&ak, host_k_pool) != cudaSuccess ||
      cudaPointerGetAttributes(&av, host_v_pool) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_NOT_PINNED;
  }
  if (ak.type != cudaMemoryTypeHost || av.type != cudaMemoryTypeHost) return LSA_ERR_NOT_PINNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint8_t* pk = static_cast<const uint8_t*>(host_k_pool);
  const uint8_t* pv = static_cast<const uint8_t*>(host_v_pool);
  uint8_t* bk = static_cast<uint8_t*>(k_buf);
  uint8_t* bv = static_cast<uint8_t*>(v_buf);
  for (int b = 0; b < B; ++b) {
    const int c0 = cu_kept_host[b], n = cu_kept_host[b + 1] - c0;
    const int32_t* kb = kept_host + static_cast<int64_t>(b) * max_kept;
    auto slot_of = [&](int j) -> int64_t {
      return chunk_table_host ? chunk_table_host[static_cast<int64_t>(b) * max_chunks + kb[j]]
                              : static_cast<int64_t>(b) * max_chunks + kb[j];
    };
    for (int j = 0; j < n;) {
      const int64_t s0 = slot_of(j);
      int r = 1;
      while (j + r < n && slot_of(j + r) == s0 + r) ++r;   // adjacent in the pool (and in the buffer)
      if (copy_run(pk, bk, s0, c0 + j, r, buf_chunks, s) != cudaSuccess ||
          copy_run(pv, bv, s0, c0 + j, r, buf_chunks, s) != cudaSuccess) {
        cudaGetLastError();
        return LSA_ERR_CUDA;
      }
      j += r;
    }
  }
  if (done_event && cudaEventRecord(static_cast<cudaEvent_t>(done_event), s) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

}  // extern "C"
