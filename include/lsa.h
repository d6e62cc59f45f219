/*
 * lsa.h -- C ABI of liblsa, the B200 (sm_100a) decode hot path of Lookahead
 * Sparse Attention (LSA).
 *
 * The method (pages on "FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long
 * Context via Lookahead Sparse Attention"): every tau = 64 decode steps a neural
 * memory indexer scores each 64-token chunk of the context (summary page,
 * sections 1 Introduction and 2.1 Architecture); only the chunks the coming
 * window needs are kept on the GPU (summary page, Abstract and 2.1), fetched
 * from a CPU tier when the cache lives there (summary page, 3 Experiments,
 * "Experimental Setup"; handbook page "DeepSeek-V4: Architecting for Ultra-Long
 * Contexts", "The Neural Memory Indexer", item 3); decode attention then runs
 * over the kept chunks only, as GQA with 64 query heads, 8 KV heads and head
 * dimension 128 (handbook page, "Grouped Query Attention (GQA) vs. Multi-Head
 * Attention (MHA)").
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers marked "device" are CUDA device (or managed) memory of the
 *    current device; "host" pointers are CPU memory.  The caller owns every
 *    buffer, stream and event.  The library never calls cudaMalloc; its only
 *    device memory is the static scratch array of
 *    lsa_sparse_decode_attn_noalloc (LSA_NOALLOC_SCRATCH_BYTES per GPU that
 *    loads the library) and the device status word.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every compute call only enqueues work on `stream` and returns.
 *  - Return value: LSA_OK (0) or a negative lsa_status.  Argument checks are
 *    done on the host, before anything is launched; a failed check launches
 *    nothing.  LSA_ERR_CUDA reports a launch error (cudaGetLastError).
 *  - Conditions only the device can see (a count or slot index out of range, a
 *    compact buffer too small, a bounded wait that ran out) set bits of a
 *    device status word (LSA_DEV_ERR_*) instead of trapping; the offending
 *    work item is skipped.  lsa_read_device_status() returns and clears it.
 *  - Shapes are fixed: 64 query heads, 8 KV heads, head dim 128, 64-token
 *    chunks, 16 indexer heads of dim 128.  bf16 is IEEE-style bfloat16 stored
 *    as 2 bytes; all bf16 arrays must be 16-byte aligned.
 *  - Layouts (row-major, last index fastest):
 *      KV pool                  : bf16 [slot][8 kv heads][64 tokens][128]
 *                                 (LSA_CHUNK_BYTES bytes per slot, per K or V)
 *      compact buffer           : bf16 [8 kv heads][buf_chunks][64 tokens][128]
 *                                 (head-major: the kept chunks of one KV head
 *                                 are contiguous, so the attention streams one
 *                                 contiguous range per (sequence, head))
 *      indexer keys             : bf16 [slot][128]
 *      indexer query            : bf16 [B][16][128]
 *      decode query             : bf16 [B][64][128]
 *      attention output         : fp32 [B][64][128]
 *      chunk table              : int32 [B][max_chunks], logical chunk -> slot;
 *                                 NULL means slot = b * max_chunks + c.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSA_NUM_Q_HEADS 64
#define LSA_NUM_KV_HEADS 8
#define LSA_HEAD_DIM 128
#define LSA_CHUNK_TOKENS 64
#define LSA_INDEX_HEADS 16
#define LSA_INDEX_DIM 128
/* Bytes of one chunk of K (or of V): 8 heads x 64 tokens x 128 dims x 2 B. */
#define LSA_CHUNK_BYTES 131072
/* Largest batch the attention and top-K calls accept. */
#define LSA_MAX_BATCH 4096

typedef enum {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = -1,       /* null pointer, negative size, bad value   */
  LSA_ERR_UNSUPPORTED_SHAPE = -2, /* size beyond what a kernel supports       */
  LSA_ERR_WORKSPACE = -3,         /* workspace missing or too small           */
  LSA_ERR_CUDA = -4,              /* CUDA runtime/launch error                */
  LSA_ERR_NOT_PINNED = -5,        /* host pool is not page-locked memory      */
  LSA_ERR_MISALIGNED = -6,        /* pointer not 16-byte aligned              */
  LSA_ERR_NO_DEVICE = -7          /* no usable sm_100 device                  */
} lsa_status;

/* Bits of the device status word. */
#define LSA_DEV_ERR_BAD_COUNT 1u   /* n_chunks / k_per_seq / cu_kept out of range */
#define LSA_DEV_ERR_BAD_SLOT 2u    /* chunk table entry outside [0, n_slots)     */
#define LSA_DEV_ERR_BAD_CHUNK 4u   /* kept chunk index outside [0, max_chunks)   */
#define LSA_DEV_ERR_CAPACITY 8u    /* compact buffer or kept row too small        */
#define LSA_DEV_ERR_TIMEOUT 16u    /* a bounded in-kernel wait ran out            */
#define LSA_DEV_ERR_WORKSPACE 32u  /* reserved: not raised by this version        */
#define LSA_DEV_ERR_INTERNAL 64u   /* launch-layout assumption violated (a bug)    */

/* Human-readable name of an lsa_status value. */
const char* lsa_status_string(int status);

/* ABI version of this library (major * 100 + minor). */
int lsa_version(void);

/*
 * Synchronises `stream`, stores the device status word of the current device
 * in *bits (0 = no device-side error since the last read) and clears it.
 */
int lsa_read_device_status(void* stream, unsigned int* bits);

/*
 * lsa_selftest_bounded_wait -- diagnostic of the failure detection every
 * kernel relies on (a device-side wait that cannot complete must not hang the
 * GPU).  Launches one warp that waits, through the same bounded-wait helpers
 * the kernels use, on an mbarrier nothing completes (mode 0) or until the
 * device int *flag is non-zero (mode 1; flag device memory).  After limit_us
 * microseconds (1 .. 2,000,000) a wait that has not completed sets
 * LSA_DEV_ERR_TIMEOUT in the device status word and the kernel returns; the
 * context stays usable.  Not part of the decode path.
 */
int lsa_selftest_bounded_wait(int mode, const int* flag, unsigned int limit_us, void* stream);

/*
 * lsa_index_score -- indexer scores of every chunk (the Neural Memory Indexer
 * of the summary page, 2.1 Architecture; sigmoid scoring per the review page,
 * "1. Key Terms & Definitions"):
 *
 *   scores[b*max_chunks + c] = sum_h w[h] * sigmoid(q_idx[b,h,:] . keys[slot(b,c),:] / sqrt(128))
 *
 * for c < n_chunks[b]; entries c >= n_chunks[b] are left untouched.
 *   q_idx      device bf16 [B][16][128]
 *   w          device fp32 [16]
 *   chunk_keys device bf16 [n_slots][128]
 *   chunk_table device int32 [B][max_chunks] or NULL (identity layout)
 *   n_chunks   device int32 [B], each in [0, max_chunks]
 *   scores     device fp32 [B][max_chunks]
 * Device errors: BAD_COUNT (n_chunks out of range: the sequence is skipped),
 * BAD_SLOT (that chunk's score is not written).
 */
int lsa_index_score(const void* q_idx, const float* w, const void* chunk_keys, int64_t n_slots,
                    const int32_t* chunk_table, const int32_t* n_chunks, int B, int max_chunks,
                    float* scores, void* stream);

/*
 * lsa_topk_chunks -- per-sequence selection: among chunks 0 .. n-2 keep the
 * K = k_per_seq[b] best by (score descending, chunk index ascending), then add
 * the latest chunk n-1.  kept[b*max_kept + j], j < n_kept[b], lists the kept
 * chunk indices in ascending order (the latest is last);
 * n_kept[b] = min(K, n-1) + 1 (0 when n == 0); cu_kept[0] = 0 and
 * cu_kept[b+1] = cu_kept[b] + n_kept[b] (offsets into the compact buffer, in
 * chunks).  Fixed-budget form of the recall step of the summary page, 2.1
 * Architecture.
 *   scores    device fp32 [B][max_chunks] (from lsa_index_score)
 *   n_chunks, k_per_seq  device int32 [B]
 *   kept      device int32 [B][max_kept]; n_kept device int32 [B];
 *   cu_kept   device int32 [B+1]
 * B <= LSA_MAX_BATCH.  Device errors: BAD_COUNT (negative K, n out of range:
 * the sequence keeps nothing), CAPACITY (n_kept would exceed max_kept: the
 * sequence keeps nothing).
 */
int lsa_topk_chunks(const float* scores, const int32_t* n_chunks, const int32_t* k_per_seq,
                    int B, int max_chunks, int max_kept, int32_t* kept, int32_t* n_kept,
                    int32_t* cu_kept, void* stream);

/*
 * lsa_topk_chunks_local -- lsa_topk_chunks with a recent-context window of
 * n_local >= 1 chunks (the non-offloadable recent context kept beside the
 * recalled chunks, summary page, 2.1 Architecture and 3 Experiments): the
 * latest min(n_local, n) chunks are always kept, and K are chosen among the
 * chunks before them.  n_kept[b] = min(K, n - L) + L with L = min(n_local, n).
 * lsa_topk_chunks is the n_local = 1 case.
 */
int lsa_topk_chunks_local(const float* scores, const int32_t* n_chunks, const int32_t* k_per_seq,
                          int n_local, int B, int max_chunks, int max_kept, int32_t* kept,
                          int32_t* n_kept, int32_t* cu_kept, void* stream);

/*
 * lsa_threshold_chunks -- the pages' own selection rule: sigmoid thresholding
 * in place of a fixed top-k (summary page, 2.1 Architecture; the 0.5
 * classification threshold of 2.4 Configuration).  Chunk c < n-1 is kept when
 * score_c / sum_h w[h] > threshold, i.e. when the weighted mean of the heads'
 * sigmoid probabilities exceeds it (fp32: the sum of w in head order, then
 * one division per chunk); the latest chunk n-1 is always kept.  Outputs as
 * lsa_topk_chunks: kept[b*max_kept + j] ascending with the latest last,
 * n_kept[b], cu_kept[B+1].  The kept count depends on the data, so size
 * max_kept for the worst case (max n) or accept CAPACITY.
 *   scores   device fp32 [B][max_chunks]; w device fp32 [16] (as for scoring)
 *   threshold  finite; 0.5 in the pages
 * Two kernels are launched (per-sequence compaction, then offsets); B <=
 * LSA_MAX_BATCH.  Device errors: BAD_COUNT (n out of range) and CAPACITY (the
 * kept set would exceed max_kept): that sequence keeps nothing.
 */
int lsa_threshold_chunks(const float* scores, const int32_t* n_chunks, const float* w, float threshold,
                         int B, int max_chunks, int max_kept, int32_t* kept, int32_t* n_kept,
                         int32_t* cu_kept, void* stream);

/*
 * lsa_threshold_chunks_capped -- lsa_threshold_chunks under a memory budget.
 * The point of the recall step is the cut in resident KV (summary page,
 * Abstract: the GPU KV cache shrinks by about 90%), while the threshold alone
 * can keep any number of chunks.  With cap (device int32 [B], each >= 0):
 * when more than cap[b] candidates pass the threshold, the cap[b] best passing
 * chunks are kept (score descending, chunk index ascending), plus the latest
 * chunk; otherwise the result is lsa_threshold_chunks'.  n_kept[b] is then at
 * most cap[b] + 1, so buffers sized for the budget suffice.  cap == NULL is
 * lsa_threshold_chunks.  Device errors as lsa_threshold_chunks, plus
 * BAD_COUNT for a negative cap (that sequence keeps nothing).
 */
int lsa_threshold_chunks_capped(const float* scores, const int32_t* n_chunks, const float* w, float threshold,
                                const int32_t* cap, int B, int max_chunks, int max_kept, int32_t* kept,
                                int32_t* n_kept, int32_t* cu_kept, void* stream);

/*
 * lsa_gather_chunks -- copy every kept chunk from the device KV pools into the
 * compact buffers, bit for bit: for i = cu_kept[b] + j,
 *   k_buf[g][i] = k_pool[slot(b, kept[b*max_kept + j])][g] for every KV head g, same for V.
 *   k_pool, v_pool device bf16 [n_slots][8][64][128]
 *   k_buf,  v_buf  device bf16 [8][buf_chunks][64][128]
 * Device errors: CAPACITY (cu_kept[B] > buf_chunks: nothing is copied),
 * BAD_CHUNK / BAD_SLOT (that chunk is not copied).
 */
int lsa_gather_chunks(const void* k_pool, const void* v_pool, int64_t n_slots,
                      const int32_t* chunk_table, const int32_t* kept, const int32_t* cu_kept,
                      int B, int max_chunks, int max_kept, void* k_buf, void* v_buf,
                      int64_t buf_chunks, void* stream);

/*
 * lsa_fetch_from_host -- the same copy as lsa_gather_chunks, but the pools
 * live in page-locked host memory (the CPU cold tier of the summary page,
 * 3 Experiments; prefetch over the host link, handbook page, "The Neural
 * Memory Indexer").  SM threads read the mapped host pages directly (no
 * host-side loop, no copy of `kept` to the host), so the call is fully
 * asynchronous and can run on a side stream while attention runs on another.
 *   host_k_pool, host_v_pool  page-locked host bf16 [n_slots][8][64][128]
 *                             (cudaHostAlloc / cudaHostRegister); anything
 *                             else returns LSA_ERR_NOT_PINNED.
 *   num_ctas   thread blocks used for the copy (<= 0: library default), kept
 *              small so the fetch leaves SMs to concurrent kernels.
 *   done_event optional cudaEvent_t (void*) recorded on `stream` after the copy.
 * Other arguments and device errors as lsa_gather_chunks.
 */
int lsa_fetch_from_host(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                        const int32_t* chunk_table, const int32_t* kept, const int32_t* cu_kept,
                        int B, int max_chunks, int max_kept, void* k_buf, void* v_buf,
                        int64_t buf_chunks, int num_ctas, void* stream, void* done_event);

/*
 * lsa_fetch_from_host_copy -- the same copy as lsa_fetch_from_host, through
 * the GPU's copy engines instead of SM threads (host-to-device prefetch over
 * the host link, handbook page, "The Neural Memory Indexer", item 3 and its
 * closing paragraph on PCIe/NVLink bandwidth).  The copies are planned on the
 * host, so the selection must be there: kept_host and cu_kept_host are host
 * int32 copies of kept [B][max_kept] and cu_kept [B+1] (for instance one small
 * device-to-host copy after lsa_topk_chunks), and chunk_table_host a host copy
 * of the chunk table or NULL.  Each kept chunk is one cudaMemcpy2DAsync per K
 * and V (its 8 head tiles of 16 KiB into the head-major compact buffer); a run
 * of 8 or more chunks adjacent in the pool takes 8 per-head copies instead.
 * The call returns once every copy is enqueued on `stream`; done_event, when
 * given, is recorded after them.  Unlike lsa_fetch_from_host it cannot be
 * captured in a CUDA graph with a selection that changes (the copies depend on
 * host data).  Host errors: LSA_ERR_INVALID_ARG for a count, chunk index or
 * slot out of range (checked before any copy), LSA_ERR_NOT_PINNED.
 */
int lsa_fetch_from_host_copy(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                             const int32_t* chunk_table_host, const int32_t* kept_host,
                             const int32_t* cu_kept_host, int B, int max_chunks, int max_kept, void* k_buf,
                             void* v_buf, int64_t buf_chunks, void* stream, void* done_event);

/*
 * lsa_debug_fail_fetch -- host-side fault injection for the host tier: the
 * next `calls` calls of lsa_fetch_from_host, lsa_fetch_from_host_delta and
 * lsa_fetch_from_host_copy return `status` (a negative lsa_status, normally
 * LSA_ERR_CUDA: a failed transfer) after their argument checks, without
 * touching the device.  calls = 0 disarms it.  Process-wide; for tests of the
 * caller's error handling.  Not part of the decode path.
 */
int lsa_debug_fail_fetch(int calls, int status);

/* Flags of lsa_sparse_decode_attn. */
/* The kernel that ran just before this call on `stream` did not write k_buf,
 * v_buf or cu_kept (true for every decode step of a window after the first):
 * the call may then stream K/V while that kernel is still finishing. */
#define LSA_ATTN_KV_UNCHANGED 1u

/*
 * lsa_fetch_from_host_delta -- lsa_fetch_from_host with residency across
 * windows (the eviction of non-recalled entries and the retention of recalled
 * ones, summary page, 2.1 Architecture): a kept chunk that was also kept in
 * the previous window of the same sequence is copied from that window's
 * compact buffer in device memory instead of over the host link.  The result
 * is identical to lsa_fetch_from_host.
 *   prev_kept, prev_cu_kept  device int32 [B][prev_max_kept], [B+1]: the
 *                            previous window's selection (ascending lists)
 *   prev_k_buf, prev_v_buf   device bf16 [8][prev_buf_chunks][64][128]: its
 *                            compact buffers (must not be k_buf / v_buf)
 *   reused_chunks            optional device int32 counter, incremented once
 *                            per chunk copied from the previous buffers
 * Other arguments and device errors as lsa_fetch_from_host.
 */
int lsa_fetch_from_host_delta(const void* host_k_pool, const void* host_v_pool, int64_t n_slots,
                              const int32_t* chunk_table, const int32_t* kept, const int32_t* cu_kept,
                              int B, int max_chunks, int max_kept, void* k_buf, void* v_buf,
                              int64_t buf_chunks, const int32_t* prev_kept,
                              const int32_t* prev_cu_kept, int prev_max_kept,
                              const void* prev_k_buf, const void* prev_v_buf,
                              int64_t prev_buf_chunks, int32_t* reused_chunks, int num_ctas,
                              void* stream, void* done_event);

/*
 * Bytes of workspace lsa_sparse_decode_attn needs for a batch of B sequences:
 * (B*8 + 1024) partial records of 1032 floats.  It needs no initialisation;
 * each call writes the records it reads.
 */
size_t lsa_attn_workspace_size(int B);

/*
 * lsa_sparse_decode_attn -- one decode step of GQA attention over the kept
 * chunks (handbook page, "Grouped Query Attention (GQA) vs. Multi-Head
 * Attention (MHA)": softmax(q K^T / sqrt(d_k)) V, every 8 consecutive query
 * heads sharing one KV head).  For sequence b, query head h and KV head
 * g = h / 8, the keys and values are the 64 * (cu_kept[b+1] - cu_kept[b])
 * tokens of head g in k_buf / v_buf chunks cu_kept[b] .. cu_kept[b+1]-1:
 *
 *   out[b,h,:] = sum_j softmax_j(scale * q[b,h,:] . k_j) v_j    (fp32)
 *
 * A sequence with no kept chunk gets zeros.  The work is split over all SMs
 * along the kept tokens (split-K flash decoding) and the partial results are
 * merged with their log-sum-exp weights in a fixed order, so repeated calls
 * are bit-identical.  The call enqueues two kernels on `stream`: the
 * attention grid and the merge of the pairs it split, a programmatic
 * dependent of it.
 *   q            device bf16 [B][64][128]
 *   k_buf, v_buf device bf16 [8][buf_chunks][64][128]
 *   cu_kept      device int32 [B+1]
 *   softmax_scale  usually 1/sqrt(128)
 *   out          device fp32 [B][64][128]
 *   workspace    device, >= lsa_attn_workspace_size(B) bytes; calls that
 *                may overlap on the GPU need workspaces of their own.
 *   flags        0 or LSA_ATTN_KV_UNCHANGED.  The attention grid is launched
 *                as a programmatic dependent of the preceding kernel on
 *                `stream` (its start overlaps that kernel's tail); it waits
 *                for that kernel before reading q or cu_kept (without the
 *                flag) and before writing out or the workspace.  The merge
 *                grid waits for the attention grid before it reads the
 *                workspace.
 * B <= LSA_MAX_BATCH.  Device errors: CAPACITY (cu_kept[B] > buf_chunks or
 * cu_kept decreasing: nothing is computed), TIMEOUT.
 */
int lsa_sparse_decode_attn(const void* q, const void* k_buf, const void* v_buf,
                           int64_t buf_chunks, const int32_t* cu_kept, int B,
                           float softmax_scale, float* out, void* workspace,
                           size_t workspace_bytes, unsigned int flags, void* stream);

/*
 * lsa_sparse_decode_attn_noalloc -- lsa_sparse_decode_attn without a
 * caller-provided workspace, for callers that cannot allocate device memory:
 * programs with no device allocator of their own, plug-ins inside a framework
 * that owns all device memory and forbids cudaMalloc after start-up, and
 * latency-critical loops that must not call cudaMalloc (it can synchronise the
 * device).  The pages have no counterpart of this call; it is a convenience of
 * this library.
 *
 * The split-K scratch lives in a fixed array inside the library
 * (LSA_NOALLOC_SCRATCH_BYTES of device memory, held by every GPU that loads
 * the library until the process exits).  The caller still owns and passes q,
 * the compact buffers, cu_kept and out; arguments, results and device errors
 * are those of lsa_sparse_decode_attn, and so is the launch (the same grid,
 * the same merge kernel, a programmatic dependent of the preceding kernel
 * without LSA_ATTN_KV_UNCHANGED), so the output is bit-identical to
 * lsa_sparse_decode_attn's on the same inputs.  Limits: B <= LSA_NOALLOC_MAX_BATCH
 * and a device of at most 512 SMs (one CTA per SM), otherwise
 * LSA_ERR_UNSUPPORTED_SHAPE.  The call allocates nothing (no cudaMalloc, no
 * cudaFree).  Its first call on a device looks up the array's device address
 * and sets the kernel's shared-memory limit; make that first call before any
 * stream capture.  Every call on a device uses the same array: calls whose
 * work may overlap on the GPU (other streams, other host threads) race and
 * must be serialised by the caller.
 */
#define LSA_NOALLOC_MAX_BATCH 32
#define LSA_NOALLOC_MAX_CTAS 512
/* (32*8 + 512) partial records of 1032 floats. */
#define LSA_NOALLOC_SCRATCH_BYTES 3170304
int lsa_sparse_decode_attn_noalloc(const void* q, const void* k_buf, const void* v_buf,
                                   int64_t buf_chunks, const int32_t* cu_kept, int B,
                                   float softmax_scale, float* out, void* stream);

/*
 * Tokens decoded inside the current window (the local / decoded window the
 * summary page keeps beside the recalled chunks, 3 Experiments "Experimental
 * Setup"; it makes each decode step causal).  Each sequence has one local
 * chunk, k_local / v_local device bf16 [B][8][64][128], holding the tokens
 * decoded since the window started, and a count local_len device int32 [B]
 * (0 at the start of a window; the caller resets it).
 *
 * The local chunks must hold finite values in every row (zero them once when
 * they are allocated): rows at or past local_len[b] are masked out of the
 * softmax, but still enter the P.V product with weight 0, where a NaN or an
 * infinity would poison the output.
 *
 * lsa_append_token -- writes the new token of every sequence (k_new, v_new
 * device bf16 [B][8][128]) at position local_len[b] of its local chunk and
 * increments local_len[b].  Device error CAPACITY (the local chunk already
 * holds 64 tokens: nothing is written for that sequence).
 */
int lsa_append_token(const void* k_new, const void* v_new, void* k_local, void* v_local,
                     int32_t* local_len, int B, void* stream);

/*
 * lsa_reset_local -- empties every sequence's local chunk at the start of a
 * window: local_len (device int32 [B]) is set to 0, stream-ordered (a memset
 * on `stream`, capturable in a CUDA graph; no kernel).  The local K/V rows
 * are left as they are; the attention reads only the first local_len[b].
 */
int lsa_reset_local(int32_t* local_len, int B, void* stream);

/*
 * lsa_sparse_decode_attn_local -- lsa_sparse_decode_attn over the kept chunks
 * and, after them, the first local_len[b] tokens of each sequence's local
 * chunk (every 8 query heads on their KV head, as for the kept tokens).  A
 * sequence with no kept chunk and local_len 0 gets zeros.  The local chunk is
 * read after the preceding kernel has finished (it is normally written by
 * lsa_append_token just before), also with LSA_ATTN_KV_UNCHANGED, which then
 * applies to k_buf, v_buf and cu_kept only.  local_len outside [0, 64] sets
 * BAD_COUNT and is clamped.  Other arguments as lsa_sparse_decode_attn.
 */
int lsa_sparse_decode_attn_local(const void* q, const void* k_buf, const void* v_buf,
                                 int64_t buf_chunks, const int32_t* cu_kept, int B,
                                 float softmax_scale, const void* k_local, const void* v_local,
                                 const int32_t* local_len, float* out, void* workspace,
                                 size_t workspace_bytes, unsigned int flags, void* stream);

/*
 * lsa_sparse_decode_attn_selected -- the decode attention of the token-level
 * fine stage, read in place: for each sequence, the selected positions
 * sel[b*max_sel + j], j < cu_sel[b+1] - cu_sel[b] (from lsa_topk_tokens;
 * every count a multiple of 64), position p being token p % 64 of compact
 * chunk cu_kept[b] + p / 64.  Equal to lsa_gather_tokens followed by
 * lsa_sparse_decode_attn over the packed units, bit for bit, without the
 * packed copy: the kernel copies the selected rows of k_buf / v_buf
 * (bf16 [8][buf_chunks][64][128]) straight into its pipeline.
 *   sel device int32 [B][max_sel], max_sel a multiple of 64;
 *   cu_sel device int32 [B+1]; cu_kept device int32 [B+1]
 * LSA_ATTN_KV_UNCHANGED additionally promises that sel and cu_sel were not
 * written by the preceding kernel.  Device errors: CAPACITY (cu_sel
 * inconsistent: nothing is computed), BAD_CHUNK (a position outside the
 * sequence's recalled tokens: that row is read as zeros).  Workspace as for
 * lsa_sparse_decode_attn.
 */
int lsa_sparse_decode_attn_selected(const void* q, const void* k_buf, const void* v_buf,
                                    int64_t buf_chunks, const int32_t* cu_kept, const int32_t* sel,
                                    const int32_t* cu_sel, int max_sel, int B, float softmax_scale,
                                    float* out, void* workspace, size_t workspace_bytes,
                                    unsigned int flags, void* stream);

/*
 * lsa_sparse_decode_attn_append -- one causal decode step with the append
 * fused into the attention grid: lsa_append_token followed by
 * lsa_sparse_decode_attn_local in one launch (plus the merge of split pairs
 * that every attention call enqueues).  With
 * n = local_len_in[b], the step attends the kept chunks, tokens 0 .. n-1 of
 * the local chunk and this step's own token (k_new, v_new device bf16
 * [B][8][128]) as token n; it also writes that token to row n of the local
 * chunk and sets local_len_out[b] = n + 1.  local_len_in is only read and
 * local_len_out only written (they must be different arrays; a decode loop
 * alternates the two), so no reader of this launch sees the count change.
 * n == 64 (the local chunk is full) sets CAPACITY: the token is neither
 * attended nor stored, and local_len_out[b] = 64.  Other arguments, the
 * finiteness rule for the local chunks and LSA_ATTN_KV_UNCHANGED as for
 * lsa_sparse_decode_attn_local.
 */
int lsa_sparse_decode_attn_append(const void* q, const void* k_buf, const void* v_buf,
                                  int64_t buf_chunks, const int32_t* cu_kept, int B,
                                  float softmax_scale, const void* k_new, const void* v_new,
                                  void* k_local, void* v_local, const int32_t* local_len_in,
                                  int32_t* local_len_out, float* out, void* workspace,
                                  size_t workspace_bytes, unsigned int flags, void* stream);

/*
 * Token-level fine stage.  Inside the recalled chunks, native token-level
 * scoring keeps a fine-grained top-k of entries (summary page, 2.1
 * Architecture; k = 2048 tokens for the DSA lightning indexer on the search
 * page "lightning indexer").  Every decode step:
 *   lsa_token_score   -> one score per token of the recalled chunks,
 *   lsa_topk_tokens   -> the k best token positions
 *                        (or both in one call: lsa_select_tokens),
 *   lsa_sparse_decode_attn_selected -> attention over those tokens, whose
 *                        rows it reads in place from the compact buffer.
 * A causal step (lsa_sparse_decode_attn_append, which attends whole units)
 * first packs the selected tokens into dense 64-token units with
 * lsa_gather_tokens and attends the units (buf = k_out / v_out,
 * cu_kept = cu_units).
 * Token position p of sequence b is token p % 64 of its recalled chunk
 * p / 64 (kept[b*max_kept + p/64]); positions follow the context order.  All
 * KV heads attend the same selected tokens (one score per token).
 *
 * lsa_token_score -- for p < 64 * n_kept[b]:
 *   scores[b*64*max_kept + p] = sum_h w[h] * sigmoid(q_idx[b,h,:] . tok_key(p) / sqrt(128)),
 *   tok_key(p) = token_keys[slot(b, kept[b*max_kept + p/64])][p % 64][:]
 * (the indexer's own form at token granularity), and n_tokens[b] =
 * 64 * n_kept[b].
 *   q_idx      device bf16 [B][16][128], the current decode step's indexer query
 *   w          device fp32 [16]
 *   token_keys device bf16 [n_slots][64][128], per-token indexer keys by slot
 *   chunk_table, kept, n_kept as for lsa_gather_chunks / lsa_topk_chunks
 *   scores     device fp32 [B][64 * max_kept]; n_tokens device int32 [B]
 * Device errors: BAD_COUNT (n_kept out of range: skipped, n_tokens 0),
 * BAD_CHUNK / BAD_SLOT (that token's score is not written).
 */
int lsa_token_score(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                    const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B,
                    int max_chunks, int max_kept, float* scores, int32_t* n_tokens, void* stream);

/*
 * lsa_topk_tokens -- the k best token positions of each sequence by (score
 * descending, position ascending), every position when there are at most k;
 * sel[b*max_sel + j], j < n_sel[b] = min(k, n_tokens[b]), ascending;
 * cu_sel[0] = 0, cu_sel[b+1] = cu_sel[b] + n_sel[b].  Same key as
 * lsa_topk_chunks (-0 equals +0, NaN last).
 *   scores   device fp32 [B][max_tokens] (max_tokens = 64 * max_kept of lsa_token_score)
 *   n_tokens device int32 [B]
 *   k        > 0; a multiple of 64 when the result feeds lsa_gather_tokens
 *   sel device int32 [B][max_sel]; n_sel device int32 [B]; cu_sel device int32 [B+1]
 * Device errors: BAD_COUNT, CAPACITY (n_sel would exceed max_sel): that
 * sequence selects nothing.
 */
int lsa_topk_tokens(const float* scores, const int32_t* n_tokens, int k, int B, int max_tokens,
                    int max_sel, int32_t* sel, int32_t* n_sel, int32_t* cu_sel, void* stream);

/*
 * lsa_select_tokens -- lsa_token_score followed by lsa_topk_tokens in one
 * call, with the same outputs bit for bit (scores, n_tokens, sel, n_sel,
 * cu_sel; arguments as those two calls, k and max_sel as for lsa_topk_tokens).
 * The scorer also counts each sequence's scores in 4096 bins of equal width
 * over [0, sum_h w[h]), so the selection knows the bin of the k-th best score
 * before it reads a score again: a cluster of 8 CTAs per sequence reads every
 * score once, keeps the tokens above that bin and ranks the few inside it
 * exactly.  Inputs where that does not pay (many tokens in one bin, ties
 * everywhere, more than 131072 tokens in a sequence) take the exact radix
 * select of lsa_topk_tokens inside the same launch.  The counts take the
 * scorer shared memory, which pays only when its grid (B * max_kept / 2 CTAs)
 * fits in one wave of 4 CTAs per SM; larger batches run lsa_token_score and
 * lsa_topk_tokens instead (the workspace is then not touched).  Two kernels
 * either way, both programmatic dependents of their predecessor.
 *   workspace  device, >= lsa_select_tokens_workspace_size(B) bytes (64 KiB
 *              per sequence: 4 copies of the counts, so fewer of the scorer's
 *              atomic adds meet on one address), 16-byte aligned, zero before the first call
 *              (zero it once when it is allocated): the bin counts; every
 *              call leaves it zero again.  Calls that may overlap on the GPU
 *              need workspaces of their own.
 *   flags      0 or LSA_TOKENS_UNCHANGED: nothing on `stream` has written
 *              token_keys, chunk_table, kept, n_kept or w since the previous
 *              lsa_select_tokens call on it (true for every decode step of a
 *              window after the first).  The kernels of this call start while
 *              the preceding kernel is still finishing; with the flag the
 *              scorer looks up and loads its key rows, and the selection works
 *              out its counts and offsets, before waiting for it.  q_idx is
 *              read and every output written only after it.  Without the flag
 *              both wait first.
 * Device errors as lsa_token_score and lsa_topk_tokens.
 */
#define LSA_TOKENS_UNCHANGED 1u
size_t lsa_select_tokens_workspace_size(int B);
int lsa_select_tokens(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                      const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B,
                      int max_chunks, int max_kept, int k, float* scores, int32_t* n_tokens, int32_t* sel,
                      int32_t* n_sel, int32_t* cu_sel, int max_sel, void* workspace, size_t workspace_bytes,
                      unsigned int flags, void* stream);

/*
 * lsa_gather_tokens -- pack the selected tokens into dense units, bit for bit:
 * for j < n_sel[b], with unit u = cu_sel[b]/64 + j/64 and row r = j % 64,
 *   k_out[g][u][r][:] = k_buf[g][cu_kept[b] + p/64][p % 64][:],  p = sel[b*max_sel + j],
 * for every KV head g, same for V; cu_units[b] = cu_sel[b] / 64.
 *   k_buf, v_buf  device bf16 [8][buf_chunks][64][128] (the compact buffer)
 *   cu_kept       device int32 [B+1]
 *   sel, cu_sel   from lsa_topk_tokens; max_sel a multiple of 64
 *   k_out, v_out  device bf16 [8][out_chunks][64][128] (the compact buffer's layout)
 *   cu_units      device int32 [B+1]
 * Every count must be a multiple of 64 (k a multiple of 64 guarantees it).
 * Device errors: BAD_COUNT (a count that is not, or bad cu_kept: skipped),
 * CAPACITY (a unit beyond out_chunks: skipped), BAD_CHUNK (a position outside
 * the sequence's recalled tokens: that row is written as zeros).
 */
int lsa_gather_tokens(const void* k_buf, const void* v_buf, int64_t buf_chunks, const int32_t* cu_kept,
                      const int32_t* sel, const int32_t* cu_sel, int B, int max_sel, void* k_out,
                      void* v_out, int64_t out_chunks, int32_t* cu_units, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
