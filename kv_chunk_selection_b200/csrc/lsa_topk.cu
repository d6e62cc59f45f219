// lsa_topk_chunks: per-sequence top-K of the indexer scores plus the latest chunk.
//
// Method: the recalled set is the fixed-budget form of the indexer's selection
// (summary page "FlashMemory-DeepSeek-V4 ...", 2.1 Architecture): the K best
// chunks among all but the latest, ordered by score descending then chunk
// index ascending, plus the latest chunk, listed in ascending order.
//
// B200 design: one 1024-thread CTA per sequence runs an exact radix select on
// a 32-bit key that orders scores descending (the float bits mapped to an
// order-preserving unsigned and complemented); the chunk index breaks ties
// among equal keys.  Each thread owns a contiguous run of candidates and keeps
// their keys in registers (up to 16 per thread, N <= 16384; beyond that the
// cluster kernel below takes over, and beyond 131072 this kernel re-reads the
// scores).  The bits that every key shares (found from a block-wide min
// and max) need no pass, so scores in a narrow range take 3 or fewer 8-bit
// digit passes, each a shared-memory histogram and a 256-bin scan.  The kept
// set is then written in index order with two block-wide prefix scans, so the
// output is ascending without a sort.
//
// Larger candidate sets (the token-level fine stage: 16K to 128K tokens per
// sequence) take a cluster of 8 CTAs per sequence instead: 8192 threads keep
// up to 16 keys each in registers; every radix pass builds one shared-memory
// histogram per CTA, and each CTA sums the 8 histograms through distributed
// shared memory, so all 8 reach the same boundary without touching global
// memory; a last exchange of per-CTA (less, equal) counts gives each CTA its
// output offset and its share of the boundary ties in index order.
#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

namespace lsa {
namespace topk {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

// Smaller key <=> larger score (IEEE order-preserving map, then complement).
// -0.0 and +0.0 get the same key (they are equal scores, so the chunk index
// decides), and NaN sorts after every number.
__device__ __forceinline__ uint32_t desc_key(float s) {
  if (s != s) return 0xffffffffu;
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0) u = 0;
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ~ord;
}

// Kept count of one sequence (K chosen among the chunks before the latest
// n_local, plus those n_local), or 0 with *err set when its counts are invalid.
__device__ __forceinline__ int kept_count(int n, int k, int n_local, int max_chunks, int max_kept, unsigned* err) {
  if (n < 0 || n > max_chunks || k < 0) {
    *err |= LSA_DEV_ERR_BAD_COUNT;
    return 0;
  }
  if (n == 0) return 0;
  const int n_rec = min(n_local, n);
  const int nk = min(k, n - n_rec) + n_rec;
  if (nk > max_kept) {
    *err |= LSA_DEV_ERR_CAPACITY;
    return 0;
  }
  return nk;
}

// Exclusive block-wide prefix sum of one int per thread; *total gets the sum.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int ws = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += y;
    }
    warp_sums[lane] = ws;  // inclusive
  }
  __syncthreads();
  const int excl = x - v + (warp > 0 ? warp_sums[warp - 1] : 0);
  if (total) *total = warp_sums[kWarps - 1];
  __syncthreads();
  return excl;
}

constexpr int kMaxPerThread = 16;   // candidates kept in registers per thread (N <= 16384)

// Key of candidate i: the descending key of its score.
struct ScoreKey {
  const float* sc;
  __device__ __forceinline__ uint32_t operator()(int i) const { return desc_key(ld_dep(sc + i)); }
};

// Selects the kc smallest keys among candidates 0..cand-1 (kc < cand) and
// writes their indices in ascending order to out[0..kc).  Thread t owns the
// contiguous candidates [t*per, (t+1)*per); with kCached their keys live in
// registers for all passes, otherwise they are re-read through key_at.
template <bool kCached, class KeyAt>
__device__ void select_and_write(KeyAt key_at, int cand, int kc, int per, int32_t* __restrict__ out,
                                 int* hist, int* warp_sums, int* sel) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int lo = min(cand, tid * per), hi = min(cand, lo + per);
  uint32_t kr[kCached ? kMaxPerThread : 1];
  if (kCached) {
#pragma unroll
    for (int e = 0; e < kMaxPerThread; ++e) kr[e] = (lo + e < hi) ? key_at(lo + e) : 0u;
  }
  auto key_of = [&](int e) -> uint32_t { return kCached ? kr[e] : key_at(lo + e); };
  const int n_own = hi - lo;

  // Bits shared by every candidate key need no pass: start below the highest
  // bit where the smallest and largest key differ.
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  if (kCached) {
#pragma unroll
    for (int e = 0; e < kMaxPerThread; ++e)
      if (e < n_own) { kmin = min(kmin, kr[e]); kmax = max(kmax, kr[e]); }
  } else {
    for (int e = 0; e < n_own; ++e) { const uint32_t k = key_of(e); kmin = min(kmin, k); kmax = max(kmax, k); }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
  }
  if (lane == 0) { warp_sums[tid >> 5] = static_cast<int>(kmin); hist[tid >> 5] = static_cast<int>(kmax); }
  __syncthreads();
  if (tid < 32) {
    uint32_t a = static_cast<uint32_t>(warp_sums[tid]), z = static_cast<uint32_t>(hist[tid]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, off));
      z = max(z, __shfl_xor_sync(0xffffffffu, z, off));
    }
    if (tid == 0) { sel[0] = static_cast<int>(a); sel[1] = static_cast<int>(z); }
  }
  __syncthreads();
  kmin = static_cast<uint32_t>(sel[0]);
  kmax = static_cast<uint32_t>(sel[1]);
  __syncthreads();
  const uint32_t diff = kmin ^ kmax;
  int hi_bit = diff ? 31 - __clz(diff) : -1;
  uint32_t mask = hi_bit >= 31 ? 0u : (0xffffffffu << (hi_bit + 1));
  uint32_t prefix = kmin & mask;
  int krem = kc;

  // ---- radix select of the kc-th smallest key over the remaining bits ---------
  while (hi_bit >= 0) {
    const int width = min(8, hi_bit + 1);
    const int shift = hi_bit - width + 1;
    const uint32_t dmask = (1u << width) - 1u;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    if (kCached) {
#pragma unroll
      for (int e = 0; e < kMaxPerThread; ++e)
        if (e < n_own && (kr[e] & mask) == prefix) atomicAdd(&hist[(kr[e] >> shift) & dmask], 1);
    } else {
      for (int e = 0; e < n_own; ++e) {
        const uint32_t k = key_of(e);
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & dmask], 1);
      }
    }
    __syncthreads();
    // Inclusive prefix over the bins (warps 0..7), then locate the bin that
    // holds the krem-th smallest remaining key.
    int count = 0, incl = 0;
    if (tid < 256) {
      count = hist[tid];
      incl = count;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) warp_sums[tid >> 5] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      for (int w = 0; w < (tid >> 5); ++w) incl += warp_sums[w];
      const int excl = incl - count;
      if (excl < krem && incl >= krem) {
        sel[0] = tid;
        sel[1] = krem - excl;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel[0]) << shift;
    mask |= dmask << shift;
    krem = sel[1];
    hi_bit -= width;
    __syncthreads();
  }
  const uint32_t boundary = prefix;  // the kc-th smallest key; take krem of its ties
  griddep_launch_dependents();   // the rest is the output pass

  // ---- write the kept candidates in ascending index order ---------------------
  int n_eq = 0;
  if (kCached) {
#pragma unroll
    for (int e = 0; e < kMaxPerThread; ++e) n_eq += (e < n_own && kr[e] == boundary);
  } else {
    for (int e = 0; e < n_own; ++e) n_eq += (key_of(e) == boundary);
  }
  const int eq_before = block_exclusive_scan(n_eq, warp_sums, nullptr);
  int n_sel = 0, eq_seen = eq_before;
  bool take[kCached ? kMaxPerThread : 1];
  if (kCached) {
#pragma unroll
    for (int e = 0; e < kMaxPerThread; ++e) {
      bool t = false;
      if (e < n_own) {
        if (kr[e] < boundary) t = true;
        else if (kr[e] == boundary) t = (eq_seen++ < krem);
      }
      take[e] = t;
      n_sel += t;
    }
  } else {
    for (int e = 0; e < n_own; ++e) {
      const uint32_t k = key_of(e);
      if (k < boundary) ++n_sel;
      else if (k == boundary) n_sel += (eq_seen++ < krem);
    }
  }
  int pos = block_exclusive_scan(n_sel, warp_sums, nullptr);
  if (kCached) {
#pragma unroll
    for (int e = 0; e < kMaxPerThread; ++e)
      if (take[e]) out[pos++] = lo + e;
  } else {
    eq_seen = eq_before;
    for (int e = 0; e < n_own; ++e) {
      const uint32_t k = key_of(e);
      bool t = k < boundary;
      if (k == boundary) t = (eq_seen++ < krem);
      if (t) out[pos++] = lo + e;
    }
  }
}

__global__ void __launch_bounds__(kThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ n_chunks,
            const int32_t* __restrict__ k_per_seq, int k_all, int n_local, int B, int max_chunks, int max_kept,
            int32_t* __restrict__ kept, int32_t* __restrict__ n_kept, int32_t* __restrict__ cu_kept,
            unsigned* status) {
  // k_per_seq == nullptr: every sequence has budget k_all.
  __shared__ int hist[256];
  __shared__ int warp_sums[32];
  __shared__ int sel[2];
  griddep_wait();   // the previous kernel on the stream has finished
  const int b = blockIdx.x;
  const int tid = threadIdx.x;

  // cu_kept[b+1] = sum of the kept counts of sequences 0..b.
  int part = 0;
  unsigned dummy = 0;
  for (int bb = tid; bb <= b; bb += kThreads)
    part += kept_count(ld_dep(n_chunks + bb), k_per_seq ? ld_dep(k_per_seq + bb) : k_all, n_local, max_chunks,
                       max_kept, &dummy);
  int tot = 0;
  block_exclusive_scan(part, warp_sums, &tot);
  unsigned err = 0;
  const int n = ld_dep(n_chunks + b);
  const int nk = kept_count(n, k_per_seq ? ld_dep(k_per_seq + b) : k_all, n_local, max_chunks, max_kept, &err);
  if (tid == 0) {
    cu_kept[b + 1] = tot;
    if (b == 0) cu_kept[0] = 0;
    n_kept[b] = nk;
    if (err) set_status(status, err);
  }
  if (nk == 0) return;
  int32_t* out = kept + static_cast<int64_t>(b) * max_kept;
  const int n_rec = min(n_local, n);   // the recent chunks, always kept and last
  const int cand = n - n_rec;
  const int kc = nk - n_rec;
  if (kc == cand) {  // keep every chunk
    for (int c = tid; c < n; c += kThreads) out[c] = c;
    return;
  }
  for (int i = tid; i < n_rec; i += kThreads) out[kc + i] = cand + i;
  if (kc == 0) return;
  const ScoreKey key{scores + static_cast<int64_t>(b) * max_chunks};
  const int per = (cand + kThreads - 1) / kThreads;
  if (per <= kMaxPerThread)
    select_and_write<true>(key, cand, kc, per, out, hist, warp_sums, sel);
  else
    select_and_write<false>(key, cand, kc, per, out, hist, warp_sums, sel);
}

// ---- cluster variant ------------------------------------------------------
constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = kClusterCtas * kThreads;
constexpr int kClusterMaxCand = kClusterThreads * kMaxPerThread;   // 131072
// Candidate counts above this go to the cluster kernel (one CTA re-reads the
// scores every pass beyond it).
constexpr int kClusterMinCand = kThreads * kMaxPerThread;          // 16384

// The cluster's exact radix select: the kc smallest keys of candidates
// 0 .. cand-1 (kc < cand, cand <= 8192 * kPer) of the scores at sc, written to
// out[0 .. kc) in ascending index order.  Every thread of every CTA of the
// cluster calls it; rank r's threads own the contiguous candidates
// [gtid * per, (gtid + 1) * per), gtid = r * 1024 + thread, with their keys
// in registers.
template <int kPer>
__device__ void cluster_select_and_write(const float* __restrict__ sc, int cand, int kc, int32_t* __restrict__ out) {
  // Two histograms, alternating between passes: pass p clears the one that
  // pass p-1's remote reads used two passes back, and the cluster barrier of
  // pass p-1 orders those reads before this clear, so a pass needs one
  // cluster barrier instead of two.
  __shared__ int hist[2][256];
  __shared__ int warp_sums[32];
  __shared__ uint32_t warp_max[32];
  __shared__ int sel[2];
  __shared__ uint32_t xmm[2 * kClusterCtas];   // [rank] min key, [8 + rank] max key, pushed by each rank
  __shared__ int xcnt[2 * kClusterCtas];       // [rank] keys below the boundary, [8 + rank] keys equal to it
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int gtid = static_cast<int>(rank) * kThreads + tid;
  const int per = (cand + kClusterThreads - 1) / kClusterThreads;
  // Announce this CTA to the cluster, load the keys, and wait for every CTA
  // before the first remote store.
  cluster_arrive_relaxed();
  const int lo = min(cand, gtid * per), hi = min(cand, lo + per);
  const int n_own = hi - lo;
  uint32_t kr[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) kr[e] = (e < n_own) ? desc_key(ld_dep(sc + lo + e)) : 0u;

  // ---- smallest and largest key of the whole cluster ------------------------
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int e = 0; e < kPer; ++e)
    if (e < n_own) { kmin = min(kmin, kr[e]); kmax = max(kmax, kr[e]); }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
  }
  if (lane == 0) { warp_sums[tid >> 5] = static_cast<int>(kmin); warp_max[tid >> 5] = kmax; }
  __syncthreads();
  uint32_t cta_min = 0u, cta_max = 0u;   // valid in warp 0 (every lane, after the xor reduction)
  if (tid < 32) {
    cta_min = static_cast<uint32_t>(warp_sums[tid]);
    cta_max = warp_max[tid];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      cta_min = min(cta_min, __shfl_xor_sync(0xffffffffu, cta_min, off));
      cta_max = max(cta_max, __shfl_xor_sync(0xffffffffu, cta_max, off));
    }
  }
  cluster_wait();        // every CTA of the cluster is running
  if (tid < kClusterCtas) {   // warp 0 pushes this CTA's extremes to every rank
    st_cluster_u32(cluster_map(&xmm[rank], tid), cta_min);
    st_cluster_u32(cluster_map(&xmm[kClusterCtas + rank], tid), cta_max);
  }
  cluster_sync_all();
  kmin = 0xffffffffu;
  kmax = 0u;
#pragma unroll
  for (int r = 0; r < kClusterCtas; ++r) {
    kmin = min(kmin, xmm[r]);
    kmax = max(kmax, xmm[kClusterCtas + r]);
  }
  const uint32_t diff = kmin ^ kmax;
  int hi_bit = diff ? 31 - __clz(diff) : -1;
  uint32_t mask = hi_bit >= 31 ? 0u : (0xffffffffu << (hi_bit + 1));
  uint32_t prefix = kmin & mask;
  int krem = kc;

  // ---- radix select over the cluster ------------------------------------------
  // Buffer 0 is cleared here; buffer (p + 1) & 1 right after pass p's cluster
  // barrier, which orders every remote read of it (made in pass p - 1) first.
  if (tid < 256) hist[0][tid] = 0;
  __syncthreads();
  int pass = 0;
  while (hi_bit >= 0) {
    const int width = min(8, hi_bit + 1);
    const int shift = hi_bit - width + 1;
    const uint32_t dmask = (1u << width) - 1u;
    int* h = hist[pass & 1];
#pragma unroll
    for (int e = 0; e < kPer; ++e)
      if (e < n_own && (kr[e] & mask) == prefix) atomicAdd(&h[(kr[e] >> shift) & dmask], 1);
    cluster_sync_all();   // every rank's histogram of this pass is complete
    if (tid < 256) hist[(pass + 1) & 1][tid] = 0;   // published by the block barriers below
    int count = 0, incl = 0;
    if (tid < 256) {
#pragma unroll
      for (int r = 0; r < kClusterCtas; ++r) count += static_cast<int>(ld_cluster_u32(cluster_map(&h[tid], r)));
      incl = count;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) warp_sums[tid >> 5] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      for (int w = 0; w < (tid >> 5); ++w) incl += warp_sums[w];
      const int excl = incl - count;
      if (excl < krem && incl >= krem) {
        sel[0] = tid;
        sel[1] = krem - excl;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel[0]) << shift;
    mask |= dmask << shift;
    krem = sel[1];
    hi_bit -= width;
    ++pass;
    __syncthreads();   // sel is rewritten by the next pass
  }
  const uint32_t boundary = prefix;   // the kc-th smallest key; krem of its ties are taken
  griddep_launch_dependents();   // the rest is the count exchange and the output pass

  // ---- offsets of this CTA: keys below the boundary and ties of lower ranks ---
  int n_less = 0, n_eq = 0;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    n_less += (e < n_own && kr[e] < boundary);
    n_eq += (e < n_own && kr[e] == boundary);
  }
  // one block scan for both counts: equal keys in the high half, smaller ones
  // in the low half (at most 16 per thread and 8192 per CTA each)
  int cta_both = 0;
  const int both_before = block_exclusive_scan((n_eq << 16) | n_less, warp_sums, &cta_both);
  const int eq_before = both_before >> 16;
  const int cta_eq = cta_both >> 16, cta_less = cta_both & 0xffff;
  if (tid < kClusterCtas) {
    st_cluster_u32(cluster_map(&xcnt[rank], tid), static_cast<uint32_t>(cta_less));
    st_cluster_u32(cluster_map(&xcnt[kClusterCtas + rank], tid), static_cast<uint32_t>(cta_eq));
  }
  // The last cluster-wide step: every remote read of a histogram above was
  // consumed before this barrier, and only local reads follow it.
  cluster_sync_all();
  int eq_off = 0, out_off = 0;
  for (int r = 0; r < static_cast<int>(rank); ++r) {
    const int eq_r = xcnt[kClusterCtas + r];
    out_off += xcnt[r] + min(max(krem - eq_off, 0), eq_r);
    eq_off += eq_r;
  }
  int eq_seen = eq_off + eq_before, n_sel = 0;
  bool take[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    bool t = false;
    if (e < n_own) {
      if (kr[e] < boundary) t = true;
      else if (kr[e] == boundary) t = (eq_seen++ < krem);
    }
    take[e] = t;
    n_sel += t;
  }
  int pos = out_off + block_exclusive_scan(n_sel, warp_sums, nullptr);
#pragma unroll
  for (int e = 0; e < kPer; ++e)
    if (take[e]) out[pos++] = lo + e;
}


// kPer: register slots per thread (4, 8 or 16), the smallest that holds the
// candidates; dead slots still cost issue slots in every pass.
template <int kPer>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kThreads)
topk_cluster_kernel(const float* __restrict__ scores, const int32_t* __restrict__ n_chunks,
                    const int32_t* __restrict__ k_per_seq, int k_all, int n_local, int B, int max_chunks,
                    int max_kept, int32_t* __restrict__ kept, int32_t* __restrict__ n_kept,
                    int32_t* __restrict__ cu_kept, unsigned* status) {
  __shared__ int warp_sums[32];
  griddep_wait();   // the previous kernel on the stream has finished
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();

  // Counts: identical in every CTA of the cluster, written by rank 0.  Every
  // early return below depends on them only, so the whole cluster takes it.
  int part = 0;
  unsigned dummy = 0;
  for (int bb = tid; bb <= b; bb += kThreads)
    part += kept_count(ld_dep(n_chunks + bb), k_per_seq ? ld_dep(k_per_seq + bb) : k_all, n_local, max_chunks,
                       max_kept, &dummy);
  int tot = 0;
  block_exclusive_scan(part, warp_sums, &tot);
  unsigned err = 0;
  const int n = ld_dep(n_chunks + b);
  const int nk = kept_count(n, k_per_seq ? ld_dep(k_per_seq + b) : k_all, n_local, max_chunks, max_kept, &err);
  if (rank == 0 && tid == 0) {
    cu_kept[b + 1] = tot;
    if (b == 0) cu_kept[0] = 0;
    n_kept[b] = nk;
    if (err) set_status(status, err);
  }
  if (nk == 0) return;
  int32_t* out = kept + static_cast<int64_t>(b) * max_kept;
  const int n_rec = min(n_local, n);
  const int cand = n - n_rec;
  const int kc = nk - n_rec;
  const int gtid = static_cast<int>(rank) * kThreads + tid;
  if (kc == cand) {
    for (int c = gtid; c < n; c += kClusterThreads) out[c] = c;
    return;
  }
  for (int i = gtid; i < n_rec; i += kClusterThreads) out[kc + i] = cand + i;
  if (kc == 0) return;
  const int per = (cand + kClusterThreads - 1) / kClusterThreads;
  if (per > kPer) {   // the host never launches this case
    if (rank == 0 && tid == 0) set_status(status, LSA_DEV_ERR_INTERNAL);
    return;
  }
  cluster_select_and_write<kPer>(scores + static_cast<int64_t>(b) * max_chunks, cand, kc, out);
}

// ---- token selection from the scorer's score-bin counts ---------------------
// lsa_select_tokens: the token scorer also counts every sequence's scores in
// kScoreBins bins of equal width (lsa_common.cuh), in kScoreBinReplicas copies
// so that fewer of its atomic adds meet on one address; the bin that holds
// the k-th best score is then known before any score is read again.  A
// cluster of 8 CTAs per sequence, each owning an eighth of the positions:
//   1. what the scorer does not write (the bin scale from the head weights,
//      the token counts from the kept counts as the scorer computes them, the
//      output offsets), before the grid dependency wait when the caller
//      promises those inputs settled; after the wait every thread issues its
//      loads at once: up to kPer scores of its CTA's slice (in registers) and
//      four bins of the counts;
//   2. every CTA sums the count copies and finds that boundary bin b* (one
//      block scan; all reach the same answer from the same counts);
//   3. each CTA classifies its slice: a token in a bin above b* is selected
//      (its bit is set in the CTA's bitmap, one ballot per 32 positions), a
//      token in b* is a candidate (key and position; the bins are narrow, so
//      there are few);
//   4. each CTA pushes its count of selected tokens and its candidates into
//      every CTA's shared memory, and one cluster barrier publishes them; then
//      every CTA ranks all candidates by (key, position) the same way (one warp
//      per candidate, its lanes comparing it against 32 others per ballot),
//      takes the r best (r = k - tokens above b*), and knows its own output
//      offset;
//   5. each CTA writes its slice's positions in ascending order.
// Every token above b* outscores every token in or below it, so this is the
// exact top-k.  When the counts cannot be trusted (they do not add up to the
// sequence's tokens, or b* does not split the tokens at k), the candidates do
// not fit the lists, or the sequence is longer than the slices, the cluster
// runs the exact radix select instead (one CTA re-reading the scores beyond
// 131072 tokens).  The result is the same either way.
constexpr int kSelMaxTokens = kClusterMaxCand;                       // 131072: 16 per thread
constexpr int kSelSliceWords = kSelMaxTokens / kClusterCtas / 32;    // 512 bitmap words per CTA
constexpr int kSelMaxCand = 128;                                     // candidates of one CTA
static_assert(kThreads * 4 == kScoreBins, "one int4 of bin counts per thread");
static_assert(kScoreBinReplicas * kScoreBins / 4 == kClusterCtas * 512, "each CTA clears 512 int4 of the counts");

template <int kPer>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kThreads, 1)
select_tokens_kernel(const float* __restrict__ scores, const int32_t* __restrict__ n_kept, int max_kept,
                     const float* __restrict__ w, int k, int max_tokens, int max_sel, int32_t* __restrict__ hist,
                     int32_t* __restrict__ sel, int32_t* __restrict__ n_sel, int32_t* __restrict__ cu_sel,
                     unsigned* status, int kept_stable) {
  __shared__ uint32_t bits[kSelSliceWords];
  __shared__ uint32_t all_key[kClusterCtas * kSelMaxCand];   // [rank r][i]: CTA r's candidates, pushed by r
  __shared__ int all_pos[kClusterCtas * kSelMaxCand];
  __shared__ int x_above[kClusterCtas], x_cand[kClusterCtas];  // pushed by each rank
  __shared__ int warp_sums[32];
  __shared__ int hist_s[256];
  __shared__ int sel2[2];
  __shared__ int s_bstar, s_above, s_ncand, s_earlier;
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const float* sc = scores + static_cast<int64_t>(b) * max_tokens;
  int4* hrow = reinterpret_cast<int4*>(hist + static_cast<int64_t>(b) * kScoreBinReplicas * kScoreBins);

  // ---- 1. what the scorer does not write; then every load at once ------------------
  // The bin scale, the token counts as the scorer writes them (64 n_kept[b];
  // 0 when n_kept is out of range) and the offsets, as lsa_topk_tokens
  // computes them from those: min(k, n) positions per sequence (rank 0's
  // warp 0 sums them over sequences 0 .. b).  With kept_stable (the caller's promise that no
  // kernel still running writes w or the kept counts) they are worked out
  // before the grid dependency wait, while the scorer runs.
  float scale = 0.f;
  int tot = 0, n = 0, nk = 0;
  unsigned err = 0;
  auto counts = [&]() {
    // Every load first, so that they take one round trip: this sequence's
    // kept count, the head weights, and (for the lanes of rank 0's warp 0,
    // which alone needs the offsets) the kept counts of sequences 0 .. b.
    const bool lead = rank == 0 && warp == 0;
    const int m_own = ld_dep(n_kept + b);
    float wv[kIndexHeads];
#pragma unroll
    for (int h = 0; h < kIndexHeads; ++h) wv[h] = ld_dep(w + h);
    const int m_lane = (lead && lane <= b) ? ld_dep(n_kept + lane) : 0;
    float wsum = 0.f;
#pragma unroll
    for (int h = 0; h < kIndexHeads; ++h) wsum += wv[h];
    scale = score_bin_scale_of_sum(wsum);
    auto tokens_of = [&](int m) { return (m < 0 || m > max_kept) ? 0 : m * kChunkTokens; };
    n = tokens_of(m_own);
    nk = kept_count(n, k, 0, max_tokens, max_sel, &err);
    if (lead) {   // warp-uniform
      unsigned dummy = 0;
      int part = lane <= b ? kept_count(tokens_of(m_lane), k, 0, max_tokens, max_sel, &dummy) : 0;
      for (int bb = lane + 32; bb <= b; bb += 32)
        part += kept_count(tokens_of(ld_dep(n_kept + bb)), k, 0, max_tokens, max_sel, &dummy);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      tot = part;
    }
  };
  if (kept_stable) counts();
  griddep_wait();   // the scorer has finished: scores and the bin counts are final, the outputs free
  if (!kept_stable) counts();
  // This CTA's slice of positions, in whole bitmap words, sized from the row
  // length (so the loads need not wait for the token count): thread t holds
  // positions lo + j * 1024 + t, j < kPer.
  const int slice = ((max_tokens + kClusterCtas - 1) / kClusterCtas + 31) / 32 * 32;
  const int lo = min(max_tokens, static_cast<int>(rank) * slice);
  const int hi_row = min(max_tokens, lo + slice);
  const bool sliced = slice <= kPer * kThreads;                      // the slice fits the registers
  float v[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int p = lo + j * kThreads + tid;
    v[j] = (sliced && p < hi_row) ? ld_dep(sc + p) : 0.f;
  }
  int c4[4] = {0, 0, 0, 0};   // bins 4 tid .. 4 tid + 3, summed over the copies
#pragma unroll
  for (int rep = 0; rep < kScoreBinReplicas; ++rep) {
    const int4 x = hrow[rep * (kScoreBins / 4) + tid];
    c4[0] += x.x; c4[1] += x.y; c4[2] += x.z; c4[3] += x.w;
  }
  auto clear_counts = [&]() {   // this CTA's eighth of the counts, zero for the next call
    if (tid < 512) hrow[rank * 512 + tid] = make_int4(0, 0, 0, 0);
  };
  if (rank == 0 && tid == 0) {   // (rank 0 writes the offsets)
    cu_sel[b + 1] = tot;
    if (b == 0) cu_sel[0] = 0;
    n_sel[b] = nk;
    if (err) set_status(status, err);
  }
  int32_t* out = sel + static_cast<int64_t>(b) * max_sel;
  if (nk == 0 || nk == n) {   // nothing, or every position (cluster-uniform: no count is needed)
    clear_counts();
    for (int c = static_cast<int>(rank) * kThreads + tid; c < nk; c += kClusterThreads) out[c] = c;
    return;
  }
  cluster_arrive_relaxed();   // (A) this CTA runs; waited on before the first remote store

  // ---- 2. the boundary bin ----------------------------------------------------------
  const int own = c4[0] + c4[1] + c4[2] + c4[3];
  int total = 0;
  const int below = block_exclusive_scan(own, warp_sums, &total);   // tokens in bins under 4 tid
  if (tid == 0) { s_bstar = -1; s_above = 0; s_ncand = 0; s_earlier = 0; }
  __syncthreads();
  if (total == n && sliced && scale > 0.f) {                         // cluster-uniform
    int above = total - below - own;                                 // tokens in bins over 4 tid + 3
#pragma unroll
    for (int j = 3; j >= 0; --j) {
      if (above < nk && above + c4[j] >= nk) s_bstar = 4 * tid + j;
      above += c4[j];
    }
  }
  __syncthreads();
  const int bstar = s_bstar;
  bool fast = bstar >= 0;                                            // cluster-uniform
  const int hi = min(n, hi_row);

  // ---- 3. classify this CTA's slice -------------------------------------------------
  if (fast) {
    int above_w = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (lo + j * kThreads < hi) {   // block-uniform
        const int p = lo + j * kThreads + tid;
        const int bi = p < hi ? score_bin(v[j], scale) : -1;
        const uint32_t up = __ballot_sync(0xffffffffu, bi > bstar);
        const uint32_t eq = __ballot_sync(0xffffffffu, bi == bstar);
        if (lane == 0) bits[j * (kThreads / 32) + warp] = up;
        above_w += __popc(up);
        if (eq) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&s_ncand, __popc(eq));
          base = __shfl_sync(0xffffffffu, base, 0);
          if ((eq >> lane) & 1u) {
            const int slot = base + __popc(eq & ((1u << lane) - 1u));
            if (slot < kSelMaxCand) {
              all_key[rank * kSelMaxCand + slot] = desc_key(v[j]);
              all_pos[rank * kSelMaxCand + slot] = p;
            }
          }
        }
      }
    }
    if (lane == 0 && above_w) atomicAdd(&s_above, above_w);
  }
  __syncthreads();

  // ---- 4. push counts and candidates to every CTA; one barrier publishes them -------
  cluster_wait();   // (A): every CTA of the cluster runs
  if (fast) {
    const int m_own = min(s_ncand, kSelMaxCand);
    if (tid < kClusterCtas) {
      st_cluster_u32(cluster_map(&x_above[rank], tid), static_cast<uint32_t>(s_above));
      st_cluster_u32(cluster_map(&x_cand[rank], tid), static_cast<uint32_t>(s_ncand));
    }
    for (int t = tid; t < kClusterCtas * m_own; t += kThreads) {
      const int r = t / m_own, i = t - r * m_own;
      if (r != static_cast<int>(rank)) {
        st_cluster_u32(cluster_map(&all_key[rank * kSelMaxCand + i], r), all_key[rank * kSelMaxCand + i]);
        st_cluster_u32(cluster_map(&all_pos[rank * kSelMaxCand + i], r),
                       static_cast<uint32_t>(all_pos[rank * kSelMaxCand + i]));
      }
    }
  }
  cluster_sync_all();   // #1: every push is visible, and every CTA has read the counts
  clear_counts();

  if (fast) {
    int mt = 0, above_all = 0, off = 0;
#pragma unroll
    for (int r = 0; r < kClusterCtas; ++r) {
      fast = fast && x_cand[r] <= kSelMaxCand;
      mt += x_cand[r];
      above_all += x_above[r];
      if (r < static_cast<int>(rank)) off += x_above[r];
    }
    const int r_take = nk - above_all;
    fast = fast && r_take >= 0 && r_take <= mt;                      // cluster-uniform
    if (fast) {
      // Candidate f of the flat list (the CTAs' lists in rank order) is slot
      // (r, f - start[r]) of the slotted arrays.  Warp w ranks candidates
      // w, w + 32, ...: its lanes compare the candidate with 32 others per
      // ballot, and the count of candidates before it decides.
      int start[kClusterCtas + 1];
      start[0] = 0;
#pragma unroll
      for (int r = 0; r < kClusterCtas; ++r) start[r + 1] = start[r] + x_cand[r];
      auto slot_of = [&](int f) {   // the last list that starts at or before f (start is non-decreasing)
        int r = 0, base = 0;
#pragma unroll
        for (int q = 1; q < kClusterCtas; ++q)
          if (f >= start[q]) { r = q; base = start[q]; }
        return r * kSelMaxCand + (f - base);
      };
      for (int f = warp; f < mt; f += kThreads / 32) {
        const int si = slot_of(f);
        const uint32_t ki = all_key[si];
        const int pi = all_pos[si];
        int before = 0;
        for (int j0 = 0; j0 < mt; j0 += 32) {
          bool bj = false;
          if (j0 + lane < mt) {
            const int sj = slot_of(j0 + lane);
            const uint32_t kj = all_key[sj];
            bj = (kj < ki) || (kj == ki && all_pos[sj] < pi);
          }
          before += __popc(__ballot_sync(0xffffffffu, bj));
        }
        if (lane == 0 && before < r_take) {
          const int r = si / kSelMaxCand;
          if (r < static_cast<int>(rank)) atomicAdd(&s_earlier, 1);
          if (r == static_cast<int>(rank)) atomicOr(&bits[(pi - lo) >> 5], 1u << ((pi - lo) & 31));
        }
      }
      __syncthreads();   // the bits and the count of earlier ranks' taken candidates
      off += s_earlier;
      // ---- 5. this slice's positions, ascending ---------------------------------------
      griddep_launch_dependents();
      const int words = hi > lo ? (hi - lo + 31) >> 5 : 0;
      const uint32_t x0 = tid < words ? bits[tid] : 0u;
      int pos = off + block_exclusive_scan(__popc(x0), warp_sums, nullptr);
      uint32_t x = x0;
      while (x) {
        out[pos++] = lo + (tid << 5) + (__ffs(x) - 1);
        x &= x - 1u;
      }
      return;
    }
  }

  // ---- the exact path --------------------------------------------------------------
  if (n <= kClusterThreads * kPer) {
    cluster_select_and_write<kPer>(sc, n, nk, out);
  } else if (rank == 0) {   // beyond the cluster's registers: one CTA re-reads the scores
    select_and_write<false>(ScoreKey{sc}, n, nk, (n + kThreads - 1) / kThreads, out, hist_s, warp_sums, sel2);
  }
}

// One CTA per sequence up to kClusterMinCand candidates, a cluster of 8 up to
// kClusterMaxCand, one CTA re-reading the scores beyond.
int launch_topk(bool pdl, const float* scores, const int32_t* n_count, const int32_t* k_per_seq, int k_all,
                int n_local, int B, int max_count, int max_kept, int32_t* kept, int32_t* n_kept, int32_t* cu_kept,
                cudaStream_t s) {
  if (max_count > kClusterMinCand && max_count <= kClusterMaxCand) {
    const dim3 grid(kClusterCtas, B);
    unsigned* st = lsa_device_status_ptr();
    auto kernel = max_count <= kClusterThreads * 4   ? topk_cluster_kernel<4>
                  : max_count <= kClusterThreads * 8 ? topk_cluster_kernel<8>
                                                     : topk_cluster_kernel<16>;
    launch_pdl(pdl, kernel, grid, dim3(kThreads), 0, s, scores, n_count, k_per_seq, k_all, n_local, B, max_count,
               max_kept, kept, n_kept, cu_kept, st);
  } else {
    launch_pdl(pdl, topk_kernel, dim3(B), dim3(kThreads), 0, s, scores, n_count, k_per_seq, k_all, n_local, B, max_count,
               max_kept, kept, n_kept, cu_kept, lsa_device_status_ptr());
  }
  return launch_status();
}

}  // namespace topk
}  // namespace lsa

extern "C" int lsa_topk_chunks_local(const float* scores, const int32_t* n_chunks, const int32_t* k_per_seq,
                                     int n_local, int B, int max_chunks, int max_kept, int32_t* kept,
                                     int32_t* n_kept, int32_t* cu_kept, void* stream) {
  using namespace lsa;
  if (!scores || !n_chunks || !k_per_seq || !kept || !n_kept || !cu_kept || B <= 0 || max_chunks <= 0 ||
      max_kept <= 0 || n_local <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(B) * max_kept >= (int64_t{1} << 31)) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  return topk::launch_topk(false, scores, n_chunks, k_per_seq, 0, n_local, B, max_chunks, max_kept, kept, n_kept,
                           cu_kept, static_cast<cudaStream_t>(stream));
}

// Token-level fine top-k (summary page, 2.1 Architecture): the k best token
// positions of each sequence's recalled chunks, same key and tie rule, no
// recent window (every position is a candidate), ascending output.
extern "C" int lsa_topk_tokens(const float* scores, const int32_t* n_tokens, int k, int B, int max_tokens,
                               int max_sel, int32_t* sel, int32_t* n_sel, int32_t* cu_sel, void* stream) {
  using namespace lsa;
  if (!scores || !n_tokens || !sel || !n_sel || !cu_sel || B <= 0 || max_tokens <= 0 || max_sel <= 0 || k <= 0)
    return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(B) * max_sel >= (int64_t{1} << 31) ||
      static_cast<int64_t>(B) * max_tokens >= (int64_t{1} << 40))
    return LSA_ERR_UNSUPPORTED_SHAPE;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  return topk::launch_topk(true, scores, n_tokens, nullptr, k, 0, B, max_tokens, max_sel, sel, n_sel, cu_sel,
                           static_cast<cudaStream_t>(stream));
}

extern "C" size_t lsa_select_tokens_workspace_size(int B) {
  if (B <= 0 || B > LSA_MAX_BATCH) return 0;
  return static_cast<size_t>(B) * lsa::kScoreBinReplicas * lsa::kScoreBins * sizeof(int32_t);
}

// lsa_token_score followed by lsa_topk_tokens, with the selection driven by
// the scorer's score-bin counts (summary page, 2.1 Architecture: native
// token-level scoring keeps a fine-grained top-k inside the recalled subset).
extern "C" int lsa_select_tokens(const void* q_idx, const float* w, const void* token_keys, int64_t n_slots,
                                 const int32_t* chunk_table, const int32_t* kept, const int32_t* n_kept, int B,
                                 int max_chunks, int max_kept, int k, float* scores, int32_t* n_tokens, int32_t* sel,
                                 int32_t* n_sel, int32_t* cu_sel, int max_sel, void* workspace,
                                 size_t workspace_bytes, unsigned int flags, void* stream) {
  using namespace lsa;
  // Every check of both kernels comes before the first launch.
  if (!sel || !n_sel || !cu_sel || k <= 0 || max_sel <= 0 || B <= 0 || max_kept <= 0) return LSA_ERR_INVALID_ARG;
  if (flags & ~static_cast<unsigned>(LSA_TOKENS_UNCHANGED)) return LSA_ERR_INVALID_ARG;
  const int keys_unchanged = (flags & LSA_TOKENS_UNCHANGED) ? 1 : 0;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(B) * max_sel >= (int64_t{1} << 31) ||
      static_cast<int64_t>(max_kept) * kChunkTokens >= (int64_t{1} << 31))
    return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!workspace || workspace_bytes < lsa_select_tokens_workspace_size(B)) return LSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return LSA_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = device_sm_count();
  if (sms <= 0) return LSA_ERR_NO_DEVICE;
  const int max_tokens = max_kept * kChunkTokens;
  // The bin counts cost the scorer shared memory (four CTAs per SM instead of
  // five), which only pays when its grid runs in one wave: then the step waits
  // on the selection's latency, which the counts cut.  Larger grids take the
  // scorer without counts and the radix select (lsa_token_score +
  // lsa_topk_tokens), with the same result.
  const int64_t score_ctas = static_cast<int64_t>(B) * ((max_tokens + 127) / 128);
  if (score_ctas > static_cast<int64_t>(4) * sms) {
    const int st = score::launch_token_score(q_idx, w, token_keys, n_slots, chunk_table, kept, n_kept, B, max_chunks,
                                             max_kept, scores, n_tokens, nullptr, keys_unchanged, s);
    if (st != LSA_OK) return st;
    return topk::launch_topk(true, scores, n_tokens, nullptr, k, 0, B, max_tokens, max_sel, sel, n_sel, cu_sel, s);
  }
  int32_t* hist = static_cast<int32_t*>(workspace);
  const int st = score::launch_token_score(q_idx, w, token_keys, n_slots, chunk_table, kept, n_kept, B, max_chunks,
                                           max_kept, scores, n_tokens, hist, keys_unchanged, s);
  if (st != LSA_OK) return st;
  auto kernel = max_tokens <= topk::kClusterThreads * 4   ? topk::select_tokens_kernel<4>
                : max_tokens <= topk::kClusterThreads * 8 ? topk::select_tokens_kernel<8>
                                                          : topk::select_tokens_kernel<16>;
  launch_pdl(true, kernel, dim3(topk::kClusterCtas, B), dim3(topk::kThreads), 0, s, scores, n_kept, max_kept, w, k,
             max_tokens, max_sel, hist, sel, n_sel, cu_sel, lsa_device_status_ptr(), keys_unchanged);
  return launch_status();
}

extern "C" int lsa_topk_chunks(const float* scores, const int32_t* n_chunks, const int32_t* k_per_seq, int B,
                               int max_chunks, int max_kept, int32_t* kept, int32_t* n_kept, int32_t* cu_kept,
                               void* stream) {
  return lsa_topk_chunks_local(scores, n_chunks, k_per_seq, 1, B, max_chunks, max_kept, kept, n_kept, cu_kept,
                               stream);
}

// ---------------------------------------------------------------------------
// lsa_threshold_chunks: the pages' own selection rule, sigmoid thresholding in
// place of a fixed top-k (summary page, 2.1 Architecture and 2.4
// Configuration): chunk c < n-1 is kept when score_c / sum_h w_h (the weighted
// mean of the heads' sigmoid probabilities) exceeds the threshold; the latest
// chunk is always kept.  The kept count is data-dependent, so a first kernel
// compacts each sequence (one CTA per sequence, contiguous candidate runs per
// thread, one block scan, index order preserved) and a second one-CTA kernel
// turns the counts into cu_kept.
// ---------------------------------------------------------------------------
namespace lsa {
namespace topk {

// Key of candidate i for the capped threshold rule: a chunk that passes the
// threshold keeps its descending score key; one that does not gets the largest
// key, which only NaN scores share (and NaN never passes), so every passing
// chunk ranks before every other one.
struct PassKey {
  const float* sc;
  float wsum, threshold;
  __device__ __forceinline__ uint32_t operator()(int i) const {
    const float s = __ldg(sc + i);
    return (s / wsum > threshold) ? desc_key(s) : 0xffffffffu;
  }
};

__global__ void __launch_bounds__(kThreads)
threshold_kernel(const float* __restrict__ scores, const int32_t* __restrict__ n_chunks,
                 const float* __restrict__ w, float threshold, const int32_t* __restrict__ cap, int max_chunks,
                 int max_kept, int32_t* __restrict__ kept, int32_t* __restrict__ n_kept, unsigned* status) {
  __shared__ int warp_sums[32];
  __shared__ int hist[256];
  __shared__ int sel[2];
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  griddep_wait();                 // the previous kernel on the stream has finished
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n = __ldg(n_chunks + b);
  if (n < 0 || n > max_chunks) {
    if (tid == 0) { n_kept[b] = 0; set_status(status, LSA_DEV_ERR_BAD_COUNT); }
    return;
  }
  if (n == 0) {
    if (tid == 0) n_kept[b] = 0;
    return;
  }
  float wsum = 0.f;   // fixed order: every thread gets the same fp32 sum
#pragma unroll
  for (int h = 0; h < kIndexHeads; ++h) wsum += __ldg(w + h);
  const float* sc = scores + static_cast<int64_t>(b) * max_chunks;
  const int cand = n - 1;
  const int per = (cand + kThreads - 1) / kThreads;
  const int lo = min(cand, tid * per), hi = min(cand, lo + per);
  int cnt = 0;
  for (int i = lo; i < hi; ++i) cnt += (__ldg(sc + i) / wsum > threshold);
  int total = 0;
  int pos = block_exclusive_scan(cnt, warp_sums, &total);
  const int cap_b = cap ? __ldg(cap + b) : total;
  if (cap_b < 0) {
    if (tid == 0) { n_kept[b] = 0; set_status(status, LSA_DEV_ERR_BAD_COUNT); }
    return;
  }
  if (min(total, cap_b) + 1 > max_kept) {
    if (tid == 0) { n_kept[b] = 0; set_status(status, LSA_DEV_ERR_CAPACITY); }
    return;
  }
  int32_t* out = kept + static_cast<int64_t>(b) * max_kept;
  if (total > cap_b) {
    // More chunks pass than the budget allows: keep the cap_b best passing
    // chunks (score descending, chunk index ascending), in index order.
    if (cap_b > 0) {
      const PassKey key{sc, wsum, threshold};
      const int per_t = (cand + kThreads - 1) / kThreads;
      if (per_t <= kMaxPerThread)
        select_and_write<true>(key, cand, cap_b, per_t, out, hist, warp_sums, sel);
      else
        select_and_write<false>(key, cand, cap_b, per_t, out, hist, warp_sums, sel);
    }
    if (tid == 0) {
      out[cap_b] = n - 1;
      n_kept[b] = cap_b + 1;
    }
    return;
  }
  for (int i = lo; i < hi; ++i)
    if (__ldg(sc + i) / wsum > threshold) out[pos++] = i;
  if (tid == 0) {
    out[total] = n - 1;
    n_kept[b] = total + 1;
  }
}

// cu_kept[0] = 0, cu_kept[b+1] = cu_kept[b] + n_kept[b]  (one CTA, B <= 4096).
__global__ void __launch_bounds__(kThreads)
offsets_kernel(const int32_t* __restrict__ n_kept, int B, int32_t* __restrict__ cu_kept) {
  __shared__ int warp_sums[32];
  griddep_launch_dependents();   // let the next kernel launch; its CTAs wait for this grid
  griddep_wait();                 // the previous kernel on the stream has finished
  const int tid = threadIdx.x;
  constexpr int kPer = (LSA_MAX_BATCH + kThreads - 1) / kThreads;   // 4
  int v[kPer], s = 0;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int b = tid * kPer + e;
    v[e] = b < B ? n_kept[b] : 0;
    s += v[e];
  }
  int run = block_exclusive_scan(s, warp_sums, nullptr);
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int b = tid * kPer + e;
    run += v[e];
    if (b < B) cu_kept[b + 1] = run;
  }
  if (tid == 0) cu_kept[0] = 0;
}

}  // namespace topk
}  // namespace lsa

extern "C" int lsa_threshold_chunks(const float* scores, const int32_t* n_chunks, const float* w, float threshold,
                                    int B, int max_chunks, int max_kept, int32_t* kept, int32_t* n_kept,
                                    int32_t* cu_kept, void* stream) {
  return lsa_threshold_chunks_capped(scores, n_chunks, w, threshold, nullptr, B, max_chunks, max_kept, kept,
                                     n_kept, cu_kept, stream);
}

extern "C" int lsa_threshold_chunks_capped(const float* scores, const int32_t* n_chunks, const float* w,
                                           float threshold, const int32_t* cap, int B, int max_chunks,
                                           int max_kept, int32_t* kept, int32_t* n_kept, int32_t* cu_kept,
                                           void* stream) {
  using namespace lsa;
  if (!scores || !n_chunks || !w || !kept || !n_kept || !cu_kept || B <= 0 || max_chunks <= 0 || max_kept <= 0)
    return LSA_ERR_INVALID_ARG;
  if (!isfinite(threshold)) return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(B) * max_kept >= (int64_t{1} << 31)) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (device_sm_count() <= 0) return LSA_ERR_NO_DEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  launch_pdl(false, topk::threshold_kernel, dim3(B), dim3(topk::kThreads), 0, s, scores, n_chunks, w, threshold, cap,
             max_chunks, max_kept, kept, n_kept, lsa_device_status_ptr());
  int st = launch_status();
  if (st != LSA_OK) return st;
  launch_pdl(false, topk::offsets_kernel, dim3(1), dim3(topk::kThreads), 0, s, n_kept, B, cu_kept);
  return launch_status();
}
