// lsa_sparse_decode_attn: one GQA decode step over the kept chunks.
//
// Method: softmax(q K^T / sqrt(d)) V per query head, 8 consecutive query heads
// per KV head (handbook page "DeepSeek-V4: Architecting for Ultra-Long
// Contexts", section "Grouped Query Attention (GQA) vs. Multi-Head Attention
// (MHA)"), over only the chunks kept for the window (summary page
// "FlashMemory-DeepSeek-V4 ...", Abstract and 2.1 Architecture).
//
// B200 design
// -----------
// * Work unit = one (sequence b, KV head g, kept chunk j) tile: 64 tokens of K
//   and of V, 16 KiB each, contiguous in the compact buffer.  The units of all
//   (b, g) pairs are laid end to end, and the grid (one CTA per SM) cuts that
//   list into equal contiguous ranges (split-K over the kept tokens, balanced
//   to within one unit per CTA for any batch mix).
// * A producer warp streams units into a 4-stage shared-memory ring with TMA
//   (cp.async.bulk.tensor, 128-byte swizzle, evict-first L2 hint) completing
//   on mbarriers.  Two groups of 4 consumer warps take alternate units; each
//   warp of a group takes 16 of the unit's 64 tokens.
// * Per warp, scores are computed transposed, S^T = K Q^T, on the tensor
//   cores (mma.sync m16n8k16: M = 16 tokens, N = the 8 query heads of the
//   group, K = 128), so no MMA row is padding.  The online softmax runs in
//   fp32 (exp2 domain); probabilities are split into two bf16 parts
//   (P = P_hi + P_lo, about 16 mantissa bits), transposed in registers with
//   movmatrix and used as the B operands of O^T += V^T P^T (M = 128 dims,
//   N = 8 heads, K = 16 tokens, V^T read once with ldmatrix.trans).
// * At the end of each (b, g) segment the 8 warps combine their (max, sum,
//   acc) in shared memory.  A segment that covers the whole pair writes the
//   output; otherwise it writes a normalised partial and its log-sum-exp, and
//   the CTA is done: no tickets, fences or merges on the attention grid's
//   tail.  A small second kernel, launched as a programmatic dependent, folds
//   the partials of each split pair in CTA order once the grid has finished,
//   spread over the SMs of the pair's contributors, so the result does not
//   depend on timing.
// * Launched as a programmatic dependent of the previous kernel: when the
//   caller states that K/V did not change, the producer starts streaming
//   before the previous kernel has finished.
// * Variants on the same pipeline: a per-sequence local chunk of decoded
//   tokens as one more masked unit per KV head (with the step's own token
//   optionally written into it by the consumer warp that owns its row), and
//   units of 64 selected tokens (the token-level fine stage) whose rows the
//   producer warp copies straight from the compact buffer with cp.async.
#include <math.h>

#include <mutex>

#include "lsa_common.cuh"
#include "lsa_runtime.cuh"

namespace lsa {
namespace attn {

constexpr int kGroups = 2;                   // consumer warp groups, taking alternate units
constexpr int kWarpsPerGroup = 4;            // each warp of a group takes 16 of a unit's 64 tokens
constexpr int kConsumerWarps = kGroups * kWarpsPerGroup;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kConsumerThreads = kConsumerWarps * 32;
#ifndef LSA_ATTN_STAGES
#define LSA_ATTN_STAGES 4
#endif
constexpr int kStages = LSA_ATTN_STAGES;     // TMA ring depth (32 KiB per stage)
// Unit i goes to stage i % kStages and to group i % kGroups.  With kStages a
// multiple of kGroups every stage belongs to one group, which waits on its
// phases strictly in order; otherwise a group could wait on a phase two ahead
// of the barrier's and the parity test would succeed early.
static_assert(kStages % kGroups == 0, "each stage must belong to a single consumer group");
constexpr int kCtasPerSm = 1;                // one CTA per SM: 8 consumer warps
constexpr int kBoxBytes = 8192;              // 64 tokens x 64 dims of bf16
constexpr int kStageBytes = 4 * kBoxBytes;   // K dims 0-63, K dims 64-127, V lo, V hi
constexpr int kAccStride = 132;              // padded row of the combine buffer
constexpr int kRecFloats = kGroup * kHeadDim + kGroup;  // partial o[8][128] + lse[8]
constexpr int kMaxCtas = 1024;
static_assert(kRecFloats * 4 % 16 == 0, "records are copied in 16-byte pieces");
constexpr int kSmemBytes = kStages * kStageBytes +
                           kConsumerWarps * kGroup * kAccStride * 4 + 2 * kConsumerWarps * kGroup * 4 +
                           2 * kStages * 8 + 16;

// T units cut into G contiguous ranges: the first `rem` CTAs take base + 1
// units, the others base (base = T / G, rem = T % G).  Everything is 32-bit
// (T <= 8 * 2^22).  When T < G the CTAs c >= T are empty and sit after every
// non-empty one, so the CTAs between the first and last owner of any unit
// range all own part of it.
struct Partition {
  int base, rem;
  __device__ Partition(int T, int G) : base(T / G), rem(T % G) {}
  __device__ int start(int c) const { return c * base + min(c, rem); }
  __device__ int cta_of(int u) const {
    const int big = rem * (base + 1);
    return u < big ? u / (base + 1) : rem + (u - big) / base;
  }
};

// Sequence offsets counted in 64-token units: an array of chunk offsets
// (shift 0: cu_kept), or of token offsets that are multiples of 64 (shift 6:
// cu_sel of the token-level fine stage, read without a packed copy).  An
// earlier kernel on the stream may have written them (ld_dep).
struct Offsets {
  const int32_t* p;
  int shift;
  __device__ __forceinline__ int raw(int i) const { return ld_dep(p + i); }
  __device__ __forceinline__ int operator()(int i) const { return raw(i) >> shift; }
};

// Verdict on the sequence offsets, the same in every thread of the block: the
// first is 0, none decreases, the total fits `cap`; indexed offsets are token
// offsets, multiples of 64 and at most max_sel apart.
__device__ __forceinline__ bool offsets_bad(Offsets cu, int B, int64_t cap, bool indexed, int max_sel) {
  const int total = cu(B);
  int bad = (cu.raw(0) != 0 || total < 0 || static_cast<int64_t>(total) > cap) ? 1 : 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    bad |= (cu(b + 1) < cu(b));
    if (indexed) bad |= ((cu.raw(b + 1) & 63) != 0) | (cu.raw(b + 1) - cu.raw(b) > max_sel);
  }
  return __syncthreads_or(bad) != 0;
}

// Units of sequence b: its kept chunks plus E local chunks (E = 1 when the
// window's decoded tokens are attended), for each of the 8 KV heads.  The
// units of sequence b start at 8 * (cu[b] + E * b).
__device__ __forceinline__ int64_t seq_unit_base(Offsets cu, int E, int b) {
  return 8 * (static_cast<int64_t>(cu(b)) + static_cast<int64_t>(E) * b);
}
__device__ __forceinline__ int units_of(Offsets cu, int E, int b) { return cu(b + 1) - cu(b) + E; }
// Largest b in [0, B) whose units start at or before u (the sequence of unit u).
__device__ __forceinline__ int seq_of_unit(Offsets cu, int E, int B, int64_t u) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_unit_base(cu, E, mid) <= u) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct UnitCursor {
  int b, g, j;
  __device__ void start(Offsets cu, int E, int B, int64_t u) {
    b = seq_of_unit(cu, E, B, u);
    const int64_t r = u - seq_unit_base(cu, E, b);
    const int n = units_of(cu, E, b);
    g = static_cast<int>(r / n);
    j = static_cast<int>(r - static_cast<int64_t>(g) * n);
  }
  __device__ void advance(Offsets cu, int E, int B, int n_b) {
    if (++j == n_b) {
      j = 0;
      if (++g == kNumKVHeads) {
        g = 0;
        ++b;
        while (b < B && units_of(cu, E, b) == 0) ++b;
      }
    }
  }
};

// The decode step's own token, appended inside the step (all null otherwise):
// position n = local_len[b] of the local chunk receives it and is attended as
// token n; the new count n + 1 goes to a second array, so that no reader of
// this grid sees the count change.
struct AppendArgs {
  const uint4* k_new;   // [B][8 KV heads][16 x 16 B]: one token
  const uint4* v_new;
  uint4* k_local;       // [B][8][64 tokens][16 x 16 B]: the local chunks
  uint4* v_local;
  int32_t* len_out;     // [B]
};

// The token-level fine stage read in place (all null otherwise): unit j of
// (b, g) holds the 64 selected positions sel[b][64 j .. 64 j + 63]; position
// p is row p % 64 of compact chunk ck[b] + p / 64 of KV head g.  The producer
// copies those rows straight into the stage instead of reading a packed copy.
struct SelectArgs {
  const int32_t* sel;   // [B][max_sel]
  const int32_t* ck;    // [B + 1]: chunk offsets of the compact buffer (cu_kept)
  int max_sel;
  int64_t ck_chunks;    // chunks in the compact buffer
  const uint4* k_buf;   // the compact buffer, head-major [8][ck_chunks][64][16 x 16 B]
  const uint4* v_buf;
};

// Grid: kCtasPerSm CTAs per SM, capped at kMaxCtas.
inline int grid_for(int sms) { return sms * kCtasPerSm < kMaxCtas ? sms * kCtasPerSm : kMaxCtas; }

// Smallest share of units worth a CTA of its own.  A launch over few units
// (the token-level fine stage: 32 units per KV head) runs on fewer CTAs, so
// each (sequence, KV head) pair is split fewer ways and its merge folds fewer
// partials; large launches keep one CTA per SM.
constexpr int64_t kMinUnitsPerCta = 4;
constexpr int64_t kMinIndexedUnitsPerCta = 2;   // the in-place fine stage: more CTAs issue its row copies
constexpr int kPosAhead = 2;                     // units whose positions the in-place producer loads ahead (4: no gain)
inline int grid_for_units(int sms, int64_t max_units, int64_t per_cta = kMinUnitsPerCta) {
  const int64_t want = (max_units + per_cta - 1) / per_cta;
  const int full = grid_for(sms);
  return want < 1 ? 1 : (want < full ? static_cast<int>(want) : full);
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
sparse_decode_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_kl, const __grid_constant__ CUtensorMap tm_vl,
                          const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ cu_raw, int B,
                          int64_t buf_chunks, const int32_t* __restrict__ local_len, float scale_log2,
                          float* __restrict__ out, float* __restrict__ records,
                          unsigned* status, int kv_unchanged, AppendArgs app, SelectArgs sa) {
  const bool indexed = sa.sel != nullptr;
  const Offsets cu{cu_raw, indexed ? 6 : 0};
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte TMA swizzle pattern repeats every 1024 bytes and the fragment
  // addressing below assumes each box starts on such a boundary.
  if (smem_u32(smem_raw) & 1023u) {
    griddep_wait();   // every CTA waits before it ends
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(status, LSA_DEV_ERR_INTERNAL);
    return;
  }
  uint8_t* smem = smem_raw;
  float* accbuf = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  float* mbuf = accbuf + kConsumerWarps * kGroup * kAccStride;
  float* lbuf = mbuf + kConsumerWarps * kGroup;
  uint64_t* full = reinterpret_cast<uint64_t*>(lbuf + kConsumerWarps * kGroup);
  uint64_t* empty = full + kStages;
  int* flags = reinterpret_cast<int*>(empty + kStages);  // [0] abort

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // With kv_unchanged the caller guarantees that the preceding kernel on the
  // stream did not write k_buf, v_buf or cu_kept, so those may be read before
  // it has finished; everything else (q, out, the workspace) waits for it.
  if (!kv_unchanged) griddep_wait();

  // ---- validate cu_kept (every thread reaches the same verdict) -------------
  // (Indexed: token offsets, multiples of 64, at most max_sel per sequence;
  // buf_chunks is then the unit capacity B * max_sel / 64.)
  if (offsets_bad(cu, B, buf_chunks, indexed, sa.max_sel)) {
    if (kv_unchanged) griddep_wait();   // every CTA waits before it ends
    if (blockIdx.x == 0 && tid == 0) set_status(status, LSA_DEV_ERR_CAPACITY);
    return;
  }
  const int E = local_len ? 1 : 0;   // one local unit per (b, g) when decoded tokens are attended
  const int T = 8 * (cu(B) + E * B);
  const int G = gridDim.x;
  const Partition part(T, G);
  const int64_t u0 = part.start(blockIdx.x), u1 = part.start(blockIdx.x + 1);

  // Sequences without kept chunks get zeros (written after the wait).
  auto zero_empty = [&](int first, int stride) {
    for (int b = blockIdx.x; b < B; b += G) {
      if (units_of(cu, E, b) == 0) {
        float4* o = reinterpret_cast<float4*>(out + static_cast<int64_t>(b) * kNumQHeads * kHeadDim);
        for (int i = first; i < kNumQHeads * kHeadDim / 4; i += stride) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  if (u0 >= u1) {
    if (kv_unchanged) griddep_wait();
    zero_empty(tid, kThreads);
    griddep_launch_dependents();
    return;
  }

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], indexed ? 32 : 1);   // indexed: one cp.async arrival per producer lane
      mbar_init(&empty[s], kWarpsPerGroup);   // a stage is consumed by one warp group
    }
    flags[0] = 0;
    mbar_fence_init();
  }
  __syncthreads();
  griddep_launch_dependents();
  volatile int* abort_flag = flags;

  if (warp == kConsumerWarps && indexed) {
    // ============ producer warp, fine stage: selected rows in place ==========
    // Lane l resolves the addresses of rows l and l + 32 of the unit; then the
    // warp copies two rows per instruction, lanes 0-15 the 16 pieces of 16
    // bytes of one row and lanes 16-31 those of the next (each row's address
    // taken from the lane that resolved it), so one instruction touches two
    // 256-byte rows instead of 32 scattered pieces.  The pieces land at their
    // swizzled places in the stage; each lane arrives on the stage's full
    // barrier when its copies have landed.  A position outside the sequence's
    // recalled tokens is written as zeros.  The positions of a unit are
    // loaded kPosAhead units ahead, while the units before it wait for their
    // stages and issue their copies, so their L2 round trips are off the
    // producer's path.
    UnitCursor cur;
    cur.start(cu, E, B, u0);
    const int64_t n_units = u1 - u0;
    const uint32_t smem_base_p = smem_u32(smem);
    int at_b = -1, n_b = 0;
    int64_t ckb = 0, n_pos = 0;
    auto load_pos = [&](const UnitCursor& c, int* p) {   // positions lane and lane + 32 of unit c
#pragma unroll
      for (int h = 0; h < 2; ++h)
        p[h] = ld_dep(sa.sel + static_cast<int64_t>(c.b) * sa.max_sel + c.j * kChunkTokens + lane + 32 * h);
    };
    // The look-ahead cursor `la` is the unit whose positions load next; la_nb
    // is the unit count of its sequence.
    UnitCursor la = cur;
    int la_nb = n_units > 0 ? units_of(cu, E, la.b) : 0;
    auto la_next = [&](int* p) {
      load_pos(la, p);
      const int prev = la.b;
      la.advance(cu, E, B, la_nb);
      if (la.b != prev && la.b < B) la_nb = units_of(cu, E, la.b);
    };
    int pq[kPosAhead + 1][2] = {};   // positions of units i .. i + kPosAhead
#pragma unroll
    for (int q = 0; q < kPosAhead; ++q)
      if (q < n_units) la_next(pq[q]);
    for (int64_t i = 0; i < n_units; ++i) {
      const int s = static_cast<int>(i % kStages);
      const int b = cur.b, g = cur.g;
      if (b != at_b) {   // the sequence's compact-buffer offset and recalled positions, once per sequence
        at_b = b;
        n_b = units_of(cu, E, b);
        ckb = ld_dep(sa.ck + b);
        n_pos = (static_cast<int64_t>(ld_dep(sa.ck + b + 1)) - ckb) * kChunkTokens;
      }
      if (i + kPosAhead < n_units) la_next(pq[kPosAhead]);
      if (i >= kStages) {
        const unsigned par = static_cast<unsigned>(((i / kStages) - 1) & 1);
        int okw = 1;
        if (lane == 0) okw = mbar_wait_bounded(&empty[s], par, abort_flag) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) {
          if (lane == 0) {
            if (!*abort_flag) set_status(status, LSA_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          break;
        }
      }
      const uint32_t st = smem_base_p + s * kStageBytes;
      int64_t row_of[2];   // rows lane and lane + 32: compact-buffer row, or -1 (zeros)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int p = pq[0][h];
        const bool okp = p >= 0 && p < n_pos && ckb + p / kChunkTokens < sa.ck_chunks;
        if (!okp) set_status(status, LSA_DEV_ERR_BAD_CHUNK);
        row_of[h] = okp ? (g * sa.ck_chunks + ckb + p / kChunkTokens) * kChunkTokens + p % kChunkTokens : -1;
      }
      const int x = lane & 15;   // this lane's 16-byte piece of its row
#pragma unroll
      for (int it = 0; it < kChunkTokens / 2; ++it) {
        const int r = 2 * it + (lane >> 4);                       // the row this lane copies
        const int64_t row = __shfl_sync(0xffffffffu, row_of[it >> 4], r & 31);   // rows 0-31 in h = 0
        const uint32_t nb = row >= 0 ? 16u : 0u;
        const int64_t src = row >= 0 ? row * 16 + x : 0;
        const uint32_t off = (x >> 3) * kBoxBytes + r * 128 + (((x & 7) ^ (r & 7)) << 4);
        cp_async_16_zfill(st + off, sa.k_buf + src, nb);
        cp_async_16_zfill(st + 2 * kBoxBytes + off, sa.v_buf + src, nb);
      }
      cp_async_mbar_arrive_noinc(&full[s]);
      cur.advance(cu, E, B, n_b);
#pragma unroll
      for (int q = 0; q < kPosAhead; ++q) {
        pq[q][0] = pq[q + 1][0];
        pq[q][1] = pq[q + 1][1];
      }
    }
    cp_async_wait_all();   // every copy this lane issued has landed before the warp leaves
    return;
  }

  if (warp == kConsumerWarps) {
    // ====================== producer warp: TMA stream ========================
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t policy = l2_policy_evict_first();
      UnitCursor cur;
      cur.start(cu, E, B, u0);
      const int64_t n_units = u1 - u0;
      int64_t issued = 0;
      bool waited = !kv_unchanged;   // the local chunks are written by the preceding kernel
      int at_b = -1, cb = 0, n_kept_b = 0;
      for (int64_t i = 0; i < n_units; ++i) {
        const int s = static_cast<int>(i % kStages);
        if (i >= kStages) {
          const unsigned par = static_cast<unsigned>(((i / kStages) - 1) & 1);
          if (!mbar_wait_bounded(&empty[s], par, abort_flag)) {
            if (!*abort_flag) set_status(status, LSA_DEV_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
        if (cur.b != at_b) {   // the sequence's offsets, once per sequence
          at_b = cur.b;
          cb = cu(cur.b);
          n_kept_b = cu(cur.b + 1) - cb;
        }
        const bool local = E && cur.j == n_kept_b;
        uint8_t* st = smem + s * kStageBytes;
        if (local && !waited) {
          griddep_wait();
          waited = true;
        }
        // compact buffer: head-major rows (g, chunk, token); local chunks: (b, g, token)
        const int row = local ? (cur.b * kNumKVHeads + cur.g) * kChunkTokens
                              : (cur.g * static_cast<int>(buf_chunks) + cb + cur.j) * kChunkTokens;
        const CUtensorMap* mk = local ? &tm_kl : &tm_k;
        const CUtensorMap* mv = local ? &tm_vl : &tm_v;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        tma_load_2d(st, mk, 0, row, &full[s], policy);
        tma_load_2d(st + kBoxBytes, mk, 64, row, &full[s], policy);
        tma_load_2d(st + 2 * kBoxBytes, mv, 0, row, &full[s], policy);
        tma_load_2d(st + 3 * kBoxBytes, mv, 64, row, &full[s], policy);
        issued = i + 1;
        cur.advance(cu, E, B, n_kept_b + E);
      }
      if (*abort_flag) {
        // Let every copy already issued land before the CTA exits.
        int never = 0;
        for (int64_t i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
          mbar_wait_bounded(&full[i % kStages], static_cast<unsigned>((i / kStages) & 1), &never);
      }
    }
    return;
  }

  // ========================= consumer warps ==================================
  UnitCursor cur;
  cur.start(cu, E, B, u0);
  // While the previous kernel finishes, bring the first segment's 8 query rows
  // (2 KiB) into L2, so that the loads after the wait hit L2.  A prefetch puts
  // nothing in registers and L2 sees the previous kernel's stores, so this is
  // safe even if that kernel writes q.
  if (kv_unchanged && tid < 16)
    prefetch_l2(q + (static_cast<int64_t>(cur.b) * kNumQHeads + cur.g * kGroup) * kHeadDim + tid * 64);
  if (kv_unchanged) griddep_wait();
  zero_empty(tid, kConsumerThreads);
  const int grp = warp / kWarpsPerGroup;   // takes the units with unit_i % 2 == grp
  const int wig = warp % kWarpsPerGroup;   // 16-token slice of a unit
  const int gl = lane >> 2;   // row group of the mma fragments
  const int c4 = lane & 3;    // column pair of the mma fragments
  const int mi = lane >> 3, r8 = lane & 7;
  // ldmatrix row addresses of this lane (see the fragment maps in the header comment)
  const int krow = wig * 16 + r8 + ((mi & 1) << 3);
  const int kx = mi >> 1;
  const int vrow = wig * 16 + r8 + ((mi >> 1) << 3);
  const int vx = mi & 1;
  const uint32_t smem_base = smem_u32(smem);
  // Swizzled byte offsets of this lane's ldmatrix rows within a stage, for the
  // 8 k-steps of S^T (K boxes) and the 8 dim tiles of O^T (V boxes).
  uint32_t kofs[8], vofs[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    kofs[t] = (t >> 2) * kBoxBytes + krow * 128 + ((((t & 3) * 2 + kx) ^ (krow & 7)) << 4);
    vofs[t] = 2 * kBoxBytes + (t >> 2) * kBoxBytes + vrow * 128 + ((((t & 3) * 2 + vx) ^ (vrow & 7)) << 4);
  }

  const int hh = tid >> 5;          // combine: head within the group (warp-uniform)
  const int d0 = (tid & 31) * 4;    // 4 consecutive dims

  int64_t u = u0;
  int64_t unit_i = 0;
  while (u < u1) {
    const int b = cur.b, g = cur.g;
    const int cb = cu(b);
    const int n_kept_b = cu(b + 1) - cb;
    const int n_b = n_kept_b + E;   // units of the pair
    // Valid tokens of the pair's local unit (its last unit, when E = 1), and
    // the row that receives this step's own token (-1: none).
    int valid_local = 64, new_row = -1;
    if (E) {
      valid_local = ld_dep(local_len + b);
      if (valid_local < 0 || valid_local > kChunkTokens) {
        if (tid == 0 && g == 0) set_status(status, LSA_DEV_ERR_BAD_COUNT);
        valid_local = min(max(valid_local, 0), kChunkTokens);
      }
      if (app.k_new) {
        if (valid_local < kChunkTokens) {
          new_row = valid_local;
          valid_local += 1;
        } else if (tid == 0 && g == 0) {
          set_status(status, LSA_DEV_ERR_CAPACITY);   // the local chunk is full: the token is not appended
        }
      }
    }
    const int j0 = cur.j;
    const int64_t seg_cap = static_cast<int64_t>(j0) + (u1 - u);
    const int jend = seg_cap < n_b ? static_cast<int>(seg_cap) : n_b;
    const bool whole_pair = (j0 == 0 && jend == n_b);

    // Q^T fragments (B operand of S^T = K Q^T): head 8g+gl, dims 16t + 2c4 (+8).
    uint32_t bq[8][2];
    {
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          q + (static_cast<int64_t>(b) * kNumQHeads + g * kGroup + gl) * kHeadDim);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        bq[t][0] = ld_dep(qrow + 8 * t + c4);
        bq[t][1] = ld_dep(qrow + 8 * t + 4 + c4);
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    for (int jj = j0; jj < jend; ++jj, ++unit_i) {
      if (static_cast<int>(unit_i & 1) != grp) continue;   // the other group's unit
      const int s = static_cast<int>(unit_i % kStages);
      bool ok = !*abort_flag;
      if (ok) {
        ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((unit_i / kStages) & 1), abort_flag);
        if (!ok) {
          if (!*abort_flag) set_status(status, LSA_DEV_ERR_TIMEOUT);
          *abort_flag = 1;
        }
      }
      if (ok) {
        const uint32_t sbase = smem_base + s * kStageBytes;
        if (E && jj == n_kept_b && app.k_new) {
          if (wig == 0 && lane == 0 && g == 0) app.len_out[b] = valid_local;   // one writer per sequence
          if (new_row >= 0 && (new_row >> 4) == wig) {
            // This warp owns row new_row: lanes 0-15 write the token's K row,
            // lanes 16-31 its V row, into the tile (128-byte swizzle, as the
            // ldmatrix offsets read it) and into the local chunk in memory.
            const int kv = lane >> 4, x = lane & 15;
            const int64_t pg = static_cast<int64_t>(b) * kNumKVHeads + g;
            const uint4 val = ld_dep((kv ? app.v_new : app.k_new) + pg * 16 + x);
            const uint32_t off = (2 * kv + (x >> 3)) * kBoxBytes + new_row * 128 + (((x & 7) ^ (new_row & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sbase + off), "r"(val.x), "r"(val.y),
                         "r"(val.z), "r"(val.w)
                         : "memory");
            (kv ? app.v_local : app.k_local)[(pg * kChunkTokens + new_row) * 16 + x] = val;
            fence_proxy_async_smem();   // ordered before the TMA that refills this stage
            __syncwarp();
          }
        }
        // ---- S^T[16 tokens x 8 heads] = K[16 x 128] Q^T[128 x 8] ----------
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(sbase + kofs[t], a0, a1, a2, a3);
          mma_bf16_16816((t & 1) ? sb : sa, a0, a1, a2, a3, bq[t][0], bq[t][1]);
        }
        // s[0]: (token gl, head 2c4)  s[1]: (gl, 2c4+1)  s[2]: (gl+8, 2c4)  s[3]: (gl+8, 2c4+1)
        float s0 = (sa[0] + sb[0]) * scale_log2, s1 = (sa[1] + sb[1]) * scale_log2;
        float s2 = (sa[2] + sb[2]) * scale_log2, s3 = (sa[3] + sb[3]) * scale_log2;
        if (E && jj == n_kept_b) {   // local unit: tokens not yet decoded are masked
          const int tok = wig * 16 + gl;
          if (tok >= valid_local) s0 = s1 = -INFINITY;
          if (tok + 8 >= valid_local) s2 = s3 = -INFINITY;
        }
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        // Reference for the exponentials: the new max, or 0 while every score
        // seen is masked (keeps alpha and p at 0 instead of NaN).
        const float rf0 = mn0 == -INFINITY ? 0.f : mn0, rf1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = fast_exp2(m0 - rf0), al1 = fast_exp2(m1 - rf1);
        m0 = mn0;
        m1 = mn1;
        const float p0 = fast_exp2(s0 - rf0), p1 = fast_exp2(s1 - rf1);
        const float p2 = fast_exp2(s2 - rf0), p3 = fast_exp2(s3 - rf1);
        // P as a sum of two bf16 parts (P_hi + P_lo carries about 16 bits of
        // mantissa): a single bf16 rounding of P is too coarse when a softmax
        // spans only a few tokens.
        const uint32_t ptop = pack_bf16(p0, p1), pbot = pack_bf16(p2, p3);
        const uint32_t ptop_lo = pack_bf16(p0 - bf16_lo(ptop), p1 - bf16_hi(ptop));
        const uint32_t pbot_lo = pack_bf16(p2 - bf16_lo(pbot), p3 - bf16_hi(pbot));
        l0 = l0 * al0 + p0 + p2;
        l1 = l1 * al1 + p1 + p3;
        // Rescale only when some running max moved (warp-uniform branch); once
        // the maxima settle, alpha is exactly 1 and the 32 multiplies are skipped.
        if (__any_sync(0xffffffffu, (al0 != 1.f) | (al1 != 1.f))) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[i][0] *= al0;
            acc[i][1] *= al1;
            acc[i][2] *= al0;
            acc[i][3] *= al1;
          }
        }
        // P^T as the B operand (k = token, n = head): transpose the 8x8 blocks.
        const uint32_t pb0 = movmatrix_trans(ptop), pb1 = movmatrix_trans(pbot);
        const uint32_t pl0 = movmatrix_trans(ptop_lo), pl1 = movmatrix_trans(pbot_lo);
        // ---- O^T[128 dims x 8 heads] += V^T[128 x 16 tokens] (P_hi + P_lo)^T ---
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(sbase + vofs[i], a0, a1, a2, a3);
          mma_bf16_16816(acc[i], a0, a1, a2, a3, pb0, pb1);
          mma_bf16_16816(acc[i], a0, a1, a2, a3, pl0, pl1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- end of segment: combine the 8 warps --------------------------------
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    if (gl == 0) {
      mbuf[warp * kGroup + 2 * c4] = m0;
      mbuf[warp * kGroup + 2 * c4 + 1] = m1;
      lbuf[warp * kGroup + 2 * c4] = l0;
      lbuf[warp * kGroup + 2 * c4 + 1] = l1;
    }
    {
      float* ab = accbuf + warp * kGroup * kAccStride;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ab[(2 * c4) * kAccStride + 16 * i + gl] = acc[i][0];
        ab[(2 * c4 + 1) * kAccStride + 16 * i + gl] = acc[i][1];
        ab[(2 * c4) * kAccStride + 16 * i + gl + 8] = acc[i][2];
        ab[(2 * c4 + 1) * kAccStride + 16 * i + gl + 8] = acc[i][3];
      }
    }
    named_barrier(1, kConsumerThreads);

    float mw[kConsumerWarps], M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      mw[w] = mbuf[w * kGroup + hh];
      M = fmaxf(M, mw[w]);
    }
    float L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    const float Mref = M == -INFINITY ? 0.f : M;   // every score of the segment masked: o = 0
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float sc = fast_exp2(mw[w] - Mref);   // 0 for a warp that saw no unit of this segment
      L += sc * lbuf[w * kGroup + hh];
      const float4 x = *reinterpret_cast<const float4*>(accbuf + (w * kGroup + hh) * kAccStride + d0);
      o.x += sc * x.x; o.y += sc * x.y; o.z += sc * x.z; o.w += sc * x.w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int p = b * kNumKVHeads + g;
    if (whole_pair) {
      float* dst = out + (static_cast<int64_t>(b) * kNumQHeads + g * kGroup + hh) * kHeadDim + d0;
      *reinterpret_cast<float4*>(dst) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    } else {
      float* rec = records + static_cast<int64_t>(p + blockIdx.x) * kRecFloats;
      *reinterpret_cast<float4*>(rec + hh * kHeadDim + d0) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if ((tid & 31) == 0) rec[kGroup * kHeadDim + hh] = M + __log2f(L);
      // attn_merge_kernel folds the records of the pair once this grid is done.
    }
    named_barrier(1, kConsumerThreads);   // combine buffer free for the next segment

    // Move the cursor to the unit after this segment.
    u += jend - j0;
    cur.j = jend - 1;
    cur.advance(cu, E, B, n_b);
  }
}

// ---- split-K merge -----------------------------------------------------------
// A (sequence, KV head) pair whose units the grid split over CTAs
// [c_lo, c_hi] left one normalised partial per contributing CTA c (record
// p + c: o[8 heads][128] and the log-sum-exp of each head).  attn_merge_kernel
// runs as a programmatic dependent of the attention launch with the same grid
// size G: its CTA c takes, for each split pair that attention CTA c
// contributed to, the heads h with h = c - c_lo (mod n), n = c_hi - c_lo + 1,
// so the 8 heads of a pair are folded on up to 8 SMs at once.  Its CTAs start
// as attention CTAs exit and fix their tasks from the offsets while the
// slowest attention CTAs still stream; then they wait for the grid, stage the
// needed rows of the records in shared memory with one round of asynchronous
// copies (the log-sum-exps too, so no thread stalls on a load while issuing)
// and fold each (pair, head) in CTA order, so the result does not depend on
// timing.  256 threads, at most 64 registers each, 34 KiB.
constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergeItems = 64;       // (task, record) rows staged per round
// A CTA meets at most two split pairs (those of its first and last unit), and
// takes at most 4 heads of each (a split pair has n >= 2 contributors): at
// most 8 tasks, one per warp.
constexpr int kMergeTasks = kMergeWarps;

__global__ void __launch_bounds__(kMergeThreads, 4)
attn_merge_kernel(const int32_t* __restrict__ cu_raw, int shift, int E, int B, int64_t cap, int max_sel,
                  const float* __restrict__ records, float* __restrict__ out) {
  // Per staged row: 32 x 16 B of o, then the 16 B of the record that hold its
  // log-sum-exp (4 heads' worth; the row's head picks one).
  __shared__ __align__(16) float4 s_o[kMergeItems * 33];
  __shared__ int s_off[kMergeItems], s_loff[kMergeItems];   // float4 offsets from `records`
  __shared__ int t_rec[kMergeTasks], t_h[kMergeTasks], t_out[kMergeTasks], t_item0[kMergeTasks + 1];
  __shared__ int s_ntasks;
  griddep_launch_dependents();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // The offsets were final before the attention grid started (it waits for
  // their writer before it lets this grid launch, or they did not change); they
  // are read before the wait.
  const Offsets cu{cu_raw, shift};
  const bool bad = offsets_bad(cu, B, cap, shift != 0, max_sel);
  if (tid == 0) {
    int nt = 0, items = 0;
    const int T = bad ? 0 : 8 * (cu(B) + E * B);
    const Partition part(T, gridDim.x);
    const int c = blockIdx.x;
    const int u0 = part.start(c), u1 = part.start(c + 1);
    int prev_a = -1;
    for (int side = 0; side < 2 && u0 < u1; ++side) {
      const int u = side == 0 ? u0 : u1 - 1;
      const int b = seq_of_unit(cu, E, B, u);
      const int base = static_cast<int>(seq_unit_base(cu, E, b));
      const int n_b = units_of(cu, E, b);
      const int g = (u - base) / n_b;
      const int a_p = base + g * n_b;
      if (a_p == prev_a) break;          // the same pair at both ends of the range
      prev_a = a_p;
      const int lo = part.cta_of(a_p), hi = part.cta_of(a_p + n_b - 1);
      if (lo == hi) continue;            // whole in one CTA: written by the attention kernel
      const int n = hi - lo + 1;
      for (int h = c - lo; h < kGroup && nt < kMergeTasks; h += n) {
        t_rec[nt] = (b * kNumKVHeads + g) + lo;
        t_h[nt] = h;
        t_out[nt] = b * kNumQHeads + g * kGroup + h;
        t_item0[nt] = items;
        items += n;
        ++nt;
      }
    }
    t_item0[nt] = items;
    s_ntasks = nt;
  }
  __syncthreads();
  const int nt = s_ntasks;
  if (nt == 0) {
    griddep_wait();   // every CTA waits, so this grid never completes before the attention grid
    return;
  }
  const int items = t_item0[nt];
  // Source offsets of the rows of round i0, in float4 units: the row's o and
  // the 16-byte piece holding its log-sum-exp.
  auto fill = [&](int i0) {
    const int ni = min(kMergeItems, items - i0);
    for (int it = tid; it < ni; it += kMergeThreads) {
      const int gi = i0 + it;
      int t = 0;
      while (t + 1 < nt && t_item0[t + 1] <= gi) ++t;
      const int base = (t_rec[t] + (gi - t_item0[t])) * (kRecFloats / 4);
      s_off[it] = base + t_h[t] * (kHeadDim / 4);
      s_loff[it] = base + (kGroup * kHeadDim) / 4 + (t_h[t] >> 2);
    }
  };
  // Everything that does not need the records is done before the wait: the
  // code after it runs with cold instruction caches (the attention grid's
  // stream evicts them between launches), and every further stretch of code
  // costs a fetch round trip.
  fill(0);
  __syncthreads();
  griddep_wait();   // every CTA waits, so this grid never completes before the attention grid
  const float4* rec4 = reinterpret_cast<const float4*>(records);
  const int my0 = warp < nt ? t_item0[warp] : 0, my1 = warp < nt ? t_item0[warp + 1] : 0;
  const int hl = warp < nt ? (t_h[warp] & 3) : 0;   // this warp's log-sum-exp within its 16-byte piece
  float m = -INFINITY, den = 0.f;
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i0 = 0; i0 < items; i0 += kMergeItems) {
    if (i0 > 0) {   // rounds after the first (more than kMergeItems rows)
      fill(i0);
      __syncthreads();
    }
    const int ni = min(kMergeItems, items - i0);
    // One round of asynchronous 16-byte copies: per row its o and its lse piece.
    for (int x = tid; x < ni * 33; x += kMergeThreads) {
      const int it = x / 33, qd = x - it * 33;
      cp_async_16_cg(smem_u32(s_o + x), rec4 + (qd < 32 ? s_off[it] + qd : s_loff[it]));
    }
    cp_async_wait_all();
    __syncthreads();
    // Warp t folds task t's rows of this round, in CTA order.
    const int a = max(my0, i0), e = min(my1, i0 + ni);
    for (int gi = a; gi < e; ++gi) {
      const float4* row = s_o + (gi - i0) * 33;
      const float l = reinterpret_cast<const float*>(row + 32)[hl];
      const float m_new = fmaxf(m, l);
      const float mref = m_new == -INFINITY ? 0.f : m_new;   // every partial so far empty
      const float sc = fast_exp2(m - mref), w = fast_exp2(l - mref);
      const float4 x = row[lane];
      den = den * sc + w;
      r.x = r.x * sc + w * x.x;
      r.y = r.y * sc + w * x.y;
      r.z = r.z * sc + w * x.z;
      r.w = r.w * sc + w * x.w;
      m = m_new;
    }
    __syncthreads();
  }
  if (warp < nt) {
    const float id = den > 0.f ? 1.f / den : 0.f;
    reinterpret_cast<float4*>(out + static_cast<int64_t>(t_out[warp]) * kHeadDim)[lane] =
        make_float4(r.x * id, r.y * id, r.z * id, r.w * id);
  }
}

// Workspace: fp32 records[(B*8 + kMaxCtas)][kRecFloats], one slot per
// (pair p, contributing CTA c) at index p + c.  Each launch writes the slots it
// reads, so the contents left between calls do not matter.
size_t workspace_bytes(int B) {
  return (static_cast<size_t>(B) * kNumKVHeads + kMaxCtas) * kRecFloats * sizeof(float);
}

// Kernel attributes, set once per device.  The carve-out is left to the
// driver: the one it picks for the attention CTA's 166 KB leaves no room for a
// merge CTA beside it, so merge CTAs start as attention CTAs exit.  Asking for
// the largest carve-out lets them sit side by side, which gained 0.1 us per
// 500K step but cost 0.8 us per step of the token-level fine stage, whose next
// kernels then also start early and wait on the SMs.
inline cudaError_t set_kernel_attributes() {
  return cudaFuncSetAttribute(sparse_decode_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

// The merge of split pairs, as a programmatic dependent of the attention
// launch just issued on `stream` with `grid` CTAs.
inline cudaError_t launch_merge(int grid, const int32_t* cu, int shift, int E, int B, int64_t cap, int max_sel,
                                const float* records, float* out, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_merge_kernel, cu, shift, E, B, cap, max_sel, records, out);
}

}  // namespace attn
}  // namespace lsa

namespace {
std::mutex g_attn_mu;
bool g_attn_attr_set[64] = {};

int encode_kv_map(CUtensorMap* map, const void* base, int64_t buf_chunks) {
  lsa::EncodeTiledFn enc = lsa::tensor_map_encoder();
  if (!enc) return LSA_ERR_NO_DEVICE;
  // 2-D view of the compact buffer: rows = (chunk, KV head, token), 128 bf16 per row.
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(lsa::kHeadDim),
                              static_cast<cuuint64_t>(buf_chunks) * lsa::kNumKVHeads * lsa::kChunkTokens};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(lsa::kHeadDim) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(lsa::kChunkTokens)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LSA_OK : LSA_ERR_CUDA;
}
}  // namespace

extern "C" {

size_t lsa_attn_workspace_size(int B) {
  if (B <= 0 || B > LSA_MAX_BATCH) return 0;
  return lsa::attn::workspace_bytes(B);
}

}  // extern "C"

namespace {
// Shared launcher of every attention entry point: lsa_sparse_decode_attn,
// lsa_sparse_decode_attn_local (k_local == nullptr: no local units),
// lsa_sparse_decode_attn_append, lsa_sparse_decode_attn_selected and
// lsa_sparse_decode_attn_noalloc.  `records` (records_bytes long) holds the
// split-K partials: it must have room for (B * 8 + max_grid) records, and a
// launch whose grid would exceed max_grid is refused.
int attn_launch_records(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks,
                        const int32_t* cu_kept, int B, float softmax_scale, const void* k_local, const void* v_local,
                        const int32_t* local_len, float* out, float* records, size_t records_bytes, int max_grid,
                        unsigned int flags, void* stream, const lsa::attn::AppendArgs& app,
                        const lsa::attn::SelectArgs& sa) {
  using namespace lsa;
  if (!q || !k_buf || !v_buf || !cu_kept || !out || B <= 0 || buf_chunks <= 0) return LSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return LSA_ERR_INVALID_ARG;
  if (flags & ~static_cast<unsigned>(LSA_ATTN_KV_UNCHANGED)) return LSA_ERR_INVALID_ARG;
  const bool local = k_local != nullptr;
  if (local && (!v_local || !local_len)) return LSA_ERR_INVALID_ARG;
  if (B > LSA_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  // TMA row coordinates are 32-bit: (buf_chunks * 512) rows must fit.
  if (buf_chunks > (int64_t{1} << 22)) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(k_buf) || !aligned16(v_buf) || !aligned16(out) || !aligned16(records))
    return LSA_ERR_MISALIGNED;
  if (local && (!aligned16(k_local) || !aligned16(v_local))) return LSA_ERR_MISALIGNED;
  const size_t need = (static_cast<size_t>(B) * kNumKVHeads + static_cast<size_t>(max_grid)) * attn::kRecFloats *
                      sizeof(float);
  if (!records || records_bytes < need) return LSA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return LSA_ERR_NO_DEVICE;
  // buf_chunks bounds the kept total (cu_kept[B] lives on the device).
  const int grid = attn::grid_for_units(sms, static_cast<int64_t>(kNumKVHeads) * (buf_chunks + (local ? B : 0)),
                                        sa.sel ? attn::kMinIndexedUnitsPerCta : attn::kMinUnitsPerCta);
  if (grid > max_grid) return LSA_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(g_attn_mu);
    if (dev < 64 && !g_attn_attr_set[dev]) {
      if (attn::set_kernel_attributes() != cudaSuccess) {
        cudaGetLastError();
        return LSA_ERR_CUDA;
      }
      g_attn_attr_set[dev] = true;
    }
  }
  CUtensorMap tm_k, tm_v, tm_kl, tm_vl;
  int st = encode_kv_map(&tm_k, k_buf, buf_chunks);
  if (st != LSA_OK) return st;
  st = encode_kv_map(&tm_v, v_buf, buf_chunks);
  if (st != LSA_OK) return st;
  if (local) {   // the local chunks: [B][8][64][128], one chunk per sequence
    st = encode_kv_map(&tm_kl, k_local, B);
    if (st != LSA_OK) return st;
    st = encode_kv_map(&tm_vl, v_local, B);
    if (st != LSA_OK) return st;
  } else {
    tm_kl = tm_k;
    tm_vl = tm_v;
  }
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  // Launched as a programmatic dependent of the preceding kernel: its
  // prologue (and, with LSA_ATTN_KV_UNCHANGED, its K/V stream) overlaps the
  // tail of that kernel; the kernel waits for it before touching its outputs.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(attn::kThreads);
  cfg.dynamicSmemBytes = attn::kSmemBytes;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int kv_unchanged = (flags & LSA_ATTN_KV_UNCHANGED) ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, attn::sparse_decode_attn_kernel, tm_k, tm_v, tm_kl, tm_vl,
                         static_cast<const __nv_bfloat16*>(q), cu_kept, B, buf_chunks,
                         local ? local_len : static_cast<const int32_t*>(nullptr), scale_log2, out, records,
                         lsa_device_status_ptr(), kv_unchanged, app, sa) != cudaSuccess ||
      attn::launch_merge(static_cast<int>(cfg.gridDim.x), cu_kept, sa.sel ? 6 : 0, local ? 1 : 0, B, buf_chunks,
                         sa.max_sel, records, out, cfg.stream) != cudaSuccess) {
    cudaGetLastError();
    return LSA_ERR_CUDA;
  }
  return launch_status();
}

// The workspace entry points: the records live in the caller's workspace.
int attn_launch(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks, const int32_t* cu_kept,
                int B, float softmax_scale, const void* k_local, const void* v_local, const int32_t* local_len,
                float* out, void* workspace, size_t workspace_bytes, unsigned int flags, void* stream,
                const lsa::attn::AppendArgs& app = lsa::attn::AppendArgs{},
                const lsa::attn::SelectArgs& sa = lsa::attn::SelectArgs{}) {
  return attn_launch_records(q, k_buf, v_buf, buf_chunks, cu_kept, B, softmax_scale, k_local, v_local, local_len,
                             out, static_cast<float*>(workspace), workspace_bytes, lsa::attn::kMaxCtas, flags,
                             stream, app, sa);
}
}  // namespace

extern "C" {

int lsa_sparse_decode_attn(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks,
                           const int32_t* cu_kept, int B, float softmax_scale, float* out, void* workspace,
                           size_t workspace_bytes, unsigned int flags, void* stream) {
  return attn_launch(q, k_buf, v_buf, buf_chunks, cu_kept, B, softmax_scale, nullptr, nullptr, nullptr, out,
                     workspace, workspace_bytes, flags, stream);
}

int lsa_sparse_decode_attn_local(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks,
                                 const int32_t* cu_kept, int B, float softmax_scale, const void* k_local,
                                 const void* v_local, const int32_t* local_len, float* out, void* workspace,
                                 size_t workspace_bytes, unsigned int flags, void* stream) {
  if (!k_local) return LSA_ERR_INVALID_ARG;
  return attn_launch(q, k_buf, v_buf, buf_chunks, cu_kept, B, softmax_scale, k_local, v_local, local_len, out,
                     workspace, workspace_bytes, flags, stream);
}

int lsa_sparse_decode_attn_selected(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks,
                                    const int32_t* cu_kept, const int32_t* sel, const int32_t* cu_sel, int max_sel,
                                    int B, float softmax_scale, float* out, void* workspace, size_t workspace_bytes,
                                    unsigned int flags, void* stream) {
  using namespace lsa;
  if (!sel || !cu_sel || !cu_kept || !k_buf || !v_buf || max_sel <= 0 || B <= 0 || buf_chunks <= 0)
    return LSA_ERR_INVALID_ARG;
  if (max_sel % kChunkTokens != 0) return LSA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * max_sel >= (int64_t{1} << 31)) return LSA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(k_buf) || !aligned16(v_buf)) return LSA_ERR_MISALIGNED;
  const attn::SelectArgs sa{sel, cu_kept, max_sel, buf_chunks, static_cast<const uint4*>(k_buf),
                            static_cast<const uint4*>(v_buf)};
  // The kernel walks units of 64 selected tokens (cu_sel / 64); their number
  // is at most B * max_sel / 64, which stands in for the buffer size.
  const int64_t unit_cap = static_cast<int64_t>(B) * (max_sel / kChunkTokens);
  return attn_launch(q, k_buf, v_buf, unit_cap, cu_sel, B, softmax_scale, nullptr, nullptr, nullptr, out, workspace,
                     workspace_bytes, flags, stream, attn::AppendArgs{}, sa);
}

int lsa_sparse_decode_attn_append(const void* q, const void* k_buf, const void* v_buf, int64_t buf_chunks,
                                  const int32_t* cu_kept, int B, float softmax_scale, const void* k_new,
                                  const void* v_new, void* k_local, void* v_local, const int32_t* local_len_in,
                                  int32_t* local_len_out, float* out, void* workspace, size_t workspace_bytes,
                                  unsigned int flags, void* stream) {
  using namespace lsa;
  if (!k_local || !v_local || !k_new || !v_new || !local_len_in || !local_len_out) return LSA_ERR_INVALID_ARG;
  if (static_cast<const void*>(local_len_in) == static_cast<const void*>(local_len_out)) return LSA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new)) return LSA_ERR_MISALIGNED;
  const attn::AppendArgs app{static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
                             static_cast<uint4*>(k_local), static_cast<uint4*>(v_local), local_len_out};
  return attn_launch(q, k_buf, v_buf, buf_chunks, cu_kept, B, softmax_scale, k_local, v_local, local_len_in, out,
                     workspace, workspace_bytes, flags, stream, app);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// lsa_sparse_decode_attn_noalloc: the same decode step for callers that cannot
// allocate device memory.  Some callers have no device allocator of their own
// (a plain C host program, or a plug-in living inside a framework that owns
// all device memory and forbids cudaMalloc once it has started), and some
// cannot allocate at the moment they call (cudaMalloc may synchronise the
// device, which a latency-critical decode loop must not do).  For them the
// split-K scratch (the partial results) lives in a fixed
// array inside this library instead of a caller-provided workspace.
//
// The array is a file-scope __device__ variable of LSA_NOALLOC_SCRATCH_BYTES
// bytes: every GPU that loads the library holds it until the process exits.
// Its size fixes the limits: at most LSA_NOALLOC_MAX_BATCH sequences and a
// grid of at most LSA_NOALLOC_MAX_CTAS CTAs (one per SM); larger requests are
// rejected with LSA_ERR_UNSUPPORTED_SHAPE.  All calls on a device share the
// one array, so calls whose kernels may overlap on the GPU (different
// streams, or different host threads) race with each other and must be
// serialised by the caller.  Each launch writes the records it reads, so
// leftovers of an earlier call do not matter.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes =
    (static_cast<size_t>(LSA_NOALLOC_MAX_BATCH) * lsa::kNumKVHeads + LSA_NOALLOC_MAX_CTAS) * lsa::attn::kRecFloats *
    sizeof(float);
static_assert(kNoAllocScratchBytes == LSA_NOALLOC_SCRATCH_BYTES, "header constant out of date");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the scratch array for the current device.  The host-side
// symbol is only a stand-in, so the address is looked up once per device
// (with that device current) through cudaGetSymbolAddress.
int noalloc_setup(int dev, void** scratch) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return LSA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *scratch = g_noalloc_ptr[dev];
  return LSA_OK;
}
}  // namespace

extern "C" int lsa_sparse_decode_attn_noalloc(const void* q, const void* k_buf, const void* v_buf,
                                              int64_t buf_chunks, const int32_t* cu_kept, int B,
                                              float softmax_scale, float* out, void* stream) {
  using namespace lsa;
  if (!q || !k_buf || !v_buf || !cu_kept || !out || B <= 0 || buf_chunks <= 0) return LSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !isfinite(softmax_scale)) return LSA_ERR_INVALID_ARG;
  if (B > LSA_NOALLOC_MAX_BATCH) return LSA_ERR_UNSUPPORTED_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LSA_ERR_NO_DEVICE;
  }
  void* scratch = nullptr;
  const int st = noalloc_setup(dev, &scratch);
  if (st != LSA_OK) return st;
  // The same launch as lsa_sparse_decode_attn (grid, programmatic dependent
  // launch, merge), with the records in the static array; a grid beyond
  // LSA_NOALLOC_MAX_CTAS (a device of more than 512 SMs) is refused.
  return attn_launch_records(q, k_buf, v_buf, buf_chunks, cu_kept, B, softmax_scale, nullptr, nullptr, nullptr, out,
                             static_cast<float*>(scratch), kNoAllocScratchBytes, LSA_NOALLOC_MAX_CTAS, 0, stream,
                             attn::AppendArgs{}, attn::SelectArgs{});
}
