"""Plain fp64 CPU oracle for the Lookahead Sparse Attention (LSA) decode step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library and imports
nothing from it.  Every input arrives as a numpy array (bf16 values already
widened exactly to float32/float64 by the caller, or raw integers for the byte
copies); every floating-point step runs in float64.

What it computes, and the passages it follows
---------------------------------------------
Sources are the web pages about "FlashMemory-DeepSeek-V4: Lightning Index
Ultra-Long Context via Lookahead Sparse Attention" (cited below as *FM-DS-V4
summary*, with its section), the handbook page "DeepSeek-V4: Architecting for
Ultra-Long Contexts" (*DS-V4 handbook*, with its section) and the Korean review
of the same paper (*FM-DS-V4 review*, with its section).

1. ``index_scores`` -- the Neural Memory Indexer.  Every tau decode steps the
   indexer scores each historical chunk from the current query state against
   the chunk's cached indexer key (FM-DS-V4 summary, 1 Introduction and
   2.1 Architecture; DS-V4 handbook, "The Neural Memory Indexer", items 2-3),
   through a sigmoid (FM-DS-V4 review, 1. Key Terms, "Neural Memory Indexer")
   over a dot product (FM-DS-V4 summary, 3 Experiments "Limitations").  The
   specified form is score_c = sum_h w_h * sigmoid(q_h . k_c / sqrt(d_I)) over
   H_I = 16 indexer heads, d_I = 128.
2. ``topk_chunks`` -- keep the K highest-scoring chunks among all but the latest
   one, ordered by (score descending, chunk index ascending), and always keep
   the latest chunk (the non-offloadable recent context of FM-DS-V4 summary,
   2.1 Architecture).  The kept list is returned in ascending chunk order.
3. ``gather_chunks`` -- copy the kept chunks, in kept order, into one compact
   buffer, so that only the chunks the query needs stay resident on the GPU
   (FM-DS-V4 summary, Abstract and 2.1 Architecture).
4. ``sparse_decode_attn`` -- GQA decode attention over the kept tokens only:
   softmax(Q K^T / sqrt(d_k)) V per query head (DS-V4 handbook, "Grouped Query
   Attention (GQA) vs. Multi-Head Attention (MHA)", the attention equation), 64
   query heads sharing 8 KV heads, head dimension 128, every 8 consecutive query
   heads on one KV head (same section, the DeepSeek-V4 configuration list).
   Plain two-pass softmax, no splitting.
5. ``threshold_chunks`` -- the pages' own selection rule: sigmoid thresholding
   at 0.5 in place of a fixed top-k (FM-DS-V4 summary, 2.1 Architecture and
   2.4 Configuration), read as score_c / sum_h w_h > 0.5, latest chunk kept.
6. ``topk_chunks(..., n_local=L)`` -- the non-offloadable recent context kept
   beside the recalled chunks (FM-DS-V4 summary, 2.1 Architecture; the local
   window of 3 Experiments) generalised from the latest chunk to the latest L.
7. ``sparse_decode_attn(..., k_local, v_local, local_len)`` -- the tokens
   decoded inside the current window (the decoded window of FM-DS-V4 summary,
   3 Experiments) are appended before each step attends: attention then runs
   over the kept chunks plus the first local_len[b] tokens of the sequence's
   local chunk.
8. ``token_scores`` / ``topk_tokens`` / ``fine_decode_attn`` -- the second,
   token-level stage: native token-level scoring picks a fine-grained top-k of
   entries inside the recalled subset instead of the whole context (FM-DS-V4
   summary, 2.1 Architecture), k = 2048 tokens in the DSA lightning indexer
   (search page "lightning indexer", the Multi-layer Indexer abstract).  Every
   decode step scores each token of its sequence's recalled chunks with the
   step's indexer query, keeps the k best, and attends only those.

Readings taken where the pages are silent are listed in the design notes of
this repository and marked "Reading:" at the point of use.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, special cases reducing to library routines, brute force).
"""
from __future__ import annotations

import math

import numpy as np

# Shapes fixed by the method (DS-V4 handbook, GQA section: 64 query heads,
# 8 KV heads, head dim 128).  Indexer heads and dims: H_I = 16, d_I = 128.
# Chunk length: 64 tokens.
NUM_Q_HEADS = 64
NUM_KV_HEADS = 8
HEAD_DIM = 128
GROUP = NUM_Q_HEADS // NUM_KV_HEADS
CHUNK_TOKENS = 64
INDEX_HEADS = 16
INDEX_DIM = 128


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns (uint16/int16) to float64."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def _slot(chunk_table, b: int, c: int, max_chunks: int) -> int:
    # Reading: a missing table means the identity layout, slot = b*max_chunks + c.
    if chunk_table is None:
        return b * max_chunks + c
    return int(chunk_table[b, c])


def index_scores(q_idx, w, chunk_keys, chunk_table, n_chunks, max_chunks=None):
    """Indexer scores for every chunk of every sequence.

    q_idx      [B, H_I, d_I]  indexer query of the window (one per sequence).
    w          [H_I]          per-head indexer weights.
    chunk_keys [n_slots, d_I] cached indexer key of each physical chunk slot.
    chunk_table[B, max_chunks] logical chunk -> physical slot, or None.
    n_chunks   [B]            number of chunks in each sequence.

    Returns float64 [B, max_chunks]; entries c >= n_chunks[b] are NaN.
    score[b, c] = sum_h w_h * sigmoid(q_idx[b, h] . k[slot(b, c)] / sqrt(d_I)).
    """
    q_idx = np.asarray(q_idx, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    keys = np.asarray(chunk_keys, dtype=np.float64)
    n_chunks = np.asarray(n_chunks).astype(np.int64)
    B = q_idx.shape[0]
    if max_chunks is None:
        max_chunks = int(chunk_table.shape[1]) if chunk_table is not None else int(n_chunks.max(initial=0))
    out = np.full((B, max_chunks), np.nan, dtype=np.float64)
    for b in range(B):
        n = int(n_chunks[b])
        if n == 0:
            continue
        slots = np.array([_slot(chunk_table, b, c, max_chunks) for c in range(n)], dtype=np.int64)
        logits = q_idx[b] @ keys[slots].T / math.sqrt(INDEX_DIM)      # [H_I, n]
        sig = 1.0 / (1.0 + np.exp(-logits))                             # sigmoid, fp64 libm exp
        out[b, :n] = w @ sig                                            # weighted sum over heads
    return out


def topk_chunks(scores, n_chunks, k_per_seq, n_local=1):
    """Per-sequence kept chunk lists.

    The latest ``n_local`` chunks are always kept (the recent context; one
    chunk, the latest, by default).  Candidates are the chunks before them,
    0 .. n-1-n_local.  They are ordered by score descending, then chunk index
    ascending; the first K are kept, the recent chunks are added, and the list
    is returned in ascending order.  Reading: the recent chunks are outside the
    K budget, so exactly min(K, n-L) + L chunks are kept with L = min(n_local, n);
    K >= n-L keeps every chunk; n == 0 keeps none.
    """
    scores = np.asarray(scores, dtype=np.float64)
    out = []
    for b in range(len(n_chunks)):
        n = int(n_chunks[b])
        k = int(k_per_seq[b])
        if n == 0:
            out.append(np.zeros(0, dtype=np.int64))
            continue
        n_rec = min(int(n_local), n)
        cand = np.arange(n - n_rec, dtype=np.int64)
        s = scores[b, : n - n_rec]
        # np.lexsort sorts by the last key first: primary key -score, then index.
        order = np.lexsort((cand, -s))
        chosen = cand[order[: max(0, min(k, n - n_rec))]]
        recent = np.arange(n - n_rec, n, dtype=np.int64)
        kept = np.sort(np.concatenate([chosen, recent]))
        out.append(kept)
    return out


def threshold_chunks(scores, n_chunks, w, threshold=0.5, cap=None):
    """The pages' sigmoid-threshold selection (FM-DS-V4 summary, 2.1 and 2.4).

    Reading: a chunk is recalled when its weighted mean sigmoid probability
    score_c / sum_h w_h exceeds the threshold; the latest chunk is always kept.

    ``cap`` (one budget per sequence, optional): the pages want the resident
    KV cut to about a tenth (FM-DS-V4 summary, Abstract) but give the threshold
    no bound.  Reading: when more than cap[b] chunks pass, the cap[b] passing
    chunks with the highest scores are kept, by score descending then chunk
    index ascending (the tie rule of ``topk_chunks``), listed ascending.
    """
    scores = np.asarray(scores, dtype=np.float64)
    wsum = float(np.sum(np.asarray(w, dtype=np.float64)))
    out = []
    for b in range(len(n_chunks)):
        n = int(n_chunks[b])
        if n == 0:
            out.append(np.zeros(0, dtype=np.int64))
            continue
        cand = np.arange(n - 1, dtype=np.int64)
        chosen = cand[scores[b, : n - 1] / wsum > threshold]
        if cap is not None and len(chosen) > int(cap[b]):
            ranked = sorted(chosen.tolist(), key=lambda c: (-scores[b, c], c))
            chosen = np.sort(np.array(ranked[: int(cap[b])], dtype=np.int64))
        out.append(np.concatenate([chosen, np.array([n - 1], dtype=np.int64)]))
    return out


def cumulative_kept(kept_lists):
    """cu_kept[B+1]: start of each sequence's kept chunks in the compact buffer."""
    cu = np.zeros(len(kept_lists) + 1, dtype=np.int64)
    for b, k in enumerate(kept_lists):
        cu[b + 1] = cu[b] + len(k)
    return cu


def gather_chunks(k_pool, v_pool, chunk_table, kept_lists, max_chunks=None):
    """Copy kept chunks into the compact buffers, sequence by sequence, in kept order.

    Pools are [n_slots, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM] of any dtype; the
    copy is element-exact.  Returns (k_buf, v_buf, cu_kept).
    """
    if max_chunks is None and chunk_table is not None:
        max_chunks = chunk_table.shape[1]
    cu = cumulative_kept(kept_lists)
    total = int(cu[-1])
    k_buf = np.empty((total,) + tuple(k_pool.shape[1:]), dtype=k_pool.dtype)
    v_buf = np.empty((total,) + tuple(v_pool.shape[1:]), dtype=v_pool.dtype)
    for b, kept in enumerate(kept_lists):
        for j, c in enumerate(kept):
            s = _slot(chunk_table, b, int(c), max_chunks)
            k_buf[cu[b] + j] = k_pool[s]
            v_buf[cu[b] + j] = v_pool[s]
    return k_buf, v_buf, cu


def attend_one(q_h, K, V, scale):
    """softmax(q K^T * scale) V for one query vector over T tokens (two-pass)."""
    s = (K @ q_h) * scale          # [T]
    m = np.max(s)
    p = np.exp(s - m)
    return (p @ V) / np.sum(p)


def sparse_decode_attn(q, k_buf, v_buf, cu_kept, scale=None, seqs=None, heads=None,
                       k_local=None, v_local=None, local_len=None):
    """GQA decode attention of each query head over its sequence's kept tokens.

    q      [B, 64, 128]
    k_buf  [total_kept, 8, 64, 128], v_buf the same
    cu_kept[B+1]
    k_local, v_local [B, 8, 64, 128] and local_len [B] (optional): the tokens
    decoded in the current window; the first local_len[b] of them are attended
    after the kept chunks.
    Query head h reads KV head h // 8 (8 consecutive query heads per KV head).
    Returns float64 [B, 64, 128]; a sequence with no token to attend gives
    zeros (Reading: the empty softmax is defined as a zero output).
    ``seqs``/``heads`` restrict the work to a sample; other rows stay NaN.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    q = np.asarray(q, dtype=np.float64)
    B = q.shape[0]
    out = np.full((B, NUM_Q_HEADS, HEAD_DIM), np.nan, dtype=np.float64)
    seqs = range(B) if seqs is None else seqs
    heads = range(NUM_Q_HEADS) if heads is None else heads
    for b in seqs:
        lo, hi = int(cu_kept[b]), int(cu_kept[b + 1])
        n_loc = 0 if local_len is None else int(local_len[b])
        if hi == lo and n_loc == 0:
            out[b, list(heads)] = 0.0
            continue
        for g in range(NUM_KV_HEADS):
            group_heads = [h for h in heads if h // GROUP == g]
            if not group_heads:
                continue
            K = np.asarray(k_buf[lo:hi, g], dtype=np.float64).reshape(-1, HEAD_DIM)
            V = np.asarray(v_buf[lo:hi, g], dtype=np.float64).reshape(-1, HEAD_DIM)
            if n_loc:
                K = np.concatenate([K, np.asarray(k_local[b, g, :n_loc], dtype=np.float64)])
                V = np.concatenate([V, np.asarray(v_local[b, g, :n_loc], dtype=np.float64)])
            for h in group_heads:
                out[b, h] = attend_one(q[b, h], K, V, scale)
    return out


def token_scores(q_idx, w, token_keys, chunk_table, kept_lists, max_chunks=None):
    """Token-level indexer scores inside the recalled chunks of each sequence.

    q_idx      [B, H_I, d_I]         indexer query of the current decode step.
    token_keys [n_slots, 64, d_I]    cached indexer key of every token, by chunk slot.
    kept_lists                        recalled chunks of each sequence, ascending.
    Returns one float64 array per sequence of length 64 * len(kept): position
    p = 64 j + i is token i of the j-th recalled chunk (so positions follow
    the context order), and
        score[b, p] = sum_h w_h * sigmoid(q_idx[b, h] . key(p) / sqrt(d_I)).
    Reading: the pages name the token-level stage but not its formula; it is
    taken to be the indexer's own weighted-sigmoid form applied per token.
    """
    q_idx = np.asarray(q_idx, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    if max_chunks is None and chunk_table is not None:
        max_chunks = chunk_table.shape[1]
    out = []
    for b, kept in enumerate(kept_lists):
        if len(kept) == 0:
            out.append(np.zeros(0, dtype=np.float64))
            continue
        rows = [np.asarray(token_keys[_slot(chunk_table, b, int(c), max_chunks)], dtype=np.float64)
                for c in kept]
        K = np.concatenate(rows)                                        # [64 * n_kept, d_I]
        logits = q_idx[b] @ K.T / math.sqrt(INDEX_DIM)                  # [H_I, 64 * n_kept]
        out.append(w @ (1.0 / (1.0 + np.exp(-logits))))
    return out


def topk_tokens(scores_list, k):
    """The k best token positions of each sequence, by score descending then
    position ascending, returned ascending; every position when there are at
    most k (Reading: the same tie rule as the chunk selection)."""
    out = []
    for sc in scores_list:
        n = len(sc)
        if n <= k:
            out.append(np.arange(n, dtype=np.int64))
            continue
        order = sorted(range(n), key=lambda p: (-sc[p], p))
        out.append(np.sort(np.array(order[:k], dtype=np.int64)))
    return out


def fine_decode_attn(q, k_buf, v_buf, cu_kept, selected, scale=None, seqs=None, heads=None):
    """GQA decode attention over the selected tokens only.

    Token position p of sequence b is row p % 64 of compact chunk
    cu_kept[b] + p // 64; every KV head attends the same selected positions
    (one indexer score per token).  Other conventions as ``sparse_decode_attn``.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(HEAD_DIM)
    q = np.asarray(q, dtype=np.float64)
    B = q.shape[0]
    out = np.full((B, NUM_Q_HEADS, HEAD_DIM), np.nan, dtype=np.float64)
    seqs = range(B) if seqs is None else seqs
    heads = range(NUM_Q_HEADS) if heads is None else heads
    for b in seqs:
        sel = np.asarray(selected[b], dtype=np.int64)
        if sel.size == 0:
            out[b, list(heads)] = 0.0
            continue
        chunk = int(cu_kept[b]) + sel // CHUNK_TOKENS
        row = sel % CHUNK_TOKENS
        for g in range(NUM_KV_HEADS):
            group_heads = [h for h in heads if h // GROUP == g]
            if not group_heads:
                continue
            K = np.asarray(k_buf[chunk, g, row], dtype=np.float64)       # [n_sel, 128]
            V = np.asarray(v_buf[chunk, g, row], dtype=np.float64)
            for h in group_heads:
                out[b, h] = attend_one(q[b, h], K, V, scale)
    return out


def decode_window(q_idx, w, chunk_keys, chunk_table, n_chunks, k_per_seq,
                  k_pool, v_pool, q_steps, max_chunks=None, steps=None,
                  n_local=1, k_new=None, v_new=None):
    """One lookahead window: score, select, gather, then attention for each step.

    q_steps [T, B, 64, 128]: the decode-step queries of the window.
    n_local: recent chunks always kept (``topk_chunks``).
    k_new, v_new [T, B, 8, 128] (optional): the token each step decodes.  When
    given, the window is causal: step t first appends its own token to the
    sequence's local chunk, then attends the kept chunks plus the t + 1 tokens
    decoded so far in this window (FM-DS-V4 summary, 3 Experiments, the decoded
    window; Reading: the local chunk starts empty at every window).
    Returns (scores, kept_lists, cu_kept, outputs[T, B, 64, 128]).
    """
    scores = index_scores(q_idx, w, chunk_keys, chunk_table, n_chunks, max_chunks)
    kept = topk_chunks(scores, n_chunks, k_per_seq, n_local=n_local)
    k_buf, v_buf, cu = gather_chunks(k_pool, v_pool, chunk_table, kept, max_chunks)
    steps = range(q_steps.shape[0]) if steps is None else steps
    if k_new is None:
        outs = {t: sparse_decode_attn(q_steps[t], k_buf, v_buf, cu) for t in steps}
        return scores, kept, cu, outs
    T, B = q_steps.shape[0], q_steps.shape[1]
    # local chunk [B, 8, 64, 128]: token t of the window at position t
    k_loc = np.zeros((B, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM))
    v_loc = np.zeros_like(k_loc)
    k_loc[:, :, :T] = np.transpose(np.asarray(k_new, dtype=np.float64), (1, 2, 0, 3))
    v_loc[:, :, :T] = np.transpose(np.asarray(v_new, dtype=np.float64), (1, 2, 0, 3))
    outs = {t: sparse_decode_attn(q_steps[t], k_buf, v_buf, cu, k_local=k_loc, v_local=v_loc,
                                  local_len=[t + 1] * B) for t in steps}
    return scores, kept, cu, outs
