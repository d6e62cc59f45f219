"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test ties one oracle function to something other than its own formula:
a closed form, a special case that reduces to a library routine (scipy's
``expit``, torch's ``scaled_dot_product_attention``, Python's ``sorted``), an
invariant, or brute force on tiny inputs.  They are chosen so that a plausible
slip (a dropped scale, a sign, a head mapped to the wrong KV head, a transposed
operand, a wrong tie order, a lost latest chunk) fails at least one of them.
CPU only.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle

RNG = np.random.default_rng(1234)


def bf16_round(x):
    """Round float values to bf16 (nearest even) and widen back to float64."""
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


# ----------------------------------------------------------------- scoring ---

def test_score_zero_query_is_half_weight_sum():
    """q_I = 0: every logit is 0, sigmoid(0) = 1/2, so score = sum(w)/2 for every chunk."""
    B, N = 2, 7
    q = np.zeros((B, 16, 128))
    w = RNG.uniform(0, 1, 16)
    keys = bf16_round(RNG.standard_normal((B * N, 128)))
    s = oracle.index_scores(q, w, keys, None, [N, N], max_chunks=N)
    np.testing.assert_allclose(s, np.full((B, N), w.sum() / 2), rtol=1e-15, atol=0)


def test_score_closed_form_scale_and_head_weights():
    """q_h = a_h * ones, k = ones/8: q_h.k / sqrt(128) = a_h * 16 / sqrt(128) = a_h*sqrt(2).

    The score is then sum_h w_h * expit(a_h * sqrt(2)), computed here with scipy's
    expit.  Pins the 1/sqrt(d_I) scale (not 1/d_I, not none), the sigmoid sign and
    that head h uses weight w_h.
    """
    a = np.array([0, 1, -1, 2, -2, 3, 0.5, -0.5, 1, 0, -3, 2, 1, -1, 0.25, 4], dtype=np.float64)
    q = np.ones((1, 16, 128)) * a[None, :, None]
    keys = np.full((3, 128), 0.125)
    w = RNG.uniform(0, 1, 16)
    s = oracle.index_scores(q, w, keys, None, [3], max_chunks=3)
    expect = float(np.dot(w, expit(a * math.sqrt(2.0))))
    np.testing.assert_allclose(s[0], [expect] * 3, rtol=1e-14)
    # one-hot weights isolate each head
    for h in range(16):
        e = np.zeros(16)
        e[h] = 1.0
        s = oracle.index_scores(q, e, keys, None, [3], max_chunks=3)
        np.testing.assert_allclose(s[0, 0], expit(a[h] * math.sqrt(2.0)), rtol=1e-14)


def test_score_sigmoid_root2_high_precision():
    """sigmoid(sqrt 2) evaluated with 40-digit decimal arithmetic, independent of numpy."""
    from decimal import Decimal, getcontext
    getcontext().prec = 40
    expect = float(1 / (1 + (-Decimal(2).sqrt()).exp()))
    q = np.ones((1, 16, 128))
    keys = np.full((1, 128), 0.125)
    e = np.zeros(16)
    e[0] = 1.0
    s = oracle.index_scores(q, e, keys, None, [1], max_chunks=1)
    assert abs(s[0, 0] - expect) < 2e-16


def test_score_chunk_table_indirection():
    """score[b, c] depends only on the key in slot table[b, c].

    Slot s holds the key x_s * ones with x_s = s/64 (exact in bf16), so with q = ones
    on head 0 and w = e_0 the score of a slot is expit(sqrt(128) * x_s) in closed form.
    """
    B, M, S = 3, 6, 18
    keys = np.repeat((np.arange(S) / 64.0)[:, None], 128, axis=1)
    table = RNG.permutation(S)[: B * M].reshape(B, M)
    n = [6, 4, 0]
    q = np.zeros((B, 16, 128))
    q[:, 0, :] = 1.0
    e = np.zeros(16)
    e[0] = 1.0
    s = oracle.index_scores(q, e, keys, table, n)
    for b in range(B):
        for c in range(M):
            if c < n[b]:
                np.testing.assert_allclose(s[b, c], expit(math.sqrt(128) * table[b, c] / 64.0), rtol=1e-14)
            else:
                assert np.isnan(s[b, c])


def test_score_range_invariant():
    """0 < score < sum(w) on random bf16 inputs."""
    B, N = 2, 50
    q = bf16_round(RNG.standard_normal((B, 16, 128)))
    keys = bf16_round(RNG.standard_normal((B * N, 128)))
    w = RNG.uniform(0, 1, 16)
    s = oracle.index_scores(q, w, keys, None, [N, N], max_chunks=N)
    assert np.all(s > 0) and np.all(s < w.sum())


def test_score_brute_force_loops():
    """Independent triple loop with math.exp on a tiny paged case."""
    B, M = 2, 5
    q = bf16_round(RNG.standard_normal((B, 16, 128)))
    keys = bf16_round(RNG.standard_normal((12, 128)))
    table = RNG.permutation(12)[:10].reshape(B, M)
    w = RNG.uniform(0, 1, 16)
    s = oracle.index_scores(q, w, keys, table, [5, 3])
    for b in range(B):
        for c in range([5, 3][b]):
            tot = 0.0
            for h in range(16):
                dot = sum(q[b, h, i] * keys[table[b, c], i] for i in range(128))
                tot += w[h] * (1.0 / (1.0 + math.exp(-dot / math.sqrt(128))))
            assert abs(s[b, c] - tot) <= 1e-13 * abs(tot)


# ------------------------------------------------------------------- top-K ---

def _brute_topk(scores_row, n, k):
    if n == 0:
        return []
    cand = sorted(range(n - 1), key=lambda c: (-scores_row[c], c))
    return sorted(cand[: max(0, min(k, n - 1))] + [n - 1])


@pytest.mark.parametrize("trial", range(30))
def test_topk_matches_full_sort(trial):
    rng = np.random.default_rng(trial)
    B = int(rng.integers(1, 5))
    M = int(rng.integers(1, 65))
    n = rng.integers(0, M + 1, B)
    k = rng.integers(0, M + 2, B)
    if trial % 3 == 0:      # many exact ties
        scores = rng.integers(0, 4, (B, M)).astype(np.float64)
    else:
        scores = rng.standard_normal((B, M))
    got = oracle.topk_chunks(scores, n, k)
    for b in range(B):
        assert list(got[b]) == _brute_topk(list(scores[b]), int(n[b]), int(k[b]))


def test_topk_all_ties_closed_form():
    """All scores equal: the lowest indices win: kept = {0..K-1} + {N-1}."""
    N, K = 40, 9
    got = oracle.topk_chunks(np.full((1, N), 0.37), [N], [K])
    assert list(got[0]) == list(range(K)) + [N - 1]


def test_topk_boundaries():
    s = RNG.standard_normal((1, 10))
    assert list(oracle.topk_chunks(s, [10], [9])[0]) == list(range(10))      # K = N-1
    assert list(oracle.topk_chunks(s, [10], [50])[0]) == list(range(10))     # K > N-1
    assert list(oracle.topk_chunks(s, [1], [4])[0]) == [0]                   # only the latest
    assert list(oracle.topk_chunks(s, [0], [4])[0]) == []                    # empty sequence
    assert list(oracle.topk_chunks(s, [10], [0])[0]) == [9]                  # K = 0


def test_topk_latest_not_double_counted():
    """The latest chunk has the highest score: it is kept once, plus K others."""
    s = np.arange(12, dtype=np.float64)[None, :]          # latest (11) scores highest
    got = oracle.topk_chunks(s, [12], [3])[0]
    assert list(got) == [8, 9, 10, 11]
    s2 = -np.arange(12, dtype=np.float64)[None, :]        # latest scores lowest
    assert list(oracle.topk_chunks(s2, [12], [3])[0]) == [0, 1, 2, 11]


@pytest.mark.parametrize("trial", range(12))
def test_topk_local_window_matches_full_sort(trial):
    """Recent context of L chunks: brute force with Python's sorted()."""
    rng = np.random.default_rng(100 + trial)
    M = int(rng.integers(1, 50))
    n = int(rng.integers(0, M + 1))
    k = int(rng.integers(0, M + 2))
    L = int(rng.integers(1, 6))
    scores = rng.integers(0, 3, (1, M)).astype(np.float64) if trial % 2 else rng.standard_normal((1, M))
    got = list(oracle.topk_chunks(scores, [n], [k], n_local=L)[0])
    if n == 0:
        assert got == []
        return
    r = min(L, n)
    cand = sorted(range(n - r), key=lambda c: (-scores[0, c], c))
    assert got == sorted(cand[: max(0, min(k, n - r))] + list(range(n - r, n)))


def test_topk_local_window_default_is_latest_chunk():
    s = RNG.standard_normal((2, 30))
    a = oracle.topk_chunks(s, [30, 7], [5, 2])
    b = oracle.topk_chunks(s, [30, 7], [5, 2], n_local=1)
    assert all(list(x) == list(y) for x, y in zip(a, b))


def test_attention_local_tokens_equal_an_appended_chunk():
    """A full local chunk (64 decoded tokens) attends exactly like one more kept
    chunk at the end of the compact buffer; local_len = 0 changes nothing."""
    rng = np.random.default_rng(31)
    k_buf, v_buf = _rand_bufs(3, rng)
    kl, vl = _rand_bufs(2, rng)           # [B=2][8][64][128]
    q = bf16_round(rng.standard_normal((2, 64, 128)))
    cu = [0, 2, 3]
    full = oracle.sparse_decode_attn(q, k_buf, v_buf, cu, k_local=kl, v_local=vl, local_len=[64, 64])
    k_cat = np.concatenate([k_buf[0:2], kl[0:1], k_buf[2:3], kl[1:2]])
    v_cat = np.concatenate([v_buf[0:2], vl[0:1], v_buf[2:3], vl[1:2]])
    ref = oracle.sparse_decode_attn(q, k_cat, v_cat, [0, 3, 5])
    np.testing.assert_allclose(full, ref, rtol=1e-12, atol=1e-15)
    none = oracle.sparse_decode_attn(q, k_buf, v_buf, cu, k_local=kl, v_local=vl, local_len=[0, 0])
    np.testing.assert_array_equal(none, oracle.sparse_decode_attn(q, k_buf, v_buf, cu))


def test_attention_local_tokens_only_closed_form():
    """No kept chunk, local_len = 3 tokens with keys (0, s, 2s) along e_0 and values e_j:
    the output is the softmax of (0, s, 2s)/sqrt(128) over the first 3 dims."""
    kl = np.zeros((1, 8, 64, 128))
    vl = np.zeros((1, 8, 64, 128))
    for j in range(3):
        kl[0, :, j, 0] = 4.0 * j
        vl[0, :, j, j] = 1.0
    kl[0, :, 3:, 0] = 1e3                 # beyond local_len: must be ignored
    q = np.zeros((1, 64, 128))
    q[0, :, 0] = 1.0
    got = oracle.sparse_decode_attn(q, np.zeros((0, 8, 64, 128)), np.zeros((0, 8, 64, 128)), [0, 0],
                                    k_local=kl, v_local=vl, local_len=[3])
    e = np.array([math.exp(4.0 * j / math.sqrt(128)) for j in range(3)])
    np.testing.assert_allclose(got[0, 17, :3], e / e.sum(), rtol=1e-13)
    assert np.all(got[0, :, 3:] == 0)


def test_threshold_rule():
    w = np.array([0.5, 1.5] + [0.0] * 14)
    s = np.array([[0.2, 1.2, 1.0, 1.01, 0.0]]) * 1.0     # score / sum(w) = s / 2
    got = oracle.threshold_chunks(s, [5], w)[0]
    assert list(got) == [1, 3, 4]                           # 0.6 and 0.505 pass; latest kept


def test_threshold_extremes_and_nesting():
    """The weighted mean of sigmoids lies strictly between 0 and 1, so threshold 0
    keeps every chunk and threshold 1 keeps only the latest; a higher threshold
    never keeps a chunk a lower one dropped; a sequence of one chunk keeps it and
    an empty one keeps nothing.  Scores come from the oracle's own indexer on
    random queries and keys."""
    rng = np.random.default_rng(77)
    B, N = 3, 40
    q = bf16_round(rng.standard_normal((B, 16, 128)) * 3.0)
    keys = bf16_round(rng.standard_normal((B * N, 128)))
    w = rng.uniform(0, 1, 16)
    n = [N, 1, 0]
    s = oracle.index_scores(q, w, keys, None, n, max_chunks=N)
    assert list(oracle.threshold_chunks(s, n, w, threshold=0.0)[0]) == list(range(N))
    assert list(oracle.threshold_chunks(s, n, w, threshold=1.0)[0]) == [N - 1]
    prev = set(range(N))
    for t in np.linspace(0.05, 0.95, 19):
        got = oracle.threshold_chunks(s, n, w, threshold=float(t))
        assert list(got[1]) == [0] and list(got[2]) == []
        cur = set(got[0].tolist())
        assert N - 1 in cur and cur <= prev
        prev = cur
    assert len(prev) < N          # the random queries spread the scores across thresholds


@pytest.mark.parametrize("trial", range(6))
def test_threshold_cap_matches_full_sort(trial):
    """Under a budget the capped rule keeps the cap best passing chunks: a full
    Python sort of the passing chunks by (score descending, index ascending),
    on random scores with heavy ties; a cap at or above the passing count
    changes nothing, and cap 0 keeps only the latest chunk."""
    rng = np.random.default_rng(300 + trial)
    B, N = 5, 60
    w = rng.uniform(0, 1, 16)
    s = rng.integers(0, 9, size=(B, N)) * (w.sum() / 8.0)     # score / sum(w) in {0, 1/8, ..., 1}: ties
    n = [60, 45, 2, 1, 0]
    t = 0.3
    plain = oracle.threshold_chunks(s, n, w, threshold=t)
    for cap in ([0, 0, 0, 0, 0], [7, 3, 1, 5, 2], [100] * 5, [len(p) - 1 for p in plain]):
        cap = [max(c, 0) for c in cap]
        got = oracle.threshold_chunks(s, n, w, threshold=t, cap=cap)
        for b in range(B):
            if n[b] == 0:
                assert list(got[b]) == []
                continue
            passing = [c for c in range(n[b] - 1) if s[b, c] / w.sum() > t]
            best = sorted(passing, key=lambda c: (-s[b, c], c))[: cap[b]]
            assert list(got[b]) == sorted(best) + [n[b] - 1]
            if cap[b] >= len(passing):
                assert list(got[b]) == list(plain[b])


def test_threshold_cap_is_topk_when_the_budget_binds():
    """Every passing chunk outscores every other, so when more pass than the
    budget the capped rule equals the top-K rule with K = cap."""
    rng = np.random.default_rng(310)
    w = rng.uniform(0, 1, 16)
    s = rng.uniform(0.0, w.sum(), size=(3, 200))
    n, cap = [200, 150, 90], [20, 5, 60]
    got = oracle.threshold_chunks(s, n, w, threshold=0.2, cap=cap)
    ref = oracle.topk_chunks(s, n, cap)
    for b in range(3):
        assert list(got[b]) == list(ref[b])


# ------------------------------------------------------------------ gather ---

def test_gather_closed_form_positions():
    """Pools filled with their own flat index: the gathered element at
    (i = cu[b] + j, h, t, d) must equal the flat index of (table[b, kept_j], h, t, d)."""
    S, B, M = 11, 2, 5
    shape = (S, 8, 64, 128)
    k_pool = np.arange(np.prod(shape), dtype=np.int64).reshape(shape)
    v_pool = -k_pool
    table = RNG.permutation(S)[: B * M].reshape(B, M)
    kept = [np.array([0, 3, 4]), np.array([1, 4])]
    k_buf, v_buf, cu = oracle.gather_chunks(k_pool, v_pool, table, kept)
    assert list(cu) == [0, 3, 5]
    h, t, d = np.meshgrid(np.arange(8), np.arange(64), np.arange(128), indexing="ij")
    for b in range(B):
        for j, c in enumerate(kept[b]):
            flat = ((table[b, c] * 8 + h) * 64 + t) * 128 + d
            assert np.array_equal(k_buf[cu[b] + j], flat)
            assert np.array_equal(v_buf[cu[b] + j], -flat)


# --------------------------------------------------------------- attention ---

def _rand_bufs(n_chunks, rng):
    k = bf16_round(rng.standard_normal((n_chunks, 8, 64, 128)))
    v = bf16_round(rng.standard_normal((n_chunks, 8, 64, 128)))
    return k, v


def test_attention_all_chunks_equals_dense_sdpa():
    """With every chunk kept, the result is dense GQA attention: torch's fp64
    scaled_dot_product_attention with K/V repeated 8x per KV head."""
    rng = np.random.default_rng(7)
    B, n = 2, [3, 2]
    cu = np.array([0, 3, 5])
    k_buf, v_buf = _rand_bufs(5, rng)
    q = bf16_round(rng.standard_normal((B, 64, 128)))
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, cu)
    for b in range(B):
        K = torch.from_numpy(k_buf[cu[b]:cu[b + 1]]).permute(1, 0, 2, 3).reshape(8, -1, 128)
        V = torch.from_numpy(v_buf[cu[b]:cu[b + 1]]).permute(1, 0, 2, 3).reshape(8, -1, 128)
        K = K.repeat_interleave(8, dim=0)
        V = V.repeat_interleave(8, dim=0)
        Q = torch.from_numpy(q[b]).reshape(64, 1, 128)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).reshape(64, 128).numpy()
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-14)


def test_attention_identical_keys_give_mean_of_v():
    rng = np.random.default_rng(8)
    k_buf, v_buf = _rand_bufs(3, rng)
    k_buf[:] = k_buf[0, 0, 0]               # every key equal
    q = bf16_round(rng.standard_normal((1, 64, 128)))
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, [0, 3])
    for h in range(64):
        g = h // 8
        np.testing.assert_allclose(got[0, h], v_buf[:, g].reshape(-1, 128).mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_single_chunk_closed_form():
    """q = e_0, k_j = (s_j, 0, ...), v_j = e_j (j < 64): o_h[j] = softmax_j(s_j / sqrt(128))."""
    s_int = (np.arange(64) % 7) - 3.0
    k = np.zeros((1, 8, 64, 128))
    k[0, :, :, 0] = s_int
    v = np.zeros((1, 8, 64, 128))
    for j in range(64):
        v[0, :, j, j] = 1.0
    q = np.zeros((1, 64, 128))
    q[0, :, 0] = 1.0
    got = oracle.sparse_decode_attn(q, k, v, [0, 1])
    e = np.array([math.exp(x / math.sqrt(128)) for x in s_int])
    expect = np.zeros(128)
    expect[:64] = e / e.sum()
    for h in range(64):
        np.testing.assert_allclose(got[0, h], expect, rtol=1e-13, atol=1e-16)


def test_attention_gqa_head_mapping():
    """V of KV head g is the constant g+1: every query head h must return h // 8 + 1."""
    rng = np.random.default_rng(9)
    k_buf, v_buf = _rand_bufs(2, rng)
    for g in range(8):
        v_buf[:, g] = g + 1.0
    q = bf16_round(rng.standard_normal((1, 64, 128)))
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, [0, 2])
    for h in range(64):
        np.testing.assert_allclose(got[0, h], np.full(128, h // 8 + 1.0), rtol=1e-13)


def test_attention_scale_pin_two_tokens():
    """Two tokens with logits 0 and 1 after scaling: weights 1/(1+e) and e/(1+e)."""
    k = np.zeros((1, 8, 64, 128))
    v = np.zeros((1, 8, 64, 128))
    # token 0: k = 0, v = (1, 0, ..); token 1: k = sqrt(128) e_0, v = (0, 1, ..);
    # tokens 2..63 get a very negative logit (k = -sqrt(128)*40 e_0) and v = 0.
    k[0, :, 1, 0] = math.sqrt(128)
    k[0, :, 2:, 0] = -math.sqrt(128) * 40
    v[0, :, 0, 0] = 1.0
    v[0, :, 1, 1] = 1.0
    q = np.zeros((1, 64, 128))
    q[0, :, 0] = 1.0
    got = oracle.sparse_decode_attn(q, k, v, [0, 1])
    np.testing.assert_allclose(got[0, 5, 0], 1 / (1 + math.e), rtol=1e-13)
    np.testing.assert_allclose(got[0, 5, 1], math.e / (1 + math.e), rtol=1e-13)


def test_attention_large_logits_stay_finite():
    """Logits 1000 and 1001 (scaled): the softmax is shift-invariant, so the weights are
    still 1/(1+e) and e/(1+e); an implementation without the max shift overflows."""
    k = np.zeros((1, 8, 64, 128))
    v = np.zeros((1, 8, 64, 128))
    k[0, :, 0, 0] = 1000 * math.sqrt(128)
    k[0, :, 1, 0] = 1001 * math.sqrt(128)
    k[0, :, 2:, 0] = -1000 * math.sqrt(128)
    v[0, :, 0, 0] = 1.0
    v[0, :, 1, 1] = 1.0
    q = np.zeros((1, 64, 128))
    q[0, :, 0] = 1.0
    got = oracle.sparse_decode_attn(q, k, v, [0, 1])
    np.testing.assert_allclose(got[0, 63, :2], [1 / (1 + math.e), math.e / (1 + math.e)], rtol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_attention_split_and_lse_merge_equal_one_pass(seed):
    """Split-K invariant (rows a6 + a7): cutting the kept tokens of a (sequence,
    KV head) pair at arbitrary points, normalising each part by its own softmax,
    and folding the parts in order with base-2 log-sum-exp weights and a running
    maximum (an empty part included) gives the oracle's one-pass attention to
    rounding, for any number of parts, parts of one token among them."""
    rng = np.random.default_rng(100 + seed)
    n = 3
    k_buf, v_buf = _rand_bufs(n, rng)
    q = bf16_round(rng.standard_normal((1, 64, 128)))
    ref = oracle.sparse_decode_attn(q, k_buf, v_buf, [0, n])
    T = 64 * n
    c = 1.0 / math.sqrt(128) / math.log(2.0)          # logits in base 2
    for h in (0, 9, 63):
        g = h // 8
        K = k_buf[:, g].reshape(T, 128)
        V = v_buf[:, g].reshape(T, 128)
        cuts = sorted(set(rng.integers(1, T, 2 + 3 * seed).tolist()) | {1, T - 1})
        bounds = [0] + cuts + [T]
        parts = []
        for a, b in zip(bounds[:-1], bounds[1:]):
            s = (K[a:b] @ q[0, h]) * c
            mx = s.max()
            p = np.exp2(s - mx)
            parts.append((mx + math.log2(p.sum()), (p @ V[a:b]) / p.sum()))
        parts.insert(len(parts) // 2, (-math.inf, np.zeros(128)))   # a part with no valid token
        m, den, acc = -math.inf, 0.0, np.zeros(128)
        for lse, o in parts:
            m_new = max(m, lse)
            mref = 0.0 if m_new == -math.inf else m_new
            sc, w = np.exp2(m - mref), np.exp2(lse - mref)
            den, acc, m = den * sc + w, acc * sc + w * o, m_new
        np.testing.assert_allclose(acc / den, ref[0, h], rtol=1e-12, atol=1e-14)


def test_attention_chunk_permutation_invariance():
    rng = np.random.default_rng(10)
    k_buf, v_buf = _rand_bufs(4, rng)
    q = bf16_round(rng.standard_normal((1, 64, 128)))
    a = oracle.sparse_decode_attn(q, k_buf, v_buf, [0, 4])
    p = [2, 0, 3, 1]
    b = oracle.sparse_decode_attn(q, k_buf[p], v_buf[p], [0, 4])
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_attention_empty_sequence_is_zero():
    rng = np.random.default_rng(11)
    k_buf, v_buf = _rand_bufs(2, rng)
    q = bf16_round(rng.standard_normal((3, 64, 128)))
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, [0, 2, 2, 2])
    assert np.all(got[1] == 0) and np.all(got[2] == 0)
    assert np.all(np.isfinite(got[0]))


def test_bf16_bits_widening():
    x = torch.tensor([1.0, -2.5, 3.140625, 0.0, -0.0, 65280.0]).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy()
    np.testing.assert_array_equal(oracle.bf16_bits_to_f64(bits), x.to(torch.float64).numpy())


def test_decode_window_composition():
    """A whole window equals its stages run one after another (tiny sizes)."""
    rng = np.random.default_rng(12)
    N, K = 10, 3
    keys = bf16_round(rng.standard_normal((N, 128)))
    kp, vp = _rand_bufs(N, rng)
    q_idx = bf16_round(rng.standard_normal((1, 16, 128)))
    w = rng.uniform(0, 1, 16)
    qs = bf16_round(rng.standard_normal((2, 1, 64, 128)))
    scores, kept, cu, outs = oracle.decode_window(q_idx, w, keys, None, [N], [K], kp, vp, qs, max_chunks=N)
    assert len(kept[0]) == K + 1 and kept[0][-1] == N - 1
    ref = oracle.sparse_decode_attn(qs[1], kp[kept[0]], vp[kept[0]], [0, K + 1])
    np.testing.assert_array_equal(outs[1], ref)


def test_decode_window_causal_equals_dense_sdpa_over_kept_and_decoded_tokens():
    """Causal window with a recent window of 2 chunks: step t attends exactly the
    tokens of the kept chunks followed by the t + 1 tokens decoded so far.  The
    reference is torch's fp64 scaled_dot_product_attention over that token list."""
    rng = np.random.default_rng(41)
    N, K, T = 10, 3, 5
    keys = bf16_round(rng.standard_normal((N, 128)))
    kp, vp = _rand_bufs(N, rng)
    q_idx = bf16_round(rng.standard_normal((1, 16, 128)))
    w = rng.uniform(0, 1, 16)
    qs = bf16_round(rng.standard_normal((T, 1, 64, 128)))
    k_new = bf16_round(rng.standard_normal((T, 1, 8, 128)))
    v_new = bf16_round(rng.standard_normal((T, 1, 8, 128)))
    scores, kept, cu, outs = oracle.decode_window(q_idx, w, keys, None, [N], [K], kp, vp, qs, max_chunks=N,
                                                  n_local=2, k_new=k_new, v_new=v_new)
    assert len(kept[0]) == K + 2 and list(kept[0][-2:]) == [N - 2, N - 1]
    for t in (0, 2, T - 1):
        Kc = torch.from_numpy(kp[kept[0]]).permute(1, 0, 2, 3).reshape(8, -1, 128)
        Vc = torch.from_numpy(vp[kept[0]]).permute(1, 0, 2, 3).reshape(8, -1, 128)
        Kd = torch.from_numpy(k_new[: t + 1, 0]).permute(1, 0, 2)       # [8, t+1, 128]
        Vd = torch.from_numpy(v_new[: t + 1, 0]).permute(1, 0, 2)
        Kall = torch.cat([Kc, Kd], dim=1).repeat_interleave(8, dim=0)
        Vall = torch.cat([Vc, Vd], dim=1).repeat_interleave(8, dim=0)
        Q = torch.from_numpy(qs[t, 0]).reshape(64, 1, 128)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, Kall, Vall).reshape(64, 128).numpy()
        np.testing.assert_allclose(outs[t][0], ref, rtol=1e-12, atol=1e-14)


# ------------------------------------------------- token-level fine stage ---

def _token_case(rng, n_slots=7, B=2, max_chunks=5):
    tok_keys = bf16_round(rng.standard_normal((n_slots, 64, 128)))
    table = np.array([[3, 0, 6, 1, 2], [5, 4, 0, 0, 0]], dtype=np.int64)[:B, :max_chunks]
    kept = [np.array([0, 2, 4]), np.array([1])]
    q_idx = bf16_round(rng.standard_normal((B, 16, 128)))
    w = rng.uniform(0, 1, 16)
    return tok_keys, table, kept, q_idx, w


def test_token_scores_equal_chunk_scores_of_per_token_keys():
    """Every token scored like a chunk whose indexer key is that token's key: the
    pinned chunk scorer over a table that maps position p = 64 j + i to the flat
    row 64 * slot(kept[j]) + i gives the same numbers."""
    rng = np.random.default_rng(51)
    tok_keys, table, kept, q_idx, w = _token_case(rng)
    got = oracle.token_scores(q_idx, w, tok_keys, table, kept)
    flat = tok_keys.reshape(-1, 128)
    for b in range(2):
        rows = np.array([64 * table[b, c] + i for c in kept[b] for i in range(64)])
        ref = oracle.index_scores(q_idx[b:b + 1], w, flat, rows[None, :], [len(rows)])[0]
        np.testing.assert_allclose(got[b], ref, rtol=1e-14, atol=0)


def test_token_scores_brute_force_loops():
    rng = np.random.default_rng(52)
    tok_keys, table, kept, q_idx, w = _token_case(rng)
    got = oracle.token_scores(q_idx, w, tok_keys, table, kept)
    for b, p in ((0, 0), (0, 64 + 17), (0, 191), (1, 63)):
        slot = table[b, kept[b][p // 64]]
        key = tok_keys[slot, p % 64]
        s = 0.0
        for h in range(16):
            dot = sum(float(q_idx[b, h, d]) * float(key[d]) for d in range(128))
            s += float(w[h]) / (1.0 + math.exp(-dot / math.sqrt(128)))
        assert abs(got[b][p] - s) <= 1e-12 * abs(s)
    assert len(got[0]) == 192 and len(got[1]) == 64


def test_token_scores_zero_query_is_half_weight_sum():
    rng = np.random.default_rng(53)
    tok_keys, table, kept, q_idx, w = _token_case(rng)
    got = oracle.token_scores(np.zeros_like(q_idx), w, tok_keys, table, kept)
    for b in range(2):
        np.testing.assert_allclose(got[b], 0.5 * w.sum(), rtol=1e-15)


@pytest.mark.parametrize("trial", range(4))
def test_topk_tokens_matches_rank_count_definition(trial):
    """Position p is selected iff fewer than k positions beat it, where q beats p
    when s_q > s_p or (s_q == s_p and q < p); ties are frequent on purpose."""
    rng = np.random.default_rng(60 + trial)
    n = int(rng.integers(1, 300))
    k = int(rng.integers(0, 320))
    sc = np.round(rng.uniform(0, 1, n), 1)          # about 11 distinct values
    got = oracle.topk_tokens([sc], k)[0]
    beats = [(sc > sc[p]).sum() + (sc[:p] == sc[p]).sum() for p in range(n)]
    ref = [p for p in range(n) if beats[p] < k]
    assert list(got) == ref
    assert len(got) == min(k, n)


def test_fine_attention_keeping_every_token_is_chunk_attention():
    rng = np.random.default_rng(54)
    k_buf, v_buf = _rand_bufs(4, rng)
    q = bf16_round(rng.standard_normal((2, 64, 128)))
    cu = [0, 3, 4]
    sel = [np.arange(192), np.arange(64)]
    got = oracle.fine_decode_attn(q, k_buf, v_buf, cu, sel)
    ref = oracle.sparse_decode_attn(q, k_buf, v_buf, cu)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-15)
    empty = oracle.fine_decode_attn(q, k_buf, v_buf, cu, [np.arange(0), np.arange(64)])
    assert np.all(empty[0] == 0)


def test_fine_attention_equals_dense_sdpa_over_selected_rows():
    """torch's fp64 SDPA over exactly the selected rows (KV repeated per group);
    the order of the selected list does not matter."""
    rng = np.random.default_rng(55)
    k_buf, v_buf = _rand_bufs(5, rng)
    q = bf16_round(rng.standard_normal((2, 64, 128)))
    cu = [0, 3, 5]
    sel = [np.sort(rng.choice(192, 70, replace=False)), np.sort(rng.choice(128, 9, replace=False))]
    got = oracle.fine_decode_attn(q, k_buf, v_buf, cu, sel)
    for b in range(2):
        c = cu[b] + sel[b] // 64
        r = sel[b] % 64
        K = torch.from_numpy(k_buf[c, :, r]).permute(1, 0, 2).repeat_interleave(8, dim=0)   # [64, n, 128]
        V = torch.from_numpy(v_buf[c, :, r]).permute(1, 0, 2).repeat_interleave(8, dim=0)
        Q = torch.from_numpy(q[b]).reshape(64, 1, 128)
        ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).reshape(64, 128).numpy()
        np.testing.assert_allclose(got[b], ref, rtol=1e-12, atol=1e-14)
    shuffled = [rng.permutation(s) for s in sel]
    np.testing.assert_allclose(oracle.fine_decode_attn(q, k_buf, v_buf, cu, shuffled), got, rtol=1e-12, atol=1e-15)


# ------------------------------------------------- unit-signature closed form ---
# The full-size GPU tests of the split-K partition use zero keys and one-hot
# values (tests/unit_signature.py), where attention is a ratio of token counts.
# These pins tie that closed form to the oracle's attention.

def _signature_case(n_kept, seed):
    import unit_signature as us
    cu = np.concatenate([[0], np.cumsum(n_kept)]).astype(np.int64)
    total = int(cu[-1])
    off = us.offsets(max(total, 1), seed)
    v_hm = us.compact_v(off[:, :total], "cpu").to(torch.float64)             # [8, total, 64, 128]
    v_buf = v_hm.permute(1, 0, 2, 3).numpy()                                  # chunk-major for the oracle
    k_buf = np.zeros_like(v_buf)
    q = bf16_round(np.random.default_rng(seed).standard_normal((len(n_kept), 64, 128)))
    return us, cu, off, k_buf, v_buf, q


@pytest.mark.parametrize("n_kept", [[1], [3, 0, 2], [5, 1]])
def test_unit_signature_closed_form_equals_oracle(n_kept):
    us, cu, off, k_buf, v_buf, q = _signature_case(n_kept, seed=sum(n_kept) + 7)
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, cu)
    want = us.expected_chunks(off, cu)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)
    us.assert_signature(got, want)


def test_unit_signature_closed_form_with_local_tokens_equals_oracle():
    us, cu, off, k_buf, v_buf, q = _signature_case([2, 0, 1], seed=31)
    B = 3
    offl = us.local_offsets(B, 32)
    v_loc = us.one_hot_rows(torch.from_numpy(offl)).to(torch.float64).numpy()  # [B, 8, 64, 128]
    k_loc = np.zeros_like(v_loc)
    ll = [5, 17, 0]
    got = oracle.sparse_decode_attn(q, k_buf, v_buf, cu, k_local=k_loc, v_local=v_loc, local_len=ll)
    want = us.expected_chunks(off, cu, local_off=offl, local_len=ll)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)


def test_unit_signature_closed_form_selected_equals_oracle():
    us, cu, off, k_buf, v_buf, q = _signature_case([3, 2], seed=41)
    rng = np.random.default_rng(42)
    sel = [np.sort(rng.choice(192, 128, replace=False)), np.sort(rng.choice(128, 64, replace=False))]
    got = oracle.fine_decode_attn(q, k_buf, v_buf, cu, sel)
    want = us.expected_selected(off, cu, sel)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)


def test_unit_signature_detects_a_missing_or_repeated_unit():
    """The closed form separates the right unit set from one with a unit dropped
    or read twice by far more than its tolerance (mistakes planted on the CPU)."""
    import pytest as _pt
    us, cu, off, k_buf, v_buf, q = _signature_case([40], seed=51)
    want = us.expected_chunks(off, cu)
    dropped = oracle.sparse_decode_attn(q, k_buf[:39], v_buf[:39], [0, 39])
    with _pt.raises(AssertionError):
        us.assert_signature(dropped, want)
    twice = np.concatenate([k_buf, k_buf[7:8]]), np.concatenate([v_buf, v_buf[7:8]])
    repeated = oracle.sparse_decode_attn(q, twice[0], twice[1], [0, 41])
    with _pt.raises(AssertionError):
        us.assert_signature(repeated, want)
