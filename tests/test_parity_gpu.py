"""GPU parity: every kernel of liblsa against the fp64 oracle, through the C ABI.

Sizes: full windows at the tiny workload; the 128K workload in full for
scoring, selection and gather and at sampled decode steps for attention;
hand-made ragged batches that split (sequence, KV head) pairs across CTAs and
leave ragged tails; and the 500K / batched / 1M host-tier workloads at full
size on sampled outputs.
"""
import math

import numpy as np
import pytest
import torch

import kv_chunk_selection_b200 as lsa
import oracle
import workloads
from kv_chunk_selection_b200.window import LayerWindow
from lsa_testlib import (assert_attention_close, assert_kept_matches, assert_scores_close, cm, f64, i64,
                         kept_from_gpu)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_chunk_selection_b200 import build
    build.build()
    lsa.lib()
    yield
    torch.cuda.synchronize()


def status_clean():
    bits = lsa.read_device_status()
    assert bits == 0, f"device status {lsa.decode_status(bits)}"


def score_on_gpu(inp, layer=0, window=0):
    L = inp.layers[layer]
    scores = torch.full((inp.batch, inp.max_chunks), float("nan"), device=DEV)
    lsa.lsa_index_score(L.q_idx[window], L.w, L.chunk_keys, inp.chunk_table, inp.n_chunks, scores)
    return scores


def oracle_scores(inp, layer=0, window=0):
    L = inp.layers[layer]
    return oracle.index_scores(f64(L.q_idx[window]), f64(L.w), f64(L.chunk_keys), i64(inp.chunk_table),
                               i64(inp.n_chunks), inp.max_chunks)


# ------------------------------------------------------------------ scoring --

@pytest.mark.parametrize("name", ["tiny", "128k", "500k", "1m_host", "batched"])
def test_index_score_matches_oracle(name):
    inp = workloads.make_inputs(name, DEV, pools=False, layers=1)
    for w in range(min(2, inp.workload.windows)):
        g = score_on_gpu(inp, 0, w)
        o = oracle_scores(inp, 0, w)
        assert_scores_close(g, o, i64(inp.n_chunks))
        # entries past each sequence's end are left untouched
        gh = f64(g)
        for b, n in enumerate(i64(inp.n_chunks)):
            assert np.all(np.isnan(gh[b, n:]))
    status_clean()


# ---------------------------------------------------------------- selection --

def run_topk(scores, n_chunks, k_per_seq, max_kept):
    B = scores.shape[0]
    kept = torch.full((B, max_kept), -7, dtype=torch.int32, device=DEV)
    n_kept = torch.zeros(B, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_chunks(scores, n_chunks, k_per_seq, kept, n_kept, cu)
    return kept, n_kept, cu


@pytest.mark.parametrize("name", ["tiny", "128k", "500k", "1m_host", "batched"])
def test_topk_matches_oracle(name):
    inp = workloads.make_inputs(name, DEV, pools=False, layers=1)
    n, k = i64(inp.n_chunks), i64(inp.k_per_seq)
    g = score_on_gpu(inp)
    kept, n_kept, cu = run_topk(g, inp.n_chunks, inp.k_per_seq, int(k.max()) + 1)
    got = kept_from_gpu(kept, n_kept)
    # same decision in the same precision: the oracle's selection run on the GPU's fp32 scores
    ref_same = oracle.topk_chunks(f64(g), n, k)
    for b in range(len(n)):
        assert got[b] == list(ref_same[b]), f"seq {b}"
    # against the oracle's own fp64 scores, with the tie window
    assert_kept_matches(got, oracle_scores(inp), n, k)
    assert i64(cu).tolist() == oracle.cumulative_kept(ref_same).tolist()
    if inp.layers[0].planted is not None:
        planted = set(inp.layers[0].planted.tolist())
        recall = len(planted & set(got[0])) / len(planted)
        print(f"planted-chunk recall {recall:.2f}")  # diagnostic only
    status_clean()


def test_topk_edge_cases():
    cases = [(0, 3), (1, 0), (1, 5), (2, 0), (2, 1), (5, 4), (5, 10), (64, 8), (3000, 300), (16384, 1638),
             (4097, 4095), (100, 0), (777, 776), (1025, 513), (20000, 2000), (16386, 9000), (30001, 7)]
    B = len(cases)
    M = max(c[0] for c in cases)
    rng = np.random.default_rng(5)
    scores = np.zeros((B, M), dtype=np.float32)
    for b, (n, _) in enumerate(cases):
        kind = b % 4
        if kind == 0:
            scores[b, :n] = 0.25                                     # all ties
        elif kind == 1:
            scores[b, :n] = rng.integers(-3, 4, n) * 0.5             # heavy ties, negatives
        elif kind == 2:
            scores[b, :n] = rng.standard_normal(n)
        else:
            v = rng.standard_normal(n).astype(np.float32)
            v[::7] = 0.0
            v[3::7] = -0.0                                           # signed zeros tie
            scores[b, :n] = v
    n_chunks = torch.tensor([c[0] for c in cases], dtype=torch.int32, device=DEV)
    k_per_seq = torch.tensor([c[1] for c in cases], dtype=torch.int32, device=DEV)
    kept, n_kept, cu = run_topk(torch.from_numpy(scores).to(DEV), n_chunks, k_per_seq, M)
    got = kept_from_gpu(kept, n_kept)
    ref = oracle.topk_chunks(scores.astype(np.float64), i64(n_chunks), i64(k_per_seq))
    for b in range(B):
        assert got[b] == list(ref[b]), f"case {cases[b]}"
    assert i64(cu).tolist() == oracle.cumulative_kept(ref).tolist()
    status_clean()


def test_topk_nan_and_inf_order():
    s = np.array([[1.0, np.nan, np.inf, -np.inf, 2.0, np.nan, 0.5, 0.0]], dtype=np.float32)
    n = torch.tensor([8], dtype=torch.int32, device=DEV)
    for K in range(0, 8):
        k = torch.tensor([K], dtype=torch.int32, device=DEV)
        kept, n_kept, _ = run_topk(torch.from_numpy(s).to(DEV), n, k, 8)
        ref = oracle.topk_chunks(s.astype(np.float64), [8], [K])
        assert kept_from_gpu(kept, n_kept)[0] == list(ref[0]), K
    status_clean()


def run_threshold(scores, n_chunks, w, threshold, max_kept):
    B = scores.shape[0]
    kept = torch.full((B, max_kept), -7, dtype=torch.int32, device=DEV)
    n_kept = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_threshold_chunks(scores, n_chunks, w, kept, n_kept, cu, threshold=threshold)
    return kept, n_kept, cu


def assert_threshold_matches(got, scores64, n, w64, t):
    """Exact match with the oracle's rule on the same scores, except chunks whose
    weighted mean probability is within 1e-6 (relative) of the threshold."""
    ref = oracle.threshold_chunks(scores64, n, w64, t)
    wsum = float(np.sum(w64))
    for b in range(len(n)):
        g, r = set(got[b]), set(ref[b].tolist())
        for c in g ^ r:
            assert abs(scores64[b, c] / wsum - t) <= 1e-6 * abs(t), f"seq {b}: chunk {c} differs away from the threshold"
        assert sorted(got[b]) == got[b]


@pytest.mark.parametrize("name,t", [("tiny", 0.5), ("128k", 0.5), ("128k", 0.6), ("batched", 0.55)])
def test_threshold_matches_oracle(name, t):
    inp = workloads.make_inputs(name, DEV, pools=False, layers=1)
    n = i64(inp.n_chunks)
    g = score_on_gpu(inp)
    kept, n_kept, cu = run_threshold(g, inp.n_chunks, inp.layers[0].w, t, inp.max_chunks)
    got = kept_from_gpu(kept, n_kept)
    assert_threshold_matches(got, f64(g), n, f64(inp.layers[0].w), t)
    assert i64(cu).tolist() == oracle.cumulative_kept(got).tolist()
    # the oracle's own fp64 scores give the same set outside the threshold window
    assert_threshold_matches(got, oracle_scores(inp), n, f64(inp.layers[0].w), t)
    status_clean()


def test_threshold_edge_cases():
    w = torch.full((16,), 0.5, device=DEV)                     # sum(w) = 8
    n = torch.tensor([0, 1, 5, 5, 40], dtype=torch.int32, device=DEV)
    s = torch.zeros((5, 40), device=DEV)
    s[2, :5] = 8.0                                               # every mean probability 1.0: all kept
    s[3, :5] = 1.0                                               # 0.125: only the latest kept
    s[4, :40] = torch.linspace(0, 8, 40, device=DEV)
    kept, n_kept, cu = run_threshold(s, n, w, 0.5, 40)
    got = kept_from_gpu(kept, n_kept)
    assert got[0] == [] and got[1] == [0] and got[2] == [0, 1, 2, 3, 4] and got[3] == [4]
    ref = oracle.threshold_chunks(f64(s), i64(n), f64(w), 0.5)
    assert got[4] == list(ref[4])
    assert i64(cu).tolist() == oracle.cumulative_kept(got).tolist()
    status_clean()
    # a kept set larger than max_kept: that sequence keeps nothing, CAPACITY is reported
    kept, n_kept, cu = run_threshold(s, n, w, 0.5, 4)
    assert lsa.read_device_status() & 8
    assert i64(n_kept).tolist()[2] == 0 and i64(n_kept).tolist()[1] == 1


def run_threshold_capped(scores, n_chunks, w, threshold, cap, max_kept):
    B = scores.shape[0]
    kept = torch.full((B, max_kept), -7, dtype=torch.int32, device=DEV)
    n_kept = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_threshold_chunks(scores, n_chunks, w, kept, n_kept, cu, threshold=threshold, cap=cap)
    return kept, n_kept, cu


def assert_capped_matches(got, scores64, n, w64, t, cap):
    """The oracle's capped rule on the same scores, exactly, unless a chunk lies
    within 1e-6 (relative) of the threshold, where fp32 and fp64 may differ on
    whether it passes."""
    ref = oracle.threshold_chunks(scores64, n, w64, t, cap=cap)
    wsum = float(np.sum(w64))
    for b in range(len(n)):
        if got[b] == list(ref[b]):
            continue
        near = np.abs(scores64[b, : max(int(n[b]) - 1, 0)] / wsum - t) <= 1e-6 * abs(t)
        assert near.any(), f"seq {b}: capped selection differs with no chunk at the threshold"


@pytest.mark.parametrize("name,t", [("128k", 0.5), ("128k", 0.6), ("batched", 0.55), ("500k", 0.5)])
def test_threshold_capped_matches_oracle(name, t):
    """The budget is the top-K budget K_b: at 0.5 about half the chunks pass, so
    it binds; at 0.6 fewer pass than it allows, and the result is the plain rule."""
    inp = workloads.make_inputs(name, DEV, pools=False, layers=1)
    n, cap = i64(inp.n_chunks), i64(inp.k_per_seq)
    g = score_on_gpu(inp)
    kept, n_kept, cu = run_threshold_capped(g, inp.n_chunks, inp.layers[0].w, t, inp.k_per_seq, int(cap.max()) + 1)
    status_clean()
    got = kept_from_gpu(kept, n_kept)
    assert all(len(got[b]) <= cap[b] + 1 for b in range(len(n)))
    assert_capped_matches(got, f64(g), n, f64(inp.layers[0].w), t, cap)
    assert i64(cu).tolist() == oracle.cumulative_kept(got).tolist()


def test_threshold_capped_edge_cases():
    """Budget 0 keeps only the latest chunk; a budget above the passing count
    changes nothing; ties at the budget go to the lower index; 20000 candidates
    take the path that re-reads the scores; a negative budget is BAD_COUNT."""
    w = torch.full((16,), 0.5, device=DEV)                     # sum(w) = 8
    N = 20001
    n = torch.tensor([0, 1, 40, 40, 40, N, N], dtype=torch.int32, device=DEV)
    cap = torch.tensor([3, 3, 0, 100, 5, 1500, 3000], dtype=torch.int32, device=DEV)
    s = torch.zeros((7, N), device=DEV)
    s[2:5, :40] = torch.linspace(0, 8, 40, device=DEV)
    s[4, 30:36] = 7.0                                          # six equal passing scores, budget 5
    g = torch.Generator(device=DEV).manual_seed(9)
    s[5] = torch.rand(N, generator=g, device=DEV) * 8.0
    s[6] = torch.floor(torch.rand(N, generator=g, device=DEV) * 16.0) * 0.5   # heavy ties
    kept, n_kept, cu = run_threshold_capped(s, n, w, 0.5, cap, 20001)
    status_clean()
    got = kept_from_gpu(kept, n_kept)
    ref = oracle.threshold_chunks(f64(s), i64(n), f64(w), 0.5, cap=i64(cap))
    for b in range(7):
        assert got[b] == list(ref[b]), f"seq {b}"
    assert got[2] == [39] and got[4] == [30, 31, 36, 37, 38, 39]   # 36-38 score higher than the six ties
    assert got[3] == list(oracle.threshold_chunks(f64(s), i64(n), f64(w), 0.5)[3])
    assert i64(cu).tolist() == oracle.cumulative_kept(got).tolist()
    bad = torch.tensor([3, -1, 0, 100, 5, 1500, 3000], dtype=torch.int32, device=DEV)   # on a sequence with a chunk
    run_threshold_capped(s, n, w, 0.5, bad, 20001)
    assert lsa.read_device_status() == 1                      # LSA_DEV_ERR_BAD_COUNT


def test_threshold_window_attention():
    """Threshold selection feeds the same gather and attention: whole step vs the oracle."""
    inp = workloads.make_inputs("128k", DEV, layers=1, windows=1, steps=2)
    L = inp.layers[0]
    g = score_on_gpu(inp)
    kept, n_kept, cu = run_threshold(g, inp.n_chunks, L.w, 0.6, inp.max_chunks)
    total = int(cu[-1])
    kb = torch.empty((8, total, 64, 128), dtype=torch.bfloat16, device=DEV)
    vb = torch.empty_like(kb)
    lsa.lsa_gather_chunks(L.k_pool, L.v_pool, inp.chunk_table, kept, cu, inp.max_chunks, kb, vb)
    out = torch.empty((1, 64, 128), device=DEV)
    ws = lsa.new_attn_workspace(1)
    lsa.lsa_sparse_decode_attn(L.q[0, 1], kb, vb, cu, out, ws)
    got = kept_from_gpu(kept, n_kept)
    assert_threshold_matches(got, f64(g), i64(inp.n_chunks), f64(L.w), 0.6)
    assert torch.equal(cm(kb), L.k_pool[torch.tensor(got[0], device=DEV)])
    ref = oracle.sparse_decode_attn(f64(L.q[0, 1]), f64(cm(kb)), f64(cm(vb)), i64(cu))
    assert_attention_close(out, ref)
    status_clean()


# ------------------------------------------------------------------ gather --

def paged_case(B=6, seed=3, max_chunks=40):
    rng = np.random.default_rng(seed)
    n = rng.integers(1, max_chunks + 1, B)
    n[1] = 1
    n_slots = int(n.sum()) + 5
    perm = rng.permutation(n_slots)
    table = np.zeros((B, max_chunks), dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, : n[b]] = perm[off: off + n[b]]
        off += n[b]
    k = np.array([max(0, int(x) // 3) for x in n])
    return n.astype(np.int32), k.astype(np.int32), table, n_slots


def test_gather_paged_bit_exact():
    n, k, table, n_slots = paged_case()
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(11)
    shape = (n_slots, 8, 64, 128)
    k_pool = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    scores = torch.rand((B, M), generator=g, device=DEV)
    n_t = torch.from_numpy(n).to(DEV)
    k_t = torch.from_numpy(k).to(DEV)
    tab = torch.from_numpy(table).to(DEV)
    kept, n_kept, cu = run_topk(scores, n_t, k_t, int(k.max()) + 1)
    buf_chunks = int((k + 1).sum())
    kb = torch.zeros((8, buf_chunks, 64, 128), dtype=torch.bfloat16, device=DEV)
    vb = torch.zeros_like(kb)
    lsa.lsa_gather_chunks(k_pool, v_pool, tab, kept, cu, M, kb, vb)
    kept_l = kept_from_gpu(kept, n_kept)
    rk, rv, rcu = oracle.gather_chunks(k_pool.view(torch.int16).cpu().numpy(), v_pool.view(torch.int16).cpu().numpy(),
                                       table, kept_l, M)
    total = int(rcu[-1])
    assert np.array_equal(cm(kb)[:total].view(torch.int16).cpu().numpy(), rk)
    assert np.array_equal(cm(vb)[:total].view(torch.int16).cpu().numpy(), rv)
    status_clean()


# --------------------------------------------------------------- attention --

def ragged_buffers(n_kept, seed=21):
    g = torch.Generator(device=DEV).manual_seed(seed)
    total = int(sum(n_kept))
    shape = (8, max(total, 1), 64, 128)   # head-major compact buffer
    kb = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    vb = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(n_kept)]), dtype=torch.int32, device=DEV)
    q = torch.randn((len(n_kept), 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    return q, kb, vb, cu


def run_attn(q, kb, vb, cu):
    B = q.shape[0]
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    ws = lsa.new_attn_workspace(B)
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out, ws)
    return out, ws


@pytest.mark.parametrize("n_kept", [[1], [9], [257], [1, 0, 37, 3, 150, 9], [0, 0, 5, 0], [2] * 40,
                                    [300, 1, 1, 1, 1, 1, 1, 1, 299]])
def test_attention_ragged_matches_oracle(n_kept):
    q, kb, vb, cu = ragged_buffers(n_kept)
    out, _ = run_attn(q, kb, vb, cu)
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu))
    assert_attention_close(out, ref)
    status_clean()


@pytest.mark.parametrize("n_kept,local_len", [([0, 3, 150, 9], [0, 1, 17, 64]), ([5], [64]), ([0, 0], [3, 0]),
                                               ([300, 1, 40], [63, 2, 32])])
def test_attention_local_tokens_match_oracle(n_kept, local_len):
    q, kb, vb, cu = ragged_buffers(n_kept, seed=41)
    B = len(n_kept)
    g = torch.Generator(device=DEV).manual_seed(42)
    kl = torch.randn((B, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    vl = torch.randn((B, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    ll = torch.tensor(local_len, dtype=torch.int32, device=DEV)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_local(q, kb, vb, cu, kl, vl, ll, out, lsa.new_attn_workspace(B))
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu), k_local=f64(kl), v_local=f64(vl),
                                    local_len=local_len)
    assert_attention_close(out, ref)
    status_clean()


def test_append_then_attend_is_causal():
    """A window of decode steps: each step appends its token, then attends over the
    kept chunks plus every token decoded so far (compared with the oracle)."""
    n_kept = [7, 60]
    q, kb, vb, cu = ragged_buffers(n_kept, seed=43)
    B = len(n_kept)
    g = torch.Generator(device=DEV).manual_seed(44)
    steps = 6
    k_new = torch.randn((steps, B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    v_new = torch.randn((steps, B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    qs = torch.randn((steps, B, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    kl = torch.zeros((B, 8, 64, 128), dtype=torch.bfloat16, device=DEV)
    vl = torch.zeros_like(kl)
    ll = torch.zeros(B, dtype=torch.int32, device=DEV)
    ws = lsa.new_attn_workspace(B)
    outs = torch.empty((steps, B, 64, 128), device=DEV)
    for t in range(steps):
        lsa.lsa_append_token(k_new[t], v_new[t], kl, vl, ll)
        lsa.lsa_sparse_decode_attn_local(qs[t], kb, vb, cu, kl, vl, ll, outs[t], ws, kv_unchanged=t > 0)
    torch.cuda.synchronize()
    assert i64(ll).tolist() == [steps] * B
    for t in (0, steps - 1):
        kloc = np.zeros((B, 8, 64, 128))
        vloc = np.zeros((B, 8, 64, 128))
        kloc[:, :, : t + 1] = f64(k_new[: t + 1]).transpose(1, 2, 0, 3)
        vloc[:, :, : t + 1] = f64(v_new[: t + 1]).transpose(1, 2, 0, 3)
        ref = oracle.sparse_decode_attn(f64(qs[t]), f64(cm(kb)), f64(cm(vb)), i64(cu), k_local=kloc, v_local=vloc,
                                        local_len=[t + 1] * B)
        assert_attention_close(outs[t], ref)
    status_clean()


def test_fused_append_step_matches_two_launch_path_and_oracle():
    """lsa_sparse_decode_attn_append = lsa_append_token then the local attention,
    bit for bit, and the oracle with the token at row n; the local chunk gets the
    row, the other rows are untouched, and local_len_out = n + 1."""
    n_kept, n_loc = [0, 3, 5, 1], [0, 5, 63, 17]
    B = len(n_kept)
    q, kb, vb, cu = ragged_buffers(n_kept, seed=91)
    g = torch.Generator(device=DEV).manual_seed(92)
    kl = torch.randn((B, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    vl = torch.randn((B, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    kn = torch.randn((B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    vn = torch.randn((B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    len_in = torch.tensor(n_loc, dtype=torch.int32, device=DEV)
    len_out = torch.full((B,), -5, dtype=torch.int32, device=DEV)
    kl_f, vl_f = kl.clone(), vl.clone()
    out_f = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_append(q, kb, vb, cu, kn, vn, kl_f, vl_f, len_in, len_out, out_f,
                                      lsa.new_attn_workspace(B))
    # two launches: append (in place), then the local attention
    kl_t, vl_t, len_t = kl.clone(), vl.clone(), len_in.clone()
    out_t = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_append_token(kn, vn, kl_t, vl_t, len_t)
    lsa.lsa_sparse_decode_attn_local(q, kb, vb, cu, kl_t, vl_t, len_t, out_t, lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    status_clean()
    assert len_out.tolist() == [n + 1 for n in n_loc] == len_t.tolist()
    assert torch.equal(kl_f, kl_t) and torch.equal(vl_f, vl_t)
    for b, n in enumerate(n_loc):
        assert torch.equal(kl_f[b, :, n], kn[b]) and torch.equal(vl_f[b, :, n], vn[b])
    mask = torch.ones((B, 64), dtype=torch.bool, device=DEV)
    mask[torch.arange(B), torch.tensor(n_loc)] = False
    assert torch.equal(kl_f.permute(0, 2, 1, 3)[mask], kl.permute(0, 2, 1, 3)[mask])
    assert torch.equal(out_f, out_t)
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu), k_local=f64(kl_t), v_local=f64(vl_t),
                                    local_len=[n + 1 for n in n_loc])
    assert_attention_close(out_f, ref)


def test_rejected_offsets_under_kv_unchanged_report_capacity_and_the_stream_goes_on():
    """Offsets that the attention rejects (a total beyond the compact buffer)
    make every CTA leave before any K/V read; with LSA_ATTN_KV_UNCHANGED each
    CTA first waits for the preceding kernel, so the grid still completes after
    it.  CAPACITY is reported, and the next, correct call on the stream matches
    the oracle."""
    q, kb, vb, cu = ragged_buffers([3, 1], seed=97)
    ws = lsa.new_attn_workspace(2)
    out = torch.full((2, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out, ws)
    bad = cu.clone()
    bad[-1] = kb.shape[1] + 1          # one chunk more than the buffer holds
    lsa.lsa_sparse_decode_attn(q, kb, vb, bad, out, ws, kv_unchanged=True)
    assert lsa.read_device_status() & 8          # CAPACITY
    out2 = torch.full((2, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out2, ws, kv_unchanged=True)
    torch.cuda.synchronize()
    status_clean()
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu))
    assert_attention_close(out2, ref)


def test_fused_append_full_local_chunk_reports_capacity():
    n_kept = [2]
    q, kb, vb, cu = ragged_buffers(n_kept, seed=93)
    kl = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16, device=DEV)
    vl = torch.zeros_like(kl)
    kl[:] = torch.randn((1, 8, 64, 128), generator=torch.Generator(device=DEV).manual_seed(94), device=DEV)
    kn = torch.ones((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    len_in = torch.tensor([64], dtype=torch.int32, device=DEV)
    len_out = torch.tensor([0], dtype=torch.int32, device=DEV)
    before = kl.clone()
    out = torch.empty((1, 64, 128), device=DEV)
    lsa.lsa_sparse_decode_attn_append(q, kb, vb, cu, kn, kn, kl, vl, len_in, len_out, out, lsa.new_attn_workspace(1))
    torch.cuda.synchronize()
    assert lsa.read_device_status() & 8          # CAPACITY
    assert len_out.tolist() == [64] and torch.equal(kl, before)
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu), k_local=f64(kl), v_local=f64(vl),
                                    local_len=[64])
    assert_attention_close(out, ref)


def test_append_reports_full_local_chunk():
    kl = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16, device=DEV)
    ll = torch.tensor([64], dtype=torch.int32, device=DEV)
    tok = torch.ones((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    lsa.lsa_append_token(tok, tok, kl, kl, ll)
    assert lsa.read_device_status() & 8
    assert int(ll.item()) == 64 and int(kl.abs().sum().item()) == 0


@pytest.mark.parametrize("n_local", [1, 4, 128])
def test_topk_recent_window_matches_oracle(n_local):
    inp = workloads.make_inputs("batched", DEV, pools=False, layers=1)
    n, k = i64(inp.n_chunks), i64(inp.k_per_seq)
    g = score_on_gpu(inp)
    B = inp.batch
    max_kept = int(k.max()) + n_local
    kept = torch.full((B, max_kept), -7, dtype=torch.int32, device=DEV)
    n_kept = torch.zeros(B, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_chunks(g, inp.n_chunks, inp.k_per_seq, kept, n_kept, cu, n_local=n_local)
    got = kept_from_gpu(kept, n_kept)
    ref = oracle.topk_chunks(f64(g), n, k, n_local=n_local)
    for b in range(B):
        assert got[b] == list(ref[b]), f"seq {b}"
    assert i64(cu).tolist() == oracle.cumulative_kept(ref).tolist()
    status_clean()


def test_max_batch_window_step():
    """The largest batch the calls accept (4096 sequences), tiny ragged sequences,
    some empty, through a paged table: score, select, gather and one attention
    step.  Selection bit-exact on the GPU's scores, offsets exact, gathers exact,
    attention on a sample of sequences and zeros for every empty one."""
    B, M = 4096, 5
    rng = np.random.default_rng(77)
    n = rng.integers(0, M + 1, B)
    n[:3] = [0, 1, M]
    k = rng.integers(0, 3, B)
    n_slots = int(n.sum())
    perm = rng.permutation(n_slots)
    table = np.zeros((B, M), dtype=np.int32)
    off = 0
    for b in range(B):
        table[b, : n[b]] = perm[off: off + n[b]]
        off += n[b]
    g = torch.Generator(device=DEV).manual_seed(78)
    k_pool = torch.randn((n_slots, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn((n_slots, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    keys = torch.randn((n_slots, 128), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand(16, generator=g, device=DEV)
    q_idx = torch.randn((B, 16, 128), generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn((B, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    n_t, k_t, tab = (torch.from_numpy(x.astype(np.int32)).to(DEV) for x in (n, k, table))
    lw = LayerWindow(n_t, k_t, tab, M, DEV)
    lw.select(q_idx, w, keys)
    lw.gather(k_pool, v_pool)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lw.attend(q, out)
    torch.cuda.synchronize()
    status_clean()
    sc = f64(lw.scores)
    ref = oracle.topk_chunks(sc, n, k)
    got = lw.kept_lists()
    assert all(got[b] == list(ref[b]) for b in range(B))
    cu = i64(lw.cu_kept[0])
    assert cu.tolist() == oracle.cumulative_kept(ref).tolist()
    for b in (1, 2, 4095, int(np.argmax(n))):
        for j, c in enumerate(got[b]):
            assert torch.equal(cm(lw.k_bufs[0])[cu[b] + j], k_pool[int(table[b, c])])
    empty = [b for b in range(B) if n[b] == 0]
    assert torch.all(out[empty] == 0)
    seqs = sorted(set(rng.choice(B, 48, replace=False).tolist()) | {1, 2, 4095})
    for b in seqs:   # one sequence at a time: only its own kept chunks go to the host
        lo, hi = int(cu[b]), int(cu[b + 1])
        ref_o = oracle.sparse_decode_attn(f64(q[b: b + 1]), f64(cm(lw.k_bufs[0])[lo:hi]), f64(cm(lw.v_bufs[0])[lo:hi]),
                                          [0, hi - lo])
        assert_attention_close(out[b: b + 1], ref_o)


@pytest.mark.parametrize("n_local", [1, 3])
def test_topk_long_sequences_cluster_kernel(n_local):
    """Chunk top-K beyond 16384 candidates runs on the 8-CTA cluster kernel, with a
    per-sequence K and a recent window; ragged lengths, one sequence short, one
    empty; bit-exact against the oracle's rule on the same scores."""
    n = np.array([40000, 17000, 5, 0, 23456])
    k = np.array([4000, 1700, 2, 3, 2345])
    B, M = len(n), int(n.max())
    g = torch.Generator(device=DEV).manual_seed(31 + n_local)
    scores = torch.rand((B, M), generator=g, device=DEV)
    scores[0, ::7] = 0.5                      # many exact ties
    n_t = torch.from_numpy(n.astype(np.int32)).to(DEV)
    k_t = torch.from_numpy(k.astype(np.int32)).to(DEV)
    max_kept = int(k.max()) + n_local
    kept = torch.full((B, max_kept), -7, dtype=torch.int32, device=DEV)
    n_kept = torch.zeros(B, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_chunks(scores, n_t, k_t, kept, n_kept, cu, n_local=n_local)
    torch.cuda.synchronize()
    status_clean()
    got = kept_from_gpu(kept, n_kept)
    ref = oracle.topk_chunks(f64(scores), n, k, n_local=n_local)
    for b in range(B):
        assert got[b] == list(ref[b]), f"seq {b}"
    assert i64(cu).tolist() == oracle.cumulative_kept(ref).tolist()


def test_attention_closed_forms():
    n_kept = [3, 70]
    q, kb, vb, cu = ragged_buffers(n_kept, seed=4)
    kb[:] = kb[0, 0, 0]                       # identical keys: output = mean of V
    out, _ = run_attn(q, kb, vb, cu)
    o = f64(out)
    c = i64(cu)
    for b in range(2):
        for h in (0, 13, 63):
            mean = f64(cm(vb)[c[b]: c[b + 1], h // 8]).reshape(-1, 128).mean(axis=0)
            np.testing.assert_allclose(o[b, h], mean, atol=2e-3, rtol=1e-3)
    # GQA mapping: V of KV head g is the constant g + 1
    q, kb, vb, cu = ragged_buffers(n_kept, seed=5)
    for g in range(8):
        vb[g] = g + 1.0                       # head-major: KV head g first
    out, _ = run_attn(q, kb, vb, cu)
    o = f64(out)
    for h in range(64):
        np.testing.assert_allclose(o[:, h], h // 8 + 1.0, rtol=1e-5)
    status_clean()


def test_attention_deterministic_and_workspace_reusable():
    q, kb, vb, cu = ragged_buffers([400, 3, 77])
    out1, ws = run_attn(q, kb, vb, cu)
    out2 = torch.empty_like(out1)
    for _ in range(3):
        lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out2, ws)
    assert torch.equal(out1, out2)
    # the workspace needs no initialisation: all bytes 0xFF (NaN records) give the same result
    ws.fill_(255)
    out3 = torch.empty_like(out1)
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out3, ws)
    assert torch.equal(out1, out3)
    status_clean()


def test_attention_overlapped_steps_match():
    """Steps launched with kv_unchanged (K/V streamed while the previous step's
    merge finishes) give bit-identical results, also right after a gather."""
    n, k, table, n_slots = paged_case(B=5, seed=15, max_chunks=60)
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(16)
    shape = (n_slots, 8, 64, 128)
    k_pool = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    n_t, k_t, tab = (torch.from_numpy(x).to(DEV) for x in (n, k, table))
    scores = torch.rand((B, M), generator=g, device=DEV)
    kept, n_kept, cu = run_topk(scores, n_t, k_t, int(k.max()) + 1)
    buf = int((k + 1).sum())
    kb = torch.empty((8, buf, 64, 128), dtype=torch.bfloat16, device=DEV)
    vb = torch.empty_like(kb)
    qs = torch.randn((6, B, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    ws = lsa.new_attn_workspace(B)
    ref = torch.empty((6, B, 64, 128), device=DEV)
    got = torch.empty_like(ref)
    lsa.lsa_gather_chunks(k_pool, v_pool, tab, kept, cu, M, kb, vb)
    for t in range(6):
        lsa.lsa_sparse_decode_attn(qs[t], kb, vb, cu, ref[t], ws)
    torch.cuda.synchronize()
    kb.zero_()
    vb.zero_()
    lsa.lsa_gather_chunks(k_pool, v_pool, tab, kept, cu, M, kb, vb)   # rewrite, then overlap the steps
    for t in range(6):
        lsa.lsa_sparse_decode_attn(qs[t], kb, vb, cu, got[t], ws, kv_unchanged=t > 0)
    torch.cuda.synchronize()
    assert torch.equal(ref, got)
    o = oracle.sparse_decode_attn(f64(qs[3]), f64(cm(kb)), f64(cm(vb)), i64(cu))
    assert_attention_close(got[3], o)
    status_clean()


def test_attention_scale_argument():
    q, kb, vb, cu = ragged_buffers([5])
    out = torch.empty((1, 64, 128), device=DEV)
    ws = lsa.new_attn_workspace(1)
    lsa.lsa_sparse_decode_attn(q, kb, vb, cu, out, ws, softmax_scale=0.3)
    ref = oracle.sparse_decode_attn(f64(q), f64(cm(kb)), f64(cm(vb)), i64(cu), scale=0.3)
    assert_attention_close(out, ref)


# ------------------------------------------------------------ whole window --

def f32(t: torch.Tensor) -> np.ndarray:
    """Exact float32 host copy of a bf16 tensor (half the memory of float64)."""
    return t.detach().float().cpu().numpy()


def window_parity(name, steps, layer=0, window=0, heads=None, seqs=None, **kw):
    inp = workloads.make_inputs(name, DEV, layers=1, **kw)
    L = inp.layers[layer]
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV)
    lw.select(L.q_idx[window], L.w, L.chunk_keys)
    if inp.workload.host_pool:
        lw.fetch(L.k_pool, L.v_pool)
    else:
        lw.gather(L.k_pool, L.v_pool)
    outs = {}
    for t in steps:
        out = torch.empty((inp.batch, 64, 128), device=DEV)
        lw.attend(L.q[window, t], out)
        outs[t] = out
    torch.cuda.synchronize()
    status_clean()
    # scores and selection
    n, k = i64(inp.n_chunks), i64(inp.k_per_seq)
    o_scores = oracle_scores(inp, layer, window)
    assert_scores_close(lw.scores, o_scores, n)
    got = lw.kept_lists()
    assert_kept_matches(got, o_scores, n, k)
    cu = i64(lw.cu_kept[0])
    total = int(cu[-1])
    # gather: every kept chunk equals its pool slot, bit for bit
    table = i64(inp.chunk_table)
    idx = torch.tensor([int(table[b, c]) for b in range(inp.batch) for c in got[b]], device=L.k_pool.device)
    assert torch.equal(cm(lw.k_bufs[0])[:total], L.k_pool[idx].to(DEV))
    assert torch.equal(cm(lw.v_bufs[0])[:total], L.v_pool[idx].to(DEV))
    # attention at the sampled steps: the oracle on the kept set the GPU chose
    kb, vb = f32(cm(lw.k_bufs[0])[:total]), f32(cm(lw.v_bufs[0])[:total])
    errs = []
    for t in steps:
        ref = oracle.sparse_decode_attn(f64(L.q[window, t]), kb, vb, cu, heads=heads, seqs=seqs)
        errs.append(assert_attention_close(outs[t], ref, heads=heads, seqs=seqs))
    return inp, lw, outs, errs


def test_window_tiny_full():
    """Whole window of the tiny workload, all 64 steps, against the oracle's own window."""
    inp = workloads.make_inputs("tiny", DEV)
    L = inp.layers[0]
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV)
    outs = torch.empty((64, 1, 64, 128), device=DEV)
    lw.run_window(L.q_idx[0], L.w, L.chunk_keys, L.k_pool, L.v_pool, L.q[0], outs)
    torch.cuda.synchronize()
    status_clean()
    scores, kept, cu, o_outs = oracle.decode_window(
        f64(L.q_idx[0]), f64(L.w), f64(L.chunk_keys), i64(inp.chunk_table), i64(inp.n_chunks),
        i64(inp.k_per_seq), f64(L.k_pool), f64(L.v_pool), f64(L.q[0]), inp.max_chunks)
    assert_scores_close(lw.scores, scores, i64(inp.n_chunks))
    assert lw.kept_lists()[0] == list(kept[0])
    for t in range(64):
        assert_attention_close(outs[t], o_outs[t])


def test_window_tiny_causal_recent_window():
    """Causal window (every step appends its token, then attends) with the latest
    2 chunks kept, all 64 steps, against the oracle's causal window; a second run
    of the same window must reset the local chunk and repeat it bit for bit."""
    inp = workloads.make_inputs("tiny", DEV)
    L = inp.layers[0]
    kn, vn = workloads.decoded_tokens(inp, 0, DEV)
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, n_local=2, causal=True)
    outs = torch.empty((64, 1, 64, 128), device=DEV)
    lw.run_window(L.q_idx[0], L.w, L.chunk_keys, L.k_pool, L.v_pool, L.q[0], outs, k_new=kn[0], v_new=vn[0])
    torch.cuda.synchronize()
    status_clean()
    assert int(lw.local_len[0]) == 64
    scores, kept, cu, o_outs = oracle.decode_window(
        f64(L.q_idx[0]), f64(L.w), f64(L.chunk_keys), i64(inp.chunk_table), i64(inp.n_chunks),
        i64(inp.k_per_seq), f64(L.k_pool), f64(L.v_pool), f64(L.q[0]), inp.max_chunks,
        n_local=2, k_new=f64(kn[0]), v_new=f64(vn[0]))
    assert lw.kept_lists()[0] == list(kept[0])
    for t in range(64):
        assert_attention_close(outs[t], o_outs[t])
    again = torch.empty_like(outs)
    lw.run_window(L.q_idx[0], L.w, L.chunk_keys, L.k_pool, L.v_pool, L.q[0], again, k_new=kn[0], v_new=vn[0])
    torch.cuda.synchronize()
    status_clean()
    assert torch.equal(outs, again)


def test_reset_local_empties_the_local_chunk():
    B = 3
    kl = torch.zeros((B, 8, 64, 128), dtype=torch.bfloat16, device=DEV)
    vl = torch.zeros_like(kl)
    ll = torch.tensor([5, 0, 64], dtype=torch.int32, device=DEV)
    lsa.lsa_reset_local(ll)
    assert ll.tolist() == [0, 0, 0]
    g = torch.Generator(device=DEV).manual_seed(2)
    kt = torch.randn((B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    vt = torch.randn((B, 8, 128), generator=g, device=DEV).to(torch.bfloat16)
    lsa.lsa_append_token(kt, vt, kl, vl, ll)
    assert ll.tolist() == [1, 1, 1]
    assert torch.equal(kl[:, :, 0], kt) and torch.equal(vl[:, :, 0], vt)
    status_clean()


def test_window_128k_sampled_steps():
    window_parity("128k", steps=[0, 31, 63], window=1)


@pytest.mark.slow
def test_window_500k_sampled_steps():
    window_parity("500k", steps=[0, 63], heads=[0, 9, 18, 27, 36, 45, 54, 63])


@pytest.mark.slow
def test_window_batched_one_layer_sampled():
    window_parity("batched", steps=[0, 63], heads=[0, 15, 22, 31, 36, 47, 53, 63])


@pytest.mark.slow
def test_window_1m_host_tier_sampled():
    inp, lw, outs, errs = window_parity("1m_host", steps=[0], heads=[0, 27, 63])


# ------------------------------------------------------------ host fetch ----

def test_fetch_from_host_equals_gather():
    n, k, table, n_slots = paged_case(B=4, seed=9, max_chunks=30)
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(12)
    shape = (n_slots, 8, 64, 128)
    k_dev = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    v_dev = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    k_host = k_dev.cpu().pin_memory()
    v_host = v_dev.cpu().pin_memory()
    scores = torch.rand((B, M), generator=g, device=DEV)
    n_t, k_t, tab = (torch.from_numpy(x).to(DEV) for x in (n, k, table))
    kept, n_kept, cu = run_topk(scores, n_t, k_t, int(k.max()) + 1)
    buf = int((k + 1).sum())
    a_k = torch.zeros((8, buf, 64, 128), dtype=torch.bfloat16, device=DEV)
    a_v, b_k, b_v = torch.zeros_like(a_k), torch.zeros_like(a_k), torch.zeros_like(a_k)
    lsa.lsa_gather_chunks(k_dev, v_dev, tab, kept, cu, M, a_k, a_v)
    side = torch.cuda.Stream()
    ev = torch.cuda.Event()
    side.wait_stream(torch.cuda.current_stream())
    lsa.lsa_fetch_from_host(k_host, v_host, tab, kept, cu, M, b_k, b_v, num_ctas=16, stream=side, done_event=ev)
    torch.cuda.current_stream().wait_event(ev)
    assert torch.equal(a_k, b_k) and torch.equal(a_v, b_v)
    status_clean()


@pytest.mark.parametrize("table_kind", ["paged", "identity_runs"])
def test_fetch_copy_engine_equals_gather(table_kind):
    """The copy-engine fetch (selection read on the host, one 2-D copy per kept
    chunk and per K/V, per-head copies for runs of adjacent slots) is byte-equal
    to the device gather.  The identity table with a budget of most chunks makes
    long runs of adjacent slots."""
    if table_kind == "paged":
        n, k, table, n_slots = paged_case(B=4, seed=19, max_chunks=30)
    else:
        n = np.array([40, 25, 64])
        k = np.array([36, 3, 60])
        table = np.zeros((3, 64), dtype=np.int32)
        off = 0
        for b in range(3):
            table[b, : n[b]] = np.arange(off, off + n[b])
            off += int(n[b])
        n_slots = off
        n, k = n.astype(np.int32), k.astype(np.int32)
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(13)
    shape = (n_slots, 8, 64, 128)
    k_dev = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    v_dev = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    k_host, v_host = k_dev.cpu().pin_memory(), v_dev.cpu().pin_memory()
    scores = torch.rand((B, M), generator=g, device=DEV)
    n_t, k_t, tab = (torch.from_numpy(np.ascontiguousarray(x)).to(DEV) for x in (n, k, table))
    kept, n_kept, cu = run_topk(scores, n_t, k_t, int(k.max()) + 1)
    buf = int((k + 1).sum()) + 3
    a_k = torch.zeros((8, buf, 64, 128), dtype=torch.bfloat16, device=DEV)
    a_v, b_k, b_v = torch.zeros_like(a_k), torch.zeros_like(a_k), torch.zeros_like(a_k)
    lsa.lsa_gather_chunks(k_dev, v_dev, tab, kept, cu, M, a_k, a_v)
    side = torch.cuda.Stream()
    ev = torch.cuda.Event()
    kept_h, cu_h = kept.cpu(), cu.cpu()
    side.wait_stream(torch.cuda.current_stream())
    lsa.lsa_fetch_from_host_copy(k_host, v_host, tab.cpu(), kept_h, cu_h, M, b_k, b_v, stream=side, done_event=ev)
    torch.cuda.current_stream().wait_event(ev)
    assert torch.equal(a_k, b_k) and torch.equal(a_v, b_v)
    status_clean()


def test_fetch_injected_failure_reaches_the_caller():
    """An injected transfer failure comes back from the binding as an error
    (nothing is launched), and the next fetch works."""
    n, k, table, n_slots = paged_case(B=2, seed=21, max_chunks=12)
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(14)
    k_dev = torch.randn((n_slots, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    k_host = k_dev.cpu().pin_memory()
    scores = torch.rand((B, M), generator=g, device=DEV)
    n_t, k_t, tab = (torch.from_numpy(x).to(DEV) for x in (n, k, table))
    kept, n_kept, cu = run_topk(scores, n_t, k_t, int(k.max()) + 1)
    buf = int((k + 1).sum())
    a_k = torch.zeros((8, buf, 64, 128), dtype=torch.bfloat16, device=DEV)
    b_k, b_v = torch.zeros_like(a_k), torch.zeros_like(a_k)
    lsa.lsa_gather_chunks(k_dev, k_dev, tab, kept, cu, M, a_k, torch.zeros_like(a_k))
    lsa.lsa_debug_fail_fetch(1, -4)
    with pytest.raises(lsa.LsaError) as err:
        lsa.lsa_fetch_from_host(k_host, k_host, tab, kept, cu, M, b_k, b_v)
    assert err.value.status == -4
    assert torch.count_nonzero(b_k) == 0
    lsa.lsa_fetch_from_host(k_host, k_host, tab, kept, cu, M, b_k, b_v)
    torch.cuda.synchronize()
    assert torch.equal(a_k, b_k)
    status_clean()


def test_fetch_delta_reuses_previous_window():
    """Residency across windows: chunks kept in both windows come from the previous
    compact buffer; the result equals a plain host fetch bit for bit, and the reuse
    count equals the size of the intersection of the two kept sets."""
    n, k, table, n_slots = paged_case(B=4, seed=21, max_chunks=48)
    B, M = table.shape
    g = torch.Generator(device=DEV).manual_seed(22)
    shape = (n_slots, 8, 64, 128)
    k_host = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16).cpu().pin_memory()
    v_host = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16).cpu().pin_memory()
    n_t, k_t, tab = (torch.from_numpy(x).to(DEV) for x in (n, k, table))
    s_a = torch.rand((B, M), generator=g, device=DEV)
    s_b = s_a.clone()
    s_b[:, ::3] = torch.rand((B, (M + 2) // 3), generator=g, device=DEV)   # partly different selection
    ka, na, cua = run_topk(s_a, n_t, k_t, int(k.max()) + 1)
    kb_, nb, cub = run_topk(s_b, n_t, k_t, int(k.max()) + 1)
    buf = int((k + 1).sum())
    ak = torch.zeros((8, buf, 64, 128), dtype=torch.bfloat16, device=DEV)
    av = torch.zeros_like(ak)
    lsa.lsa_fetch_from_host(k_host, v_host, tab, ka, cua, M, ak, av)                 # window A
    bk, bv, rk, rv = (torch.zeros_like(ak) for _ in range(4))
    reused = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.lsa_fetch_from_host_delta(k_host, v_host, tab, kb_, cub, M, bk, bv, ka, cua, ak, av, reused)
    lsa.lsa_fetch_from_host(k_host, v_host, tab, kb_, cub, M, rk, rv)                # plain window B
    torch.cuda.synchronize()
    assert torch.equal(bk, rk) and torch.equal(bv, rv)
    la, lb = kept_from_gpu(ka, na), kept_from_gpu(kb_, nb)
    inter = sum(len(set(x) & set(y)) for x, y in zip(la, lb))
    assert int(reused.item()) == inter and inter > 0
    status_clean()


def test_fetch_rejects_unpinned_pool():
    k_host = torch.zeros((4, 8, 64, 128), dtype=torch.bfloat16)     # pageable
    kept = torch.zeros((1, 2), dtype=torch.int32, device=DEV)
    cu = torch.tensor([0, 1], dtype=torch.int32, device=DEV)
    buf = torch.zeros((8, 2, 64, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(lsa.LsaError, match="NOT_PINNED"):
        lsa.lsa_fetch_from_host(k_host, k_host, None, kept, cu, 4, buf, buf)


# ------------------------------------------------------- device-side errors --

def test_device_errors_are_reported_not_trapped():
    shape = (4, 8, 64, 128)
    pool = torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
    buf = torch.zeros((8, 2, 64, 128), dtype=torch.bfloat16, device=DEV)
    kept = torch.tensor([[0, 9]], dtype=torch.int32, device=DEV)      # 9 >= max_chunks (4)
    cu = torch.tensor([0, 2], dtype=torch.int32, device=DEV)
    lsa.lsa_gather_chunks(pool, pool, None, kept, cu, 4, buf, buf)
    assert lsa.read_device_status() & 4                                 # BAD_CHUNK
    table = torch.tensor([[0, 1, 2, 77]], dtype=torch.int32, device=DEV)  # slot 77 >= n_slots
    kept = torch.tensor([[0, 3]], dtype=torch.int32, device=DEV)
    lsa.lsa_gather_chunks(pool, pool, table, kept, cu, 4, buf, buf)
    assert lsa.read_device_status() & 2                                 # BAD_SLOT
    cu_big = torch.tensor([0, 3], dtype=torch.int32, device=DEV)        # 3 chunks > buffer of 2
    lsa.lsa_gather_chunks(pool, pool, None, kept, cu_big, 4, buf, buf)
    assert lsa.read_device_status() & 8                                 # CAPACITY
    q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((1, 64, 128), device=DEV)
    ws = lsa.new_attn_workspace(1)
    lsa.lsa_sparse_decode_attn(q, buf, buf, cu_big, out, ws)
    assert lsa.read_device_status() & 8
    keys = torch.zeros((4, 128), dtype=torch.bfloat16, device=DEV)
    scores = torch.zeros((1, 4), device=DEV)
    lsa.lsa_index_score(torch.zeros((1, 16, 128), dtype=torch.bfloat16, device=DEV),
                        torch.ones(16, device=DEV), keys, None,
                        torch.tensor([5], dtype=torch.int32, device=DEV), scores)
    assert lsa.read_device_status() & 1                                 # BAD_COUNT
    assert lsa.read_device_status() == 0
