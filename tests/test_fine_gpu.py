"""GPU parity of the token-level fine stage against the fp64 oracle.

Inside the recalled chunks every decode step scores each token with the
step's indexer query, keeps the k best token positions (score descending,
position ascending) and attends only those (summary page
"FlashMemory-DeepSeek-V4 ...", 2.1 Architecture; k = 2048 as for the DSA
lightning indexer on the search page).  Each stage is compared with the oracle
through the C ABI: scores within 1e-4 relative, the selection bit-exact
against the oracle's selection on the GPU's own fp32 scores (and outside the
tie window against the oracle's fp64 scores), the packed units bit for bit,
and attention within the attention tolerance.
"""
import numpy as np
import pytest
import torch

import kv_chunk_selection_b200 as lsa
import oracle
import workloads
from kv_chunk_selection_b200.window import LayerWindow
from lsa_testlib import SCORE_RTOL, TIE_RTOL, assert_attention_close, cm, f64, i64, kept_from_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_chunk_selection_b200 import build
    build.build()
    lsa.lib()
    lsa.read_device_status()


def status_clean():
    bits = lsa.read_device_status()
    assert bits == 0, f"device status {lsa.decode_status(bits)}"


def recalled(name, **kw):
    """Inputs of a workload, its window-0 chunk selection on the GPU, the compact
    buffer, and the fine-stage inputs (token keys, per-step indexer queries)."""
    inp = workloads.make_inputs(name, DEV, layers=1, windows=1, **kw)
    L = inp.layers[0]
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV)
    lw.select(L.q_idx[0], L.w, L.chunk_keys)
    lw.gather(L.k_pool, L.v_pool)
    tok_keys, q_tok = workloads.fine_inputs(inp, 0, DEV, windows=1)
    torch.cuda.synchronize()
    status_clean()
    return inp, L, lw, tok_keys, q_tok


def token_scores_gpu(lw, q, w, tok_keys):
    scores = torch.full((lw.B, 64 * lw.max_kept), float("nan"), device=DEV)
    n_tok = torch.full((lw.B,), -1, dtype=torch.int32, device=DEV)
    lsa.lsa_token_score(q, w, tok_keys, lw.chunk_table, lw.kept[0], lw.n_kept[0], lw.max_chunks, scores, n_tok)
    return scores, n_tok


def topk_tokens_gpu(scores, n_tok, k, max_sel=None):
    B = scores.shape[0]
    max_sel = k if max_sel is None else max_sel
    sel = torch.full((B, max_sel), -7, dtype=torch.int32, device=DEV)
    n_sel = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_topk_tokens(scores, n_tok, k, sel, n_sel, cu)
    return sel, n_sel, cu


def assert_token_selection(got, gpu_scores, ref_scores, k):
    """Bit-exact against the oracle's rule on the GPU's fp32 scores; against the
    fp64 scores, differences only inside the tie window at the k-th score."""
    same = oracle.topk_tokens(gpu_scores, k)
    ref = oracle.topk_tokens(ref_scores, k)
    for b in range(len(got)):
        assert got[b] == list(same[b]), f"seq {b}: differs from the rule on its own scores"
        if got[b] == list(ref[b]):
            continue
        s = ref_scores[b]
        order = np.lexsort((np.arange(len(s)), -s))
        sk, sk1 = s[order[k - 1]], s[order[k]]
        for p in set(got[b]) ^ set(ref[b]):
            assert abs(s[p] - sk) <= TIE_RTOL * abs(sk) + (sk - sk1), f"seq {b}: position {p} not at the boundary"


@pytest.mark.parametrize("name,kw", [("128k", {}), ("batched", {"batch": 6, "pools": True})])
def test_token_scores_match_oracle(name, kw):
    inp, L, lw, tok_keys, q_tok = recalled(name, **kw)
    scores, n_tok = token_scores_gpu(lw, q_tok[0, 5], L.w, tok_keys)
    torch.cuda.synchronize()
    status_clean()
    kept = lw.kept_lists()
    ref = oracle.token_scores(f64(q_tok[0, 5]), f64(L.w), f64(tok_keys), i64(inp.chunk_table), kept,
                              inp.max_chunks)
    g = f64(scores)
    assert i64(n_tok).tolist() == [64 * len(k) for k in kept]
    for b in range(lw.B):
        n = len(ref[b])
        err = np.abs(g[b, :n] - ref[b])
        assert np.all(err <= SCORE_RTOL * np.abs(ref[b])), f"seq {b}: worst rel {np.max(err / np.abs(ref[b]))}"
        assert np.all(np.isnan(g[b, n:])), "entries past the recalled tokens must be left untouched"


@pytest.mark.parametrize("k", [64, 2048, 4096])
def test_token_topk_matches_oracle(k):
    inp, L, lw, tok_keys, q_tok = recalled("batched", batch=6)
    scores, n_tok = token_scores_gpu(lw, q_tok[0, 0], L.w, tok_keys)
    sel, n_sel, cu = topk_tokens_gpu(scores, n_tok, k)
    torch.cuda.synchronize()
    status_clean()
    kept = lw.kept_lists()
    ref_scores = oracle.token_scores(f64(q_tok[0, 0]), f64(L.w), f64(tok_keys), i64(inp.chunk_table), kept,
                                     inp.max_chunks)
    g = f64(scores)
    gpu_scores = [g[b, : 64 * len(kept[b])] for b in range(lw.B)]
    got = kept_from_gpu(sel, n_sel)
    assert i64(n_sel).tolist() == [min(k, 64 * len(kb)) for kb in kept]
    assert i64(cu).tolist() == np.concatenate([[0], np.cumsum(i64(n_sel))]).tolist()
    assert_token_selection(got, gpu_scores, ref_scores, k)


@pytest.mark.parametrize("n", [5000, 40000, 131072, 131073])
def test_token_topk_ties_and_signed_zero(n):
    """All-equal scores keep the first k positions; -0.0 ties with +0.0; NaN last.
    The sizes reach the one-CTA kernel, the 8-CTA cluster kernel (up to 131072
    candidates, its largest) and the one-CTA kernel that re-reads the scores."""
    B = 3
    s = torch.zeros((B, n), device=DEV)
    s[1] = -0.0
    s[1, ::2] = 0.0
    s[2] = torch.rand(n, generator=torch.Generator(device=DEV).manual_seed(3), device=DEV)
    s[2, 100:200] = float("nan")
    n_tok = torch.tensor([n, n, n], dtype=torch.int32, device=DEV)
    sel, n_sel, _ = topk_tokens_gpu(s, n_tok, 128)
    torch.cuda.synchronize()
    status_clean()
    got = kept_from_gpu(sel, n_sel)
    assert got[0] == list(range(128)) and got[1] == list(range(128))
    assert not any(100 <= p < 200 for p in got[2])
    # NaN ranks after every number: the oracle's rule on the same scores with
    # NaN mapped to -inf (4900 finite scores, so no NaN or -inf is selected)
    finite = f64(s[2])
    finite[np.isnan(finite)] = -np.inf
    assert got[2] == list(oracle.topk_tokens([finite], 128)[0])


@pytest.mark.parametrize("n,k", [(131073, 2048), (200000, 128)])
def test_token_topk_reread_path_random_scores(n, k):
    """Beyond 131072 candidates the one-CTA kernel re-reads the scores from
    memory.  Random scores (and scores quantised to 1/256, so the boundary
    falls inside a long run of ties) must select exactly what the oracle's
    rule selects on the same fp32 scores."""
    g = torch.Generator(device=DEV).manual_seed(n + k)
    s = torch.rand((3, n), generator=g, device=DEV)
    s[1] = torch.floor(s[1] * 256.0) / 256.0
    s[2] = torch.randn((n,), generator=g, device=DEV)
    lens = [n, n - 77, n - 1]
    n_tok = torch.tensor(lens, dtype=torch.int32, device=DEV)
    sel, n_sel, cu = topk_tokens_gpu(s, n_tok, k)
    torch.cuda.synchronize()
    status_clean()
    got = kept_from_gpu(sel, n_sel)
    host_scores = f64(s)
    ref = oracle.topk_tokens([host_scores[b, : lens[b]] for b in range(3)], k)
    for b in range(3):
        assert got[b] == list(ref[b]), f"seq {b}"
    assert i64(cu).tolist() == [0, k, 2 * k, 3 * k]


def two_call_selection(lw, q, w, tok_keys, k, max_sel=None):
    scores, n_tok = token_scores_gpu(lw, q, w, tok_keys)
    sel, n_sel, cu = topk_tokens_gpu(scores, n_tok, k, max_sel)
    return scores, n_tok, sel, n_sel, cu


def fused_selection(lw, q, w, tok_keys, k, ws, max_sel=None, keys_unchanged=False):
    B = lw.B
    max_sel = k if max_sel is None else max_sel
    scores = torch.full((B, 64 * lw.max_kept), float("nan"), device=DEV)
    n_tok = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    sel = torch.full((B, max_sel), -7, dtype=torch.int32, device=DEV)
    n_sel = torch.full((B,), -7, dtype=torch.int32, device=DEV)
    cu = torch.full((B + 1,), -7, dtype=torch.int32, device=DEV)
    lsa.lsa_select_tokens(q, w, tok_keys, lw.chunk_table, lw.kept[0], lw.n_kept[0], lw.max_chunks, k, scores, n_tok,
                          sel, n_sel, cu, ws, keys_unchanged=keys_unchanged)
    return scores, n_tok, sel, n_sel, cu


def assert_same_selection(a, b):
    for x, y, name in zip(a, b, ("scores", "n_tokens", "sel", "n_sel", "cu_sel")):
        if name == "sel":   # entries past n_sel are not written
            n = a[3].cpu().tolist()
            for i, m in enumerate(n):
                assert torch.equal(x[i, :m], y[i, :m]), f"sel of sequence {i}"
        else:
            assert torch.equal(torch.nan_to_num(x, nan=-9.0) if x.is_floating_point() else x,
                               torch.nan_to_num(y, nan=-9.0) if y.is_floating_point() else y), name


@pytest.mark.parametrize("name,kw,k", [("128k", {}, 2048), ("500k", {}, 2048), ("batched", {"batch": 2}, 1024),
                                       ("batched", {"batch": 2}, 64), ("batched", {"batch": 8}, 1024),
                                       ("tiny", {}, 2048)])
def test_select_tokens_equals_score_then_topk(name, kw, k):
    """lsa_select_tokens (scores counted into bins, the selection driven by the
    counts) gives the two-call path's outputs bit for bit, twice in a row (the
    bin counts are left zeroed), and the oracle's rule on its own scores.  A
    batch of 8 has a scorer grid of more than one wave and takes the two-call
    path inside the library."""
    inp, L, lw, tok_keys, q_tok = recalled(name, **kw)
    ws = lsa.new_select_tokens_workspace(lw.B)
    ref = two_call_selection(lw, q_tok[0, 3], L.w, tok_keys, k)
    for call in range(2):   # the second call loads its keys before the preceding kernel ends
        got = fused_selection(lw, q_tok[0, 3], L.w, tok_keys, k, ws, keys_unchanged=call > 0)
        torch.cuda.synchronize()
        status_clean()
        assert_same_selection(got, ref)
        assert int(torch.count_nonzero(ws)) == 0, f"call {call}: the bin counts must be left zeroed"
    kept = lw.kept_lists()
    g = f64(got[0])
    sel = kept_from_gpu(got[2], got[3])
    same = oracle.topk_tokens([g[b, : 64 * len(kept[b])] for b in range(lw.B)], k)
    for b in range(lw.B):
        assert sel[b] == list(same[b]), f"seq {b}"


def test_select_tokens_exact_path_on_ties():
    """A zero indexer query makes every token score sum(w)/2: one bin holds
    every token, so the selection takes its exact radix-select path, and keeps
    the first k positions."""
    inp, L, lw, tok_keys, q_tok = recalled("batched", batch=2)
    ws = lsa.new_select_tokens_workspace(lw.B)
    zero_q = torch.zeros_like(q_tok[0, 0])
    got = fused_selection(lw, zero_q, L.w, tok_keys, 512, ws)
    ref = two_call_selection(lw, zero_q, L.w, tok_keys, 512)
    torch.cuda.synchronize()
    status_clean()
    assert_same_selection(got, ref)
    for b, s in enumerate(kept_from_gpu(got[2], got[3])):
        assert s == list(range(len(s))), f"seq {b}"
    assert int(torch.count_nonzero(ws)) == 0


def test_select_tokens_crowded_boundary_bin():
    """An indexer query a thousand times smaller puts nearly every score in one
    or two bins: the boundary bin overflows the candidate lists and the cluster
    takes its exact path, with the two-call path's result."""
    inp, L, lw, tok_keys, q_tok = recalled("128k")
    ws = lsa.new_select_tokens_workspace(lw.B)
    small_q = (q_tok[0, 2].float() * 1e-3).to(torch.bfloat16)
    got = fused_selection(lw, small_q, L.w, tok_keys, 2048, ws)
    ref = two_call_selection(lw, small_q, L.w, tok_keys, 2048)
    torch.cuda.synchronize()
    status_clean()
    assert_same_selection(got, ref)
    assert int(torch.count_nonzero(ws)) == 0


def test_select_tokens_beyond_the_bitmap():
    """131136 recalled tokens (2049 chunks): the scorer's grid is more than one
    wave, so the library runs the two-call path; same result."""
    n_chunks = torch.tensor([2050], dtype=torch.int32, device=DEV)
    lw = LayerWindow(n_chunks, torch.tensor([2048], dtype=torch.int32, device=DEV), None, 2050, DEV, fine_k=2048)
    lw.kept[0][0] = torch.arange(2049, dtype=torch.int32, device=DEV)
    lw.n_kept[0][0] = 2049
    tok_keys = workloads.randn_bf16((2050, 64, 128), 123, DEV)
    q = workloads.randn_bf16((1, 16, 128), 124, DEV)
    w = torch.rand(16, generator=torch.Generator(device=DEV).manual_seed(125), device=DEV)
    ws = lsa.new_select_tokens_workspace(1)
    got = fused_selection(lw, q, w, tok_keys, 2048, ws)
    ref = two_call_selection(lw, q, w, tok_keys, 2048)
    torch.cuda.synchronize()
    status_clean()
    assert int(got[1][0]) == 2049 * 64
    assert_same_selection(got, ref)
    assert int(torch.count_nonzero(ws)) == 0


def test_gather_tokens_bit_exact():
    inp, L, lw, tok_keys, q_tok = recalled("batched", batch=6)
    scores, n_tok = token_scores_gpu(lw, q_tok[0, 1], L.w, tok_keys)
    k = 1024
    sel, n_sel, cu_sel = topk_tokens_gpu(scores, n_tok, k)
    units = lw.B * k // 64
    k_out = torch.zeros((8, units, 64, 128), dtype=torch.bfloat16, device=DEV)
    v_out = torch.zeros_like(k_out)
    cu_units = torch.full((lw.B + 1,), -1, dtype=torch.int32, device=DEV)
    lsa.lsa_gather_tokens(lw.k_bufs[0], lw.v_bufs[0], lw.cu_kept[0], sel, cu_sel, k_out, v_out, cu_units)
    torch.cuda.synchronize()
    status_clean()
    cs, ck = i64(cu_sel), i64(lw.cu_kept[0])
    assert i64(cu_units).tolist() == (cs // 64).tolist()
    got = kept_from_gpu(sel, n_sel)
    for b in range(lw.B):
        p = torch.tensor(got[b], device=DEV, dtype=torch.int64)
        chunk = int(ck[b]) + p // 64
        row = p % 64
        want_k = cm(lw.k_bufs[0])[chunk, :, row]                   # [n, 8, 128]
        want_v = cm(lw.v_bufs[0])[chunk, :, row]
        u0 = int(cs[b]) // 64
        n = len(got[b])
        have_k = cm(k_out)[u0: u0 + n // 64].permute(0, 2, 1, 3).reshape(n, 8, 128)
        have_v = cm(v_out)[u0: u0 + n // 64].permute(0, 2, 1, 3).reshape(n, 8, 128)
        assert torch.equal(have_k, want_k) and torch.equal(have_v, want_v), f"seq {b}"


@pytest.mark.parametrize("name,kw,k", [("128k", {}, 2048), ("batched", {"batch": 6}, 1024)])
def test_fine_step_attention_matches_oracle(name, kw, k):
    """One whole fine step through the window API: token stage, then attention over
    the selected tokens, against the oracle's attention over the GPU's selection."""
    inp, L, _, tok_keys, q_tok = recalled(name, **kw)
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, fine_k=k)
    lw.select(L.q_idx[0], L.w, L.chunk_keys)
    lw.gather(L.k_pool, L.v_pool)
    out = torch.empty((lw.B, 64, 128), device=DEV)
    lw.fine_select(q_tok[0, 7], L.w, tok_keys)
    lw.attend(L.q[0, 7], out)
    torch.cuda.synchronize()
    status_clean()
    sel = kept_from_gpu(lw.sel, lw.n_sel)
    heads = None if lw.B == 1 else [0, 9, 18, 27, 36, 45, 54, 63]
    ref = oracle.fine_decode_attn(f64(L.q[0, 7]), f64(cm(lw.k_bufs[0])), f64(cm(lw.v_bufs[0])), i64(lw.cu_kept[0]), sel,
                                  heads=heads)
    assert_attention_close(out, ref, heads=heads)


def test_select_tokens_flagged_writes_every_count_including_empty_sequences():
    """With LSA_TOKENS_UNCHANGED the scorer's CTAs that find no rows leave at
    once, but each sequence's first CTA still waits and writes its token count:
    a flagged call into fresh outputs (counts set to -1) equals the unflagged
    call bit for bit, the sequence with nothing recalled included."""
    B = 3
    n_chunks = torch.tensor([0, 3, 40], dtype=torch.int32, device=DEV)
    k_per_seq = torch.tensor([0, 2, 9], dtype=torch.int32, device=DEV)
    max_chunks = 40
    g = torch.Generator(device=DEV).manual_seed(18)
    n_slots = B * max_chunks
    keys = torch.randn((n_slots, 128), generator=g, device=DEV).to(torch.bfloat16)
    tok_keys = torch.randn((n_slots, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand(16, generator=g, device=DEV)
    q_idx = torch.randn((B, 16, 128), generator=g, device=DEV).to(torch.bfloat16)
    q_tok = torch.randn((B, 16, 128), generator=g, device=DEV).to(torch.bfloat16)
    lw = LayerWindow(n_chunks, k_per_seq, None, max_chunks, DEV, fine_k=256)
    lw.select(q_idx, w, keys)
    ws = lsa.new_select_tokens_workspace(lw.B)
    ref = fused_selection(lw, q_tok, w, tok_keys, 256, ws)
    got = fused_selection(lw, q_tok, w, tok_keys, 256, ws, keys_unchanged=True)
    torch.cuda.synchronize()
    status_clean()
    assert i64(got[1]).tolist() == [0, 192, 640]
    assert_same_selection(got, ref)


def test_fine_stage_short_and_empty_sequences():
    """A sequence with fewer recalled tokens than k keeps them all (the step then
    equals chunk attention); a sequence with nothing recalled gets zeros."""
    B = 3
    n_chunks = torch.tensor([0, 3, 40], dtype=torch.int32, device=DEV)
    k_per_seq = torch.tensor([0, 2, 9], dtype=torch.int32, device=DEV)
    max_chunks = 40
    g = torch.Generator(device=DEV).manual_seed(8)
    n_slots = B * max_chunks
    k_pool = torch.randn((n_slots, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    v_pool = torch.randn((n_slots, 8, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    keys = torch.randn((n_slots, 128), generator=g, device=DEV).to(torch.bfloat16)
    tok_keys = torch.randn((n_slots, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand(16, generator=g, device=DEV)
    q_idx = torch.randn((B, 16, 128), generator=g, device=DEV).to(torch.bfloat16)
    q_tok = torch.randn((B, 16, 128), generator=g, device=DEV).to(torch.bfloat16)
    q = torch.randn((B, 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    lw = LayerWindow(n_chunks, k_per_seq, None, max_chunks, DEV, fine_k=256)
    lw.select(q_idx, w, keys)
    lw.gather(k_pool, v_pool)
    lw.fine_select(q_tok, w, tok_keys)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lw.attend(q, out)
    torch.cuda.synchronize()
    status_clean()
    assert i64(lw.n_sel).tolist() == [0, 192, 256]
    sel = kept_from_gpu(lw.sel, lw.n_sel)
    assert sel[1] == list(range(192))
    ref = oracle.fine_decode_attn(f64(q), f64(cm(lw.k_bufs[0])), f64(cm(lw.v_bufs[0])), i64(lw.cu_kept[0]), sel)
    assert_attention_close(out, ref)
    assert torch.all(out[0] == 0)
    chunk_ref = oracle.sparse_decode_attn(f64(q), f64(cm(lw.k_bufs[0])), f64(cm(lw.v_bufs[0])), i64(lw.cu_kept[0]),
                                          seqs=[1])
    assert_attention_close(out[1:2], chunk_ref[1:2])


@pytest.mark.parametrize("keys_unchanged", [False, True])
def test_fine_steps_pipelined_select_own_scores(keys_unchanged):
    """Fine steps back to back on one stream, no host synchronisation between
    them (each kernel a programmatic dependent of the one before, as in a
    window): three windows of 64 steps, each step's selection copied aside on
    the stream, then every selection checked bit for bit against the oracle's
    top-k of that step's own fp32 scores.  A selection kernel that read its
    scores before the scorer had finished them would differ here."""
    inp = workloads.make_inputs("tiny", DEV)
    L = inp.layers[0]
    tok_keys, q_tok = workloads.fine_inputs(inp, 0, DEV)
    kn, vn = workloads.decoded_tokens(inp, 0, DEV)
    k = 256
    for _ in range(3):
        lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, fine_k=k, causal=True)
        outs = torch.empty((64, 1, 64, 128), device=DEV)
        sel_at = torch.empty((64,) + tuple(lw.sel.shape), dtype=lw.sel.dtype, device=DEV)
        nsel_at = torch.empty((64,) + tuple(lw.n_sel.shape), dtype=lw.n_sel.dtype, device=DEV)
        sc_at = torch.empty((64,) + tuple(lw.tok_scores.shape), dtype=lw.tok_scores.dtype, device=DEV)
        lw.select(L.q_idx[0], L.w, L.chunk_keys)
        lw.gather(L.k_pool, L.v_pool)
        lw.reset_local()
        for t in range(64):
            lw.append(kn[0, t], vn[0, t])
            lw.fine_select(q_tok[0, t], L.w, tok_keys, keys_unchanged=keys_unchanged and t > 0)
            lw.attend(L.q[0, t], outs[t])
            sel_at[t].copy_(lw.sel)
            nsel_at[t].copy_(lw.n_sel)
            sc_at[t].copy_(lw.tok_scores)
        torch.cuda.synchronize()
        status_clean()
        n = int(lw.n_tokens[0])
        for t in range(64):
            own = f64(sc_at[t])[0, :n]
            want = list(oracle.topk_tokens([own], k)[0])
            got = sel_at[t, 0, : int(nsel_at[t, 0])].cpu().tolist()
            assert got == want, f"step {t}: selection differs from the top-k of its own scores"


def test_window_tiny_fine_and_causal():
    """A whole tiny window with the fine stage (k = 256 of 576 recalled tokens) and
    the causal local chunk, all 64 steps, against the oracle step by step."""
    inp = workloads.make_inputs("tiny", DEV)
    L = inp.layers[0]
    tok_keys, q_tok = workloads.fine_inputs(inp, 0, DEV)
    kn, vn = workloads.decoded_tokens(inp, 0, DEV)
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, fine_k=256, causal=True)
    outs = torch.empty((64, 1, 64, 128), device=DEV)
    sels = []
    lw.select(L.q_idx[0], L.w, L.chunk_keys)
    lw.gather(L.k_pool, L.v_pool)
    lw.reset_local()
    for t in range(64):
        lw.append(kn[0, t], vn[0, t])
        lw.fine_select(q_tok[0, t], L.w, tok_keys)
        lw.attend(L.q[0, t], outs[t])
        sels.append(kept_from_gpu(lw.sel, lw.n_sel))
    torch.cuda.synchronize()
    status_clean()
    kept = lw.kept_lists()
    kb, vb, cu = f64(cm(lw.k_bufs[0])), f64(cm(lw.v_bufs[0])), i64(lw.cu_kept[0])
    k_loc, v_loc = f64(lw.k_local), f64(lw.v_local)
    for t in range(64):
        ref_scores = oracle.token_scores(f64(q_tok[0, t]), f64(L.w), f64(tok_keys), i64(inp.chunk_table), kept,
                                         inp.max_chunks)
        want = oracle.topk_tokens(ref_scores, 256)
        assert sels[t][0] == list(want[0]), f"step {t}: token selection differs"
        # fine attention over the selected tokens plus the t + 1 decoded tokens
        sel = np.asarray(sels[t][0])
        ch, row = cu[0] + sel // 64, sel % 64
        units_k = kb[ch, :, row].reshape(-1, 64, 8, 128).transpose(0, 2, 1, 3)
        units_v = vb[ch, :, row].reshape(-1, 64, 8, 128).transpose(0, 2, 1, 3)
        ref = oracle.sparse_decode_attn(f64(L.q[0, t]), units_k, units_v, [0, units_k.shape[0]], k_local=k_loc,
                                        v_local=v_loc, local_len=[t + 1])
        assert_attention_close(outs[t], ref)


def test_selected_in_place_equals_packed_path():
    """lsa_sparse_decode_attn_selected (the selected rows copied straight from the
    compact buffer) equals lsa_gather_tokens + lsa_sparse_decode_attn bit for bit;
    a position outside the recalled tokens reads as zeros and is reported."""
    inp, L, lw, tok_keys, q_tok = recalled("batched", batch=6)
    k = 1024
    scores, n_tok = token_scores_gpu(lw, q_tok[0, 3], L.w, tok_keys)
    sel, n_sel, cu_sel = topk_tokens_gpu(scores, n_tok, k)
    B = lw.B
    units = B * k // 64
    k_out = torch.zeros((8, units, 64, 128), dtype=torch.bfloat16, device=DEV)
    v_out = torch.zeros_like(k_out)
    cu_units = torch.zeros((B + 1,), dtype=torch.int32, device=DEV)
    lsa.lsa_gather_tokens(lw.k_bufs[0], lw.v_bufs[0], lw.cu_kept[0], sel, cu_sel, k_out, v_out, cu_units)
    q = L.q[0, 3]
    out_p = torch.full((B, 64, 128), float("nan"), device=DEV)
    out_s = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn(q, k_out, v_out, cu_units, out_p, lsa.new_attn_workspace(B))
    lsa.lsa_sparse_decode_attn_selected(q, lw.k_bufs[0], lw.v_bufs[0], lw.cu_kept[0], sel, cu_sel, out_s,
                                        lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    status_clean()
    assert torch.equal(out_s, out_p)
    # one corrupted position: its rows are zeros, the status says BAD_CHUNK
    bad = sel.clone()
    b0 = int(np.argmax(i64(n_sel)))
    bad[b0, 5] = 10 ** 8
    out_b = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_selected(q, lw.k_bufs[0], lw.v_bufs[0], lw.cu_kept[0], bad, cu_sel, out_b,
                                        lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    assert lsa.read_device_status() & 4          # BAD_CHUNK
    cs, ck = i64(cu_sel), i64(lw.cu_kept[0])
    n = int(cs[b0 + 1] - cs[b0])
    p = sel[b0, :n].to(torch.int64)
    K = f64(cm(lw.k_bufs[0])[int(ck[b0]) + p // 64, :, p % 64])    # [n, 8, 128], gathered on the GPU
    V = f64(cm(lw.v_bufs[0])[int(ck[b0]) + p // 64, :, p % 64])
    K[5] = 0.0
    V[5] = 0.0
    units_k = K.reshape(-1, 64, 8, 128).transpose(0, 2, 1, 3)
    units_v = V.reshape(-1, 64, 8, 128).transpose(0, 2, 1, 3)
    ref = oracle.sparse_decode_attn(f64(q[b0: b0 + 1]), units_k, units_v, [0, units_k.shape[0]])
    assert_attention_close(out_b[b0: b0 + 1], ref)


@pytest.mark.slow
def test_fine_stage_500k_full_size():
    """The token-level stage on the 500K workload as the bench runs it (52480 recalled
    tokens, k = 2048, selected tokens read in place), at steps 0 and 63: token
    scores for every recalled token, the selection, and attention on sampled heads."""
    inp = workloads.make_inputs("500k", DEV, layers=1, windows=1)
    L = inp.layers[0]
    tok_keys, q_tok = workloads.fine_inputs(inp, 0, DEV, windows=1)
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, fine_k=2048)
    lw.select(L.q_idx[0], L.w, L.chunk_keys)
    lw.gather(L.k_pool, L.v_pool)
    kept = lw.kept_lists()
    keys32 = tok_keys.float().cpu().numpy()          # exact for bf16 values
    total = int(lw.cu_kept[0][-1])
    kb, vb = cm(lw.k_bufs[0])[:total].float().cpu().numpy(), cm(lw.v_bufs[0])[:total].float().cpu().numpy()
    heads = [0, 9, 18, 27, 36, 45, 54, 63]
    for t in (0, 63):
        out = torch.empty((1, 64, 128), device=DEV)
        lw.fine_select(q_tok[0, t], L.w, tok_keys)
        lw.attend(L.q[0, t], out)
        torch.cuda.synchronize()
        status_clean()
        ref_scores = oracle.token_scores(f64(q_tok[0, t]), f64(L.w), keys32, i64(inp.chunk_table), kept,
                                         inp.max_chunks)
        n = len(ref_scores[0])
        g = f64(lw.tok_scores)[0, :n]
        err = np.abs(g - ref_scores[0])
        assert np.all(err <= SCORE_RTOL * np.abs(ref_scores[0])), f"step {t}: token scores off"
        got = kept_from_gpu(lw.sel, lw.n_sel)
        assert_token_selection(got, [g], ref_scores, 2048)
        ref = oracle.fine_decode_attn(f64(L.q[0, t]), kb, vb, i64(lw.cu_kept[0]), got, heads=heads)
        assert_attention_close(out, ref, heads=heads)


@pytest.mark.slow
def test_causal_window_500k_sampled_steps():
    """A causal 500K window as the bench runs it (the step's token appended and
    attended in one launch), all 64 steps on the GPU, steps 0 and 63 against the
    oracle on sampled heads: the kept chunks plus the first t + 1 decoded tokens."""
    inp = workloads.make_inputs("500k", DEV, layers=1, windows=1)
    L = inp.layers[0]
    kn, vn = workloads.decoded_tokens(inp, 0, DEV, windows=1)
    lw = LayerWindow(inp.n_chunks, inp.k_per_seq, inp.chunk_table, inp.max_chunks, DEV, causal=True)
    outs = torch.empty((64, 1, 64, 128), device=DEV)
    lw.run_window(L.q_idx[0], L.w, L.chunk_keys, L.k_pool, L.v_pool, L.q[0], outs, k_new=kn[0], v_new=vn[0])
    torch.cuda.synchronize()
    status_clean()
    assert int(lw.local_len[0]) == 64
    total = int(lw.cu_kept[0][-1])
    kb, vb = cm(lw.k_bufs[0])[:total].float().cpu().numpy(), cm(lw.v_bufs[0])[:total].float().cpu().numpy()
    kl, vl = f64(lw.k_local), f64(lw.v_local)
    assert np.array_equal(kl[0].transpose(1, 0, 2), f64(kn[0, :, 0]))   # token t at row t of the local chunk
    heads = [0, 9, 18, 27, 36, 45, 54, 63]
    for t in (0, 63):
        ref = oracle.sparse_decode_attn(f64(L.q[0, t]), kb, vb, i64(lw.cu_kept[0]), heads=heads, k_local=kl,
                                        v_local=vl, local_len=[t + 1])
        assert_attention_close(outs[t], ref, heads=heads)
