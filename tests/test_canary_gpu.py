"""Canary guards around every output buffer (out-of-bounds write detection).

compute-sanitizer is not used on the test machines, so out-of-bounds writes
are caught the plain way: every output buffer of every entry point is carved
out of a larger allocation whose 4 KiB on each side hold a byte pattern, and
the parts of a buffer that a call must not write (entries past a sequence's
count, compact-buffer chunks past cu_kept[B], local rows other than the
appended one) hold the same pattern.  After each call the pattern must be
intact.  The calls run at the edge sizes of the suite: an empty sequence, a
budget K >= n - 1, K = 0, a full local chunk, a token budget k larger than the
recalled tokens, and the largest batch (4096 sequences).
"""
import math

import numpy as np
import pytest
import torch

import kv_chunk_selection_b200 as lsa

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_chunk_selection_b200 import build
    build.build()
    lsa.lib()
    lsa.read_device_status()
    yield
    torch.cuda.synchronize()


class Guarded:
    """A tensor whose allocation has GUARD pattern bytes on both sides."""

    def __init__(self, shape, dtype):
        nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=DEV)
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def bytes(self):
        """The buffer itself as bytes, in its own shape with a trailing byte axis."""
        return self.raw[GUARD:-GUARD].view(tuple(self.t.shape) + (-1,))

    def check(self, what):
        assert bool(torch.all(self.raw[:GUARD] == PATTERN)), f"{what}: write before the buffer"
        assert bool(torch.all(self.raw[-GUARD:] == PATTERN)), f"{what}: write past the buffer"


def untouched(region: torch.Tensor) -> bool:
    return bool(torch.all(region == PATTERN)) if region.numel() else True


def tails_untouched(rows: torch.Tensor, counts) -> bool:
    """rows [B, n, bytes]: every entry j >= counts[b] of row b still holds the pattern."""
    c = torch.as_tensor(np.asarray(counts), device=rows.device).view(-1, 1)
    past = torch.arange(rows.shape[1], device=rows.device).view(1, -1) >= c
    return untouched(rows[past])


def status():
    return lsa.read_device_status()


def edge_batch(seed=5):
    """n_chunks / K per sequence: empty, one chunk, K >= n-1, K = 0, ordinary."""
    n = [0, 1, 2, 5, 40, 30, 64, 3]
    k = [3, 0, 5, 10, 8, 29, 0, 1]
    B = len(n)
    max_chunks = 72
    n_slots = sum(n)
    perm = torch.randperm(n_slots, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    table = torch.zeros((B, max_chunks), dtype=torch.int32)
    off = 0
    for b in range(B):
        table[b, : n[b]] = perm[off: off + n[b]]
        off += n[b]
    return n, k, max_chunks, n_slots, table


def rand_bf16(shape, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    return torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)


def test_canaries_chunk_path_edge_sizes():
    n, k, max_chunks, n_slots, table = edge_batch()
    B = len(n)
    n_t = torch.tensor(n, dtype=torch.int32, device=DEV)
    k_t = torch.tensor(k, dtype=torch.int32, device=DEV)
    table = table.to(DEV)
    q_idx = rand_bf16((B, 16, 128), 1)
    w = torch.rand(16, generator=torch.Generator(device=DEV).manual_seed(2), device=DEV)
    keys = rand_bf16((n_slots, 128), 3)
    k_pool = rand_bf16((n_slots, 8, 64, 128), 4)
    v_pool = rand_bf16((n_slots, 8, 64, 128), 5)

    scores = Guarded((B, max_chunks), torch.float32)
    lsa.lsa_index_score(q_idx, w, keys, table, n_t, scores.t)
    torch.cuda.synchronize()
    assert status() == 0
    scores.check("scores")
    assert tails_untouched(scores.bytes(), n), "scores past a sequence's chunks"

    max_kept = 32
    kept, n_kept, cu = Guarded((B, max_kept), torch.int32), Guarded((B,), torch.int32), Guarded((B + 1,), torch.int32)
    lsa.lsa_topk_chunks(scores.t, n_t, k_t, kept.t, n_kept.t, cu.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((kept, "kept"), (n_kept, "n_kept"), (cu, "cu_kept")):
        g.check(name)
    nk = n_kept.t.cpu().tolist()
    assert nk == [0 if x == 0 else min(kk, x - 1) + 1 for x, kk in zip(n, k)]
    assert tails_untouched(kept.bytes(), nk), "kept past n_kept"

    total = int(cu.t[B])
    extra = 3
    k_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    v_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    lsa.lsa_gather_chunks(k_pool, v_pool, table, kept.t, cu.t, max_chunks, k_buf.t, v_buf.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((k_buf, "k_buf"), (v_buf, "v_buf")):
        g.check(name)
        assert untouched(g.bytes()[:, total:]), f"{name}: chunks past cu_kept[B]"

    # the host tier: the same copy from page-locked pools, plain and delta
    hk, hv = k_pool.cpu().pin_memory(), v_pool.cpu().pin_memory()
    hk_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    hv_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    lsa.lsa_fetch_from_host(hk, hv, table, kept.t, cu.t, max_chunks, hk_buf.t, hv_buf.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((hk_buf, "fetched k_buf"), (hv_buf, "fetched v_buf")):
        g.check(name)
        assert untouched(g.bytes()[:, total:]), f"{name}: chunks past cu_kept[B]"
    assert torch.equal(hk_buf.t[:, :total], k_buf.t[:, :total])
    dk_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    dv_buf = Guarded((8, total + extra, 64, 128), torch.bfloat16)
    reused = torch.zeros(1, dtype=torch.int32, device=DEV)
    lsa.lsa_fetch_from_host_delta(hk, hv, table, kept.t, cu.t, max_chunks, dk_buf.t, dv_buf.t, kept.t, cu.t,
                                  k_buf.t, v_buf.t, reused)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((dk_buf, "delta k_buf"), (dv_buf, "delta v_buf")):
        g.check(name)
        assert untouched(g.bytes()[:, total:]), f"{name}: chunks past cu_kept[B]"
    assert int(reused) == total

    # attention: output and workspace
    q = rand_bf16((B, 64, 128), 6)
    out = Guarded((B, 64, 128), torch.float32)
    ws = Guarded((lsa.lsa_attn_workspace_size(B),), torch.uint8)
    lsa.lsa_sparse_decode_attn(q, k_buf.t, v_buf.t, cu.t, out.t, ws.t)
    torch.cuda.synchronize()
    assert status() == 0
    out.check("out")
    ws.check("workspace")
    assert torch.all(out.t[0] == 0), "an empty sequence gets zeros"

    out_na = Guarded((B, 64, 128), torch.float32)
    lsa.lsa_sparse_decode_attn_noalloc(q, k_buf.t, v_buf.t, cu.t, out_na.t)
    torch.cuda.synchronize()
    assert status() == 0
    out_na.check("noalloc out")
    assert torch.equal(out_na.t, out.t)

    # threshold selection
    tk, tn, tc = Guarded((B, max_chunks), torch.int32), Guarded((B,), torch.int32), Guarded((B + 1,), torch.int32)
    lsa.lsa_threshold_chunks(scores.t, n_t, w, tk.t, tn.t, tc.t, threshold=0.5)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((tk, "threshold kept"), (tn, "threshold n_kept"), (tc, "threshold cu_kept")):
        g.check(name)
    assert tails_untouched(tk.bytes(), tn.t.cpu().tolist()), "threshold kept past n_kept"


def test_canaries_local_chunk_and_fused_append():
    B = 5
    n_kept = [0, 2, 1, 0, 3]
    cu_l = np.concatenate([[0], np.cumsum(n_kept)])
    total = int(cu_l[-1])
    k_buf, v_buf = rand_bf16((8, total, 64, 128), 7), rand_bf16((8, total, 64, 128), 8)
    cu = torch.tensor(cu_l, dtype=torch.int32, device=DEV)
    q = rand_bf16((B, 64, 128), 9)
    k_loc, v_loc = Guarded((B, 8, 64, 128), torch.bfloat16), Guarded((B, 8, 64, 128), torch.bfloat16)
    k_loc.t.copy_(rand_bf16((B, 8, 64, 128), 10))
    v_loc.t.copy_(rand_bf16((B, 8, 64, 128), 11))
    len_in_l = [0, 63, 64, 5, 64]                      # empty, last free row, full, ordinary, full
    len_in = torch.tensor(len_in_l, dtype=torch.int32, device=DEV)
    len_out = Guarded((B,), torch.int32)
    k_new, v_new = rand_bf16((B, 8, 128), 12), rand_bf16((B, 8, 128), 13)
    before_k, before_v = k_loc.t.clone(), v_loc.t.clone()
    out = Guarded((B, 64, 128), torch.float32)
    ws = Guarded((lsa.lsa_attn_workspace_size(B),), torch.uint8)
    lsa.lsa_sparse_decode_attn_append(q, k_buf, v_buf, cu, k_new, v_new, k_loc.t, v_loc.t, len_in, len_out.t,
                                      out.t, ws.t)
    torch.cuda.synchronize()
    assert status() == 8, "a full local chunk reports CAPACITY"          # LSA_DEV_ERR_CAPACITY
    for g, name in ((k_loc, "k_local"), (v_loc, "v_local"), (len_out, "local_len_out"), (out, "out"),
                    (ws, "workspace")):
        g.check(name)
    assert len_out.t.cpu().tolist() == [min(x + 1, 64) for x in len_in_l]
    for b in range(B):
        for name, cur, old, new in (("k", k_loc.t, before_k, k_new), ("v", v_loc.t, before_v, v_new)):
            n = len_in_l[b]
            rows = [r for r in range(64) if r != n]
            assert torch.equal(cur[b][:, rows], old[b][:, rows]), f"{name}_local of sequence {b}: other rows"
            if n < 64:
                assert torch.equal(cur[b][:, n], new[b]), f"{name}_local of sequence {b}: appended row"

    # lsa_append_token + local attention: the same checks on the two-launch path
    k_loc.t.copy_(before_k)
    v_loc.t.copy_(before_v)
    ll = Guarded((B,), torch.int32)
    ll.t.copy_(len_in)
    lsa.lsa_append_token(k_new, v_new, k_loc.t, v_loc.t, ll.t)
    out2 = Guarded((B, 64, 128), torch.float32)
    lsa.lsa_sparse_decode_attn_local(q, k_buf, v_buf, cu, k_loc.t, v_loc.t, ll.t, out2.t, ws.t)
    torch.cuda.synchronize()
    assert status() == 8
    for g, name in ((k_loc, "k_local"), (v_loc, "v_local"), (ll, "local_len"), (out2, "out"), (ws, "workspace")):
        g.check(name)
    assert torch.equal(out2.t, out.t), "fused and two-launch causal steps agree"


def test_canaries_fine_stage_k_beyond_recalled_tokens():
    n, k, max_chunks, n_slots, table = edge_batch(seed=6)
    B = len(n)
    table = table.to(DEV)
    n_t = torch.tensor(n, dtype=torch.int32, device=DEV)
    max_kept = 32
    kept = torch.full((B, max_kept), -1, dtype=torch.int32, device=DEV)
    n_kept = torch.zeros(B, dtype=torch.int32, device=DEV)
    cu = torch.zeros(B + 1, dtype=torch.int32, device=DEV)
    scores = torch.rand((B, max_chunks), generator=torch.Generator(device=DEV).manual_seed(7), device=DEV)
    lsa.lsa_topk_chunks(scores, n_t, torch.tensor(k, dtype=torch.int32, device=DEV), kept, n_kept, cu)
    total = int(cu[B])
    k_buf, v_buf = rand_bf16((8, total, 64, 128), 8), rand_bf16((8, total, 64, 128), 9)
    tok_keys = rand_bf16((n_slots, 64, 128), 10)
    q_tok = rand_bf16((B, 16, 128), 11)
    w = torch.rand(16, generator=torch.Generator(device=DEV).manual_seed(12), device=DEV)
    tok = Guarded((B, 64 * max_kept), torch.float32)
    n_tok = Guarded((B,), torch.int32)
    lsa.lsa_token_score(q_tok, w, tok_keys, table, kept, n_kept, max_chunks, tok.t, n_tok.t)
    torch.cuda.synchronize()
    assert status() == 0
    tok.check("token scores")
    n_tok.check("n_tokens")
    nt = n_tok.t.cpu().tolist()
    assert tails_untouched(tok.bytes(), nt), "token scores past a sequence's tokens"

    kk = 256                                            # more than several sequences recall
    sel, n_sel, cu_sel = Guarded((B, kk), torch.int32), Guarded((B,), torch.int32), Guarded((B + 1,), torch.int32)
    lsa.lsa_topk_tokens(tok.t, n_tok.t, kk, sel.t, n_sel.t, cu_sel.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((sel, "sel"), (n_sel, "n_sel"), (cu_sel, "cu_sel")):
        g.check(name)
    ns = n_sel.t.cpu().tolist()
    assert ns == [min(kk, x) for x in nt]
    assert tails_untouched(sel.bytes(), ns), "sel past n_sel"

    # the same step through lsa_select_tokens (scores counted into bins, the selection driven by the counts)
    tok2 = Guarded((B, 64 * max_kept), torch.float32)
    n_tok2 = Guarded((B,), torch.int32)
    sel2, n_sel2, cu_sel2 = Guarded((B, kk), torch.int32), Guarded((B,), torch.int32), Guarded((B + 1,), torch.int32)
    ws_sel = Guarded((lsa.lib().lsa_select_tokens_workspace_size(B),), torch.uint8)
    ws_sel.t.zero_()
    lsa.lsa_select_tokens(q_tok, w, tok_keys, table, kept, n_kept, max_chunks, kk, tok2.t, n_tok2.t, sel2.t, n_sel2.t,
                          cu_sel2.t, ws_sel.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((tok2, "fused token scores"), (n_tok2, "fused n_tokens"), (sel2, "fused sel"),
                    (n_sel2, "fused n_sel"), (cu_sel2, "fused cu_sel"), (ws_sel, "selection counts")):
        g.check(name)
    assert tails_untouched(tok2.bytes(), nt), "fused token scores past a sequence's tokens"
    assert tails_untouched(sel2.bytes(), ns), "fused sel past n_sel"
    assert int(torch.count_nonzero(ws_sel.t)) == 0, "the counts are left zeroed"
    assert torch.equal(n_sel2.t, n_sel.t) and torch.equal(cu_sel2.t, cu_sel.t)

    units = sum(ns) // 64
    k_out = Guarded((8, units + 2, 64, 128), torch.bfloat16)
    v_out = Guarded((8, units + 2, 64, 128), torch.bfloat16)
    cu_units = Guarded((B + 1,), torch.int32)
    lsa.lsa_gather_tokens(k_buf, v_buf, cu, sel.t, cu_sel.t, k_out.t, v_out.t, cu_units.t)
    q = rand_bf16((B, 64, 128), 13)
    out = Guarded((B, 64, 128), torch.float32)
    ws = Guarded((lsa.lsa_attn_workspace_size(B),), torch.uint8)
    lsa.lsa_sparse_decode_attn_selected(q, k_buf, v_buf, cu, sel.t, cu_sel.t, out.t, ws.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((k_out, "packed k"), (v_out, "packed v"), (cu_units, "cu_units"), (out, "out"),
                    (ws, "workspace")):
        g.check(name)
    for g, name in ((k_out, "packed k"), (v_out, "packed v")):
        assert untouched(g.bytes()[:, units:]), f"{name}: units past cu_units[B]"


def test_canaries_largest_batch():
    B = 4096
    rng = np.random.default_rng(4096)
    n = rng.integers(0, 5, size=B)
    k = rng.integers(0, 3, size=B)
    max_chunks = 4
    n_t = torch.tensor(n, dtype=torch.int32, device=DEV)
    scores = torch.rand((B, max_chunks), generator=torch.Generator(device=DEV).manual_seed(14), device=DEV)
    max_kept = 4
    kept, n_kept, cu = Guarded((B, max_kept), torch.int32), Guarded((B,), torch.int32), Guarded((B + 1,), torch.int32)
    lsa.lsa_topk_chunks(scores, n_t, torch.tensor(k, dtype=torch.int32, device=DEV), kept.t, n_kept.t, cu.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((kept, "kept"), (n_kept, "n_kept"), (cu, "cu_kept")):
        g.check(name)
    assert tails_untouched(kept.bytes(), n_kept.t.cpu().numpy()), "kept past n_kept"
    total = int(cu.t[B])
    k_buf, v_buf = rand_bf16((8, total, 64, 128), 15), rand_bf16((8, total, 64, 128), 16)
    q = rand_bf16((B, 64, 128), 17)
    out = Guarded((B, 64, 128), torch.float32)
    ws = Guarded((lsa.lsa_attn_workspace_size(B),), torch.uint8)
    lsa.lsa_sparse_decode_attn(q, k_buf, v_buf, cu.t, out.t, ws.t)
    k_loc, v_loc = rand_bf16((B, 8, 64, 128), 18), rand_bf16((B, 8, 64, 128), 19)
    ll = torch.tensor(rng.integers(0, 65, size=B), dtype=torch.int32, device=DEV)
    out_l = Guarded((B, 64, 128), torch.float32)
    lsa.lsa_sparse_decode_attn_local(q, k_buf, v_buf, cu.t, k_loc, v_loc, ll, out_l.t, ws.t)
    torch.cuda.synchronize()
    assert status() == 0
    for g, name in ((out, "out"), (out_l, "local out"), (ws, "workspace")):
        g.check(name)
    assert bool(torch.isfinite(out.t).all()) and bool(torch.isfinite(out_l.t).all())
