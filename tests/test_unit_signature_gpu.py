"""Every attention entry point at full size, with results that identify each unit.

The split-K attention cuts the units of all (sequence, KV head) pairs into
contiguous CTA ranges with 32-bit base/remainder arithmetic and walks them
with a cursor; the merge kernel then folds each split pair.  With random keys
and values the elementwise tolerance cannot see a 64-token unit lost or read
twice at a long context (it moves an output by about 8 / T).  Here the keys
are zero and the values one-hot (tests/unit_signature.py), so the output is a
ratio of token counts known in closed form, and a unit dropped, repeated or
read from the wrong head or sequence moves it by at least 64 / T relative,
against a check at 1e-5 relative with exact zeros.  Compact-buffer chunks past
cu_kept[B] and rows that were not selected hold NaN, so a read outside the
attended set poisons the output.

Sizes: the 500K and 1M kept sets (820 and 1639 chunks, one sequence), the
batched workload's 32 ragged kept sets, 4096 sequences (the largest batch),
and launches whose grid has more CTAs than there are units.
"""
import numpy as np
import pytest
import torch

import kv_chunk_selection_b200 as lsa
import workloads
import unit_signature as us

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_chunk_selection_b200 import build
    build.build()
    lsa.lib()
    lsa.read_device_status()
    yield
    torch.cuda.synchronize()


def status_clean():
    bits = lsa.read_device_status()
    assert bits == 0, f"device status {lsa.decode_status(bits)}"


def batched_kept():
    n, k = workloads.lengths_for(workloads.WORKLOADS["batched"])
    return (np.minimum(k.numpy(), n.numpy() - 1) + 1).tolist()


def max_batch_kept():
    return np.random.default_rng(4096).integers(0, 4, size=4096).tolist()


# name -> (kept chunks per sequence, extra compact chunks past cu_kept[B])
CASES = {
    "500k": ([820], 0),
    "1m": ([1639], 0),
    "batched": (batched_kept(), 0),
    "max_batch": (max_batch_kept(), 0),
    "grid_over_units": ([3, 0, 2], 2000),          # 40 units, 148 CTAs
    "one_chunk_big_buffer": ([1], 600),            # 8 units, 148 CTAs
}


def signature_buffers(n_kept, extra, seed):
    """Zero keys, one-hot values; chunks past cu_kept[B] hold NaN in K and V."""
    cu = np.concatenate([[0], np.cumsum(n_kept)]).astype(np.int64)
    total = int(cu[-1])
    buf = total + extra
    off = us.offsets(max(buf, 1), seed)
    v = us.compact_v(off[:, :buf], DEV)
    k = torch.zeros_like(v)
    if extra:
        v[:, total:] = float("nan")
        k[:, total:] = float("nan")
    B = len(n_kept)
    q = torch.randn((B, 64, 128), generator=torch.Generator(device=DEV).manual_seed(seed), device=DEV).to(
        torch.bfloat16)
    cu_t = torch.tensor(cu, dtype=torch.int32, device=DEV)
    return q, k, v, cu_t, cu, off


def host(t):
    return t.detach().double().cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_signature_chunks(name):
    n_kept, extra = CASES[name]
    q, k, v, cu_t, cu, off = signature_buffers(n_kept, extra, seed=11)
    B = len(n_kept)
    want = us.expected_chunks(off, cu)
    ws = lsa.new_attn_workspace(B)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn(q, k, v, cu_t, out, ws)
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), want, f"{name}, first call")
    # a second step of the window: K/V streamed before the previous kernel ends
    out2 = torch.full_like(out, float("nan"))
    lsa.lsa_sparse_decode_attn(q, k, v, cu_t, out2, ws, kv_unchanged=True)
    torch.cuda.synchronize()
    status_clean()
    assert torch.equal(out, out2), f"{name}: the KV-unchanged step differs"


@pytest.mark.parametrize("name", ["500k", "batched", "max_batch", "grid_over_units"])
def test_signature_local(name):
    n_kept, extra = CASES[name]
    q, k, v, cu_t, cu, off = signature_buffers(n_kept, extra, seed=12)
    B = len(n_kept)
    offl = us.local_offsets(B, 13)
    v_loc = us.one_hot_rows(torch.from_numpy(offl).to(DEV))                 # [B, 8, 64, 128]
    k_loc = torch.zeros_like(v_loc)
    ll = np.random.default_rng(14).integers(0, 65, size=B)
    ll[0] = 37 if B == 1 else ll[0]
    ll_t = torch.tensor(ll, dtype=torch.int32, device=DEV)
    want = us.expected_chunks(off, cu, local_off=offl, local_len=ll)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_local(q, k, v, cu_t, k_loc, v_loc, ll_t, out, lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), want, name)


@pytest.mark.parametrize("name", ["500k", "batched", "grid_over_units"])
def test_signature_fused_append(name):
    n_kept, extra = CASES[name]
    q, k, v, cu_t, cu, off = signature_buffers(n_kept, extra, seed=15)
    B = len(n_kept)
    offl = us.local_offsets(B, 16)
    v_loc = us.one_hot_rows(torch.from_numpy(offl).to(DEV))
    k_loc = torch.zeros_like(v_loc)
    n_in = np.random.default_rng(17).integers(0, 64, size=B)
    n_in[0] = 63
    # this step's token is row n_in[b] of the local chunk: its one-hot continues the chunk's pattern
    rows = us.one_hot_rows(torch.from_numpy(offl).to(DEV))                  # [B, 8, 64, 128]
    idx = torch.from_numpy(n_in).to(DEV).view(B, 1, 1, 1).expand(B, 8, 1, 128)
    v_new = torch.gather(rows, 2, idx).squeeze(2).contiguous()              # [B, 8, 128]
    k_new = torch.zeros_like(v_new)
    v_loc[torch.arange(B, device=DEV), :, torch.from_numpy(n_in).to(DEV)] = 7.0   # overwritten by the step
    len_in = torch.tensor(n_in, dtype=torch.int32, device=DEV)
    len_out = torch.full((B,), -1, dtype=torch.int32, device=DEV)
    want = us.expected_chunks(off, cu, local_off=offl, local_len=n_in + 1)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_append(q, k, v, cu_t, k_new, v_new, k_loc, v_loc, len_in, len_out, out,
                                      lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), want, name)
    assert len_out.cpu().numpy().tolist() == (n_in + 1).tolist()
    stored = v_loc[torch.arange(B, device=DEV), :, torch.from_numpy(n_in).to(DEV)]
    assert torch.equal(stored, v_new), "the step's token must be stored in its local row"


def random_selection(n_kept, k, seed):
    rng = np.random.default_rng(seed)
    sel = []
    for n in n_kept:
        tokens = 64 * n
        m = min(k, tokens)
        sel.append(np.sort(rng.choice(tokens, m, replace=False)) if m else np.zeros(0, dtype=np.int64))
    return sel


# (case, selected tokens per sequence, max_sel): the last case sizes the grid
# for 2048 selected tokens per sequence but selects 64, so CTAs outnumber units.
@pytest.mark.parametrize("name,k,max_sel", [("500k", 2048, 2048), ("1m", 2048, 2048), ("batched", 2048, 2048),
                                            ("grid_over_units", 64, 2048)])
def test_signature_selected_in_place(name, k, max_sel):
    n_kept, extra = CASES[name]
    q, k_buf, v_buf, cu_t, cu, off = signature_buffers(n_kept, extra, seed=18)
    B = len(n_kept)
    sel = random_selection(n_kept, k, seed=19)
    # rows that are not selected hold NaN: reading one poisons the output
    mask = torch.ones(v_buf.shape[:3], dtype=torch.bool, device=DEV)
    for b in range(B):
        p = torch.from_numpy(sel[b]).to(DEV)
        mask[:, int(cu[b]) + p // 64, p % 64] = False
    v_buf[mask] = float("nan")
    sel_t = torch.full((B, max_sel), -1, dtype=torch.int32, device=DEV)
    for b in range(B):
        sel_t[b, : len(sel[b])] = torch.from_numpy(sel[b]).to(DEV, torch.int32)
    cu_sel = torch.tensor(np.concatenate([[0], np.cumsum([len(s) for s in sel])]), dtype=torch.int32, device=DEV)
    want = us.expected_selected(off, cu, sel)
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_selected(q, k_buf, v_buf, cu_t, sel_t, cu_sel, out, lsa.new_attn_workspace(B))
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), want, name)


@pytest.mark.parametrize("name", ["500k", "grid_over_units", "one_chunk_big_buffer"])
def test_signature_noalloc(name):
    n_kept, extra = CASES[name]
    q, k, v, cu_t, cu, off = signature_buffers(n_kept, extra, seed=20)
    B = len(n_kept)
    want = us.expected_chunks(off, cu)
    ref = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn(q, k, v, cu_t, ref, lsa.new_attn_workspace(B))
    out = torch.full((B, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_noalloc(q, k, v, cu_t, out)
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), want, name)
    assert torch.equal(out, ref), "the allocation-free call runs the same launch as the workspace call"


def test_signature_noalloc_batched():
    n_kept = batched_kept()
    assert len(n_kept) == 32
    q, k, v, cu_t, cu, off = signature_buffers(n_kept, 0, seed=21)
    out = torch.full((32, 64, 128), float("nan"), device=DEV)
    lsa.lsa_sparse_decode_attn_noalloc(q, k, v, cu_t, out)
    torch.cuda.synchronize()
    status_clean()
    us.assert_signature(host(out), us.expected_chunks(off, cu), "batched")
