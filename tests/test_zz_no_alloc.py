"""The allocation-free attention entry point against the regular one.

lsa_sparse_decode_attn_noalloc serves callers that cannot allocate device
memory (programs with no device allocator of their own, plug-ins inside a
framework that owns all device memory, loops that must not call cudaMalloc
because it can synchronise the device): its split-K scratch is a fixed array
inside the library instead of a caller-provided workspace.  This test calls it
through the C ABI (ctypes, raw pointers) twice in a row on the same inputs and
checks both results against lsa_sparse_decode_attn within the attention
tolerance of the parity tests (the two calls run the same launch, so the
results are also bit-identical), checks small batches whose kept total is far
below the buffer size against the fp64 oracle, and checks that a batch beyond
the array's limit is refused.  It builds and loads the library itself, so it passes alone
in a fresh process as well as after the other tests; the file name makes
pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_chunk_selection_b200 as lsa
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"
ATT_ATOL, ATT_RTOL = 2e-3, 1e-3
NOALLOC_MAX_BATCH = 32
UNSUPPORTED = -2


@pytest.fixture(scope="module")
def L():
    from kv_chunk_selection_b200 import build
    build.build()
    return lsa.lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(n_kept, seed, extra=0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    total = int(sum(n_kept)) + extra      # extra chunks past cu_kept[B] are never read
    shape = (8, total, 64, 128)            # head-major compact buffer
    kb = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    vb = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(n_kept)]), dtype=torch.int32, device=DEV)
    q = torch.randn((len(n_kept), 64, 128), generator=g, device=DEV).to(torch.bfloat16)
    return q, kb, vb, cu


def test_noalloc_matches_workspace_entry_point_twice(L):
    # Ragged batch: pairs split across many CTAs (merged through the scratch),
    # pairs handled whole by one CTA, and an empty sequence.
    n_kept = [1, 0, 37, 3, 150, 9, 260, 2]
    q, kb, vb, cu = _inputs(n_kept, seed=77)
    B = q.shape[0]
    scale = 1.0 / np.sqrt(128.0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    ref = torch.empty((B, 64, 128), device=DEV)
    ws = torch.zeros(L.lsa_attn_workspace_size(B), dtype=torch.uint8, device=DEV)
    assert L.lsa_sparse_decode_attn(_p(q), _p(kb), _p(vb), kb.shape[1], _p(cu), B, scale, _p(ref), _p(ws),
                                    ws.numel(), 0, stream) == 0

    for call in range(2):
        out = torch.full((B, 64, 128), float("nan"), device=DEV)
        st = L.lsa_sparse_decode_attn_noalloc(_p(q), _p(kb), _p(vb), kb.shape[1], _p(cu), B, scale, _p(out),
                                              stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        r, o = ref.double().cpu().numpy(), out.double().cpu().numpy()
        assert np.all(np.isfinite(o)), f"call {call}"
        assert np.all(np.abs(o - r) <= ATT_ATOL + ATT_RTOL * np.abs(r)), f"call {call}"
        assert torch.equal(out, ref), f"call {call}: same launch, same bits"
    bits = ctypes.c_uint(0)
    assert L.lsa_read_device_status(stream, ctypes.byref(bits)) == 0
    assert bits.value == 0


@pytest.mark.parametrize("n_kept,extra", [([1], 0), ([0, 2], 0), ([1], 300), ([0, 2, 1], 500)])
def test_noalloc_small_totals_match_oracle(L, n_kept, extra):
    # Few units against a buffer sized for many: the grid has more CTAs than
    # there are units, and the pairs are split over several of them.
    q, kb, vb, cu = _inputs(n_kept, seed=79 + extra, extra=extra)
    B = q.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full((B, 64, 128), float("nan"), device=DEV)
        st = L.lsa_sparse_decode_attn_noalloc(_p(q), _p(kb), _p(vb), kb.shape[1], _p(cu), B,
                                              1.0 / np.sqrt(128.0), _p(out), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        total = int(sum(n_kept))
        k_cm = kb.permute(1, 0, 2, 3)[:total].double().cpu().numpy()     # chunk-major for the oracle
        v_cm = vb.permute(1, 0, 2, 3)[:total].double().cpu().numpy()
        ref = oracle.sparse_decode_attn(q.double().cpu().numpy(), k_cm, v_cm, cu.cpu().numpy())
        o = out.double().cpu().numpy()
        assert np.all(np.abs(o - ref) <= ATT_ATOL + ATT_RTOL * np.abs(ref)), f"call {call}"
    bits = ctypes.c_uint(0)
    assert L.lsa_read_device_status(stream, ctypes.byref(bits)) == 0
    assert bits.value == 0


def test_noalloc_refuses_batch_beyond_its_scratch(L):
    n_kept = [1] * (NOALLOC_MAX_BATCH + 1)
    q, kb, vb, cu = _inputs(n_kept, seed=78)
    out = torch.empty((len(n_kept), 64, 128), device=DEV)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.lsa_sparse_decode_attn_noalloc(_p(q), _p(kb), _p(vb), kb.shape[1], _p(cu), len(n_kept),
                                          1.0 / np.sqrt(128.0), _p(out), stream)
    assert st == UNSUPPORTED
