"""The C-ABI library loads on a machine without a GPU, exports every function
its header declares, and rejects bad arguments on the host before launching.

Only argument errors that the host checks catch before any launch are used
here (null pointers, bad sizes, misaligned addresses), so these tests are safe
on any machine; the "no device" answers are only asserted without a GPU.
"""
import ctypes
import os
import re

import pytest
import torch

import kv_chunk_selection_b200 as lsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA, NOT_PINNED, MISALIGNED, NO_DEVICE = 0, -1, -2, -3, -4, -5, -6, -7
NO_GPU = not torch.cuda.is_available()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from kv_chunk_selection_b200 import build
    build.build()
    return lsa.lib()


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("lsa_index_score", "lsa_topk_chunks", "lsa_threshold_chunks", "lsa_gather_chunks",
                 "lsa_sparse_decode_attn",
                 "lsa_fetch_from_host", "lsa_attn_workspace_size", "lsa_read_device_status",
                 "lsa_status_string", "lsa_version"):
        assert name in fns


def test_library_exports_every_header_symbol(L):
    raw = ctypes.CDLL(lsa.LIB_PATH)
    missing = [f for f in header_functions() if not hasattr(raw, f)]
    assert missing == []


def test_status_strings_and_version(L):
    assert L.lsa_status_string(OK) == b"LSA_OK"
    assert L.lsa_status_string(NOT_PINNED) == b"LSA_ERR_NOT_PINNED"
    assert L.lsa_status_string(12345) == b"LSA_ERR_UNKNOWN"
    assert L.lsa_version() == 100


def test_workspace_size(L):
    assert L.lsa_attn_workspace_size(0) == 0
    assert L.lsa_attn_workspace_size(4097) == 0
    s1, s32 = L.lsa_attn_workspace_size(1), L.lsa_attn_workspace_size(32)
    assert 0 < s1 < s32
    # (8 + 1024) partial records of 1032 floats
    assert s1 == (8 + 1024) * 1032 * 4


def test_host_checks_null_pointers(L):
    n = None
    assert L.lsa_index_score(n, n, n, 1, n, n, 1, 1, n, n) == INVALID
    assert L.lsa_topk_chunks(n, n, n, 1, 1, 1, n, n, n, n) == INVALID
    assert L.lsa_threshold_chunks(n, n, n, ctypes.c_float(0.5), 1, 1, 1, n, n, n, n) == INVALID
    assert L.lsa_gather_chunks(n, n, 1, n, n, n, 1, 1, 1, n, n, 1, n) == INVALID
    assert L.lsa_fetch_from_host(n, n, 1, n, n, n, 1, 1, 1, n, n, 1, 0, n, n) == INVALID
    assert L.lsa_sparse_decode_attn(n, n, n, 1, n, 1, 0.1, n, n, 0, 0, n) == INVALID
    assert L.lsa_read_device_status(n, None) == INVALID
    assert L.lsa_topk_chunks_local(n, n, n, 1, 1, 1, 1, n, n, n, n) == INVALID
    assert L.lsa_append_token(n, n, n, n, n, 1, n) == INVALID
    assert L.lsa_reset_local(n, 1, n) == INVALID
    ok = ctypes.c_void_p(0x100000)
    assert L.lsa_sparse_decode_attn_append(ok, ok, ok, 4, ok, 1, ctypes.c_float(0.1), ok, ok, ok, ok, ok, ok, ok, ok,
                                           1 << 30, 0, n) == INVALID   # local_len_in == local_len_out
    assert L.lsa_sparse_decode_attn_append(ok, ok, ok, 4, ok, 1, ctypes.c_float(0.1), n, ok, ok, ok, ok,
                                           ctypes.c_void_p(0x200000), ok, ok, 1 << 30, 0, n) == INVALID
    assert L.lsa_token_score(n, n, n, 1, n, n, n, 1, 1, 1, n, n, n) == INVALID
    assert L.lsa_sparse_decode_attn_selected(n, n, n, 1, n, n, n, 64, 1, ctypes.c_float(0.1), n, n, 0, 0, n) == INVALID
    assert L.lsa_sparse_decode_attn_selected(ok, ok, ok, 4, ok, ok, ok, 100, 1, ctypes.c_float(0.1), ok, ok,
                                             1 << 30, 0, n) == INVALID   # max_sel % 64
    assert L.lsa_topk_tokens(n, n, 64, 1, 64, 64, n, n, n, n) == INVALID
    assert L.lsa_gather_tokens(n, n, 1, n, n, n, 1, 64, n, n, 1, n, n) == INVALID
    ok = ctypes.c_void_p(0x100000)
    assert L.lsa_topk_tokens(ok, ok, 0, 1, 64, 64, ok, ok, ok, n) == INVALID                # k = 0
    assert L.lsa_gather_tokens(ok, ok, 1, ok, ok, ok, 1, 100, ok, ok, 1, ok, n) == INVALID   # max_sel % 64
    assert L.lsa_gather_tokens(ok, ok, 1, ok, ok, ok, 1, 64, ctypes.c_void_p(0x100008), ok, 1, ok, n) == MISALIGNED
    assert L.lsa_token_score(ctypes.c_void_p(0x100002), ok, ok, 1, n, ok, ok, 1, 1, 1, ok, ok, n) == MISALIGNED
    assert L.lsa_reset_local(ctypes.c_void_p(0x100000), 0, n) == INVALID
    assert L.lsa_sparse_decode_attn_local(n, n, n, 1, n, 1, ctypes.c_float(0.1), n, n, n, n, n, 0, 0, n) == INVALID
    assert L.lsa_selftest_bounded_wait(1, n, 1000, n) == INVALID      # mode 1 needs a flag
    assert L.lsa_selftest_bounded_wait(0, n, 0, n) == INVALID         # zero limit
    assert L.lsa_selftest_bounded_wait(5, n, 1000, n) == INVALID      # unknown mode


def test_host_checks_of_the_later_entry_points(L):
    n, ok = None, ctypes.c_void_p(0x100000)
    f = ctypes.c_float(0.5)
    # capped threshold: null pointers; a NULL cap is allowed (it is the plain rule)
    assert L.lsa_threshold_chunks_capped(n, n, n, f, n, 1, 1, 1, n, n, n, n) == INVALID
    assert L.lsa_threshold_chunks_capped(ok, ok, ok, ctypes.c_float(float("nan")), n, 1, 4, 2, ok, ok, ok, n) == INVALID
    # fused token selection: missing outputs, k <= 0, no or a small workspace, a misaligned one
    ws = L.lsa_select_tokens_workspace_size(1)
    assert ws == 4 * 4096 * 4 and L.lsa_select_tokens_workspace_size(0) == 0
    sel_args = lambda k, w, wb, fl=0: (ok, ok, ok, 4, n, ok, ok, 1, 4, 2, k, ok, ok, ok, ok, ok, 128, w, wb, fl, n)
    assert L.lsa_select_tokens(*sel_args(0, ok, ws)) == INVALID
    assert L.lsa_select_tokens(*sel_args(64, n, ws)) == WORKSPACE
    assert L.lsa_select_tokens(*sel_args(64, ok, ws - 16)) == WORKSPACE
    assert L.lsa_select_tokens(*sel_args(64, ctypes.c_void_p(0x100008), ws)) == MISALIGNED
    assert L.lsa_select_tokens(*sel_args(64, ok, ws, 2)) == INVALID                       # unknown flag
    assert L.lsa_select_tokens(ok, ok, ok, 4, n, ok, ok, LSA_MAX_BATCH + 1, 4, 2, 64, ok, ok, ok, ok, ok, 128, ok,
                               1 << 40, 0, n) == UNSUPPORTED
    # copy-engine fetch: null pointers, misaligned pools
    assert L.lsa_fetch_from_host_copy(n, n, 1, n, n, n, 1, 1, 1, n, n, 1, n, n) == INVALID
    assert L.lsa_fetch_from_host_copy(ctypes.c_void_p(0x1001), ok, 4, n, ok, ok, 1, 4, 2, ok, ok, 2, n, n) == MISALIGNED


def test_host_checks_sizes_and_alignment(L):
    odd = ctypes.c_void_p(0x1001)         # misaligned, never dereferenced
    ok = ctypes.c_void_p(0x100000)        # aligned, never dereferenced (checks fail first)
    # non-positive sizes
    assert L.lsa_index_score(ok, ok, ok, 0, None, ok, 1, 4, ok, None) == INVALID
    assert L.lsa_index_score(ok, ok, ok, 4, None, ok, 0, 4, ok, None) == INVALID
    assert L.lsa_topk_chunks(ok, ok, ok, 1, 4, 0, ok, ok, ok, None) == INVALID
    assert L.lsa_topk_chunks(ok, ok, ok, LSA_MAX_BATCH + 1, 4, 2, ok, ok, ok, None) == UNSUPPORTED
    assert L.lsa_sparse_decode_attn(ok, ok, ok, 4, ok, 1, -1.0, ok, ok, 1 << 30, 0, None) == INVALID
    assert L.lsa_sparse_decode_attn(ok, ok, ok, 4, ok, 1, 0.1, ok, ok, 1 << 30, 2, None) == INVALID   # unknown flag
    assert L.lsa_sparse_decode_attn(ok, ok, ok, 4, ok, LSA_MAX_BATCH + 1, 0.1, ok, ok, 1 << 30, 0, None) == UNSUPPORTED
    assert L.lsa_sparse_decode_attn(ok, ok, ok, (1 << 22) + 1, ok, 1, 0.1, ok, ok, 1 << 30, 0, None) == UNSUPPORTED
    # misaligned bf16 arrays
    assert L.lsa_index_score(odd, ok, ok, 4, None, ok, 1, 4, ok, None) == MISALIGNED
    assert L.lsa_gather_chunks(ok, odd, 4, None, ok, ok, 1, 4, 2, ok, ok, 2, None) == MISALIGNED
    assert L.lsa_sparse_decode_attn(ok, ok, odd, 4, ok, 1, 0.1, ok, ok, 1 << 30, 0, None) == MISALIGNED
    assert L.lsa_fetch_from_host(odd, ok, 4, None, ok, ok, 1, 4, 2, ok, ok, 2, 0, None, None) == MISALIGNED
    # workspace too small
    assert L.lsa_sparse_decode_attn(ok, ok, ok, 4, ok, 1, 0.1, ok, ok, 16, 0, None) == WORKSPACE


LSA_MAX_BATCH = 4096


def test_fetch_fault_injection_returns_the_injected_status(L):
    """The host-side injection hook makes the host-tier fetch report a failed
    transfer without touching the device: argument errors still come first and
    do not use up an armed failure; after the armed calls the fetch goes on to
    its device checks (no device here, or an address that is not page-locked)."""
    ok = ctypes.c_void_p(0x100000)
    fetch = (ok, ok, 4, None, ok, ok, 1, 4, 2, ok, ok, 2, 0, None, None)
    prev = ctypes.c_void_p(0x200000)      # the previous window's buffers: not the target's
    delta = (ok, ok, 4, None, ok, ok, 1, 4, 2, ok, ok, 2, ok, ok, 2, prev, prev, 2, None, 0, None, None)
    kept = (ctypes.c_int32 * 2)(0, 1)
    cu = (ctypes.c_int32 * 2)(0, 2)
    copy = (ok, ok, 4, None, ctypes.cast(kept, ctypes.c_void_p), ctypes.cast(cu, ctypes.c_void_p), 1, 4, 2, ok, ok,
            2, None, None)
    try:
        assert L.lsa_debug_fail_fetch(3, CUDA) == OK
        assert L.lsa_fetch_from_host(*fetch) == CUDA
        assert L.lsa_fetch_from_host(None, *fetch[1:]) == INVALID          # argument check first, not counted
        assert L.lsa_fetch_from_host_delta(*delta) == CUDA
        assert L.lsa_fetch_from_host_copy(*copy) == CUDA
        assert L.lsa_fetch_from_host(*fetch) in (NO_DEVICE, NOT_PINNED)     # disarmed after three calls
        assert L.lsa_debug_fail_fetch(1, NOT_PINNED) == OK
        assert L.lsa_fetch_from_host(*fetch) == NOT_PINNED
        for calls, status in ((-1, CUDA), (1, OK), (1, 5), (1, NO_DEVICE - 1)):
            assert L.lsa_debug_fail_fetch(calls, status) == INVALID
    finally:
        L.lsa_debug_fail_fetch(0, CUDA)


def test_copy_engine_fetch_checks_the_selection_on_the_host(L):
    ok = ctypes.c_void_p(0x100000)

    def call(kept_vals, cu_vals, table=None, max_chunks=4, n_slots=4, buf=2):
        kept = (ctypes.c_int32 * len(kept_vals))(*kept_vals)
        cu = (ctypes.c_int32 * len(cu_vals))(*cu_vals)
        tb = None if table is None else ctypes.cast((ctypes.c_int32 * len(table))(*table), ctypes.c_void_p)
        return L.lsa_fetch_from_host_copy(ok, ok, n_slots, tb, ctypes.cast(kept, ctypes.c_void_p),
                                          ctypes.cast(cu, ctypes.c_void_p), 1, max_chunks, 2, ok, ok, buf, None, None)

    assert call([0, 4], [0, 2]) == INVALID                     # chunk index past max_chunks
    assert call([0, 1], [0, 3]) == INVALID                     # more chunks than the buffer holds
    assert call([0, 1], [1, 2]) == INVALID                     # cu_kept[0] != 0
    assert call([0, 3], [0, 2], table=[0, 1, 2, 9]) == INVALID  # slot past n_slots
    assert call([0, 1], [0, 2]) in (NO_DEVICE, NOT_PINNED)     # valid: on to the device checks


@pytest.mark.skipif(not NO_GPU, reason="asserts the answer on a machine without a GPU")
def test_no_device_answer(L):
    ok = ctypes.c_void_p(0x100000)
    ws = L.lsa_attn_workspace_size(1)
    assert L.lsa_sparse_decode_attn(ok, ok, ok, 4, ok, 1, 0.1, ok, ok, ws, 0, None) == NO_DEVICE
    assert L.lsa_gather_chunks(ok, ok, 4, None, ok, ok, 1, 4, 2, ok, ok, 2, None) == NO_DEVICE
    bits = ctypes.c_uint(0)
    assert L.lsa_read_device_status(None, ctypes.byref(bits)) == NO_DEVICE


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(lsa, "_lib", None)
    monkeypatch.setattr(lsa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="liblsa.so not found"):
        lsa.lib()
    importlib.reload(lsa)


def test_binding_takes_head_major_compact_buffers():
    """The binding reads the chunk count of a compact buffer from its head-major
    shape [8, chunks, 64, 128] and rejects any other shape, a chunk-major
    [chunks, 8, 64, 128] one included (it would pass a wrong size to the kernels)."""
    assert lsa._buf_chunks(torch.empty((8, 20, 64, 128), dtype=torch.bfloat16), "k_buf") == 20
    for bad in ((20, 8, 64, 128), (8, 20, 128, 64), (8, 20, 64), (4, 20, 64, 128)):
        with pytest.raises(ValueError, match="k_buf"):
            lsa._buf_chunks(torch.empty(bad, dtype=torch.bfloat16), "k_buf")
