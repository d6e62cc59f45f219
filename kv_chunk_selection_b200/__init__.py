"""Python binding of liblsa, the B200 decode hot path of Lookahead Sparse Attention.

Argument marshalling only: every function below checks dtypes, devices and
contiguity of torch tensors, passes raw pointers and sizes to the C ABI of the
same name (``include/lsa.h``) on the current torch CUDA stream, and raises
:class:`LsaError` on a non-zero status.  All computation happens in the CUDA
kernels of ``liblsa.so``; there is no fallback.  If the library has not been
built, importing works but the first call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "liblsa.so")

NUM_Q_HEADS = 64
NUM_KV_HEADS = 8
HEAD_DIM = 128
CHUNK_TOKENS = 64
INDEX_HEADS = 16
INDEX_DIM = 128
CHUNK_BYTES = NUM_KV_HEADS * CHUNK_TOKENS * HEAD_DIM * 2

DEV_ERR_BITS = {1: "BAD_COUNT", 2: "BAD_SLOT", 4: "BAD_CHUNK", 8: "CAPACITY", 16: "TIMEOUT", 32: "WORKSPACE",
                64: "INTERNAL"}

_lib = None


class LsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        name = _load().lsa_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{fn} failed: {name} ({status})")


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"liblsa.so not found at {LIB_PATH}; build it with `python -m kv_chunk_selection_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "lsa_status_string": ([I], ctypes.c_char_p),
        "lsa_version": ([], I),
        "lsa_read_device_status": ([P, ctypes.POINTER(ctypes.c_uint)], I),
        "lsa_selftest_bounded_wait": ([I, P, ctypes.c_uint, P], I),
        "lsa_index_score": ([P, P, P, I64, P, P, I, I, P, P], I),
        "lsa_topk_chunks": ([P, P, P, I, I, I, P, P, P, P], I),
        "lsa_topk_chunks_local": ([P, P, P, I, I, I, I, P, P, P, P], I),
        "lsa_append_token": ([P, P, P, P, P, I, P], I),
        "lsa_reset_local": ([P, I, P], I),
        "lsa_sparse_decode_attn_append": ([P, P, P, I64, P, I, F, P, P, P, P, P, P, P, P, S, ctypes.c_uint, P], I),
        "lsa_sparse_decode_attn_selected": ([P, P, P, I64, P, P, P, I, I, F, P, P, S, ctypes.c_uint, P], I),
        "lsa_token_score": ([P, P, P, I64, P, P, P, I, I, I, P, P, P], I),
        "lsa_topk_tokens": ([P, P, I, I, I, I, P, P, P, P], I),
        "lsa_select_tokens_workspace_size": ([I], S),
        "lsa_select_tokens": ([P, P, P, I64, P, P, P, I, I, I, I, P, P, P, P, P, I, P, S, ctypes.c_uint, P], I),
        "lsa_gather_tokens": ([P, P, I64, P, P, P, I, I, P, P, I64, P, P], I),
        "lsa_sparse_decode_attn_local": ([P, P, P, I64, P, I, F, P, P, P, P, P, S, ctypes.c_uint, P], I),
        "lsa_threshold_chunks": ([P, P, P, F, I, I, I, P, P, P, P], I),
        "lsa_threshold_chunks_capped": ([P, P, P, F, P, I, I, I, P, P, P, P], I),
        "lsa_gather_chunks": ([P, P, I64, P, P, P, I, I, I, P, P, I64, P], I),
        "lsa_fetch_from_host": ([P, P, I64, P, P, P, I, I, I, P, P, I64, I, P, P], I),
        "lsa_fetch_from_host_delta": ([P, P, I64, P, P, P, I, I, I, P, P, I64, P, P, I, P, P, I64, P, I, P, P], I),
        "lsa_fetch_from_host_copy": ([P, P, I64, P, P, P, I, I, I, P, P, I64, P, P], I),
        "lsa_debug_fail_fetch": ([I, I], I),
        "lsa_attn_workspace_size": ([I], S),
        "lsa_sparse_decode_attn": ([P, P, P, I64, P, I, F, P, P, S, ctypes.c_uint, P], I),
        "lsa_sparse_decode_attn_noalloc": ([P, P, P, I64, P, I, F, P, P], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def lib():
    """The loaded ctypes library (raw C ABI)."""
    return _load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _need(t: torch.Tensor, name: str, dtype, cuda=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _buf_chunks(t: torch.Tensor, name: str) -> int:
    """Chunks of a compact buffer, laid out head-major as [8 KV heads, chunks, 64, 128]."""
    if t.dim() != 4 or t.shape[0] != NUM_KV_HEADS or tuple(t.shape[2:]) != (CHUNK_TOKENS, HEAD_DIM):
        raise ValueError(f"{name} must be a compact buffer [8, chunks, 64, 128], got {tuple(t.shape)}")
    return int(t.shape[1])


def _check(fn: str, st: int):
    if st != 0:
        raise LsaError(fn, st)


def read_device_status(stream=None) -> int:
    """Synchronises the stream, returns and clears the device status bits."""
    bits = ctypes.c_uint(0)
    _check("lsa_read_device_status", _load().lsa_read_device_status(_stream(stream), ctypes.byref(bits)))
    return bits.value


def lsa_selftest_bounded_wait(mode: int, flag: Optional[torch.Tensor], limit_us: int, stream=None):
    """Runs the bounded-wait self-test (mode 0: mbarrier nothing completes; mode 1: device flag)."""
    if flag is not None:
        _need(flag, "flag", torch.int32)
    _check("lsa_selftest_bounded_wait",
           _load().lsa_selftest_bounded_wait(int(mode), _ptr(flag), int(limit_us), _stream(stream)))


def decode_status(bits: int) -> list:
    return [n for b, n in DEV_ERR_BITS.items() if bits & b]


def lsa_index_score(q_idx, w, chunk_keys, chunk_table, n_chunks, scores, stream=None):
    """scores[b, c] = sum_h w[h] sigmoid(q_idx[b,h].k[slot(b,c)] / sqrt(128)) for c < n_chunks[b]."""
    _need(q_idx, "q_idx", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(chunk_keys, "chunk_keys", torch.bfloat16)
    _need(n_chunks, "n_chunks", torch.int32)
    _need(scores, "scores", torch.float32)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    B = q_idx.shape[0]
    if tuple(q_idx.shape) != (B, INDEX_HEADS, INDEX_DIM) or scores.dim() != 2 or scores.shape[0] != B:
        raise ValueError("bad shapes")
    max_chunks = scores.shape[1]
    if chunk_table is not None and tuple(chunk_table.shape) != (B, max_chunks):
        raise ValueError("chunk_table must be [B, max_chunks]")
    n_slots = chunk_keys.shape[0]
    _check("lsa_index_score", _load().lsa_index_score(
        _ptr(q_idx), _ptr(w), _ptr(chunk_keys), n_slots, _ptr(chunk_table), _ptr(n_chunks), B, max_chunks,
        _ptr(scores), _stream(stream)))


def lsa_topk_chunks(scores, n_chunks, k_per_seq, kept, n_kept, cu_kept, stream=None, n_local=1):
    """Top-K chunks per sequence (score desc, index asc) plus the latest ``n_local``, ascending."""
    for t, n in ((scores, "scores"),):
        _need(t, n, torch.float32)
    for t, n in ((n_chunks, "n_chunks"), (k_per_seq, "k_per_seq"), (kept, "kept"), (n_kept, "n_kept"),
                 (cu_kept, "cu_kept")):
        _need(t, n, torch.int32)
    B, max_chunks = scores.shape
    max_kept = kept.shape[1]
    if kept.shape[0] != B or cu_kept.numel() != B + 1 or n_kept.numel() != B:
        raise ValueError("bad shapes")
    _check("lsa_topk_chunks_local", _load().lsa_topk_chunks_local(
        _ptr(scores), _ptr(n_chunks), _ptr(k_per_seq), int(n_local), B, max_chunks, max_kept, _ptr(kept),
        _ptr(n_kept), _ptr(cu_kept), _stream(stream)))


def lsa_threshold_chunks(scores, n_chunks, w, kept, n_kept, cu_kept, threshold=0.5, stream=None, cap=None):
    """Sigmoid-threshold selection: chunks with score / sum(w) > threshold, plus the latest, ascending.

    ``cap`` (int32 [B], optional) is a per-sequence budget: when more chunks
    pass, the ``cap[b]`` best passing chunks are kept (lsa_threshold_chunks_capped)."""
    _need(scores, "scores", torch.float32)
    _need(w, "w", torch.float32)
    for t, n in ((n_chunks, "n_chunks"), (kept, "kept"), (n_kept, "n_kept"), (cu_kept, "cu_kept")):
        _need(t, n, torch.int32)
    B, max_chunks = scores.shape
    max_kept = kept.shape[1]
    if kept.shape[0] != B or cu_kept.numel() != B + 1 or n_kept.numel() != B:
        raise ValueError("bad shapes")
    if cap is not None:
        _need(cap, "cap", torch.int32)
        if cap.numel() != B:
            raise ValueError("cap must have one entry per sequence")
    _check("lsa_threshold_chunks_capped", _load().lsa_threshold_chunks_capped(
        _ptr(scores), _ptr(n_chunks), _ptr(w), float(threshold), _ptr(cap), B, max_chunks, max_kept, _ptr(kept),
        _ptr(n_kept), _ptr(cu_kept), _stream(stream)))


def lsa_gather_chunks(k_pool, v_pool, chunk_table, kept, cu_kept, max_chunks, k_buf, v_buf, stream=None):
    """Copy the kept chunks of the device pools into the compact buffers."""
    for t, n in ((k_pool, "k_pool"), (v_pool, "v_pool"), (k_buf, "k_buf"), (v_buf, "v_buf")):
        _need(t, n, torch.bfloat16)
    for t, n in ((kept, "kept"), (cu_kept, "cu_kept")):
        _need(t, n, torch.int32)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    B, max_kept = kept.shape
    _check("lsa_gather_chunks", _load().lsa_gather_chunks(
        _ptr(k_pool), _ptr(v_pool), k_pool.shape[0], _ptr(chunk_table), _ptr(kept), _ptr(cu_kept), B,
        int(max_chunks), max_kept, _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _stream(stream)))


def lsa_fetch_from_host(host_k_pool, host_v_pool, chunk_table, kept, cu_kept, max_chunks, k_buf, v_buf,
                        num_ctas=0, stream=None, done_event: Optional[torch.cuda.Event] = None):
    """Same copy as lsa_gather_chunks from page-locked host pools (SM zero-copy reads)."""
    for t, n in ((host_k_pool, "host_k_pool"), (host_v_pool, "host_v_pool")):
        _need(t, n, torch.bfloat16, cuda=False)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf")):
        _need(t, n, torch.bfloat16)
    for t, n in ((kept, "kept"), (cu_kept, "cu_kept")):
        _need(t, n, torch.int32)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    B, max_kept = kept.shape
    ev = None
    if done_event is not None:
        if not done_event.cuda_event:
            # torch creates the CUDA event lazily on its first record
            done_event.record(stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream())
        ev = ctypes.c_void_p(done_event.cuda_event)
    _check("lsa_fetch_from_host", _load().lsa_fetch_from_host(
        _ptr(host_k_pool), _ptr(host_v_pool), host_k_pool.shape[0], _ptr(chunk_table), _ptr(kept),
        _ptr(cu_kept), B, int(max_chunks), max_kept, _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), int(num_ctas),
        _stream(stream), ev))


def lsa_fetch_from_host_delta(host_k_pool, host_v_pool, chunk_table, kept, cu_kept, max_chunks, k_buf, v_buf,
                              prev_kept, prev_cu_kept, prev_k_buf, prev_v_buf, reused_chunks=None, num_ctas=0,
                              stream=None, done_event: Optional[torch.cuda.Event] = None):
    """lsa_fetch_from_host, copying chunks the previous window also kept from its device buffers."""
    for t, n in ((host_k_pool, "host_k_pool"), (host_v_pool, "host_v_pool")):
        _need(t, n, torch.bfloat16, cuda=False)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf"), (prev_k_buf, "prev_k_buf"), (prev_v_buf, "prev_v_buf")):
        _need(t, n, torch.bfloat16)
    for t, n in ((kept, "kept"), (cu_kept, "cu_kept"), (prev_kept, "prev_kept"), (prev_cu_kept, "prev_cu_kept")):
        _need(t, n, torch.int32)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    if reused_chunks is not None:
        _need(reused_chunks, "reused_chunks", torch.int32)
    B, max_kept = kept.shape
    ev = None
    if done_event is not None:
        if not done_event.cuda_event:
            done_event.record(stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream())
        ev = ctypes.c_void_p(done_event.cuda_event)
    _check("lsa_fetch_from_host_delta", _load().lsa_fetch_from_host_delta(
        _ptr(host_k_pool), _ptr(host_v_pool), host_k_pool.shape[0], _ptr(chunk_table), _ptr(kept), _ptr(cu_kept),
        B, int(max_chunks), max_kept, _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(prev_kept),
        _ptr(prev_cu_kept), prev_kept.shape[1], _ptr(prev_k_buf), _ptr(prev_v_buf), _buf_chunks(prev_k_buf, "prev_k_buf"),
        _ptr(reused_chunks), int(num_ctas), _stream(stream), ev))


def lsa_fetch_from_host_copy(host_k_pool, host_v_pool, chunk_table_host, kept_host, cu_kept_host, max_chunks, k_buf,
                             v_buf, stream=None, done_event: Optional[torch.cuda.Event] = None):
    """lsa_fetch_from_host through the copy engines: the selection (kept_host
    [B, max_kept], cu_kept_host [B+1], chunk_table_host [B, max_chunks] or None)
    is read on the host, and each kept chunk is one 2-D copy per K and V."""
    for t, n in ((host_k_pool, "host_k_pool"), (host_v_pool, "host_v_pool")):
        _need(t, n, torch.bfloat16, cuda=False)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf")):
        _need(t, n, torch.bfloat16)
    for t, n in ((kept_host, "kept_host"), (cu_kept_host, "cu_kept_host")):
        _need(t, n, torch.int32, cuda=False)
    if chunk_table_host is not None:
        _need(chunk_table_host, "chunk_table_host", torch.int32, cuda=False)
    B, max_kept = kept_host.shape
    if cu_kept_host.numel() != B + 1:
        raise ValueError("cu_kept_host must have B + 1 entries")
    ev = None
    if done_event is not None:
        if not done_event.cuda_event:
            done_event.record(stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.current_stream())
        ev = ctypes.c_void_p(done_event.cuda_event)
    _check("lsa_fetch_from_host_copy", _load().lsa_fetch_from_host_copy(
        _ptr(host_k_pool), _ptr(host_v_pool), host_k_pool.shape[0], _ptr(chunk_table_host), _ptr(kept_host),
        _ptr(cu_kept_host), B, int(max_chunks), max_kept, _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"),
        _stream(stream), ev))


def lsa_debug_fail_fetch(calls: int, status: int = -4):
    """Host-side fault injection: the next ``calls`` host-tier fetch calls fail with ``status``."""
    _check("lsa_debug_fail_fetch", _load().lsa_debug_fail_fetch(int(calls), int(status)))


def lsa_attn_workspace_size(B: int) -> int:
    return int(_load().lsa_attn_workspace_size(int(B)))


def new_attn_workspace(B: int, device=None) -> torch.Tensor:
    """A workspace for lsa_sparse_decode_attn (it needs no initialisation)."""
    n = lsa_attn_workspace_size(B)
    if n == 0:
        raise ValueError("unsupported batch")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


ATTN_KV_UNCHANGED = 1


def lsa_sparse_decode_attn(q, k_buf, v_buf, cu_kept, out, workspace, softmax_scale=None, stream=None,
                           kv_unchanged=False):
    """out[b,h] = softmax(scale q[b,h] K^T) V over the kept tokens of KV head h // 8.

    ``kv_unchanged=True`` tells the library that the kernel just before this
    call on the stream did not write k_buf, v_buf or cu_kept (every decode step
    of a window after the first), so K/V streaming may overlap its tail."""
    _need(q, "q", torch.bfloat16)
    _need(k_buf, "k_buf", torch.bfloat16)
    _need(v_buf, "v_buf", torch.bfloat16)
    _need(cu_kept, "cu_kept", torch.int32)
    _need(out, "out", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    B = q.shape[0]
    if tuple(q.shape) != (B, NUM_Q_HEADS, HEAD_DIM) or tuple(out.shape) != (B, NUM_Q_HEADS, HEAD_DIM):
        raise ValueError("q and out must be [B, 64, 128]")
    if k_buf.shape != v_buf.shape or cu_kept.numel() != B + 1:
        raise ValueError("bad shapes")
    scale = 1.0 / math.sqrt(HEAD_DIM) if softmax_scale is None else float(softmax_scale)
    _check("lsa_sparse_decode_attn", _load().lsa_sparse_decode_attn(
        _ptr(q), _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), B, scale, _ptr(out),
        _ptr(workspace), workspace.numel(), ATTN_KV_UNCHANGED if kv_unchanged else 0, _stream(stream)))


def lsa_append_token(k_new, v_new, k_local, v_local, local_len, stream=None):
    """Appends each sequence's new token ([B, 8, 128]) at local_len[b] of its local chunk; increments it."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_local, "k_local"), (v_local, "v_local")):
        _need(t, n, torch.bfloat16)
    _need(local_len, "local_len", torch.int32)
    B = k_new.shape[0]
    if tuple(k_new.shape) != (B, NUM_KV_HEADS, HEAD_DIM) or tuple(k_local.shape) != (B, NUM_KV_HEADS,
                                                                                     CHUNK_TOKENS, HEAD_DIM):
        raise ValueError("k_new must be [B, 8, 128] and k_local [B, 8, 64, 128]")
    _check("lsa_append_token", _load().lsa_append_token(
        _ptr(k_new), _ptr(v_new), _ptr(k_local), _ptr(v_local), _ptr(local_len), B, _stream(stream)))


def lsa_reset_local(local_len, stream=None):
    """Sets local_len [B] to 0 (empties every local chunk), stream-ordered."""
    _need(local_len, "local_len", torch.int32)
    _check("lsa_reset_local", _load().lsa_reset_local(_ptr(local_len), local_len.shape[0], _stream(stream)))


def lsa_sparse_decode_attn_local(q, k_buf, v_buf, cu_kept, k_local, v_local, local_len, out, workspace,
                                 softmax_scale=None, stream=None, kv_unchanged=False):
    """Attention over the kept chunks plus the first local_len[b] tokens of each local chunk."""
    _need(q, "q", torch.bfloat16)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf"), (k_local, "k_local"), (v_local, "v_local")):
        _need(t, n, torch.bfloat16)
    _need(cu_kept, "cu_kept", torch.int32)
    _need(local_len, "local_len", torch.int32)
    _need(out, "out", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    B = q.shape[0]
    if tuple(q.shape) != (B, NUM_Q_HEADS, HEAD_DIM) or tuple(out.shape) != (B, NUM_Q_HEADS, HEAD_DIM):
        raise ValueError("q and out must be [B, 64, 128]")
    if tuple(k_local.shape) != (B, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM) or k_local.shape != v_local.shape:
        raise ValueError("k_local and v_local must be [B, 8, 64, 128]")
    scale = 1.0 / math.sqrt(HEAD_DIM) if softmax_scale is None else float(softmax_scale)
    _check("lsa_sparse_decode_attn_local", _load().lsa_sparse_decode_attn_local(
        _ptr(q), _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), B, scale, _ptr(k_local),
        _ptr(v_local), _ptr(local_len), _ptr(out), _ptr(workspace), workspace.numel(),
        ATTN_KV_UNCHANGED if kv_unchanged else 0, _stream(stream)))


def lsa_token_score(q_idx, w, token_keys, chunk_table, kept, n_kept, max_chunks, scores, n_tokens, stream=None):
    """Token-level scores inside the recalled chunks: scores[b, p] for p < 64 n_kept[b]
    (token p % 64 of recalled chunk kept[b, p // 64]); n_tokens[b] = 64 n_kept[b]."""
    _need(q_idx, "q_idx", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(token_keys, "token_keys", torch.bfloat16)
    for t, n in ((kept, "kept"), (n_kept, "n_kept"), (n_tokens, "n_tokens")):
        _need(t, n, torch.int32)
    _need(scores, "scores", torch.float32)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    B, max_kept = kept.shape
    if tuple(q_idx.shape) != (B, INDEX_HEADS, INDEX_DIM) or tuple(scores.shape) != (B, CHUNK_TOKENS * max_kept):
        raise ValueError("q_idx must be [B, 16, 128] and scores [B, 64 * max_kept]")
    if token_keys.dim() != 3 or tuple(token_keys.shape[1:]) != (CHUNK_TOKENS, INDEX_DIM):
        raise ValueError("token_keys must be [n_slots, 64, 128]")
    _check("lsa_token_score", _load().lsa_token_score(
        _ptr(q_idx), _ptr(w), _ptr(token_keys), token_keys.shape[0], _ptr(chunk_table), _ptr(kept), _ptr(n_kept),
        B, int(max_chunks), max_kept, _ptr(scores), _ptr(n_tokens), _stream(stream)))


def lsa_topk_tokens(scores, n_tokens, k, sel, n_sel, cu_sel, stream=None):
    """The k best token positions per sequence (score desc, position asc), ascending."""
    _need(scores, "scores", torch.float32)
    for t, n in ((n_tokens, "n_tokens"), (sel, "sel"), (n_sel, "n_sel"), (cu_sel, "cu_sel")):
        _need(t, n, torch.int32)
    B, max_tokens = scores.shape
    _check("lsa_topk_tokens", _load().lsa_topk_tokens(
        _ptr(scores), _ptr(n_tokens), int(k), B, max_tokens, sel.shape[1], _ptr(sel), _ptr(n_sel), _ptr(cu_sel),
        _stream(stream)))


def new_select_tokens_workspace(B: int, device=None) -> torch.Tensor:
    """The bin-count workspace of lsa_select_tokens, zeroed (every call leaves it zero)."""
    n = int(_load().lsa_select_tokens_workspace_size(int(B)))
    if n == 0:
        raise ValueError("unsupported batch")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


TOKENS_UNCHANGED = 1


def lsa_select_tokens(q_idx, w, token_keys, chunk_table, kept, n_kept, max_chunks, k, scores, n_tokens, sel, n_sel,
                      cu_sel, workspace, stream=None, keys_unchanged=False):
    """lsa_token_score then lsa_topk_tokens in one call (same outputs), the
    selection driven by the scorer's score-bin counts.

    ``keys_unchanged=True`` tells the library that nothing on the stream has
    written token_keys, chunk_table, kept, n_kept or w since the previous call
    of this function on it (every decode step of a window after the first), so
    the scorer may load its key rows, and the selection work out its counts,
    while the preceding kernel finishes."""
    _need(q_idx, "q_idx", torch.bfloat16)
    _need(w, "w", torch.float32)
    _need(token_keys, "token_keys", torch.bfloat16)
    for t, n in ((kept, "kept"), (n_kept, "n_kept"), (n_tokens, "n_tokens"), (sel, "sel"), (n_sel, "n_sel"),
                 (cu_sel, "cu_sel")):
        _need(t, n, torch.int32)
    _need(scores, "scores", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    if chunk_table is not None:
        _need(chunk_table, "chunk_table", torch.int32)
    B, max_kept = kept.shape
    if tuple(q_idx.shape) != (B, INDEX_HEADS, INDEX_DIM) or tuple(scores.shape) != (B, CHUNK_TOKENS * max_kept):
        raise ValueError("q_idx must be [B, 16, 128] and scores [B, 64 * max_kept]")
    if token_keys.dim() != 3 or tuple(token_keys.shape[1:]) != (CHUNK_TOKENS, INDEX_DIM):
        raise ValueError("token_keys must be [n_slots, 64, 128]")
    if sel.dim() != 2 or sel.shape[0] != B or cu_sel.numel() != B + 1 or n_sel.numel() != B:
        raise ValueError("sel must be [B, max_sel], n_sel [B] and cu_sel [B + 1]")
    _check("lsa_select_tokens", _load().lsa_select_tokens(
        _ptr(q_idx), _ptr(w), _ptr(token_keys), token_keys.shape[0], _ptr(chunk_table), _ptr(kept), _ptr(n_kept), B,
        int(max_chunks), max_kept, int(k), _ptr(scores), _ptr(n_tokens), _ptr(sel), _ptr(n_sel), _ptr(cu_sel),
        sel.shape[1], _ptr(workspace), workspace.numel(), TOKENS_UNCHANGED if keys_unchanged else 0,
        _stream(stream)))


def lsa_gather_tokens(k_buf, v_buf, cu_kept, sel, cu_sel, k_out, v_out, cu_units, stream=None):
    """Packs the selected tokens into dense 64-token units (the attention's compact layout)."""
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf"), (k_out, "k_out"), (v_out, "v_out")):
        _need(t, n, torch.bfloat16)
    for t, n in ((cu_kept, "cu_kept"), (sel, "sel"), (cu_sel, "cu_sel"), (cu_units, "cu_units")):
        _need(t, n, torch.int32)
    B, max_sel = sel.shape
    _check("lsa_gather_tokens", _load().lsa_gather_tokens(
        _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), _ptr(sel), _ptr(cu_sel), B, max_sel,
        _ptr(k_out), _ptr(v_out), _buf_chunks(k_out, "k_out"), _ptr(cu_units), _stream(stream)))


def lsa_sparse_decode_attn_selected(q, k_buf, v_buf, cu_kept, sel, cu_sel, out, workspace, softmax_scale=None,
                                    stream=None, kv_unchanged=False):
    """Attention over the selected tokens (sel [B, max_sel] from lsa_topk_tokens), read
    in place from the compact buffer: lsa_gather_tokens + lsa_sparse_decode_attn in one."""
    _need(q, "q", torch.bfloat16)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf")):
        _need(t, n, torch.bfloat16)
    for t, n in ((cu_kept, "cu_kept"), (sel, "sel"), (cu_sel, "cu_sel")):
        _need(t, n, torch.int32)
    _need(out, "out", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    B = q.shape[0]
    if tuple(q.shape) != (B, NUM_Q_HEADS, HEAD_DIM) or tuple(out.shape) != (B, NUM_Q_HEADS, HEAD_DIM):
        raise ValueError("q and out must be [B, 64, 128]")
    if sel.dim() != 2 or sel.shape[0] != B:
        raise ValueError("sel must be [B, max_sel]")
    scale = 1.0 / math.sqrt(HEAD_DIM) if softmax_scale is None else float(softmax_scale)
    _check("lsa_sparse_decode_attn_selected", _load().lsa_sparse_decode_attn_selected(
        _ptr(q), _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), _ptr(sel), _ptr(cu_sel), sel.shape[1], B,
        scale, _ptr(out), _ptr(workspace), workspace.numel(), ATTN_KV_UNCHANGED if kv_unchanged else 0,
        _stream(stream)))


def lsa_sparse_decode_attn_append(q, k_buf, v_buf, cu_kept, k_new, v_new, k_local, v_local, local_len_in,
                                  local_len_out, out, workspace, softmax_scale=None, stream=None,
                                  kv_unchanged=False):
    """One causal step in one launch: appends (k_new, v_new) [B, 8, 128] at row
    local_len_in[b] of the local chunk, attends the kept chunks plus the local
    tokens including it, and writes local_len_out[b] = local_len_in[b] + 1."""
    _need(q, "q", torch.bfloat16)
    for t, n in ((k_buf, "k_buf"), (v_buf, "v_buf"), (k_new, "k_new"), (v_new, "v_new"), (k_local, "k_local"),
                 (v_local, "v_local")):
        _need(t, n, torch.bfloat16)
    for t, n in ((cu_kept, "cu_kept"), (local_len_in, "local_len_in"), (local_len_out, "local_len_out")):
        _need(t, n, torch.int32)
    _need(out, "out", torch.float32)
    _need(workspace, "workspace", torch.uint8)
    B = q.shape[0]
    if tuple(q.shape) != (B, NUM_Q_HEADS, HEAD_DIM) or tuple(out.shape) != (B, NUM_Q_HEADS, HEAD_DIM):
        raise ValueError("q and out must be [B, 64, 128]")
    if tuple(k_local.shape) != (B, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM) or k_local.shape != v_local.shape:
        raise ValueError("k_local and v_local must be [B, 8, 64, 128]")
    if tuple(k_new.shape) != (B, NUM_KV_HEADS, HEAD_DIM) or k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new must be [B, 8, 128]")
    scale = 1.0 / math.sqrt(HEAD_DIM) if softmax_scale is None else float(softmax_scale)
    _check("lsa_sparse_decode_attn_append", _load().lsa_sparse_decode_attn_append(
        _ptr(q), _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), B, scale, _ptr(k_new), _ptr(v_new),
        _ptr(k_local), _ptr(v_local), _ptr(local_len_in), _ptr(local_len_out), _ptr(out), _ptr(workspace),
        workspace.numel(), ATTN_KV_UNCHANGED if kv_unchanged else 0, _stream(stream)))


def lsa_sparse_decode_attn_noalloc(q, k_buf, v_buf, cu_kept, out, softmax_scale=None, stream=None):
    """lsa_sparse_decode_attn without a workspace argument, for callers that cannot
    allocate device memory; its scratch is a fixed array inside the library, shared
    by every call on the device (calls that may overlap on the GPU must be
    serialised by the caller).  At most 32 sequences."""
    _need(q, "q", torch.bfloat16)
    _need(k_buf, "k_buf", torch.bfloat16)
    _need(v_buf, "v_buf", torch.bfloat16)
    _need(cu_kept, "cu_kept", torch.int32)
    _need(out, "out", torch.float32)
    B = q.shape[0]
    if tuple(q.shape) != (B, NUM_Q_HEADS, HEAD_DIM) or tuple(out.shape) != (B, NUM_Q_HEADS, HEAD_DIM):
        raise ValueError("q and out must be [B, 64, 128]")
    if k_buf.shape != v_buf.shape or cu_kept.numel() != B + 1:
        raise ValueError("bad shapes")
    scale = 1.0 / math.sqrt(HEAD_DIM) if softmax_scale is None else float(softmax_scale)
    _check("lsa_sparse_decode_attn_noalloc", _load().lsa_sparse_decode_attn_noalloc(
        _ptr(q), _ptr(k_buf), _ptr(v_buf), _buf_chunks(k_buf, "k_buf"), _ptr(cu_kept), B, scale, _ptr(out), _stream(stream)))


__all__ = [
    "LsaError", "lib", "read_device_status", "decode_status", "lsa_index_score", "lsa_topk_chunks",
    "lsa_threshold_chunks",
    "lsa_gather_chunks", "lsa_fetch_from_host", "lsa_fetch_from_host_delta", "lsa_fetch_from_host_copy",
    "lsa_debug_fail_fetch", "lsa_attn_workspace_size", "new_attn_workspace", "lsa_threshold_chunks",
    "lsa_sparse_decode_attn", "lsa_sparse_decode_attn_noalloc", "lsa_append_token", "lsa_reset_local",
    "lsa_token_score", "lsa_topk_tokens", "lsa_select_tokens", "new_select_tokens_workspace", "lsa_gather_tokens", "lsa_sparse_decode_attn_append",
    "lsa_sparse_decode_attn_selected",
    "lsa_sparse_decode_attn_local", "NUM_Q_HEADS", "NUM_KV_HEADS", "HEAD_DIM", "CHUNK_TOKENS", "INDEX_HEADS",
    "INDEX_DIM", "CHUNK_BYTES",
]
