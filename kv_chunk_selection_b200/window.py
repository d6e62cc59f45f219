"""The lookahead window schedule of one layer, on top of the C ABI.

Every tau = 64 decode steps the indexer scores all chunks, the selection keeps
the top-K plus the latest chunk, and the kept chunks are gathered into the
compact buffer (or fetched from a page-locked host pool); the next 64 decode
steps attend over that buffer only (summary page "FlashMemory-DeepSeek-V4 ...",
1 Introduction and 2.1 Architecture; handbook page "DeepSeek-V4: Architecting
for Ultra-Long Contexts", "The Neural Memory Indexer").

This module only owns buffers and issues the library calls in order; it does
no arithmetic of the method itself.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import (CHUNK_TOKENS, HEAD_DIM, NUM_KV_HEADS, NUM_Q_HEADS, lsa_append_token, lsa_attn_workspace_size,
               lsa_fetch_from_host, lsa_gather_chunks, lsa_gather_tokens, lsa_index_score, lsa_reset_local,
               lsa_sparse_decode_attn, lsa_sparse_decode_attn_append, lsa_sparse_decode_attn_local,
               lsa_sparse_decode_attn_selected, lsa_select_tokens, lsa_threshold_chunks, lsa_token_score,
               lsa_topk_chunks, lsa_topk_tokens, new_select_tokens_workspace)

TAU = 64


class LayerWindow:
    """Buffers and calls of one layer's decode window.

    Selection is the fixed top-K budget (``selection="topk"``) or the pages'
    sigmoid threshold (``selection="threshold"``, keep a chunk when its weighted
    mean probability exceeds ``threshold``).  Sizes: with top-K, ``max_kept`` =
    max_b K_b + n_local kept chunks per sequence row and the compact buffer
    holds ``sum_b (K_b + n_local)`` chunks (an upper bound of the kept total).
    The threshold keeps a data-dependent number of chunks; with
    ``threshold_cap`` (the default) it is held to the same budget, K_b best
    passing chunks at most, so the buffers have the top-K sizes; without it
    both are sized for every chunk.  With ``double_buffer`` two compact buffers
    alternate, so the selection of the next window can be fetched while the
    current one is read.

    ``n_local`` (top-K only) keeps the latest ``n_local`` chunks beside the K
    recalled ones.  With ``causal`` each sequence also has a local chunk of the
    tokens decoded inside the window, emptied by ``reset_local`` when a window
    starts.  ``attend_append`` runs one causal step in one launch (the step's
    token is appended and attended together); ``append`` followed by ``attend``
    does the same in two launches.  The token count lives in two arrays that
    alternate between fused steps (one is read while the other is written).

    ``fine_k`` (a multiple of 64) adds the token-level fine stage: every step
    ``fine_select`` scores each token of the recalled chunks with the step's
    indexer query and keeps the ``fine_k`` best, and ``attend`` runs over those
    tokens only, reading them in place from the compact buffer.  With
    ``causal`` too, the selected tokens are first packed into dense units (the
    fused append reads packed units).  ``fused_select`` (the default) scores and
    selects with lsa_select_tokens; without it, lsa_token_score and
    lsa_topk_tokens run one after the other (the same result).
    """

    def __init__(self, n_chunks: torch.Tensor, k_per_seq: torch.Tensor, chunk_table: Optional[torch.Tensor],
                 max_chunks: int, device="cuda", double_buffer: bool = False, selection: str = "topk",
                 threshold: float = 0.5, n_local: int = 1, causal: bool = False, fine_k: int = 0,
                 threshold_cap: bool = True, fused_select: bool = True):
        self.device = torch.device(device)
        self.n_chunks = n_chunks
        self.k_per_seq = k_per_seq
        self.chunk_table = chunk_table
        self.max_chunks = int(max_chunks)
        self.B = int(n_chunks.shape[0])
        if selection not in ("topk", "threshold"):
            raise ValueError("selection must be 'topk' or 'threshold'")
        self.selection = selection
        self.threshold = float(threshold)
        if n_local < 1 or (n_local != 1 and selection != "topk"):
            raise ValueError("n_local must be >= 1, and above 1 only with top-K selection")
        self.n_local = int(n_local)
        self.threshold_cap = bool(threshold_cap) and selection == "threshold"
        if selection == "topk" or self.threshold_cap:
            k_host = k_per_seq.to("cpu", torch.int64)
            self.max_kept = int(k_host.max()) + self.n_local
            self.buf_chunks = int((k_host + self.n_local).sum())
        else:
            n_host = n_chunks.to("cpu", torch.int64)
            self.max_kept = int(max_chunks)
            self.buf_chunks = int(n_host.sum())
        nbuf = 2 if double_buffer else 1
        shape = (NUM_KV_HEADS, self.buf_chunks, CHUNK_TOKENS, HEAD_DIM)   # head-major compact buffer
        self.k_bufs = [torch.empty(shape, dtype=torch.bfloat16, device=self.device) for _ in range(nbuf)]
        self.v_bufs = [torch.empty(shape, dtype=torch.bfloat16, device=self.device) for _ in range(nbuf)]
        self.scores = torch.empty((self.B, self.max_chunks), dtype=torch.float32, device=self.device)
        self.kept = [torch.zeros((self.B, self.max_kept), dtype=torch.int32, device=self.device) for _ in range(nbuf)]
        self.n_kept = [torch.zeros((self.B,), dtype=torch.int32, device=self.device) for _ in range(nbuf)]
        self.cu_kept = [torch.zeros((self.B + 1,), dtype=torch.int32, device=self.device) for _ in range(nbuf)]
        self.workspace = torch.zeros(lsa_attn_workspace_size(self.B), dtype=torch.uint8, device=self.device)
        self.active = 0
        self.causal = bool(causal)
        if self.causal:
            lshape = (self.B, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM)
            self.k_local = torch.zeros(lshape, dtype=torch.bfloat16, device=self.device)
            self.v_local = torch.zeros(lshape, dtype=torch.bfloat16, device=self.device)
            self._lens = [torch.zeros((self.B,), dtype=torch.int32, device=self.device) for _ in range(2)]
            self._phase = 0
        self.fine_k = int(fine_k)
        if self.fine_k:
            if self.fine_k < 0 or self.fine_k % CHUNK_TOKENS:
                raise ValueError("fine_k must be a positive multiple of 64")
            dev = self.device
            self.tok_scores = torch.empty((self.B, CHUNK_TOKENS * self.max_kept), dtype=torch.float32, device=dev)
            self.n_tokens = torch.zeros((self.B,), dtype=torch.int32, device=dev)
            self.sel = torch.zeros((self.B, self.fine_k), dtype=torch.int32, device=dev)
            self.n_sel = torch.zeros((self.B,), dtype=torch.int32, device=dev)
            self.cu_sel = torch.zeros((self.B + 1,), dtype=torch.int32, device=dev)
            self.fused_select = bool(fused_select)
            if self.fused_select:
                self.sel_workspace = new_select_tokens_workspace(self.B, dev)
            self.packs = self.causal   # the causal step reads packed units
            if self.packs:
                units = self.B * self.fine_k // CHUNK_TOKENS
                self.k_fine = torch.empty((NUM_KV_HEADS, units, CHUNK_TOKENS, HEAD_DIM), dtype=torch.bfloat16,
                                          device=dev)
                self.v_fine = torch.empty_like(self.k_fine)
                self.cu_units = torch.zeros((self.B + 1,), dtype=torch.int32, device=dev)

    def select(self, q_idx, w, chunk_keys, buf: int = 0, stream=None):
        """Indexer scores, then the selection (top-K or threshold) plus latest, into slot ``buf``."""
        lsa_index_score(q_idx, w, chunk_keys, self.chunk_table, self.n_chunks, self.scores, stream=stream)
        if self.selection == "topk":
            lsa_topk_chunks(self.scores, self.n_chunks, self.k_per_seq, self.kept[buf], self.n_kept[buf],
                            self.cu_kept[buf], stream=stream, n_local=self.n_local)
        else:
            lsa_threshold_chunks(self.scores, self.n_chunks, w, self.kept[buf], self.n_kept[buf], self.cu_kept[buf],
                                 threshold=self.threshold, stream=stream,
                                 cap=self.k_per_seq if self.threshold_cap else None)

    def gather(self, k_pool, v_pool, buf: int = 0, stream=None):
        lsa_gather_chunks(k_pool, v_pool, self.chunk_table, self.kept[buf], self.cu_kept[buf], self.max_chunks,
                          self.k_bufs[buf], self.v_bufs[buf], stream=stream)

    def fetch(self, host_k_pool, host_v_pool, buf: int = 0, num_ctas: int = 0, stream=None, done_event=None):
        lsa_fetch_from_host(host_k_pool, host_v_pool, self.chunk_table, self.kept[buf], self.cu_kept[buf],
                            self.max_chunks, self.k_bufs[buf], self.v_bufs[buf], num_ctas=num_ctas,
                            stream=stream, done_event=done_event)

    @property
    def local_len(self):
        """Tokens in each local chunk [B] int32 (the array the next step reads)."""
        return self._lens[self._phase]

    def reset_local(self, stream=None):
        """Empties every sequence's local chunk (start of a window; causal only)."""
        self._phase = 0
        lsa_reset_local(self._lens[0], stream=stream)

    def append(self, k_new, v_new, stream=None):
        """Adds this step's token (k_new, v_new [B, 8, 128] bf16) to the local chunks (causal only)."""
        lsa_append_token(k_new, v_new, self.k_local, self.v_local, self.local_len, stream=stream)

    def _attn_buffers(self, buf):
        if self.fine_k and self.packs:
            return self.k_fine, self.v_fine, self.cu_units
        return self.k_bufs[buf], self.v_bufs[buf], self.cu_kept[buf]

    def attend_append(self, q, out, k_new, v_new, buf: int = 0, stream=None, kv_unchanged: bool = False):
        """One causal step in one launch: the step's token (k_new, v_new [B, 8, 128])
        joins the local chunks and is attended with the kept (or fine-selected)
        tokens and the tokens decoded before it in this window."""
        kb, vb, cu = self._attn_buffers(buf)
        if self.fine_k:
            kv_unchanged = False
        lsa_sparse_decode_attn_append(q, kb, vb, cu, k_new, v_new, self.k_local, self.v_local,
                                      self._lens[self._phase], self._lens[1 - self._phase], out, self.workspace,
                                      stream=stream, kv_unchanged=kv_unchanged)
        self._phase = 1 - self._phase

    def fine_select(self, q_tok, w, token_keys, buf: int = 0, stream=None, keys_unchanged: bool = False):
        """Token-level stage of one step: scores of the recalled tokens from the step's
        indexer query q_tok [B, 16, 128] and the fine_k best (packed into dense
        units when the window is causal).  ``keys_unchanged``: nothing on the
        stream has written the token keys, the head weights or this window's kept
        lists since the previous step's call (true for every step but the first)."""
        if self.fused_select:
            lsa_select_tokens(q_tok, w, token_keys, self.chunk_table, self.kept[buf], self.n_kept[buf],
                              self.max_chunks, self.fine_k, self.tok_scores, self.n_tokens, self.sel, self.n_sel,
                              self.cu_sel, self.sel_workspace, stream=stream, keys_unchanged=keys_unchanged)
        else:
            lsa_token_score(q_tok, w, token_keys, self.chunk_table, self.kept[buf], self.n_kept[buf],
                            self.max_chunks, self.tok_scores, self.n_tokens, stream=stream)
            lsa_topk_tokens(self.tok_scores, self.n_tokens, self.fine_k, self.sel, self.n_sel, self.cu_sel,
                            stream=stream)
        if self.packs:
            lsa_gather_tokens(self.k_bufs[buf], self.v_bufs[buf], self.cu_kept[buf], self.sel, self.cu_sel,
                              self.k_fine, self.v_fine, self.cu_units, stream=stream)

    def attend(self, q, out, buf: int = 0, stream=None, kv_unchanged: bool = False):
        """One decode step: out[B, 64, 128] fp32 from q[B, 64, 128] bf16.

        ``kv_unchanged``: the previous kernel on the stream did not write this
        window's compact buffer or offsets (true for every step but the first;
        ignored with ``fine_k``, whose units change every step).
        With ``causal`` the tokens appended so far in the window are attended too."""
        if self.fine_k and not self.packs:   # the selected tokens, read in place
            lsa_sparse_decode_attn_selected(q, self.k_bufs[buf], self.v_bufs[buf], self.cu_kept[buf], self.sel,
                                            self.cu_sel, out, self.workspace, stream=stream)
            return
        kb, vb, cu = self._attn_buffers(buf)
        if self.fine_k:
            kv_unchanged = False
        if self.causal:
            lsa_sparse_decode_attn_local(q, kb, vb, cu, self.k_local, self.v_local, self.local_len, out,
                                         self.workspace, stream=stream, kv_unchanged=kv_unchanged)
        else:
            lsa_sparse_decode_attn(q, kb, vb, cu, out, self.workspace, stream=stream, kv_unchanged=kv_unchanged)

    def run_window(self, q_idx, w, chunk_keys, k_pool, v_pool, q_steps, outs, stream=None, k_new=None, v_new=None,
                   q_tok=None, token_keys=None):
        """Select, gather, then one attention call per step of ``q_steps`` [T, B, 64, 128].

        Causal windows take the decoded tokens ``k_new``, ``v_new`` [T, B, 8, 128]:
        step t appends its own token and attends it (one fused launch).  With ``fine_k`` every step
        first runs the token stage with ``q_tok`` [T, B, 16, 128] over
        ``token_keys`` [n_slots, 64, 128]."""
        if self.causal and (k_new is None or v_new is None):
            raise ValueError("a causal window needs k_new and v_new")
        if self.fine_k and (q_tok is None or token_keys is None):
            raise ValueError("the fine stage needs q_tok and token_keys")
        self.select(q_idx, w, chunk_keys, 0, stream)
        self.gather(k_pool, v_pool, 0, stream)
        if self.causal:
            self.reset_local(stream)
        for t in range(q_steps.shape[0]):
            if self.fine_k:
                self.fine_select(q_tok[t], w, token_keys, 0, stream, keys_unchanged=t > 0)
            if self.causal:
                self.attend_append(q_steps[t], outs[t], k_new[t], v_new[t], 0, stream, kv_unchanged=t > 0)
            else:
                self.attend(q_steps[t], outs[t], 0, stream, kv_unchanged=t > 0)

    def kept_lists(self, buf: int = 0):
        """Host copy of the kept chunk lists (for inspection and tests)."""
        kept = self.kept[buf].cpu()
        n = self.n_kept[buf].cpu()
        return [kept[b, : int(n[b])].tolist() for b in range(self.B)]
