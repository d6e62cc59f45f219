"""Attention inputs whose result identifies every 64-token unit that was read.

With every key zero, every logit is exactly 0, so the softmax gives each
attended token the same weight 1/T (handbook page "DeepSeek-V4: Architecting for
Ultra-Long Contexts", GQA section: softmax(q K^T / sqrt(d)) V).  Each token of a
compact chunk c of KV head g gets a one-hot value row at dimension
(off[g, c] + t) mod 128, t its row in the chunk, with off a seeded random
offset per (head, chunk).  Then

    out[b, h, d] = #{attended tokens of KV head h // 8 whose one-hot dim is d} / T_b

a ratio of small integers, which fp32 holds to a few ulps.  A unit read twice,
read from the wrong head or sequence, or skipped changes T_b by 64 tokens, which
moves every component of that head by about 64 / T_b relative (6e-4 at a
million-token context), far above the few-ulp error of the split-K merge;
components with no attended token must be exactly 0.
The closed form below is pinned against the oracle's attention on small inputs
(tests/test_oracle_pins.py).
"""
from __future__ import annotations

import numpy as np
import torch

HEAD_DIM = 128
CHUNK = 64
KV_HEADS = 8
GROUP = 8

# Relative bound of the exact-count check: fp32 sums of 1.0 are exact, the
# split-K merge's weights exp2(lse_s - M) go through ex2/lg2 approximations
# of about 2^-22 relative error each.
SIG_RTOL = 1e-5


def offsets(n_chunks_total: int, seed: int) -> np.ndarray:
    """off[g, c] in [0, 128): the one-hot dimension of token 0 of chunk c, head g."""
    return np.random.default_rng(seed).integers(0, HEAD_DIM, size=(KV_HEADS, n_chunks_total), dtype=np.int64)


def local_offsets(batch: int, seed: int) -> np.ndarray:
    """offl[b, g]: the same for the local chunk of sequence b."""
    return np.random.default_rng(seed).integers(0, HEAD_DIM, size=(batch, KV_HEADS), dtype=np.int64)


def one_hot_rows(off: torch.Tensor) -> torch.Tensor:
    """bf16 [..., 64, 128] with row t one-hot at (off + t) % 128; ``off`` int64 [...]."""
    t = torch.arange(CHUNK, device=off.device, dtype=torch.int64)
    idx = (off[..., None] + t) % HEAD_DIM
    v = torch.zeros(tuple(off.shape) + (CHUNK, HEAD_DIM), dtype=torch.bfloat16, device=off.device)
    v.scatter_(-1, idx[..., None], 1.0)
    return v


def compact_v(off: np.ndarray, device) -> torch.Tensor:
    """Head-major compact V buffer [8, chunks, 64, 128] for the offsets ``off`` [8, chunks]."""
    return one_hot_rows(torch.from_numpy(off).to(device))


def _counts(dims_by_head, batch_of, B):
    cnt = np.zeros((B, KV_HEADS, HEAD_DIM), dtype=np.int64)
    for g in range(KV_HEADS):
        np.add.at(cnt[:, g], (batch_of, dims_by_head[g]), 1)
    return cnt


def expected_chunks(off: np.ndarray, cu_kept, local_off=None, local_len=None) -> np.ndarray:
    """float64 [B, 64, 128]: attention over the kept chunks (and the first
    local_len[b] local tokens) with zero keys and the one-hot values."""
    cu = np.asarray(cu_kept, dtype=np.int64)
    B = len(cu) - 1
    total = int(cu[-1])
    chunk_seq = np.repeat(np.arange(B), np.diff(cu))                      # sequence of each compact chunk
    t = np.arange(CHUNK)
    batch_of = np.repeat(chunk_seq, CHUNK)                                # per token
    dims = [((off[g, :total, None] + t) % HEAD_DIM).reshape(-1) for g in range(KV_HEADS)]
    cnt = _counts(dims, batch_of, B)
    tokens = np.diff(cu) * CHUNK
    if local_off is not None:
        ll = np.asarray(local_len, dtype=np.int64)
        for b in range(B):
            for g in range(KV_HEADS):
                d = (local_off[b, g] + np.arange(ll[b])) % HEAD_DIM
                np.add.at(cnt[b, g], d, 1)
        tokens = tokens + ll
    return _normalise(cnt, tokens)


def expected_selected(off: np.ndarray, cu_kept, selected) -> np.ndarray:
    """float64 [B, 64, 128]: attention over the selected positions only
    (position p is row p % 64 of compact chunk cu_kept[b] + p // 64)."""
    cu = np.asarray(cu_kept, dtype=np.int64)
    B = len(cu) - 1
    cnt = np.zeros((B, KV_HEADS, HEAD_DIM), dtype=np.int64)
    tokens = np.zeros(B, dtype=np.int64)
    for b in range(B):
        p = np.asarray(selected[b], dtype=np.int64)
        tokens[b] = p.size
        chunk = cu[b] + p // CHUNK
        for g in range(KV_HEADS):
            np.add.at(cnt[b, g], (off[g, chunk] + p % CHUNK) % HEAD_DIM, 1)
    return _normalise(cnt, tokens)


def _normalise(cnt, tokens):
    B = cnt.shape[0]
    out = np.zeros((B, KV_HEADS * GROUP, HEAD_DIM), dtype=np.float64)
    for b in range(B):
        if tokens[b] == 0:
            continue
        per_head = cnt[b] / float(tokens[b])                             # [8, 128]
        out[b] = np.repeat(per_head, GROUP, axis=0)
    return out


def assert_signature(got: np.ndarray, want: np.ndarray, what: str = ""):
    """Exact zeros where no token maps, SIG_RTOL relative elsewhere."""
    assert got.shape == want.shape
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    zero = want == 0.0
    bad0 = np.argwhere(zero & (got != 0.0))
    assert bad0.size == 0, f"{what}: {len(bad0)} components should be exactly 0, first {bad0[:3].tolist()}"
    rel = np.abs(got[~zero] - want[~zero]) / want[~zero]
    assert rel.max(initial=0.0) <= SIG_RTOL, (
        f"{what}: worst relative error {rel.max():.3e} (a unit missing or read twice moves it by >= 1/T)")
