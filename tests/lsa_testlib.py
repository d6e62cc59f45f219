"""Helpers shared by the GPU parity tests: tolerances, host copies, comparisons.

Tolerances (the stated parity bar of this library):
  * indexer scores: |gpu - oracle| <= 1e-4 * |oracle|
  * kept sets and gathers: exact, except at a boundary where the oracle's K-th
    and (K+1)-th scores differ by less than 1e-5 relative; there either chunk
    is accepted and attention is checked against the oracle run on the GPU's
    own kept set
  * attention outputs (fp32): |gpu - oracle| <= 2e-3 + 1e-3 * |oracle|
"""
import numpy as np
import torch

import oracle

SCORE_RTOL = 1e-4
TIE_RTOL = 1e-5
ATT_ATOL = 2e-3
ATT_RTOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def cm(t: torch.Tensor) -> torch.Tensor:
    """Chunk-major view [chunks, 8, 64, 128] of a head-major compact buffer [8, chunks, 64, 128].

    The kernels keep compact buffers head-major; the oracle and the tests index them chunk first.
    The permutation is its own inverse, so cm() also turns a chunk-major view back into the
    head-major storage the kernels take."""
    return t.permute(1, 0, 2, 3)


def i64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.int64).numpy()


def assert_scores_close(gpu_scores, oracle_scores, n_chunks):
    g = f64(gpu_scores)
    for b, n in enumerate(n_chunks):
        n = int(n)
        err = np.abs(g[b, :n] - oracle_scores[b, :n])
        bound = SCORE_RTOL * np.abs(oracle_scores[b, :n])
        bad = np.nonzero(err > bound)[0]
        assert bad.size == 0, f"seq {b}: {bad.size} scores off, worst rel {np.max(err / np.abs(oracle_scores[b, :n]))}"


def kept_from_gpu(kept, n_kept):
    k = i64(kept)
    n = i64(n_kept)
    return [k[b, : n[b]].tolist() for b in range(len(n))]


def assert_kept_matches(gpu_kept, oracle_scores, n_chunks, k_per_seq):
    """Exact match with the oracle's selection, except inside the tie window."""
    ref = oracle.topk_chunks(oracle_scores, n_chunks, k_per_seq)
    for b, (g, r) in enumerate(zip(gpu_kept, ref)):
        g, r = list(g), list(r)
        assert len(g) == len(r), f"seq {b}: kept {len(g)} vs {len(r)}"
        if g == r:
            continue
        n, k = int(n_chunks[b]), int(k_per_seq[b])
        s = oracle_scores[b, : n - 1]
        order = np.lexsort((np.arange(n - 1), -s))
        sk, sk1 = s[order[k - 1]], s[order[k]]
        assert (sk - sk1) < TIE_RTOL * abs(sk), f"seq {b}: kept sets differ outside a tie"
        diff = set(g) ^ set(r)
        for c in diff:
            assert abs(s[c] - sk) <= TIE_RTOL * abs(sk) + (sk - sk1), f"seq {b}: chunk {c} not at the boundary"


def assert_attention_close(gpu_out, ref, heads=None, seqs=None):
    g = f64(gpu_out)
    sel = (slice(None) if seqs is None else list(seqs), slice(None) if heads is None else list(heads))
    gg = g[sel[0]][:, sel[1]]
    rr = ref[sel[0]][:, sel[1]]
    assert np.all(np.isfinite(gg))
    err = np.abs(gg - rr)
    bound = ATT_ATOL + ATT_RTOL * np.abs(rr)
    assert np.all(err <= bound), f"attention off: max err {err.max():.3e}, worst excess {(err - bound).max():.3e}"
    return float(err.max())
