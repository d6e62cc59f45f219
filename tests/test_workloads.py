"""The seeded input recipe (CPU only).

The pages measure on long-context benchmarks whose items are not used here;
synthetic inputs stand in for them at the same context lengths.  The batched
workload takes ragged lengths: each sequence's length is drawn uniformly in
[32768, 262144] tokens and floored to whole 64-token chunks (never below
32768), with K = floor(N / 8) kept chunks besides the latest one (the 12.5%
recall ratio)."""
import torch

import workloads


def test_batched_lengths_recipe():
    wl = workloads.WORKLOADS["batched"]
    n, k = workloads.lengths_for(wl)
    assert n.numel() == wl.batch == 32
    tokens = n.to(torch.int64) * 64
    assert int(tokens.min()) >= 32768 and int(tokens.max()) <= 262144
    assert torch.equal(k, torch.div(n, 8, rounding_mode="floor"))
    assert int(n.min()) < int(n.max())                      # ragged


def test_lengths_are_seeded():
    wl = workloads.WORKLOADS["batched"]
    n1, _ = workloads.lengths_for(wl)
    n2, _ = workloads.lengths_for(wl)
    n3, _ = workloads.lengths_for(wl, base_seed=workloads.BASE_SEED + 1)
    assert torch.equal(n1, n2) and not torch.equal(n1, n3)


def test_fixed_length_workloads():
    for name, chunks, k in (("500k", 8192, 819), ("128k", 2048, 256), ("1m_host", 16384, 1638)):
        n, kk = workloads.lengths_for(workloads.WORKLOADS[name])
        assert n.tolist() == [chunks] and kk.tolist() == [k]


def test_query_drift_keeps_the_distribution_and_correlates_windows():
    """Drift d: window w's indexer query is sqrt(1 - d^2) times window w-1's plus
    d times a fresh draw, so elements stay N(0, 1), consecutive windows correlate
    by about sqrt(1 - d^2), window 0 is unchanged, and d = 1 is the plain draw."""
    import math
    import torch
    plain = workloads.make_inputs("128k", "cpu", windows=4, pools=False).layers[0].q_idx.float()
    drift = workloads.make_inputs("128k", "cpu", windows=4, pools=False, query_drift=0.3).layers[0].q_idx.float()
    assert torch.equal(plain[0], drift[0])
    for w in range(4):
        assert abs(float(drift[w].std()) - 1.0) < 0.05
    for w in range(3):
        c = float(torch.nn.functional.cosine_similarity(drift[w].flatten(), drift[w + 1].flatten(), dim=0))
        assert abs(c - math.sqrt(1 - 0.09)) < 0.03
    same = workloads.make_inputs("128k", "cpu", windows=4, pools=False, query_drift=1.0).layers[0].q_idx
    assert torch.equal(same, plain.to(torch.bfloat16))
