"""The bench's algorithmic byte count against per-configuration figures fixed by
the method's sizes (CPU only).

Per decoded token a window moves the indexer key of every chunk once (256 B
per chunk, amortised over the 64 steps) and per step the kept chunks' K and V
(256 KiB per chunk: 8 KV heads x 64 tokens x 128 dims x 2 bytes, twice), the
bf16 query (16 KiB) and the fp32 output (32 KiB).  The sizes follow from the
GQA shape of the handbook page ("Grouped Query Attention (GQA) vs. Multi-Head
Attention (MHA)": 64 query heads, 8 KV heads, head dim 128) and the kept
fractions of the summary page (3 Experiments), written out here by hand."""
import pytest
import torch

import bench

MB = 1e6


@pytest.mark.parametrize("chunks,kept,per_token_mb", [
    (2048, 257, 67.43),     # 128K: 256 + latest
    (8192, 820, 215.04),    # 500K: 819 + latest
    (16384, 1639, 429.77),  # 1M: 1638 + latest
])
def test_window_bytes_per_token(chunks, kept, per_token_mb):
    n = torch.tensor([chunks], dtype=torch.int32)
    per_window, per_step, total_chunks = bench.window_bytes(n, kept, layers=1)
    assert total_chunks == chunks
    # one attention launch: kept K/V, the query and the output
    assert per_step == kept * 2 * 8 * 64 * 128 * 2 + 64 * 128 * 2 + 64 * 128 * 4
    # a window: 64 steps plus the chunk keys, the indexer query and the head weights once
    assert per_window == 64 * per_step + 256 * chunks + 16 * 128 * 2 + 16 * 4
    assert abs(per_window / 64 / MB - per_token_mb) < 0.01


def test_window_bytes_scale_with_layers_and_batch():
    n = torch.tensor([100, 0, 37], dtype=torch.int32)
    one, step, _ = bench.window_bytes(n, 20, layers=1)
    four, step4, _ = bench.window_bytes(n, 20, layers=4)
    assert four == 4 * one and step4 == step
    assert step == 20 * 262144 + 3 * (64 * 128 * 2 + 64 * 128 * 4)


def test_attention_call_launches_two_kernels():
    # the split-K attention grid and the merge of the pairs it split
    assert bench.ATTN_LAUNCHES == 2
