"""The configuration the pages fix, read from tests/golden/page_constants.txt
(each line cites its page and section), against the oracle, the library's
binding and the workloads.  These pin constants to the pages rather than to the
code that uses them."""
import inspect
import os

import pytest

import kv_chunk_selection_b200 as lsa
import oracle
import workloads
from kv_chunk_selection_b200.window import TAU, LayerWindow

HERE = os.path.dirname(os.path.abspath(__file__))


def page_constants():
    out = {}
    for line in open(os.path.join(HERE, "golden", "page_constants.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, cite = line.split("|", 1)
        name, value = head.split()
        assert cite.strip(), f"{name}: no citation"
        out[name] = float(value)
    return out


C = page_constants()


def test_gqa_shape_and_window_length():
    assert oracle.NUM_Q_HEADS == lsa.NUM_Q_HEADS == C["query_heads"]
    assert oracle.NUM_KV_HEADS == lsa.NUM_KV_HEADS == C["kv_heads"]
    assert oracle.HEAD_DIM == lsa.HEAD_DIM == C["head_dim"]
    assert TAU == workloads.TAU == C["tau"]


def test_threshold_default():
    assert inspect.signature(oracle.threshold_chunks).parameters["threshold"].default == C["threshold"]
    assert inspect.signature(LayerWindow).parameters["threshold"].default == C["threshold"]


def test_fine_budget_is_whole_units():
    assert C["fine_k"] % lsa.CHUNK_TOKENS == 0      # packs into whole 64-token units


@pytest.mark.parametrize("name,key", [("500k", "kept_fraction_500k"), ("1m_host", "kept_fraction_1m")])
def test_kept_fraction_matches_the_pages(name, key):
    n, k = workloads.lengths_for(workloads.WORKLOADS[name])
    kept = (k + 1).sum().item() / n.sum().item()
    assert abs(kept - C[key]) < 0.002


def test_local_window_is_whole_chunks():
    assert C["local_window_tokens"] % lsa.CHUNK_TOKENS == 0
    assert C["local_window_tokens"] // lsa.CHUNK_TOKENS == 128   # the recent window of 128 chunks the tests cover
