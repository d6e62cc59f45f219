"""Seeded synthetic inputs for the LSA decode step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CUDA path (through the tests and ``bench.py``)
and the fp64 oracle consume what it produces: the oracle always receives a host
copy of exactly the bytes the GPU reads.

Workloads (sizes follow the method: 64-token chunks, GQA 64 query heads over
8 KV heads of dimension 128, an indexer of 16 heads of dimension 128, a
lookahead window of tau = 64 decode steps):

=========  ====  =============  ==========  =======  ======================
name       B     chunks / seq   K           windows  notes
=========  ====  =============  ==========  =======  ======================
tiny       1     64             8           1        parity case
128k       1     2048           256         4        16 planted chunks
500k       1     8192           819         2        2 GiB pool in HBM
1m_host    1     16384          1638        2        4 GiB pool, pinned host
1m         1     16384          1638        2        4 GiB pool in HBM
batched    32    512..4096      N_b // 8    2        4 layers, paged table
=========  ====  =============  ==========  =======  ======================

Distributions: K, V, indexer keys and queries are N(0,1) drawn in float32 and
rounded to bf16 (round to nearest even); indexer head weights are U(0,1) kept
in float32.  Every tensor has its own seed derived from one base seed, so a
workload is reproducible on the device it was drawn on.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

NUM_Q_HEADS = 64
NUM_KV_HEADS = 8
HEAD_DIM = 128
CHUNK_TOKENS = 64
INDEX_HEADS = 16
INDEX_DIM = 128
TAU = 64
BASE_SEED = 20260608

# Bytes of one chunk of K (or V): 8 heads x 64 tokens x 128 dims x 2 bytes.
CHUNK_BYTES_ONE = NUM_KV_HEADS * CHUNK_TOKENS * HEAD_DIM * 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    description: str
    batch: int
    chunks: Optional[int]            # fixed chunks per sequence (None: ragged)
    k_fraction: Optional[float]      # K = floor(fraction * N) when chunks are ragged
    k_fixed: Optional[int]
    windows: int
    layers: int = 1
    planted: int = 0
    host_pool: bool = False
    ragged_tokens: tuple = ()        # (lo, hi) context length range for ragged batches
    max_chunks: Optional[int] = None


WORKLOADS = {
    "tiny": Workload(
        "tiny", "tiny LSA decode, 1 layer: B=1, L=4096 (64 chunks), K=8 + latest, 1 window",
        batch=1, chunks=64, k_fraction=None, k_fixed=8, windows=1),
    "128k": Workload(
        "128k", "128K single-sequence decode, 1 layer: B=1, L=131072 (2048 chunks), K=256 + latest, "
        "4 windows, 16 planted chunks", batch=1, chunks=2048, k_fraction=None, k_fixed=256,
        windows=4, planted=16),
    "500k": Workload(
        "500k", "500K decode, 1 layer: B=1, L=524288 (8192 chunks), K=819 + latest, 2 windows, "
        "pool resident in HBM", batch=1, chunks=8192, k_fraction=None, k_fixed=819, windows=2),
    "1m_host": Workload(
        "1m_host", "1M decode with host-tier KV pool, 1 layer: B=1, L=1048576 (16384 chunks), "
        "K=1638 + latest, 2 windows, KV pool in pinned host memory", batch=1, chunks=16384,
        k_fraction=None, k_fixed=1638, windows=2, host_pool=True),
    # The 1M sizes with the pool resident in HBM (4 GiB per K/V): the HBM side of
    # the 1M decode step, beside the host tier that the host link bounds.
    "1m": Workload(
        "1m", "1M decode, 1 layer: B=1, L=1048576 (16384 chunks), K=1638 + latest, 2 windows, "
        "pool resident in HBM", batch=1, chunks=16384, k_fraction=None, k_fixed=1638, windows=2),
    "batched": Workload(
        "batched", "batched ragged serving, 4 layers: B=32, L~U[32K,256K] rounded down to 64, "
        "K_b = floor(0.125 N_b) + latest, paged chunk table, 2 windows",
        batch=32, chunks=None, k_fraction=0.125, k_fixed=None, windows=2, layers=4,
        ragged_tokens=(32768, 262144), max_chunks=262144 // CHUNK_TOKENS),
}

# Per-tensor seed offsets.
_OFF = {"lengths": 1, "slots": 2, "w": 10, "keys": 20, "kpool": 30, "vpool": 40,
        "qidx": 50, "q": 60, "planted": 70, "knew": 80, "vnew": 90, "tokkeys": 100, "qtok": 110}


def _seed(base: int, name: str, layer: int = 0, extra: int = 0) -> int:
    return (base * 1_000_003 + _OFF[name] * 10_007 + layer * 101 + extra) % (2 ** 62)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, seed: int, device, out: Optional[torch.Tensor] = None,
               slice_elems: int = 1 << 27) -> torch.Tensor:
    """N(0,1) in float32, rounded to bf16, drawn in slices along dim 0.

    Each slice has its own generator (seed, slice index), which bounds the
    float32 temporary for pools of many GiB.  ``out`` may live elsewhere (for
    instance pinned host memory); slices are then drawn on ``device`` and copied.
    """
    shape = tuple(int(s) for s in shape)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    row = math.prod(shape[1:]) if len(shape) > 1 else 1
    rows_per = max(1, slice_elems // max(1, row))
    for i, r0 in enumerate(range(0, shape[0], rows_per)):
        r1 = min(shape[0], r0 + rows_per)
        g = _gen(seed * 7919 + i, device)
        t = torch.randn((r1 - r0,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        out[r0:r1].copy_(t.to(torch.bfloat16))
        del t
    return out


@dataclasses.dataclass
class LayerInputs:
    k_pool: torch.Tensor          # [n_slots, 8, 64, 128] bf16 (device or pinned host)
    v_pool: torch.Tensor
    chunk_keys: torch.Tensor      # [n_slots, 128] bf16
    w: torch.Tensor               # [16] float32
    q_idx: torch.Tensor           # [windows, B, 16, 128] bf16
    q: torch.Tensor               # [windows, TAU, B, 64, 128] bf16
    planted: Optional[torch.Tensor] = None   # planted chunk ids (diagnostic only)


@dataclasses.dataclass
class Inputs:
    workload: Workload
    n_chunks: torch.Tensor        # [B] int32
    k_per_seq: torch.Tensor       # [B] int32
    chunk_table: torch.Tensor     # [B, max_chunks] int32
    max_chunks: int
    n_slots: int
    layers: list
    steps: int

    @property
    def batch(self) -> int:
        return int(self.n_chunks.shape[0])


def lengths_for(wl: Workload, base_seed: int = BASE_SEED):
    """Per-sequence chunk counts and K for a workload (host tensors)."""
    if wl.chunks is not None:
        n = torch.full((wl.batch,), wl.chunks, dtype=torch.int32)
        k = torch.full((wl.batch,), wl.k_fixed, dtype=torch.int32)
        return n, k
    lo, hi = wl.ragged_tokens
    g = _gen(_seed(base_seed, "lengths"), "cpu")
    tokens = torch.randint(lo, hi + 1, (wl.batch,), generator=g, dtype=torch.int64)
    tokens = torch.clamp((tokens // CHUNK_TOKENS) * CHUNK_TOKENS, min=lo)
    n = (tokens // CHUNK_TOKENS).to(torch.int32)
    k = torch.floor(n.to(torch.float64) * wl.k_fraction).to(torch.int32)
    return n, k


def make_inputs(name_or_wl, device="cuda", base_seed: int = BASE_SEED, layers: Optional[int] = None,
                windows: Optional[int] = None, steps: int = TAU, chunks: Optional[int] = None,
                k: Optional[int] = None, batch: Optional[int] = None, pools: bool = True,
                query_drift: Optional[float] = None) -> Inputs:
    """Draw every input of a workload.  ``chunks``/``k``/``batch`` override the
    sizes (used for reduced parity cases with the same distributions); with
    ``pools=False`` the KV pools are left out (scoring and selection only).

    ``query_drift`` d in [0, 1] correlates the indexer queries of consecutive
    windows: the query of window w > 0 is sqrt(1 - d^2) times that of window
    w - 1 plus d times a fresh N(0, 1) draw (in float32, then rounded to bf16),
    so every element stays N(0, 1) and d = 1 (or None) gives independent windows.
    Small d stands in for the temporal locality of real decoding, where the
    hidden state moves little from one window to the next."""
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    if chunks is not None or k is not None or batch is not None:
        wl = dataclasses.replace(
            wl, chunks=chunks if chunks is not None else wl.chunks,
            k_fixed=k if k is not None else wl.k_fixed,
            batch=batch if batch is not None else wl.batch)
    n_layers = wl.layers if layers is None else layers
    n_windows = wl.windows if windows is None else windows
    n_chunks, k_per_seq = lengths_for(wl, base_seed)
    B = int(n_chunks.shape[0])
    max_chunks = int(wl.max_chunks or int(n_chunks.max()))
    n_slots = int(n_chunks.sum())
    # Physical slot of each logical chunk: identity for one sequence, a seeded
    # permutation of all slots for a batch (a paged cache).
    table = torch.zeros((B, max_chunks), dtype=torch.int32)
    if B == 1:
        table[0, : int(n_chunks[0])] = torch.arange(int(n_chunks[0]), dtype=torch.int32)
    else:
        perm = torch.randperm(n_slots, generator=_gen(_seed(base_seed, "slots"), "cpu")).to(torch.int32)
        off = 0
        for b in range(B):
            nb = int(n_chunks[b])
            table[b, :nb] = perm[off: off + nb]
            off += nb
    layer_list = []
    for l in range(n_layers):
        gw = _gen(_seed(base_seed, "w", l), "cpu")
        w = torch.rand((INDEX_HEADS,), generator=gw, dtype=torch.float32).to(device)
        q_idx = randn_bf16((n_windows, B, INDEX_HEADS, INDEX_DIM), _seed(base_seed, "qidx", l), device)
        if query_drift is not None and query_drift < 1.0:
            d = float(query_drift)
            prev = q_idx[0].float()
            for wi in range(1, n_windows):
                prev = math.sqrt(1.0 - d * d) * prev + d * q_idx[wi].float()
                q_idx[wi] = prev.to(torch.bfloat16)
        q = randn_bf16((n_windows, steps, B, NUM_Q_HEADS, HEAD_DIM), _seed(base_seed, "q", l), device)
        planted = None
        if wl.planted:
            # Planted structure: a few random non-latest chunks get +2.0 along the
            # unit mean direction of all indexer queries of the run, added in
            # float32 before the keys are rounded to bf16.
            gk = _gen(_seed(base_seed, "keys", l), device)
            keys32 = torch.randn((n_slots, INDEX_DIM), generator=gk, device=device, dtype=torch.float32)
            u = q_idx.float().reshape(-1, INDEX_DIM).mean(dim=0)
            u = u / torch.linalg.vector_norm(u)
            gp = _gen(_seed(base_seed, "planted", l), "cpu")
            cand = int(n_chunks[0]) - 1
            planted = torch.randperm(cand, generator=gp)[: wl.planted].sort().values
            slots = table[0, planted].long().to(device)
            keys32[slots] += 2.0 * u
            chunk_keys = keys32.to(torch.bfloat16)
            del keys32
        else:
            chunk_keys = randn_bf16((n_slots, INDEX_DIM), _seed(base_seed, "keys", l), device)
        shape = (n_slots, NUM_KV_HEADS, CHUNK_TOKENS, HEAD_DIM)
        if not pools:
            k_pool = v_pool = None
        elif wl.host_pool:
            k_pool = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            v_pool = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
            randn_bf16(shape, _seed(base_seed, "kpool", l), device, out=k_pool)
            randn_bf16(shape, _seed(base_seed, "vpool", l), device, out=v_pool)
        else:
            k_pool = randn_bf16(shape, _seed(base_seed, "kpool", l), device)
            v_pool = randn_bf16(shape, _seed(base_seed, "vpool", l), device)
        layer_list.append(LayerInputs(k_pool, v_pool, chunk_keys, w, q_idx, q, planted))
    dev = torch.device(device)
    return Inputs(wl, n_chunks.to(dev), k_per_seq.to(dev), table.to(dev), max_chunks, n_slots,
                  layer_list, steps)


def decoded_tokens(inp: Inputs, layer: int, device, base_seed: int = BASE_SEED, windows: Optional[int] = None):
    """K and V of the token each decode step produces, for the causal window:
    two bf16 tensors [windows, TAU, B, 8, 128] drawn N(0, 1) like the pools."""
    n_windows = inp.workload.windows if windows is None else windows
    shape = (n_windows, inp.steps, inp.batch, NUM_KV_HEADS, HEAD_DIM)
    return (randn_bf16(shape, _seed(base_seed, "knew", layer), device),
            randn_bf16(shape, _seed(base_seed, "vnew", layer), device))


def fine_inputs(inp: Inputs, layer: int, device, base_seed: int = BASE_SEED, windows: Optional[int] = None):
    """Inputs of the token-level fine stage: per-token indexer keys by chunk slot,
    bf16 [n_slots, 64, 128], and one indexer query per decode step, bf16
    [windows, TAU, B, 16, 128]; both N(0, 1) like the chunk-level ones."""
    n_windows = inp.workload.windows if windows is None else windows
    keys = randn_bf16((inp.n_slots, CHUNK_TOKENS, INDEX_DIM), _seed(base_seed, "tokkeys", layer), device)
    q_tok = randn_bf16((n_windows, inp.steps, inp.batch, INDEX_HEADS, INDEX_DIM), _seed(base_seed, "qtok", layer),
                       device)
    return keys, q_tok
