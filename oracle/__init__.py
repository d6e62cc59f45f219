"""fp64 CPU oracle of the LSA decode step: test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library.
"""
from .lsa_oracle import *  # noqa: F401,F403
from .lsa_oracle import (attend_one, bf16_bits_to_f64, cumulative_kept, decode_window,  # noqa: F401
                         gather_chunks, index_scores, sparse_decode_attn, threshold_chunks,
                         topk_chunks, token_scores, topk_tokens, fine_decode_attn)
