"""CPU oracle for the Lightning Indexer hot path -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, fp64 restatement of what the indexer computes.
It exists so that the CUDA path can be checked against an implementation that
shares no code with it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it; the
product path (the package ``sparse_attention_token_02_b200``) never does.

Modules
-------
fp8_e4m3   OCP FP8 E4M3 codec (decode table, RNE + satfinite encode) and the
           per-row absmax quantiser.
indexer    scores I[t,s], causal mask, top-k with a fixed tie-break, and the
           prefill / decode drivers over ragged sequences (also over an
           m-compressed key cache).
rope       the rotary embedding applied to indexer keys and queries.
after_select  what consumers do with a selection: latent-row gather, int64
           cache rows, sorted order.

Every function here is pinned by ``tests/test_oracle_*.py`` against closed forms,
hand-summed literals, invariants, brute force on tiny rows, and (for the codec)
torch's own float8 conversion.  See each function's docstring for the passage it
follows.
"""

from .fp8_e4m3 import (  # noqa: F401
    E4M3_MAX,
    bf16_bits_to_f64,
    e4m3_decode,
    e4m3_encode,
    e4m3_value_table,
    quantize_rows,
)
from .indexer import (  # noqa: F401
    decode_oracle,
    prefill_oracle,
    query_positions,
    row_scores,
    topk_row,
)
