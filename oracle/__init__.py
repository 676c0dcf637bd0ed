"""CPU oracle for the chunked H2O KV-cache attention path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or calls
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.

The oracle is a plain, slow, float64 restatement of what the paper
"Learning how to Forget: Fine-tuning for Long-Context Sparse Attention"
(KeysAndValues) defines for one attention layer with a fixed-capacity KV cache:
fill left to right, the token-position causal mask, SDPA, the attention weights
summed over the query axis (and over the query heads of a GQA group), the
cumulative H2O score and lowest-score eviction.  It shares no code with the CUDA
path; see ``oracle/h2o_oracle.py`` for the per-function citations.
"""

from .h2o_oracle import (  # noqa: F401
    EMPTY_POS,
    QMAX,
    SCORE_MODES,
    OracleCache,
    attend_head,
    attend_head_backward,
    dequantize_rows,
    pack_int4,
    quantize_rows,
    select_slots,
    selection_keys,
    unpack_int4,
)
