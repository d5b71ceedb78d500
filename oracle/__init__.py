"""Float64 CPU oracle for Block-Union KV selection and paged chunk attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never calls it, and it shares no code with the CUDA library: it is a
plain restatement of what the method computes, written from

  "CompactAttention: Accelerating Chunked Prefill with Block-Union KV
   Selection", Abstract:
   * 2D block-sparse masks are KV-selection signals, not sparse-kernel plans;
   * they become GQA-aware per-group KV block tables by a Q-block union and an
     intra-group union;
   * the tables are the minimal ones that keep every selected KV block under
     paged execution, and the selected blocks are read in place.

Where the abstract is silent (scale, log base, head-to-group map, padding,
empty rows) the readings are those listed in the repository's design notes:
scale 1/sqrt(d), natural-log LSE, group g(h) = h // (Hq/Hkv), table padding -1,
an empty key set gives O = 0 and LSE = -inf.

Every function here is pinned by tests/test_oracle_*.py against brute force,
closed forms, library routines (torch SDPA in float64) and invariants.
Nothing here is "parity unpinned".
"""
from .tables import oracle_tables, brute_force_tables, unpack_mask_bits, oracle_tables_bits  # noqa: F401
from .attention import (  # noqa: F401
    depage,
    oracle_chunk_attention,
    oracle_rows,
    brute_force_attention,
    lse_combine,
    oracle_append_kv,
    oracle_varlen,
)
from .fp8 import (  # noqa: F401,E402
    decode_e4m3,
    dequantize_pages,
    oracle_chunk_attention_fp8,
    oracle_rows_fp8,
)
