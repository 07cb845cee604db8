"""Test infrastructure: a plain, slow, fp64 CPU oracle for MLA decode over a paged KV cache.

Nothing on the product path may import this package.  Only the tests, the smoke
check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` use it.  It
shares no code with the CUDA library (``attention_mla_get_b200``): it reads the
same seeded inputs (``mla_inputs``) and computes the result straight from the
definition, with no splits, no online softmax and no tiling.

Modules
  mla_decode_ref     -- gather pages, scaled scores, causal mask, softmax, O and LSE (fp64);
                        the token-sparse variant over an index list per query position, and
                        sparse prefill over one contiguous cache
  fp8_format         -- decode of the 656-byte FP8 token (e4m3 codes, fp32 scales, bf16 RoPE)
  tile_scheduler_ref -- the integer rule that splits requests into (request, block-range)
                        chunks over the SM parts, and the num_splits prefix

Pinned by tests/test_oracle_pins.py, tests/test_fp8_format.py and
tests/test_scheduler_ref.py (brute force, closed forms, invariants, library
routines).  No function here is "parity unpinned".
"""
from .mla_decode_ref import (bf16_to_f64, gather_request_keys, attend_rows,
                             mla_decode_reference, mla_sparse_decode_reference,
                             mla_sparse_prefill_reference, visible_keys)
from .fp8_format import e4m3_table, decode_fp8_tokens
from .tile_scheduler_ref import (BLOCK_TOKENS, FIXED_SPLIT_COST, schedule, num_sm_parts_for,
                                 row_groups_for, iterate_part)

__all__ = [
    "bf16_to_f64", "gather_request_keys", "attend_rows", "mla_decode_reference",
    "mla_sparse_decode_reference", "mla_sparse_prefill_reference", "visible_keys",
    "e4m3_table", "decode_fp8_tokens",
    "BLOCK_TOKENS", "FIXED_SPLIT_COST", "schedule", "num_sm_parts_for", "row_groups_for", "iterate_part",
]
