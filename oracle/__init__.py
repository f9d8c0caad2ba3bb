"""CPU oracle for paged-KV attention (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this
package.  The CUDA library never imports it and it never imports the CUDA library.
"""

from .paged_attention import (  # noqa: F401
    PAD_SLOT,
    attend,
    bf16_to_f64,
    blocks_for_tokens,
    causal_mask,
    gather_kv,
    group_size,
    lse_combine,
    paged_decode_attention,
    slot_to_block_row,
    store_kvcache,
    varlen_prefill_attention,
)
