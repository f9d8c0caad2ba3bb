"""Seeded synthetic inputs for the paged-KV attention path.

This package builds the inputs that both the oracle and the CUDA library consume:
block-paged K/V pools (as bf16 bit patterns), block tables, context lengths,
cumulative sequence lengths, slot mappings and the new tokens' Q/K/V.  It holds
none of the attention arithmetic: it plays the part of the engine's scheduler and
block manager, which in Nano-vLLM produce exactly these tensors on the CPU
(Nano-vLLM part 1, Neutree AI, section 4 "Block Manager" and section 5.2
"preparation before the model call").
"""

from .workloads import (  # noqa: F401
    POISON_BF16,
    DecodeStep,
    PagedPool,
    PrefillStep,
    WORKLOADS,
    bf16_bits_from_f32,
    make_decode_step,
    make_prefill_step,
    decode_tiny,
    decode_mid,
    decode_batch512_shared_prefix,
    prefill_varlen_prefix_hits,
    decode_long_fragmented,
)
