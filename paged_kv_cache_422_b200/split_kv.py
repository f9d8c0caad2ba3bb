"""Split-KV decode across devices: each rank attends over its share of every sequence's
keys, the ranks exchange their partials, and each rank merges them by log-sum-exp.

This is the one sharding of the decode that has an exchange step: for long contexts a
sequence's blocks are spread over the ranks (rank r holds a contiguous run of each
sequence's blocks in its own cache), every rank computes (o_r, lse_r) for all sequences
with `nvpa_paged_decode_partial`, the parts are all-gathered (one [B, Hq, D] fp32 and one
[B, Hq] fp32 per rank: B * Hq * (D + 1) * 4 bytes, small next to the key/value bytes
read), and `nvpa_lse_combine` merges them.  The merge is the split-KV combine of the
single-GPU decode applied across devices ("Nano-vLLM part 1" section 5.2 decode).

The collective is torch.distributed's all-gather (NCCL over NVLink on GPUs, gloo on CPU
for the tests); the compute steps are the library's kernels unless the caller passes
others (the CPU tests pass stand-ins).
"""

from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import api


def shard_block_tables(block_tables, context_lens, block_size, world, rank):
    """Rank `rank`'s view of a batch whose keys are split over `world` ranks.

    Sequence b's ceil(ctx_b / block_size) blocks are cut into `world` contiguous runs of
    whole blocks; rank r gets run r: blocks [floor(r n / W), floor((r + 1) n / W)).
    Returns (local_block_tables [B, max_local_blocks] int32 padded with -1,
    local_context_lens [B] int32, first_key [B] int64): the local keys are the sequence's
    keys first_key[b] .. first_key[b] + local_context_lens[b] - 1, in order.
    """
    bt = np.asarray(block_tables)
    ctx = np.asarray(context_lens, np.int64)
    if not 0 <= rank < world:
        raise ValueError("rank outside [0, world)")
    B = ctx.shape[0]
    nblk = -(-ctx // block_size)
    lo = (rank * nblk) // world
    hi = ((rank + 1) * nblk) // world
    width = max(1, int((hi - lo).max())) if B else 1
    local_bt = np.full((B, width), -1, np.int32)
    local_ctx = np.zeros(B, np.int32)
    for b in range(B):
        n = int(hi[b] - lo[b])
        if n == 0:
            continue
        local_bt[b, :n] = bt[b, lo[b]:hi[b]]
        local_ctx[b] = int(min(ctx[b], hi[b] * block_size) - lo[b] * block_size)
    return local_bt, local_ctx, lo * block_size


def _all_gather(t, group):
    world = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        outp = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(outp, t.contiguous(), group=group)
        return outp
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def split_kv_decode(q, k_cache, v_cache, local_block_tables, local_context_lens, max_context_len,
                    softmax_scale, group=None, partial_fn=None, combine_fn=None,
                    return_lse=False):
    """Decode attention of sequences whose keys are split over the ranks of `group`.

    Every rank passes the same q and its own cache, local block tables and local context
    lengths (see shard_block_tables); every rank gets the full result.  `partial_fn` and
    `combine_fn` default to the library's nvpa_paged_decode_partial / nvpa_lse_combine.
    """
    partial_fn = partial_fn or (lambda *a: api.paged_decode_partial(*a))
    combine_fn = combine_fn or (lambda o, l: api.lse_combine(o, l, return_lse=True))
    o_part, lse_part = partial_fn(q, k_cache, v_cache, local_block_tables, local_context_lens,
                                  max_context_len, softmax_scale)
    o_all = _all_gather(o_part, group)
    lse_all = _all_gather(lse_part, group)
    out, lse = combine_fn(o_all, lse_all)
    return (out, lse) if return_lse else out
