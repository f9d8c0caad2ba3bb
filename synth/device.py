"""Move generated workloads into device memory (torch does the allocation and copies).

The full pools are allocated on the device filled with the bf16 NaN that stands for
stale rows; only the blocks the workload uses are copied over.  No arithmetic of the
method happens here.
"""

from __future__ import annotations

import numpy as np
import torch

from .workloads import POISON_BF16, DecodeStep, PagedPool, PrefillStep


def bf16_tensor(bits: np.ndarray, device=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def bits_of(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16 tensor (copied to the host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def i32(a, device=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32))
    return t.to(device) if device is not None else t


def pool_to_device(pool: PagedPool, device) -> torch.Tensor:
    full = torch.full(pool.shape, np.int16(np.uint16(POISON_BF16).view(np.int16)),
                      dtype=torch.int16, device=device)
    ids, data = pool.stored_blocks()
    if len(ids):
        step = 256
        for i in range(0, len(ids), step):
            idx = torch.from_numpy(np.asarray(ids[i:i + step], np.int64)).to(device)
            blk = torch.from_numpy(np.ascontiguousarray(data[i:i + step]).view(np.int16)).to(device)
            full.index_copy_(0, idx, blk)
    return full.view(torch.bfloat16)


def decode_to_device(step: DecodeStep, device) -> dict:
    return dict(
        q=bf16_tensor(step.q, device),
        k_new=bf16_tensor(step.k_new, device),
        v_new=bf16_tensor(step.v_new, device),
        slot_mapping=i32(step.slot_mapping, device),
        block_tables=i32(step.block_tables, device),
        context_lens=i32(step.context_lens, device),
        k_cache=pool_to_device(step.k_pool, device),
        v_cache=pool_to_device(step.v_pool, device),
    )


def prefill_to_device(step: PrefillStep, device) -> dict:
    return dict(
        q=bf16_tensor(step.q, device),
        k_new=bf16_tensor(step.k_new, device),
        v_new=bf16_tensor(step.v_new, device),
        slot_mapping=i32(step.slot_mapping, device),
        block_tables=i32(step.block_tables, device),
        cu_seqlens_q=i32(step.cu_seqlens_q, device),
        cu_seqlens_k=i32(step.cu_seqlens_k, device),
        k_cache=pool_to_device(step.k_pool, device),
        v_cache=pool_to_device(step.v_pool, device),
    )
