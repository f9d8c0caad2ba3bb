"""split_kv_decode end to end on the device: a one-rank NCCL process group on cuda:0.

The multi-rank exchange is covered by the gloo test on CPU and the kernels by the
emulated-rank test; this one runs the path exactly as a rank would: its default partial
and combine functions (nvpa_paged_decode_partial, nvpa_lse_combine) and the NCCL branch
of the all-gather (all_gather_into_tensor), against the oracle over the whole context.
Two ranks cannot share one GPU under NCCL, so the group has one rank.
"""

import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from paged_kv_cache_422_b200 import split_kv
from paged_kv_cache_422_b200.split_kv import shard_block_tables
from synth import WORKLOADS, make_decode_step
from synth.device import decode_to_device, i32
from tests.helpers import assert_attention_close, assert_lse_close, oracle_after_store

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture
def nccl_group(cuda_device):
    if dist.is_initialized():
        pytest.skip("a default process group already exists in this process")
    os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=timedelta(seconds=60), device_id=cuda_device)
    try:
        assert dist.get_backend() == "nccl"
        yield dist.group.WORLD
    finally:
        torch.cuda.synchronize(cuda_device)
        dist.destroy_process_group()


def _stored(step):
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    step.k_pool, step.v_pool = kc, vc
    return step


def test_split_kv_decode_nccl_one_rank(cuda_device, nccl_group):
    step = _stored(make_decode_step(21, [1, 17, 256, 700, 2049, 5000, 0, 3], num_q_heads=16,
                                    num_kv_heads=4, head_dim=128, block_size=64))
    t = decode_to_device(step, cuda_device)
    lbt, lctx, first = shard_block_tables(step.block_tables, step.context_lens, step.block_size,
                                          1, 0)
    assert np.array_equal(lctx, step.context_lens) and not first.any()
    out, lse = split_kv.split_kv_decode(t["q"], t["k_cache"], t["v_cache"], i32(lbt, cuda_device),
                                        i32(lctx, cuda_device), step.max_context_len, step.scale,
                                        group=nccl_group, return_lse=True)
    torch.cuda.synchronize(cuda_device)
    ref, ref_lse = oracle.paged_decode_attention(step.q, step.k_pool, step.v_pool,
                                                 step.block_tables, step.context_lens, step.scale)
    assert_attention_close(out, ref, "split-KV decode over NCCL (one rank)")
    assert_lse_close(lse, ref_lse, "split-KV decode over NCCL (one rank)")


def test_split_kv_decode_nccl_long_context(cuda_device, nccl_group):
    """The long-context workload (8 x 32768 keys, block size 16, group 4) through the same
    path; all 8 sequences against the oracle."""
    step = _stored(WORKLOADS["decode_long_b8_ctx32k_bs16"]())
    t = decode_to_device(step, cuda_device)
    out = split_kv.split_kv_decode(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                   t["context_lens"], step.max_context_len, step.scale,
                                   group=nccl_group)
    torch.cuda.synchronize(cuda_device)
    ref, _ = oracle.paged_decode_attention(step.q, step.k_pool, step.v_pool, step.block_tables,
                                           step.context_lens, step.scale)
    assert_attention_close(out, ref, "long-context split-KV over NCCL")
