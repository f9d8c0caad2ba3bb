"""Error behaviour on the GPU: host-side statuses and device-side flags (no faults)."""

import time

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from paged_kv_cache_422_b200 import NvpaError
from synth import make_decode_step, make_prefill_step
from synth.device import decode_to_device, i32, prefill_to_device
from tests.helpers import assert_attention_close, oracle_after_store

pytestmark = pytest.mark.gpu


def test_unsupported_head_dim_is_rejected(cuda_device):
    q = torch.zeros((2, 4, 96), dtype=torch.bfloat16, device=cuda_device)
    kc = torch.zeros((4, 16, 2, 96), dtype=torch.bfloat16, device=cuda_device)
    bt = torch.zeros((2, 1), dtype=torch.int32, device=cuda_device)
    ctx = torch.ones(2, dtype=torch.int32, device=cuda_device)
    with pytest.raises(NvpaError) as ei:
        nvpa.paged_decode_attention(q, kc, kc, bt, ctx, 16, 0.1)
    assert ei.value.status == 2


def test_workspace_too_small_is_rejected(cuda_device):
    step = make_decode_step(1, [4000, 10], num_q_heads=4, num_kv_heads=2, head_dim=128,
                            block_size=256)
    t = decode_to_device(step, cuda_device)
    ws = torch.empty(64, dtype=torch.uint8, device=cuda_device)
    with pytest.raises(NvpaError) as ei:
        nvpa.paged_decode_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                    t["context_lens"], 4000, step.scale, workspace=ws)
    assert ei.value.status == 4


def test_bad_block_id_is_flagged_not_read(cuda_device):
    step = make_decode_step(2, [40, 40], num_q_heads=4, num_kv_heads=2, head_dim=64,
                            block_size=16)
    t = decode_to_device(step, cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    t["block_tables"][1, 1] = step.num_blocks + 5
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = nvpa.paged_decode_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                      t["context_lens"], 40, step.scale, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()


def test_context_longer_than_declared_is_flagged(cuda_device):
    step = make_decode_step(3, [100, 20], num_q_heads=4, num_kv_heads=2, head_dim=64,
                            block_size=16)
    t = decode_to_device(step, cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = nvpa.paged_decode_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                      t["context_lens"], 50, step.scale, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_LENGTH
    assert torch.isfinite(out.float()).all()


def test_prefill_more_queries_than_keys_is_flagged(cuda_device):
    step = make_prefill_step(4, [50, 30], num_q_heads=4, num_kv_heads=2, head_dim=64,
                             block_size=16)
    t = prefill_to_device(step, cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    bad_cu_k = i32([0, 40, 70], cuda_device)       # sequence 0 now has Lq 50 > Lk 40
    out = torch.full_like(t["q"], 7.0)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nvpa.varlen_prefill_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                  t["cu_seqlens_q"], bad_cu_k, 50, 50, step.scale, out=out,
                                  err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_LENGTH
    assert torch.all(out[:50] == 7.0)                 # rows of the bad sequence untouched
    assert torch.isfinite(out[50:].float()).all() and not torch.all(out[50:] == 7.0)


def test_prefill_bad_block_id_is_flagged_and_stays_finite(cuda_device):
    """A block id out of range in one sequence's table is flagged, that piece is not read
    (zero-filled), the output stays finite, and the other sequences are unaffected."""
    import oracle
    from tests.helpers import assert_attention_close, oracle_after_store
    step = make_prefill_step(5, [300, 140], cached_blocks=[1, 0], num_q_heads=4, num_kv_heads=2,
                             head_dim=64, block_size=16)
    t = prefill_to_device(step, cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    t["block_tables"][0, 3] = step.num_blocks + 7
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = nvpa.varlen_prefill_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                        t["cu_seqlens_q"], t["cu_seqlens_k"], step.max_seqlen_q,
                                        step.max_seqlen_k, step.scale, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    ref, _ = oracle.varlen_prefill_attention(step.q, kc, vc, step.block_tables, step.cu_seqlens_q,
                                             step.cu_seqlens_k, step.scale)
    q1 = int(step.cu_seqlens_q[1])
    assert_attention_close(out[q1:], ref[q1:], "prefill, sequence with a valid table")



def test_bounded_wait_runs_out_with_a_status(cuda_device):
    """A wait that cannot complete (a barrier nothing arrives at, waited on with the
    tensor-core kernels' own bounded wait) gives up after about 2 s, flags
    NVPA_FLAG_TIMEOUT and returns; the next prefill on the same context, whose kernel
    uses the same waits, completes with no flag and matches the oracle."""
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    nvpa.check_bounded_wait(err)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert err.item() == nvpa.NVPA_FLAG_TIMEOUT
    assert 1.5 < elapsed < 60.0
    assert nvpa.lib().nvpa_check_bounded_wait(None, None) == 1   # null err_flag: INVALID_ARG

    step = make_prefill_step(300, [200, 90], cached_blocks=[1, 0], num_q_heads=8, num_kv_heads=2,
                             head_dim=128, block_size=64)
    t = prefill_to_device(step, cuda_device)
    err2 = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                       err_flag=err2)
    out = nvpa.varlen_prefill_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                        t["cu_seqlens_q"], t["cu_seqlens_k"], step.max_seqlen_q,
                                        step.max_seqlen_k, step.scale, err_flag=err2)
    torch.cuda.synchronize()
    assert err2.item() == 0
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    ref, _ = oracle.varlen_prefill_attention(step.q, kc, vc, step.block_tables, step.cu_seqlens_q,
                                             step.cu_seqlens_k, step.scale)
    assert_attention_close(out, ref, "prefill after a timed-out wait")
