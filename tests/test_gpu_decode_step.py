"""nvpa_decode_step (store + decode in one call) on the GPU against the oracle's store
followed by the oracle's decode: bit-exact cache pools after the step, attention within
the usual tolerance."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from synth import WORKLOADS, make_decode_step
from synth.device import decode_to_device, i32
from tests.helpers import (assert_attention_close, assert_lse_close, assert_pool_equal,
                           oracle_after_store)

pytestmark = pytest.mark.gpu


def _step_inputs(step, t):
    """One new token per sequence: rows and slots of the real tokens, in sequence order."""
    real = np.nonzero(step.slot_mapping >= 0)[0] if step.num_tokens > step.batch else np.arange(step.batch)
    if step.num_tokens > step.batch:      # drop padding tokens that belong to no sequence
        sel = torch.as_tensor(real[:step.batch], device=t["q"].device)
        return t["k_new"][sel].contiguous(), t["v_new"][sel].contiguous(), t["slot_mapping"][sel].contiguous()
    return t["k_new"], t["v_new"], t["slot_mapping"]


def _run_and_check(step, dev, num_splits=0, seqs=None):
    t = decode_to_device(step, dev)
    k_new, v_new, slots = _step_inputs(step, t)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out, lse = nvpa.decode_step(t["q"], k_new, v_new, t["k_cache"], t["v_cache"], slots,
                                t["block_tables"], t["context_lens"], step.max_context_len,
                                step.scale, num_splits=num_splits, err_flag=err, return_lse=True)
    torch.cuda.synchronize()
    assert err.item() == 0
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    assert_pool_equal(t["k_cache"], kc, f"{step.name} k_cache after step")
    assert_pool_equal(t["v_cache"], vc, f"{step.name} v_cache after step")
    seqs = np.arange(step.batch) if seqs is None else np.asarray(seqs)
    ref, ref_lse = oracle.paged_decode_attention(step.q[seqs], kc, vc, step.block_tables[seqs],
                                                 step.context_lens[seqs], step.scale)
    sel = torch.as_tensor(seqs, device=dev)
    assert_attention_close(out[sel], ref, f"{step.name} decode_step")
    assert_lse_close(lse[sel], ref_lse, f"{step.name} decode_step")
    return t, out


@pytest.mark.parametrize("name,seqs", [
    ("decode_tiny_b4", None),
    ("decode_mid_b64", None),
    ("decode_b512_shared_prefix", None),
    ("decode_long_b8_ctx32k_bs16", None),
])
def test_decode_step_workloads(cuda_device, name, seqs):
    _run_and_check(WORKLOADS[name](), cuda_device, seqs=seqs)


@pytest.mark.parametrize("num_splits", [1, 3, 0])
@pytest.mark.parametrize("lens,hq,hkv,d,bs", [
    ([1, 16, 17, 300], 4, 2, 64, 16),
    ([256, 257, 1000, 5], 16, 8, 128, 256),
    ([33, 700], 6, 2, 128, 32),
])
def test_decode_step_small_shapes(cuda_device, lens, hq, hkv, d, bs, num_splits):
    step = make_decode_step(7 + len(lens), lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                            block_size=bs)
    _run_and_check(step, cuda_device, num_splits=num_splits)


def test_decode_step_padded_entries_are_not_stored(cuda_device):
    """A padded batch entry (context length 0, slot -1) stores nothing and outputs zeros."""
    step = make_decode_step(12, [40, 0, 90], num_q_heads=4, num_kv_heads=2, head_dim=64,
                            block_size=16)
    assert step.slot_mapping[1] == -1
    t, out = _run_and_check(step, cuda_device)
    assert torch.all(out[1] == 0)


def test_decode_step_bad_slot_is_flagged(cuda_device):
    step = make_decode_step(13, [40, 50], num_q_heads=4, num_kv_heads=2, head_dim=64,
                            block_size=16)
    t = decode_to_device(step, cuda_device)
    slots = t["slot_mapping"].clone()
    slots[0] = step.num_blocks * step.block_size + 3
    before = t["k_cache"].clone()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nvpa.decode_step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], slots,
                     t["block_tables"], t["context_lens"], step.max_context_len, step.scale,
                     err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_SLOT
    # sequence 1's row was written, nothing else changed
    changed = (t["k_cache"].view(torch.int16) != before.view(torch.int16)).view(
        step.num_blocks * step.block_size, -1).any(dim=1)
    assert changed.nonzero().flatten().tolist() == [int(step.slot_mapping[1])]


def test_decode_step_in_cuda_graph(cuda_device):
    step = make_decode_step(14, [100, 2000, 513, 7], num_q_heads=16, num_kv_heads=8, head_dim=128,
                            block_size=256)
    dev = cuda_device
    t = decode_to_device(step, dev)
    out = torch.empty_like(t["q"])
    ws = torch.empty(nvpa.paged_decode_workspace_size(step.batch, 16, 8, 128, step.max_context_len,
                                                      256), dtype=torch.uint8, device=dev)

    def fn():
        nvpa.decode_step(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                         t["slot_mapping"], t["block_tables"], t["context_lens"],
                         step.max_context_len, step.scale, out=out, workspace=ws)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize(dev)
    kc, vc, _ = oracle_after_store(step)
    ref, _ = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables, step.context_lens,
                                           step.scale)
    assert_attention_close(out, ref, "decode_step graph replay")
    del g
