"""Decode captured in CUDA graphs and replayed with new inputs (Nano-vLLM part 1, section
5.3: decode graphs are captured ahead of time for batch sizes 1, 2, 4, 8, 16 ... 512).

The library's launch configuration depends only on host-side arguments (batch, bounds,
split count), never on the device-side lengths, and it allocates nothing, so one
capture serves every replay whose inputs are rewritten in place."""

import os

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from synth import make_decode_step
from synth.device import bf16_tensor, i32, pool_to_device
from tests.helpers import assert_attention_close, oracle_after_store

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "cuda_graph_batch_sizes.txt")


def _graph_batch_sizes():
    first, last = [], None
    for line in open(GOLDEN):
        if line.startswith("first"):
            first = [int(x) for x in line.split()[1:]]
        elif line.startswith("last"):
            last = int(line.split()[1])
    return first + list(range(first[-1] + 16, last + 1, 16))


def test_golden_ladder_reading():
    sizes = _graph_batch_sizes()
    assert sizes[:5] == [1, 2, 4, 8, 16] and sizes[-1] == 512 and sizes[5] == 32


@pytest.mark.parametrize("batch", [1, 2, 8, 16, 48, 512])
def test_decode_graph_replay_with_new_inputs(cuda_device, batch):
    assert batch in _graph_batch_sizes()
    hq, hkv, d, bs, max_ctx = 16, 8, 128, 256, 2048
    rng = np.random.default_rng(batch)
    # two steps with different lengths but the same shapes: capture on the first, replay
    # on the second after rewriting the device inputs in place
    steps = []
    for k in range(2):
        lens = rng.integers(1, max_ctx + 1, size=batch)
        steps.append(make_decode_step(1000 * batch + k, lens, num_q_heads=hq, num_kv_heads=hkv,
                                      head_dim=d, block_size=bs,
                                      num_blocks=batch * (max_ctx // bs) + 4))
    maxblk = max_ctx // bs
    dev = cuda_device

    def padded_bt(step):
        bt = np.full((batch, maxblk), -1, np.int32)
        bt[:, :step.block_tables.shape[1]] = step.block_tables
        return bt

    s0 = steps[0]
    kc = pool_to_device(s0.k_pool, dev)
    vc = pool_to_device(s0.v_pool, dev)
    q = bf16_tensor(s0.q, dev)
    k_new = bf16_tensor(s0.k_new, dev)
    v_new = bf16_tensor(s0.v_new, dev)
    slots = i32(s0.slot_mapping, dev)
    bt = i32(padded_bt(s0), dev)
    ctx = i32(s0.context_lens, dev)
    out = torch.empty_like(q)
    ws = torch.empty(nvpa.paged_decode_workspace_size(batch, hq, hkv, d, max_ctx, bs),
                     dtype=torch.uint8, device=dev)

    def step_fn():
        nvpa.store_kvcache(k_new, v_new, kc, vc, slots)
        nvpa.paged_decode_attention(q, kc, vc, bt, ctx, max_ctx, s0.scale, out=out, workspace=ws)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step_fn()                     # warm-up outside the capture (one-time set-up)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step_fn()

    for step in steps:
        # rewrite every input in place (pools, tokens, slots, tables, lengths)
        kc.copy_(pool_to_device(step.k_pool, dev))
        vc.copy_(pool_to_device(step.v_pool, dev))
        q.copy_(bf16_tensor(step.q, dev))
        k_new.copy_(bf16_tensor(step.k_new, dev))
        v_new.copy_(bf16_tensor(step.v_new, dev))
        slots.copy_(i32(step.slot_mapping, dev))
        bt.copy_(i32(padded_bt(step), dev))
        ctx.copy_(i32(step.context_lens, dev))
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize(dev)
        kco, vco, _ = oracle_after_store(step)
        sample = np.arange(batch) if batch <= 16 else np.linspace(0, batch - 1, 16).astype(int)
        ref, _ = oracle.paged_decode_attention(step.q[sample], kco, vco, step.block_tables[sample],
                                               step.context_lens[sample], step.scale)
        assert_attention_close(out[torch.as_tensor(sample, device=dev)], ref,
                               f"graph replay batch {batch}")
    del g
