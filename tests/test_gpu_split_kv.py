"""Split-KV decode across devices, emulated on one GPU: nvpa_paged_decode_partial over each
rank's share of the keys (shard_block_tables), then nvpa_lse_combine of the parts, against
the oracle's decode over the whole context.  (The ranks run one after another on the
one device; only the all-gather between them is left out, and that is covered by the gloo
test on CPU.)
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from paged_kv_cache_422_b200.split_kv import shard_block_tables
from synth import WORKLOADS, make_decode_step
from synth.device import decode_to_device, i32
from tests.helpers import assert_attention_close, assert_lse_close, oracle_after_store

pytestmark = pytest.mark.gpu


def _stored(step):
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    step.k_pool, step.v_pool = kc, vc
    return step


def _parts(step, t, world, dev, num_splits=0):
    o_parts, lse_parts = [], []
    for r in range(world):
        lbt, lctx, _ = shard_block_tables(step.block_tables, step.context_lens, step.block_size,
                                          world, r)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        o, lse = nvpa.paged_decode_partial(t["q"], t["k_cache"], t["v_cache"], i32(lbt, dev),
                                           i32(lctx, dev), step.max_context_len, step.scale,
                                           num_splits=num_splits, err_flag=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        o_parts.append(o)
        lse_parts.append(lse)
    return torch.stack(o_parts), torch.stack(lse_parts)


def test_partial_matches_oracle_on_its_keys(cuda_device):
    step = _stored(make_decode_step(3, [1, 40, 300, 1000, 0], num_q_heads=8, num_kv_heads=2,
                                    head_dim=128, block_size=32))
    t = decode_to_device(step, cuda_device)
    o, lse = nvpa.paged_decode_partial(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                       t["context_lens"], step.max_context_len, step.scale)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.paged_decode_attention(step.q, step.k_pool, step.v_pool,
                                                 step.block_tables, step.context_lens, step.scale)
    # fp32 output: well inside the bf16 tolerance
    assert np.max(np.abs(o.cpu().numpy() - ref)) < 2e-3
    assert torch.all(o[4] == 0)
    assert_lse_close(lse, ref_lse, "partial lse")


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("num_splits", [0, 3])
def test_split_kv_over_emulated_ranks(cuda_device, world, num_splits):
    step = _stored(make_decode_step(9 + world, [17, 256, 700, 2049, 5000, 3], num_q_heads=16,
                                    num_kv_heads=4, head_dim=128, block_size=64))
    t = decode_to_device(step, cuda_device)
    o_all, lse_all = _parts(step, t, world, cuda_device, num_splits)
    out, lse = nvpa.lse_combine(o_all, lse_all, return_lse=True)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.paged_decode_attention(step.q, step.k_pool, step.v_pool,
                                                 step.block_tables, step.context_lens, step.scale)
    assert_attention_close(out, ref, f"split-KV over {world} ranks")
    assert_lse_close(lse, ref_lse, f"split-KV over {world} ranks")


def test_split_kv_long_context_workload(cuda_device):
    """The long-context workload (8 x 32768 keys, block size 16) over 2 emulated ranks,
    checked on two sequences."""
    step = _stored(WORKLOADS["decode_long_b8_ctx32k_bs16"]())
    t = decode_to_device(step, cuda_device)
    o_all, lse_all = _parts(step, t, 2, cuda_device)
    out = nvpa.lse_combine(o_all, lse_all)
    torch.cuda.synchronize()
    seqs = [0, 5]
    ref, _ = oracle.paged_decode_attention(step.q[seqs], step.k_pool, step.v_pool,
                                           step.block_tables[seqs], step.context_lens[seqs],
                                           step.scale)
    assert_attention_close(out[seqs], ref, "long-context split-KV")


def test_partial_fp32_output_at_batch_512(cuda_device):
    """The partial entry point (fp32 output and lse) on the batch-512 workload: 8192 rows of
    several partitions each, more than the combine's CTAs cover in one wave; sampled
    sequences against the oracle."""
    step = _stored(WORKLOADS["decode_b512_shared_prefix"]())
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    o, lse = nvpa.paged_decode_partial(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                       t["context_lens"], step.max_context_len, step.scale,
                                       err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    seqs = list(range(0, 512, 29)) + [int(np.argmax(step.context_lens))]
    ref, ref_lse = oracle.paged_decode_attention(step.q[seqs], step.k_pool, step.v_pool,
                                                 step.block_tables[seqs], step.context_lens[seqs],
                                                 step.scale)
    sel = torch.as_tensor(seqs, device=cuda_device)
    assert np.max(np.abs(o[sel].cpu().numpy() - ref)) < 2e-3
    assert_lse_close(lse[sel], ref_lse, "batch-512 partial lse")


def test_lse_combine_weights_and_empty_rows(cuda_device):
    """Closed forms: equal lse -> plain mean of the parts; a -inf part weighs nothing; a
    row of -inf parts gives 0 and -inf."""
    dev = cuda_device
    R, B, H, D = 3, 2, 4, 64
    g = torch.Generator().manual_seed(0)
    o = torch.randn((R, B, H, D), generator=g).to(dev)
    lse = torch.zeros((R, B, H), device=dev)
    lse[1, 1] = float("-inf")
    lse[:, 0, 3] = float("-inf")
    out, lo = nvpa.lse_combine(o.contiguous(), lse.contiguous(), return_lse=True)
    torch.cuda.synchronize()
    o64 = o.double().cpu()
    exp = o64.mean(0)
    exp[1] = (o64[0, 1] + o64[2, 1]) / 2
    exp[0, 3] = 0
    got = out.double().cpu()
    assert torch.allclose(got, exp, atol=1e-2, rtol=1e-2)
    assert torch.isneginf(lo[0, 3]).item()
    assert abs(lo[0, 0].item() - np.log(3)) < 1e-5
    assert abs(lo[1, 0].item() - np.log(2)) < 1e-5
