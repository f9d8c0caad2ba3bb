"""Paged decode attention on the GPU against the float64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from synth import WORKLOADS, make_decode_step
from synth.device import decode_to_device
from tests.helpers import assert_attention_close, assert_lse_close, oracle_after_store

pytestmark = pytest.mark.gpu

_HOST_CACHE = {}


def _workload(name):
    if name not in _HOST_CACHE:
        _HOST_CACHE.clear()
        step = WORKLOADS[name]()
        kc, vc, _ = oracle_after_store(step)
        _HOST_CACHE[name] = (step, kc, vc)
    return _HOST_CACHE[name]


def _run(step, t, num_splits=0, max_context_len=None, err=None):
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                       err_flag=err)
    mcl = step.max_context_len if max_context_len is None else max_context_len
    out, lse = nvpa.paged_decode_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                           t["context_lens"], mcl, step.scale,
                                           num_splits=num_splits, err_flag=err, return_lse=True)
    torch.cuda.synchronize()
    return out, lse


def _check(step, kc, vc, out, lse, seqs, what):
    seqs = np.asarray(seqs)
    ora_out, ora_lse = oracle.paged_decode_attention(step.q[seqs], kc, vc, step.block_tables[seqs],
                                                     step.context_lens[seqs], step.scale)
    assert_attention_close(out[torch.as_tensor(seqs, device=out.device)], ora_out, what)
    assert_lse_close(lse[torch.as_tensor(seqs, device=lse.device)], ora_lse, what)


def test_decode_tiny(cuda_device):
    step, kc, vc = _workload("decode_tiny_b4")
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = _run(step, t, err=err)
    assert err.item() == 0
    _check(step, kc, vc, out, lse, range(step.batch), "decode_tiny_b4")


def test_decode_mid_all_sequences(cuda_device):
    step, kc, vc = _workload("decode_mid_b64")
    t = decode_to_device(step, cuda_device)
    out, lse = _run(step, t)
    _check(step, kc, vc, out, lse, range(step.batch), "decode_mid_b64")


@pytest.mark.parametrize("num_splits", [1, 2, 7, 0, 256])
def test_decode_split_count_does_not_change_result(cuda_device, num_splits):
    step, kc, vc = _workload("decode_mid_b64")
    t = decode_to_device(step, cuda_device)
    out, lse = _run(step, t, num_splits=num_splits)
    _check(step, kc, vc, out, lse, list(range(0, 64, 5)), f"num_splits={num_splits}")


def test_decode_b512_shared_prefix_sampled(cuda_device):
    step, kc, vc = _workload("decode_b512_shared_prefix")
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = _run(step, t, err=err)
    assert err.item() == 0
    ctx = step.context_lens
    shared = np.any(np.isin(step.block_tables, step.shared_blocks), axis=1)
    picks = set(np.argsort(ctx)[:8]) | set(np.argsort(ctx)[-8:])
    picks |= set(np.nonzero(shared)[0][:12]) | set(np.nonzero(~shared)[0][:12])
    picks |= set(range(0, 512, 37))
    _check(step, kc, vc, out, lse, sorted(picks), "decode_b512_shared_prefix")
    assert torch.isfinite(out.float()).all()
    # sequences sharing the prefix read the same 4 physical blocks
    assert len(step.shared_blocks) == 4 and shared.sum() == 256


def test_decode_many_rows_head_dim_64(cuda_device):
    """1600 sequences x 4 query heads (6400 rows, head_dim 64) with 700-900 keys each: every
    row has two or three 352-key partitions, more rows than the combine's CTAs cover in one
    wave of residents (one warp per row)."""
    lens = [700 + (37 * i) % 201 for i in range(1600)]
    step = make_decode_step(17, lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16)
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = _run(step, t, err=err)
    assert err.item() == 0
    _check(step, kc, vc, out, lse, list(range(0, 1600, 53)) + [1599], "1600 x 4 rows, head_dim 64")


def test_decode_long_context_block16(cuda_device):
    step, kc, vc = _workload("decode_long_b8_ctx32k_bs16")
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = _run(step, t, err=err)
    assert err.item() == 0
    _check(step, kc, vc, out, lse, range(step.batch), "decode_long_b8_ctx32k_bs16")


CASES = [
    # (context lens, Hq, Hkv, D, block size)
    ([1, 2, 15, 16, 17], 4, 4, 64, 16),
    ([0, 1, 300, 33], 8, 4, 64, 32),
    ([64, 65, 127, 128, 129], 6, 2, 128, 64),
    ([1000, 5, 257], 8, 1, 128, 128),
    ([511, 512, 513, 1], 16, 2, 128, 256),
    ([77, 300], 5, 1, 64, 16),
    ([2000, 31], 24, 8, 128, 16),
]


@pytest.mark.parametrize("lens,hq,hkv,d,bs", CASES)
def test_decode_small_shapes(cuda_device, lens, hq, hkv, d, bs):
    step = make_decode_step(sum(lens) + hq, lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                            block_size=bs, pad_positions=(1,))
    t = decode_to_device(step, cuda_device)
    kc, vc, _ = oracle_after_store(step)
    for ns in (0, 1, 3):
        out, lse = _run(step, t, num_splits=ns)
        _check(step, kc, vc, out, lse, range(step.batch), f"{lens} splits={ns}")
    zero = np.nonzero(step.context_lens == 0)[0]
    for b in zero:
        assert torch.all(out[b] == 0) and torch.all(torch.isneginf(lse[b]))


def test_decode_shared_blocks_equal_duplicated_blocks(cuda_device):
    share = np.array([True, True, False, True])
    step = make_decode_step(31, [700, 600, 90, 1025], num_q_heads=8, num_kv_heads=4,
                            head_dim=128, block_size=128, shared_prefix_blocks=4, share=share,
                            num_blocks=64)
    t = decode_to_device(step, cuda_device)
    out, _ = _run(step, t)
    bt = step.block_tables.copy()
    used = set(int(x) for x in bt.ravel() if x >= 0)
    free = [i for i in range(step.num_blocks) if i not in used]
    kcache, vcache = t["k_cache"], t["v_cache"]
    for b in np.nonzero(share)[0]:
        for j in range(4):
            new = free.pop()
            kcache[new] = kcache[int(bt[b, j])]
            vcache[new] = vcache[int(bt[b, j])]
            bt[b, j] = new
    t["block_tables"] = torch.as_tensor(bt, device=cuda_device)
    out2 = nvpa.paged_decode_attention(t["q"], kcache, vcache, t["block_tables"],
                                       t["context_lens"], step.max_context_len, step.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_decode_invariant_under_block_relabelling(cuda_device):
    step = make_decode_step(32, [300, 41, 900], num_q_heads=8, num_kv_heads=2, head_dim=128,
                            block_size=32, num_blocks=80)
    t = decode_to_device(step, cuda_device)
    out, _ = _run(step, t)
    perm = torch.as_tensor(np.random.default_rng(1).permutation(step.num_blocks),
                           device=cuda_device)
    k2 = torch.empty_like(t["k_cache"])
    v2 = torch.empty_like(t["v_cache"])
    k2[perm] = t["k_cache"]
    v2[perm] = t["v_cache"]
    bt = t["block_tables"].long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).to(torch.int32)
    out2 = nvpa.paged_decode_attention(t["q"], k2, v2, bt2, t["context_lens"],
                                       step.max_context_len, step.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_decode_constant_values_give_the_value(cuda_device):
    step = make_decode_step(33, [5, 400, 1], num_q_heads=4, num_kv_heads=2, head_dim=64,
                            block_size=16, q_mult=4.0)
    t = decode_to_device(step, cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    row = torch.linspace(-3, 3, 64, device=cuda_device).to(torch.bfloat16)
    t["v_cache"][:] = row
    out = nvpa.paged_decode_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                      t["context_lens"], step.max_context_len, step.scale)
    torch.cuda.synchronize()
    ref = row.double().cpu().numpy()
    assert_attention_close(out, np.broadcast_to(ref, out.shape), "constant V")
