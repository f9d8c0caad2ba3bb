"""nvpa_decode_step_shared_prefix on the GPU against the oracle.

Prefix caching ("Nano-vLLM part 1" section 4.2) maps the cached prompt of many sequences
to the same physical blocks.  The shared-prefix decode attends such a prefix once per
group of sequences on the tensor cores and the rest of each context on the worker; the
result must be the oracle's paged decode attention, whatever the grouping.  The plan's
counters (groups, members, prefix tiles) are checked too, so that a test cannot pass on
a silent fall-back to the ungrouped schedule.
"""

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


def _share(step, donor, members, nblocks):
    """Point the first nblocks table entries of `members` at the donor's blocks (the
    blocks stay wholly before every member's newest token and hold live rows)."""
    bs = step.block_size
    assert (int(step.context_lens[donor]) - 1) // bs >= nblocks
    for m in members:
        assert (int(step.context_lens[m]) - 1) // bs >= nblocks, m
        step.block_tables[m, :nblocks] = step.block_tables[donor, :nblocks]
    return step


def _prefix_chunk(batch, hkv, max_ctx, block_size):
    """Prefix keys per partition of the shared-prefix step with automatic partitioning: the
    decode partition (the header's rule for num_splits = 0), rounded up to 128."""
    target = 148 * 3 * 4                      # resident worker warps of a 148-SM B200
    per = max(1, batch) * max(1, hkv)
    ctx = max(1, max_ctx)
    r16 = lambda k: -(-k // 16) * 16          # noqa: E731
    fill = r16(-(-ctx // -(-target // per)))  # one item per warp
    if fill < 256:
        chunk = max(64, fill)
    elif per * 8 > target:
        chunk = 352
    else:                                     # about two rounds of items, <= 32 blocks
        cap = min(1024, max(128, 32 * block_size))
        chunk = min(cap, max(128, r16(-(-ctx // -(-2 * target // per)))))
    return -(-chunk // 128) * 128


def _counters(ws):
    return ws[:20].view(torch.int32).cpu().tolist()[2:5]


def _run(step, dev, store=True, num_splits=0, min_group=0, seqs=None):
    t = decode_to_device(step, dev)
    ws = torch.empty(nvpa.decode_shared_prefix_workspace_size(
        step.batch, step.num_q_heads, step.num_kv_heads, step.head_dim, step.max_context_len,
        step.block_size, num_splits, min_group), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    if store and step.num_tokens > step.batch:
        # a padded token list (slot -1 entries beyond the batch): the step takes one new
        # row per sequence, the rows of the real tokens in sequence order
        real = np.nonzero(step.slot_mapping >= 0)[0][:step.batch]
        assert len(real) == step.batch
        sel = torch.as_tensor(real, device=dev)
        kn, vn, sm = (t[k][sel].contiguous() for k in ("k_new", "v_new", "slot_mapping"))
    elif store:
        assert step.num_tokens == step.batch
        kn, vn, sm = t["k_new"], t["v_new"], t["slot_mapping"]
    else:
        kn = vn = sm = None
    out, lse = nvpa.decode_step_shared_prefix(
        t["q"], kn, vn, t["k_cache"], t["v_cache"], sm, t["block_tables"], t["context_lens"],
        step.max_context_len, step.scale, workspace=ws, num_splits=num_splits,
        min_group_size=min_group, err_flag=err, return_lse=True)
    torch.cuda.synchronize()
    assert err.item() == 0
    if store:
        kc, vc, bad = oracle_after_store(step)
        assert bad == []
        assert_pool_equal(t["k_cache"], kc, f"{step.name} k_cache after step")
        assert_pool_equal(t["v_cache"], vc, f"{step.name} v_cache after step")
    else:
        kc, vc = step.k_pool, step.v_pool   # the step's rows are in the pools already
    seqs = np.arange(step.batch) if seqs is None else np.asarray(seqs)
    ref, ref_lse = oracle.paged_decode_attention(step.q[seqs], kc, vc, step.block_tables[seqs],
                                                 step.context_lens[seqs], step.scale)
    sel = torch.as_tensor(seqs, device=dev)
    assert_attention_close(out[sel], ref, f"{step.name} shared-prefix step")
    assert_lse_close(lse[sel], ref_lse, f"{step.name} shared-prefix step")
    return _counters(ws), t, out


def _stored(step):
    """The step with its new rows already in the pools (for attention-only calls)."""
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    step.k_pool, step.v_pool = kc, vc
    return step


def test_batch512_shared_prefix_workload(cuda_device):
    """The benchmarked step, as bench.py calls it: all 512 sequences against the oracle,
    both pools bit-exact after the step."""
    step = WORKLOADS["decode_b512_shared_prefix"]()
    shared = np.all(step.block_tables[:, :4] == step.shared_blocks[None, :4], axis=1)
    (groups, members, tiles), _, _ = _run(step, cuda_device)
    assert groups == 1
    assert members == int(shared.sum())
    # 1024 prefix keys in partitions of pchunk; 64 members per query tile (2 query heads
    # each), query tiles in pairs
    pchunk = _prefix_chunk(step.batch, step.num_kv_heads, step.max_context_len, step.block_size)
    assert tiles == -(-1024 // pchunk) * (((members + 63) // 64 + 1) // 2)


@pytest.mark.parametrize("name", ["decode_tiny_b4", "decode_mid_b64", "decode_long_b8_ctx32k_bs16"])
def test_shared_prefix_api_on_the_other_decode_workloads(cuda_device, name):
    """bench.py times every decode workload through this entry point: the workloads
    without shared blocks (no group forms, every key goes to the worker), every sequence
    against the oracle and both pools bit-exact."""
    step = WORKLOADS[name]()
    (groups, members, tiles), _, _ = _run(step, cuda_device)
    assert (groups, members, tiles) == (0, 0, 0)


@pytest.mark.parametrize("store", [True, False])
@pytest.mark.parametrize("lens,hq,hkv,d,bs,nshared,nblk", [
    # 12 of 20 share 3 blocks of 16 (48 keys: a ragged key tile); group 2
    ([60 + 7 * i for i in range(20)], 4, 2, 64, 16, 12, 3),
    # 70 members: two query tiles of 64; prefix of 512 keys in two partitions
    ([513 + 37 * i for i in range(80)], 16, 8, 128, 256, 70, 2),
    # group of 3 query heads (not a power of two: one head per tile row)
    ([100 + 3 * i for i in range(24)], 6, 2, 128, 32, 20, 3),
    # group 8: 16 members per tile; 320 prefix keys (partitions of 128, the last one 64)
    ([330 + 11 * i for i in range(40)], 32, 4, 128, 16, 40, 20),
])
def test_shared_prefix_shapes(cuda_device, lens, hq, hkv, d, bs, nshared, nblk, store):
    share = np.zeros(len(lens), bool)
    share[np.random.default_rng(5).permutation(len(lens))[:nshared]] = True
    step = make_decode_step(21 + len(lens), lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                            block_size=bs, shared_prefix_blocks=nblk, share=share)
    if not store:
        step = _stored(step)
    (groups, members, tiles), _, _ = _run(step, cuda_device, store=store, min_group=4)
    assert (groups, members) == (1, nshared)
    tq = 128 // (hq // hkv if (hq // hkv) & (hq // hkv - 1) == 0 else 1)
    pchunk = _prefix_chunk(step.batch, hkv, step.max_context_len, step.block_size)
    assert tiles == -(-nblk * bs // pchunk) * ((-(-nshared // tq) + 1) // 2)   # query-tile pairs


def test_prefix_partitions_of_two_key_tiles(cuda_device):
    """16 contexts up to 4096 keys with 8 KV heads get 160-key decode partitions, so the
    prefix partitions are 256 keys: every prefix tile unit runs two key tiles, one in each
    of the kernel's two S buffers, before its epilogue."""
    lens = [4096 - 37 * i for i in range(16)]
    share = np.array([i % 4 != 3 for i in range(16)])
    step = make_decode_step(33, lens, num_q_heads=16, num_kv_heads=8, head_dim=128,
                            block_size=64, shared_prefix_blocks=8, share=share)
    pchunk = _prefix_chunk(step.batch, 8, step.max_context_len, step.block_size)
    assert pchunk == 256
    (groups, members, tiles), _, _ = _run(step, cuda_device, min_group=4)
    assert (groups, members) == (1, 12)
    # 512 prefix keys in two partitions, 12 members in one query tile (a pair of one)
    assert tiles == 2


def test_prefix_units_beyond_three_per_sm(cuda_device):
    """512 sequences that all share a 3072-token prefix: 8 query tiles of 64 members, 8
    prefix partitions of 384 keys and 8 head groups make 512 single-tile units, more than
    three for each CTA of the one-per-SM prefix grid, so every CTA takes units (at batch
    512 with a 1024-token prefix only the first 32 do and the worker streams on the other
    SMs).  Both pools bit-exact; 47 sampled sequences against the oracle."""
    lens = [3073 + (7 * i) % 227 for i in range(512)]
    step = make_decode_step(35, lens, num_q_heads=16, num_kv_heads=8, head_dim=128,
                            block_size=256, num_blocks=600, shared_prefix_blocks=12,
                            share=np.ones(512, bool))
    pchunk = _prefix_chunk(step.batch, 8, step.max_context_len, step.block_size)
    assert pchunk == 384
    (groups, members, tiles), _, _ = _run(step, cuda_device, seqs=list(range(0, 512, 11)))
    assert (groups, members) == (1, 512)
    assert tiles == (3072 // pchunk) * (512 // 64 // 2)
    assert tiles * 8 * 2 > 3 * 148


def test_two_groups_and_a_short_common_run(cuda_device):
    """Two groups with different donors; one member of the second group shares only two
    of the donor's four blocks, so that group's prefix is two blocks."""
    lens = [200 + 13 * i for i in range(30)]
    step = make_decode_step(31, lens, num_q_heads=8, num_kv_heads=2, head_dim=128,
                            block_size=32)
    _share(step, 0, range(1, 10), 5)
    _share(step, 10, range(11, 20), 4)
    step.block_tables[19, 2:4] = step.block_tables[20, 2:4]   # 19: common run of 2
    (groups, members, tiles), _, _ = _run(step, cuda_device, min_group=4)
    assert (groups, members) == (2, 20)
    # one query tile (pair) per group; prefixes of 160 and 64 keys in partitions of pchunk
    pchunk = _prefix_chunk(step.batch, 2, step.max_context_len, step.block_size)
    assert tiles == -(-160 // pchunk) + -(-64 // pchunk)


def test_member_whose_private_part_is_its_new_token(cuda_device):
    """context = prefix + 1: the private partition holds only the token stored now."""
    bs = 16
    lens = [4 * bs + 1] * 6 + [4 * bs + 40] * 6 + [30, 77]
    share = np.array([True] * 12 + [False] * 2)
    step = make_decode_step(41, lens, num_q_heads=4, num_kv_heads=1, head_dim=64, block_size=bs,
                            shared_prefix_blocks=4, share=share)
    (groups, members, _), _, _ = _run(step, cuda_device, min_group=4)
    assert (groups, members) == (1, 12)


def test_small_buckets_are_not_groups(cuda_device):
    lens = [90 + i for i in range(12)]
    share = np.array([True] * 5 + [False] * 7)
    step = make_decode_step(51, lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                            shared_prefix_blocks=2, share=share)
    (groups, members, tiles), _, _ = _run(step, cuda_device, min_group=6)
    assert (groups, members, tiles) == (0, 0, 0)
    (groups, members, _), _, _ = _run(step, cuda_device, min_group=5)
    assert (groups, members) == (1, 5)


def test_batch_below_the_smallest_group_runs_as_a_plain_step(cuda_device):
    """A batch of 5 that all share a prefix, with groups of at least 6: no group can form,
    so the call runs as the plain decode step (no plan table, no prefix launch) and its
    workspace is the plain step's size."""
    lens = [90 + 7 * i for i in range(5)]
    step = make_decode_step(53, lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                            shared_prefix_blocks=3, share=np.ones(5, bool))
    args = (step.batch, step.num_q_heads, step.num_kv_heads, step.head_dim, step.max_context_len,
            step.block_size, 0)
    assert nvpa.decode_shared_prefix_workspace_size(*args, 6) == nvpa.paged_decode_workspace_size(*args)
    (groups, members, tiles), _, _ = _run(step, cuda_device, min_group=6)
    assert (groups, members, tiles) == (0, 0, 0)
    (groups, members, _), _, _ = _run(step, cuda_device, min_group=5)
    assert (groups, members) == (1, 5)


@pytest.mark.parametrize("num_splits", [1, 2, 7])
def test_shared_prefix_with_explicit_splits(cuda_device, num_splits):
    lens = [700 + 29 * i for i in range(24)]
    share = np.array([i % 3 != 0 for i in range(24)])
    step = make_decode_step(61, lens, num_q_heads=16, num_kv_heads=8, head_dim=128,
                            block_size=64, shared_prefix_blocks=9, share=share)
    (groups, members, _), _, _ = _run(step, cuda_device, num_splits=num_splits, min_group=4)
    assert (groups, members) == (1, int(share.sum()))


def test_batch_above_plan_table_runs_ungrouped(cuda_device):
    lens = [20 + (i % 13) for i in range(2100)]
    share = np.array([i % 2 == 0 for i in range(2100)])
    step = make_decode_step(71, lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                            shared_prefix_blocks=1, share=share)
    (groups, members, tiles), _, _ = _run(step, cuda_device, seqs=list(range(0, 2100, 97)))
    assert (groups, members, tiles) == (0, 0, 0)


def test_padded_entries_and_bad_slot(cuda_device):
    bs = 16
    lens = [50] * 10 + [0, 33]
    share = np.array([True] * 10 + [False] * 2)
    step = make_decode_step(81, lens, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=bs,
                            shared_prefix_blocks=3, share=share)
    assert step.slot_mapping[10] == -1
    (groups, _, _), t, out = _run(step, cuda_device, min_group=4)
    assert groups == 1
    assert torch.all(out[10] == 0)
    # a bad slot is flagged and not written; the attention still runs
    t = decode_to_device(step, cuda_device)
    slots = t["slot_mapping"].clone()
    slots[3] = step.num_blocks * bs + 5
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nvpa.decode_step_shared_prefix(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
                                   slots, t["block_tables"], t["context_lens"],
                                   step.max_context_len, step.scale, min_group_size=4,
                                   err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & nvpa.NVPA_FLAG_BAD_SLOT


def test_shared_prefix_in_cuda_graph(cuda_device):
    lens = [600 + 41 * i for i in range(48)]
    share = np.array([i % 4 != 1 for i in range(48)])
    step = make_decode_step(91, lens, num_q_heads=16, num_kv_heads=8, head_dim=128,
                            block_size=256, shared_prefix_blocks=2, share=share)
    dev = cuda_device
    t = decode_to_device(step, dev)
    out = torch.empty_like(t["q"])
    ws = torch.empty(nvpa.decode_shared_prefix_workspace_size(48, 16, 8, 128, step.max_context_len,
                                                              256), dtype=torch.uint8, device=dev)

    def fn():
        nvpa.decode_step_shared_prefix(t["q"], t["k_new"], t["v_new"], t["k_cache"], t["v_cache"],
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
    assert _counters(ws)[:2] == [1, int(share.sum())]
    kc, vc, _ = oracle_after_store(step)
    ref, _ = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables, step.context_lens,
                                           step.scale)
    assert_attention_close(out, ref, "shared-prefix graph replay")
    del g
