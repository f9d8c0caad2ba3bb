"""Split-KV decode across ranks, host side (no GPU): the key sharding, and the exchange
and merge run by two gloo ranks with the oracle standing in for the kernels.

The merged result must equal the oracle's decode over the whole context: the sharding
must hand every key to exactly one rank, in order, and the exchange must keep the parts
of each rank together.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from paged_kv_cache_422_b200.split_kv import shard_block_tables


def _keys_of(bt_row, ctx, bs):
    return [int(bt_row[j // bs]) * bs + j % bs for j in range(ctx)]


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_sharding_hands_every_key_to_one_rank_in_order(world):
    rng = np.random.default_rng(world)
    bs = 16
    ctx = np.array([0, 1, 15, 16, 17, 100, 333, 1000], np.int64)
    nb = -(-ctx // bs)
    bt = np.full((len(ctx), int(nb.max())), -1, np.int32)
    perm = rng.permutation(int(nb.sum()) + 5)
    c = 0
    for b, n in enumerate(nb):
        bt[b, :n] = perm[c:c + n]
        c += n
    shards = [shard_block_tables(bt, ctx, bs, world, r) for r in range(world)]
    for b in range(len(ctx)):
        keys = []
        for r in range(world):
            lbt, lctx, first = shards[r]
            assert first[b] == len(keys)
            assert first[b] % bs == 0                     # runs of whole blocks
            keys += _keys_of(lbt[b], int(lctx[b]), bs)
            assert np.all(lbt[b, -(-int(lctx[b]) // bs):] == -1)   # padding past the run
        assert keys == _keys_of(bt[b], int(ctx[b]), bs)


def test_sharding_rejects_bad_rank():
    with pytest.raises(ValueError):
        shard_block_tables(np.zeros((1, 1), np.int32), [5], 16, 2, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    import oracle
    from paged_kv_cache_422_b200.split_kv import split_kv_decode
    from synth import make_decode_step

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        step = make_decode_step(5, [3, 40, 129, 300, 16], num_q_heads=4, num_kv_heads=2,
                                head_dim=64, block_size=16)
        kc, vc = step.k_pool.copy(), step.v_pool.copy()
        oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
        lbt, lctx, _ = shard_block_tables(step.block_tables, step.context_lens, step.block_size,
                                          world, rank)

        def partial_fn(q, k_cache, v_cache, bt, ctx, max_ctx, scale):
            o, lse = oracle.paged_decode_attention(q, k_cache, v_cache, bt, ctx, scale)
            return torch.from_numpy(o.astype(np.float32)), torch.from_numpy(lse.astype(np.float32))

        def combine_fn(o_all, lse_all):
            R, B, H, D = o_all.shape
            out = np.zeros((B, H, D))
            lse = np.zeros((B, H))
            for b in range(B):
                for h in range(H):
                    out[b, h], lse[b, h] = oracle.lse_combine(o_all[:, b, h].numpy(),
                                                              lse_all[:, b, h].numpy())
            return out, lse

        out, lse = split_kv_decode(step.q, kc, vc, lbt, lctx, step.max_context_len, step.scale,
                                   partial_fn=partial_fn, combine_fn=combine_fn, return_lse=True)
        ref, ref_lse = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables,
                                                     step.context_lens, step.scale)
        results[rank] = (float(np.max(np.abs(out - ref))),
                         float(np.max(np.abs(np.nan_to_num(lse - ref_lse)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_split_kv_exchange_gloo(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert len(results) == world
    for r in range(world):
        err_out, err_lse = results[r]
        assert err_out < 1e-5 and err_lse < 1e-5, (r, err_out, err_lse)
