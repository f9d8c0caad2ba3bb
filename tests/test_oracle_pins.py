"""Pins for the CPU oracle: every check here fixes the oracle to something other than itself.

What each pin guards against (a plausible slip in the oracle that would fail it):
  * worked example (Nano-vLLM part 1, section 4.1): off-by-one block counts or rows;
  * brute force against torch's float64 scaled_dot_product_attention on contiguous
    K/V: a wrong GQA mapping, a dropped or doubled scale, a wrong block/row index, a
    transposed operand, a wrong causal alignment;
  * relabelling physical blocks: reading the logical instead of the physical block id;
  * shared vs duplicated prefix blocks (section 4.2, refcounted reuse);
  * closed forms: weights sum to one, constant V, one key, zero query;
  * log-sum-exp split identity: the merge formula used to check split-KV decode;
  * decode = last row of causal prefill; prefix-cached prefill = tail of full prefill.
"""

import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

import oracle
from synth import (POISON_BF16, bf16_bits_from_f32, decode_tiny, make_decode_step,
                   make_prefill_step)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = [int(x) for x in v] if len(v) > 1 else int(v[0])
    return vals


def _bf16(x):
    return bf16_bits_from_f32(np.asarray(x, np.float32))


def _f64(bits):
    # Independent of the oracle's decoder: torch's own bf16 -> float64 conversion.
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def _scatter_contiguous(seqs, block_size, num_blocks, rng):
    """Put contiguous per-sequence rows into a paged pool under random block tables.

    Written with numpy fancy indexing (not the oracle's loops): pool[bt[p // bs], p % bs].
    """
    Hkv, D = seqs[0].shape[1:]
    pool = np.full((num_blocks, block_size, Hkv, D), POISON_BF16, np.uint16)
    perm = rng.permutation(num_blocks)
    width = max(1, max(-(-len(s) // block_size) for s in seqs))
    bt = np.full((len(seqs), width), -1, np.int32)
    cur = 0
    for b, s in enumerate(seqs):
        n = -(-len(s) // block_size)
        bt[b, :n] = perm[cur:cur + n]
        cur += n
        pos = np.arange(len(s))
        pool[bt[b, pos // block_size], pos % block_size] = s
    return pool, bt


def _sdpa(q, k, v, scale, mask=None, is_causal=False):
    """torch CPU float64 attention; q [Hq, Lq, D], k/v [Hkv, Lk, D] expanded to Hq heads."""
    g = q.shape[0] // k.shape[0]
    k = torch.as_tensor(k).repeat_interleave(g, dim=0)
    v = torch.as_tensor(v).repeat_interleave(g, dim=0)
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.as_tensor(q), k, v, attn_mask=None if mask is None else torch.as_tensor(mask),
        is_causal=is_causal, scale=scale)
    return out.numpy()


# ----------------------------------------------------------------------------------
# bf16 decoding
# ----------------------------------------------------------------------------------

def test_bf16_decode_matches_torch_on_every_pattern():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(bits)
    ref = _f64(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


# ----------------------------------------------------------------------------------
# worked example and block arithmetic (section 4.1)
# ----------------------------------------------------------------------------------

def test_worked_example_700_tokens():
    g = _read_golden("block_split_700.txt")
    nblk, last, idle = oracle.blocks_for_tokens(g["tokens"], g["block_size"])
    assert nblk == g["blocks"]
    assert nblk - 1 == g["full_blocks"]
    assert last == g["tokens_in_last_block"]
    assert idle == g["idle_slots_in_last_block"]
    assert (nblk - 1) * g["tokens_in_full_block"] + last == g["tokens"]


def test_worked_example_in_tiny_decode_workload():
    """The 700-token sequence of the tiny workload: three blocks, the newest token lands
    on row 187 of the third block, rows 188.. of that block are never read."""
    step = decode_tiny()
    b = 3
    assert step.context_lens[b] == 700
    bs = step.block_size
    kc = step.k_pool.copy()
    vc = step.v_pool.copy()
    bad = oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    assert bad == []
    third = int(step.block_tables[b, 2])
    assert np.array_equal(kc[third][187], step.k_new[b])
    assert np.all(kc[third][188:] == POISON_BF16)     # idle rows untouched
    rows = oracle.gather_kv(kc, step.block_tables[b], 700)
    assert rows.shape[0] == 700
    assert not np.any(rows == POISON_BF16)              # nothing idle was gathered
    assert np.array_equal(rows[699], step.k_new[b])


def test_slot_to_block_row():
    assert oracle.slot_to_block_row(0, 256) == (0, 0)
    assert oracle.slot_to_block_row(255, 256) == (0, 255)
    assert oracle.slot_to_block_row(256, 256) == (1, 0)
    assert oracle.slot_to_block_row(3 * 16 + 5, 16) == (3, 5)


# ----------------------------------------------------------------------------------
# store_kvcache
# ----------------------------------------------------------------------------------

def test_store_writes_exact_rows_and_skips_padding():
    rng = np.random.default_rng(11)
    nb, bs, hkv, d = 6, 4, 2, 8
    kc = np.full((nb, bs, hkv, d), POISON_BF16, np.uint16)
    vc = kc.copy()
    k = rng.integers(0, 1 << 15, size=(5, hkv, d)).astype(np.uint16)
    v = rng.integers(0, 1 << 15, size=(5, hkv, d)).astype(np.uint16)
    slots = np.array([7, -1, 0, 23, 9], np.int32)
    k0, v0 = kc.copy(), vc.copy()
    assert oracle.store_kvcache(kc, vc, k, v, slots) == []
    expect = k0.reshape(nb * bs, hkv, d).copy()
    for t, s in enumerate(slots):
        if s >= 0:
            expect[s] = k[t]
    assert np.array_equal(kc.reshape(nb * bs, hkv, d), expect)
    # the padding token's bytes appear nowhere
    flat = kc.reshape(nb * bs, -1)
    assert not any(np.array_equal(r, k[1].ravel()) for r in flat)
    assert np.array_equal(vc.reshape(nb * bs, hkv, d)[23], v[3])
    assert np.sum(np.any(kc != k0, axis=(2, 3))) == 4


def test_store_reports_out_of_range_slots():
    kc = np.zeros((2, 4, 1, 2), np.uint16)
    vc = kc.copy()
    k = np.ones((4, 1, 2), np.uint16)
    bad = oracle.store_kvcache(kc, vc, k, k, np.array([8, -2, 3, 100], np.int32))
    assert bad == [0, 1, 3]
    assert kc.reshape(8, 2)[3].tolist() == [1, 1]
    assert kc.sum() == 2


# ----------------------------------------------------------------------------------
# brute force against contiguous-cache attention
# ----------------------------------------------------------------------------------

def _random_decode(rng, lens, hq, hkv, d, bs):
    seqs_k = [_bf16(rng.standard_normal((L, hkv, d))) for L in lens]
    seqs_v = [_bf16(rng.standard_normal((L, hkv, d))) for L in lens]
    nb = sum(-(-L // bs) for L in lens) + 2
    kpool, bt = _scatter_contiguous(seqs_k, bs, nb, np.random.default_rng(rng.integers(1 << 30)))
    vpool = np.full_like(kpool, POISON_BF16)
    for b, s in enumerate(seqs_v):
        pos = np.arange(len(s))
        vpool[bt[b, pos // bs], pos % bs] = s
    q = _bf16(rng.standard_normal((len(lens), hq, d)))
    return q, kpool, vpool, bt, seqs_k, seqs_v


@pytest.mark.parametrize("lens,hq,hkv,d,bs", [
    ([1, 5, 16, 17], 4, 2, 16, 4),
    ([33, 7], 8, 2, 32, 16),
    ([64], 6, 6, 8, 8),
    ([300, 700, 17], 4, 2, 64, 256),
])
def test_decode_matches_contiguous_sdpa(lens, hq, hkv, d, bs):
    rng = np.random.default_rng(len(lens) * 1000 + d)
    q, kpool, vpool, bt, sk, sv = _random_decode(rng, lens, hq, hkv, d, bs)
    scale = 1.0 / math.sqrt(d)
    out, lse = oracle.paged_decode_attention(q, kpool, vpool, bt, np.array(lens), scale)
    for b, L in enumerate(lens):
        qq = _f64(q[b])[:, None, :]                                    # [Hq, 1, D]
        kk = _f64(sk[b]).transpose(1, 0, 2)                            # [Hkv, L, D]
        vv = _f64(sv[b]).transpose(1, 0, 2)
        ref = _sdpa(qq, kk, vv, scale)[:, 0, :]
        np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-12)
        g = hq // hkv
        for h in range(hq):
            s = scale * (_f64(sk[b])[:, h // g, :] @ _f64(q[b, h]))
            np.testing.assert_allclose(lse[b, h], np.log(np.sum(np.exp(s))), rtol=1e-12)


@settings(max_examples=25, deadline=None)
@given(st.data())
def test_decode_fuzz_against_sdpa(data):
    bs = data.draw(st.sampled_from([1, 2, 4, 16]))
    hkv = data.draw(st.integers(1, 3))
    g = data.draw(st.integers(1, 4))
    d = data.draw(st.sampled_from([4, 8, 16]))
    lens = data.draw(st.lists(st.integers(1, 40), min_size=1, max_size=4))
    seed = data.draw(st.integers(0, 1 << 20))
    rng = np.random.default_rng(seed)
    q, kpool, vpool, bt, sk, sv = _random_decode(rng, lens, hkv * g, hkv, d, bs)
    scale = data.draw(st.floats(0.05, 2.0))
    out, _ = oracle.paged_decode_attention(q, kpool, vpool, bt, np.array(lens), scale)
    for b in range(len(lens)):
        ref = _sdpa(_f64(q[b])[:, None, :], _f64(sk[b]).transpose(1, 0, 2),
                    _f64(sv[b]).transpose(1, 0, 2), scale)[:, 0, :]
        np.testing.assert_allclose(out[b], ref, rtol=1e-11, atol=1e-11)


def _random_prefill(rng, lens, cached_tokens, hq, hkv, d, bs):
    """Sequences given as full contiguous K/V; the last len-cached rows are queries."""
    sk = [_bf16(rng.standard_normal((L, hkv, d))) for L in lens]
    sv = [_bf16(rng.standard_normal((L, hkv, d))) for L in lens]
    sq = [_bf16(rng.standard_normal((L, hq, d))) for L in lens]
    nb = sum(-(-L // bs) for L in lens) + 1
    kpool, bt = _scatter_contiguous(sk, bs, nb, np.random.default_rng(rng.integers(1 << 30)))
    vpool = np.full_like(kpool, POISON_BF16)
    for b, s in enumerate(sv):
        pos = np.arange(len(s))
        vpool[bt[b, pos // bs], pos % bs] = s
    lq = [L - c for L, c in zip(lens, cached_tokens)]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = np.concatenate([s[c:] for s, c in zip(sq, cached_tokens)])
    return q, kpool, vpool, bt, cu_q, cu_k, sq, sk, sv


@pytest.mark.parametrize("lens,hq,hkv,d,bs", [
    ([5, 16, 33], 4, 2, 16, 4),
    ([40], 3, 1, 8, 16),
    ([1, 2, 3], 2, 2, 8, 2),
])
def test_prefill_square_matches_sdpa_is_causal(lens, hq, hkv, d, bs):
    """No cached prefix (Lq = Lk): torch's own causal mask applies unchanged."""
    rng = np.random.default_rng(sum(lens))
    q, kp, vp, bt, cu_q, cu_k, sq, sk, sv = _random_prefill(rng, lens, [0] * len(lens),
                                                            hq, hkv, d, bs)
    scale = 0.7 / math.sqrt(d)
    out, _ = oracle.varlen_prefill_attention(q, kp, vp, bt, cu_q, cu_k, scale)
    for i, L in enumerate(lens):
        ref = _sdpa(_f64(sq[i]).transpose(1, 0, 2), _f64(sk[i]).transpose(1, 0, 2),
                    _f64(sv[i]).transpose(1, 0, 2), scale, is_causal=True)
        np.testing.assert_allclose(out[cu_q[i]:cu_q[i + 1]], ref.transpose(1, 0, 2),
                                   rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("lens,cached,bs", [
    ([20, 33, 9], [8, 16, 0], 8),
    ([64, 100], [48, 96], 16),
    ([7], [6], 1),
])
def test_prefix_cached_prefill_equals_tail_of_full_prefill(lens, cached, bs):
    """A prompt whose first tokens are already cached must give its suffix queries the
    outputs they would get in a prefill of the whole prompt (torch's square causal
    attention on contiguous K/V).  This pins the bottom-right causal alignment."""
    rng = np.random.default_rng(7 + bs)
    hq, hkv, d = 4, 2, 16
    q, kp, vp, bt, cu_q, cu_k, sq, sk, sv = _random_prefill(rng, lens, cached, hq, hkv, d, bs)
    scale = 1.0 / math.sqrt(d)
    out, lse = oracle.varlen_prefill_attention(q, kp, vp, bt, cu_q, cu_k, scale)
    for i, (L, c) in enumerate(zip(lens, cached)):
        full = _sdpa(_f64(sq[i]).transpose(1, 0, 2), _f64(sk[i]).transpose(1, 0, 2),
                     _f64(sv[i]).transpose(1, 0, 2), scale, is_causal=True)
        np.testing.assert_allclose(out[cu_q[i]:cu_q[i + 1]], full.transpose(1, 0, 2)[c:],
                                   rtol=1e-12, atol=1e-12)
    assert np.all(np.isfinite(lse))


@settings(max_examples=20, deadline=None)
@given(st.data())
def test_prefill_fuzz_against_sdpa(data):
    bs = data.draw(st.sampled_from([1, 4, 16]))
    hkv = data.draw(st.integers(1, 2))
    g = data.draw(st.integers(1, 3))
    d = data.draw(st.sampled_from([4, 8]))
    lens = data.draw(st.lists(st.integers(1, 30), min_size=1, max_size=3))
    cached = [data.draw(st.integers(0, L - 1)) for L in lens]
    rng = np.random.default_rng(data.draw(st.integers(0, 1 << 20)))
    q, kp, vp, bt, cu_q, cu_k, sq, sk, sv = _random_prefill(rng, lens, cached, hkv * g, hkv,
                                                            d, bs)
    scale = 1.0 / math.sqrt(d)
    out, _ = oracle.varlen_prefill_attention(q, kp, vp, bt, cu_q, cu_k, scale)
    for i, (L, c) in enumerate(zip(lens, cached)):
        full = _sdpa(_f64(sq[i]).transpose(1, 0, 2), _f64(sk[i]).transpose(1, 0, 2),
                     _f64(sv[i]).transpose(1, 0, 2), scale, is_causal=True)
        np.testing.assert_allclose(out[cu_q[i]:cu_q[i + 1]], full.transpose(1, 0, 2)[c:],
                                   rtol=1e-11, atol=1e-11)


# ----------------------------------------------------------------------------------
# invariances and closed forms
# ----------------------------------------------------------------------------------

def test_decode_invariant_under_physical_block_relabelling():
    step = make_decode_step(5, [30, 64, 1, 47], block_size=8)
    kd, vd = step.k_pool.dense(), step.v_pool.dense()
    oracle.store_kvcache(kd, vd, step.k_new, step.v_new, step.slot_mapping)
    out, lse = oracle.paged_decode_attention(step.q, kd, vd, step.block_tables,
                                             step.context_lens, step.scale)
    perm = np.random.default_rng(3).permutation(step.num_blocks)
    k2 = np.empty_like(kd)
    v2 = np.empty_like(vd)
    k2[perm] = kd
    v2[perm] = vd
    bt2 = np.where(step.block_tables >= 0, perm[np.maximum(step.block_tables, 0)], -1)
    out2, lse2 = oracle.paged_decode_attention(step.q, k2, v2, bt2, step.context_lens, step.scale)
    assert np.all(np.isfinite(out))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_shared_prefix_block_equals_duplicated_blocks():
    share = np.array([True, False, True, True])
    step = make_decode_step(9, [40, 23, 33, 65], block_size=8, shared_prefix_blocks=3,
                            share=share, num_blocks=64)
    kd, vd = step.k_pool.dense(), step.v_pool.dense()
    oracle.store_kvcache(kd, vd, step.k_new, step.v_new, step.slot_mapping)
    out, lse = oracle.paged_decode_attention(step.q, kd, vd, step.block_tables,
                                             step.context_lens, step.scale)
    assert np.all(np.isfinite(out))
    # duplicate: give every sharing sequence a private copy of the shared blocks
    bt = step.block_tables.copy()
    used = set(int(x) for x in bt.ravel() if x >= 0)
    free = [i for i in range(step.num_blocks) if i not in used]
    for b in np.nonzero(share)[0]:
        for j in range(3):
            new = free.pop()
            kd[new] = kd[bt[b, j]]
            vd[new] = vd[bt[b, j]]
            bt[b, j] = new
    assert len(set(bt[share, :3].ravel().tolist())) == 9
    out2, lse2 = oracle.paged_decode_attention(step.q, kd, vd, bt, step.context_lens, step.scale)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_softmax_weights_sum_to_one():
    step = make_decode_step(2, [1, 9, 100], block_size=4, num_q_heads=6, num_kv_heads=3)
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    _, _, w = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables,
                                            step.context_lens, step.scale, return_weights=True)
    for b in range(3):
        for h in range(6):
            assert len(w[b][h]) == step.context_lens[b]
            assert abs(np.sum(w[b][h]) - 1.0) < 1e-12
            assert np.all(w[b][h] >= 0)


def test_constant_v_gives_v():
    step = make_decode_step(4, [13, 50], block_size=16)
    vconst = _bf16(np.linspace(-2, 3, step.head_dim))
    kc = step.k_pool.copy()
    vd = step.v_pool.dense()
    oracle.store_kvcache(kc, vd, step.k_new, step.v_new, step.slot_mapping)
    vd[:] = vconst
    out, _ = oracle.paged_decode_attention(step.q, kc, vd, step.block_tables,
                                           step.context_lens, step.scale)
    np.testing.assert_allclose(out, np.broadcast_to(_f64(vconst), out.shape), rtol=0, atol=1e-12)


def test_single_key_gives_its_value_exactly():
    step = make_decode_step(6, [1, 1, 1], block_size=4, num_q_heads=4, num_kv_heads=1)
    out, lse = oracle.paged_decode_attention(step.q, step.k_pool, step.v_pool, step.block_tables,
                                             step.context_lens, step.scale)
    for b in range(3):
        blk = step.block_tables[b, 0]
        # before the step the row is NaN; write the new token as store would, by hand
        assert np.all(step.v_pool[blk][0] == POISON_BF16)
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    out, lse = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables,
                                             step.context_lens, step.scale)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[b, h], _f64(step.v_new[b, 0]))
            assert lse[b, h] == pytest.approx(step.scale * float(_f64(step.k_new[b, 0])
                                                                 @ _f64(step.q[b, h])), rel=1e-14)


def test_zero_query_gives_mean_of_values():
    step = make_decode_step(8, [7, 64], block_size=8)
    q0 = np.zeros_like(step.q)
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    out, lse = oracle.paged_decode_attention(q0, kc, vc, step.block_tables,
                                             step.context_lens, step.scale)
    g = step.num_q_heads // step.num_kv_heads
    for b, L in enumerate(step.context_lens):
        pos = np.arange(L)
        rows = _f64(vc.dense()[step.block_tables[b, pos // 8], pos % 8])   # [L, Hkv, D]
        for h in range(step.num_q_heads):
            np.testing.assert_allclose(out[b, h], rows[:, h // g].mean(axis=0), atol=1e-13)
            assert lse[b, h] == pytest.approx(math.log(L), rel=1e-14)


@pytest.mark.parametrize("cuts", [[0, 1], [0, 5, 17], [0, 1, 2, 3, 40], [0, 39]])
def test_lse_split_identity(cuts):
    rng = np.random.default_rng(len(cuts))
    L, d = 41, 16
    keys = _f64(_bf16(rng.standard_normal((L, d))))
    vals = _f64(_bf16(rng.standard_normal((L, d))))
    q = _f64(_bf16(2 * rng.standard_normal(d)))
    full_o, full_l, _ = oracle.attend(q, keys, vals, 0.25)
    bounds = list(cuts) + [L]
    parts = [oracle.attend(q, keys[a:b], vals[a:b], 0.25) for a, b in zip(bounds, bounds[1:])]
    o, l = oracle.lse_combine([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(o, full_o, rtol=1e-12, atol=1e-13)
    assert l == pytest.approx(full_l, rel=1e-13)


def test_lse_combine_ignores_empty_parts():
    o, l = oracle.lse_combine([[1.0, 2.0], [5.0, 5.0]], [0.3, -np.inf])
    assert np.array_equal(o, [1.0, 2.0]) and l == pytest.approx(0.3)
    o, l = oracle.lse_combine([[1.0, 2.0]], [-np.inf])
    assert np.array_equal(o, [0.0, 0.0]) and l == -np.inf


def test_decode_equals_last_row_of_causal_prefill():
    rng = np.random.default_rng(21)
    lens = [9, 31]
    q, kp, vp, bt, cu_q, cu_k, sq, sk, sv = _random_prefill(rng, lens, [0, 0], 4, 2, 16, 4)
    out_p, lse_p = oracle.varlen_prefill_attention(q, kp, vp, bt, cu_q, cu_k, 0.3)
    qd = np.stack([sq[i][-1] for i in range(2)])
    out_d, lse_d = oracle.paged_decode_attention(qd, kp, vp, bt, np.array(lens), 0.3)
    for i in range(2):
        np.testing.assert_allclose(out_d[i], out_p[cu_q[i + 1] - 1], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse_d[i], lse_p[cu_q[i + 1] - 1], rtol=1e-13)


def test_poisoned_rows_are_never_read_in_workload():
    step = make_prefill_step(3, [70, 40, 129], cached_blocks=[2, 0, 4], block_size=32)
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    assert oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping) == []
    out, lse = oracle.varlen_prefill_attention(step.q, kc, vc, step.block_tables,
                                               step.cu_seqlens_q, step.cu_seqlens_k, step.scale)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    # without the store, the suffix rows are still NaN and show up in the output
    out_bad, _ = oracle.varlen_prefill_attention(step.q, step.k_pool, step.v_pool,
                                                 step.block_tables, step.cu_seqlens_q,
                                                 step.cu_seqlens_k, step.scale)
    assert np.isnan(out_bad).any()
