"""Varlen (prefix-cached) causal prefill attention on the GPU against the float64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from synth import make_decode_step, make_prefill_step, prefill_varlen_prefix_hits
from synth.device import bf16_tensor, decode_to_device, i32, prefill_to_device
from tests.helpers import assert_attention_close, assert_lse_close, oracle_after_store

pytestmark = pytest.mark.gpu


def _run(step, t, causal=True, err=None):
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                       err_flag=err)
    out, lse = nvpa.varlen_prefill_attention(
        t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["cu_seqlens_q"],
        t["cu_seqlens_k"], step.max_seqlen_q, step.max_seqlen_k, step.scale, causal=causal,
        err_flag=err, return_lse=True)
    torch.cuda.synchronize()
    return out, lse


def _oracle(step, causal=True):
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    return oracle.varlen_prefill_attention(step.q, kc, vc, step.block_tables, step.cu_seqlens_q,
                                           step.cu_seqlens_k, step.scale, causal=causal)


def test_prefill_prefix_hits_full_size(cuda_device):
    step = prefill_varlen_prefix_hits()
    assert (step.cached_blocks > 0).sum() > 0
    t = prefill_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out, lse = _run(step, t, err=err)
    assert err.item() == 0
    ora_out, ora_lse = _oracle(step)
    assert_attention_close(out, ora_out, "prefill_varlen_prefix_hits_b32")
    assert_lse_close(lse, ora_lse, "prefill_varlen_prefix_hits_b32")


CASES = [
    # (total lengths, cached blocks, Hq, Hkv, D, block size)
    ([1, 2, 17, 64], [0, 0, 0, 0], 4, 2, 64, 16),
    ([300, 129, 40], [2, 1, 0], 8, 8, 128, 64),
    ([513, 256, 1000], [1, 1, 3], 16, 8, 128, 256),
    ([64, 64], [4, 0], 6, 2, 128, 16),          # first sequence fully cached: Lq = 0
    ([200, 31, 77], [3, 0, 2], 12, 4, 64, 32),
    ([700], [1], 8, 1, 128, 128),
    ([450, 97], [2, 0], 8, 2, 128, 64),           # group 4: four heads per tile row block
    ([1500, 5], [5, 0], 16, 8, 128, 128),         # many query-tile pairs, prefix of 640 keys
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("lens,cached,hq,hkv,d,bs", CASES)
def test_prefill_small_shapes(cuda_device, lens, cached, hq, hkv, d, bs, causal):
    step = make_prefill_step(sum(lens) + bs, lens, cached_blocks=cached, num_q_heads=hq,
                             num_kv_heads=hkv, head_dim=d, block_size=bs)
    t = prefill_to_device(step, cuda_device)
    out, lse = _run(step, t, causal=causal)
    ora_out, ora_lse = _oracle(step, causal=causal)
    assert_attention_close(out, ora_out, f"prefill {lens} causal={causal}")
    assert_lse_close(lse, ora_lse, f"prefill {lens} causal={causal}")


@pytest.mark.parametrize("scale", [-0.125, 0.0, 0.6])
def test_prefill_scale_sign_and_size(cuda_device, scale):
    """A negative softmax scale (the kernel flips the sign of Q K^T on the tensor cores and
    scales by its magnitude), a zero scale (uniform weights over the visible keys) and a
    large one (sharp rows whose running maximum moves often)."""
    step = make_prefill_step(55, [700, 300, 129], cached_blocks=[1, 0, 0], num_q_heads=8,
                             num_kv_heads=2, head_dim=128, block_size=64, scale=scale)
    assert step.scale == scale
    t = prefill_to_device(step, cuda_device)
    out, lse = _run(step, t)
    ora_out, ora_lse = _oracle(step)
    assert_attention_close(out, ora_out, f"prefill scale {scale}")
    assert_lse_close(lse, ora_lse, f"prefill scale {scale}")


def test_prefill_last_row_equals_decode(cuda_device):
    """The last query row of a causal prefill sees the whole context: decode of the same
    token over the same cache gives the same attention."""
    step = make_prefill_step(40, [333, 90], cached_blocks=[2, 1], num_q_heads=8, num_kv_heads=2,
                             head_dim=128, block_size=32)
    t = prefill_to_device(step, cuda_device)
    out_p, _ = _run(step, t)
    last = torch.as_tensor(step.cu_seqlens_q[1:] - 1, device=cuda_device, dtype=torch.long)
    q_last = t["q"][last].contiguous()
    out_d = nvpa.paged_decode_attention(q_last, t["k_cache"], t["v_cache"], t["block_tables"],
                                        i32(step.seq_lens, cuda_device), int(step.seq_lens.max()),
                                        step.scale)
    torch.cuda.synchronize()
    diff = (out_p[last].float() - out_d.float()).abs().max().item()
    assert diff <= 2e-2


def _pack(step):
    """Query heads per 128-row tile: the GQA group when it is a power of two up to 8."""
    group = step.num_q_heads // step.num_kv_heads
    return min(group, 8) if group & (group - 1) == 0 else 1


def _expected_pairs(step):
    """(sequence, tile A, tile B or -1) -> key tiles visited, from the tiling the kernel
    uses: 128-row query tiles of 128/P tokens x P heads, pairs (2w, 2w + 1) counted from
    the sequence start, causal bottom-right alignment, 128-key tiles."""
    tq = 128 // _pack(step)
    pairs = {}
    for i in range(step.batch):
        lq = int(step.cu_seqlens_q[i + 1] - step.cu_seqlens_q[i])
        lk = int(step.cu_seqlens_k[i + 1] - step.cu_seqlens_k[i])
        cnt = -(-lq // tq)

        def nkv(qt):
            tok0, ntok = qt * tq, min(tq, lq - qt * tq)
            return min(-(-lk // 128), (lk - lq + tok0 + ntok - 1) // 128 + 1)

        for w in range((cnt + 1) // 2):
            b = 2 * w + 1 if 2 * w + 1 < cnt else -1
            pairs[(i, 2 * w, b)] = nkv(b if b >= 0 else 2 * w)
    return pairs


@pytest.mark.parametrize("which", ["full", "group4_bs16"])
def test_prefill_plan_lists_every_pair_longest_first(cuda_device, which):
    """The plan in the workspace lists each query-tile pair exactly once, sorted by the key
    tiles it visits, most first (the order inside one count is free)."""
    if which == "full":
        step = prefill_varlen_prefix_hits()
    else:
        step = make_prefill_step(7, [900, 37, 1, 400, 260], cached_blocks=[10, 0, 0, 3, 16],
                                 num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16)
    t = prefill_to_device(step, cuda_device)
    ws = torch.zeros(nvpa.varlen_prefill_workspace_size(step.batch, step.total_q), dtype=torch.uint8,
                     device=cuda_device)
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
    nvpa.varlen_prefill_attention(t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                  t["cu_seqlens_q"], t["cu_seqlens_k"], step.max_seqlen_q,
                                  step.max_seqlen_k, step.scale, workspace=ws)
    torch.cuda.synchronize()
    head = ws[:8].view(torch.int32).cpu().numpy()
    n = int(head[0])
    entries = ws[256:256 + 16 * n].view(torch.int32).cpu().numpy().reshape(n, 4)
    expected = _expected_pairs(step)
    got = [(int(e[0]), int(e[1]), int(e[2])) for e in entries]
    assert sorted(got) == sorted(expected), "the plan must list every pair exactly once"
    assert all(int(e[3]) == 0 for e in entries)
    counts = [expected[g] for g in got]
    assert all(a >= b for a, b in zip(counts, counts[1:])), "pairs must come most key tiles first"
    # every unit (pair x head group) was claimed: the counter ran at least to the end
    assert int(head[1]) >= n * (step.num_q_heads // _pack(step))
