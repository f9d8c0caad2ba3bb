"""store_kvcache and gather_kv on the GPU against the oracle: bit-exact, whole pools."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_422_b200 as nvpa
from synth import (POISON_BF16, WORKLOADS, bf16_bits_from_f32, decode_tiny, make_decode_step,
                   make_prefill_step)
from synth.device import bf16_tensor, bits_of, decode_to_device, i32, prefill_to_device
from tests.helpers import assert_pool_equal, cu_from_lens, oracle_after_store

pytestmark = pytest.mark.gpu


def _to_device(step, dev):
    return prefill_to_device(step, dev) if hasattr(step, "cu_seqlens_q") else decode_to_device(step, dev)


def _store(t, err):
    nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"],
                       err_flag=err)


def test_store_tiny_whole_pool(cuda_device):
    step = decode_tiny()
    t = decode_to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _store(t, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    assert np.array_equal(bits_of(t["k_cache"]), kc.dense())
    assert np.array_equal(bits_of(t["v_cache"]), vc.dense())
    # the padding token (index 4) was written nowhere
    pad = step.k_new[4].ravel()
    flat = bits_of(t["k_cache"]).reshape(-1, pad.size)
    assert not (flat == pad).all(axis=1).any()


@pytest.mark.parametrize("name", ["decode_mid_b64", "decode_b512_shared_prefix",
                                  "prefill_varlen_prefix_hits_b32", "decode_long_b8_ctx32k_bs16"])
def test_store_full_size_workloads(cuda_device, name):
    step = WORKLOADS[name]()
    t = _to_device(step, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    _store(t, err)
    torch.cuda.synchronize()
    assert err.item() == 0
    kc, vc, bad = oracle_after_store(step)
    assert bad == []
    assert_pool_equal(t["k_cache"], kc, f"{name} k_cache")
    assert_pool_equal(t["v_cache"], vc, f"{name} v_cache")


def test_store_strided_token_rows(cuda_device):
    """k and v as views into a packed [N, (Hq + 2 Hkv) * D] qkv buffer."""
    rng = np.random.default_rng(5)
    n, hq, hkv, d, nb, bs = 37, 8, 2, 64, 12, 16
    qkv = bf16_bits_from_f32(rng.standard_normal((n, (hq + 2 * hkv) * d), dtype=np.float32))
    qkv_t = bf16_tensor(qkv, cuda_device)
    k = qkv_t[:, hq * d:(hq + hkv) * d].view(n, hkv, d)
    v = qkv_t[:, (hq + hkv) * d:].view(n, hkv, d)
    slots = rng.permutation(nb * bs)[:n].astype(np.int32)
    slots[[3, 17]] = -1
    kc = torch.full((nb, bs, hkv, d), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    vc = kc.clone()
    nvpa.store_kvcache(k, v, kc, vc, i32(slots, cuda_device))
    torch.cuda.synchronize()
    ok = np.full((nb, bs, hkv, d), POISON_BF16, np.uint16)
    ov = ok.copy()
    kbits = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d)
    vbits = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d)
    assert oracle.store_kvcache(ok, ov, kbits, vbits, slots) == []
    assert np.array_equal(bits_of(kc), ok)
    assert np.array_equal(bits_of(vc), ov)


def test_store_out_of_range_slots_flagged_and_skipped(cuda_device):
    rng = np.random.default_rng(6)
    n, hkv, d, nb, bs = 6, 2, 128, 4, 16
    k = bf16_bits_from_f32(rng.standard_normal((n, hkv, d), dtype=np.float32))
    v = bf16_bits_from_f32(rng.standard_normal((n, hkv, d), dtype=np.float32))
    slots = np.array([0, nb * bs, 5, -7, -1, nb * bs - 1], np.int32)
    kc = torch.zeros((nb, bs, hkv, d), dtype=torch.bfloat16, device=cuda_device)
    vc = kc.clone()
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    nvpa.store_kvcache(bf16_tensor(k, cuda_device), bf16_tensor(v, cuda_device), kc, vc,
                       i32(slots, cuda_device), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == nvpa.NVPA_FLAG_BAD_SLOT
    ok = np.zeros((nb, bs, hkv, d), np.uint16)
    ov = ok.copy()
    assert oracle.store_kvcache(ok, ov, k, v, slots) == [1, 3]
    assert np.array_equal(bits_of(kc), ok)
    assert np.array_equal(bits_of(vc), ov)


def test_store_zero_tokens_is_a_noop(cuda_device):
    kc = torch.zeros((2, 16, 1, 64), dtype=torch.bfloat16, device=cuda_device)
    e = torch.empty((0, 1, 64), dtype=torch.bfloat16, device=cuda_device)
    nvpa.store_kvcache(e, e, kc, kc.clone(), torch.empty(0, dtype=torch.int32, device=cuda_device))
    torch.cuda.synchronize()
    assert kc.abs().sum().item() == 0


def _gather_check(step, kc_dev, vc_dev, kc, vc, lens, seqs=None):
    seqs = list(range(len(lens))) if seqs is None else seqs
    bt = step.block_tables[seqs]
    sub_lens = np.asarray(lens)[seqs]
    cu = cu_from_lens(sub_lens)
    dev = kc_dev.device
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    gk = nvpa.gather_kv(kc_dev, i32(bt, dev), i32(cu, dev), int(cu[-1]), err_flag=err)
    gv = nvpa.gather_kv(vc_dev, i32(bt, dev), i32(cu, dev), int(cu[-1]), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    gk, gv = bits_of(gk), bits_of(gv)
    for j, b in enumerate(seqs):
        L = int(sub_lens[j])
        assert np.array_equal(gk[cu[j]:cu[j + 1]], oracle.gather_kv(kc, step.block_tables[b], L))
        assert np.array_equal(gv[cu[j]:cu[j + 1]], oracle.gather_kv(vc, step.block_tables[b], L))
    assert not np.any(gk == POISON_BF16)


@pytest.mark.parametrize("name,seqs", [
    ("decode_tiny_b4", None),
    ("decode_mid_b64", None),
    ("decode_b512_shared_prefix", list(range(0, 512, 16))),
    ("decode_long_b8_ctx32k_bs16", [0, 5]),
])
def test_gather_bit_exact_after_store(cuda_device, name, seqs):
    step = WORKLOADS[name]()
    t = decode_to_device(step, cuda_device)
    _store(t, None)
    kc, vc, _ = oracle_after_store(step)
    _gather_check(step, t["k_cache"], t["v_cache"], kc, vc, step.context_lens, seqs)


@pytest.mark.parametrize("bs", [16, 32, 64, 128, 256])
def test_gather_block_sizes(cuda_device, bs):
    step = make_decode_step(bs, [1, bs - 1, bs, bs + 1, 3 * bs + 7], num_q_heads=4,
                            num_kv_heads=2, head_dim=64, block_size=bs)
    t = decode_to_device(step, cuda_device)
    _store(t, None)
    kc, vc, _ = oracle_after_store(step)
    _gather_check(step, t["k_cache"], t["v_cache"], kc, vc, step.context_lens)


def test_gather_prefill_workload(cuda_device):
    step = make_prefill_step(8, [300, 17, 513], cached_blocks=[1, 0, 2], num_q_heads=8,
                             num_kv_heads=4, head_dim=128, block_size=128)
    t = prefill_to_device(step, cuda_device)
    _store(t, None)
    kc, vc, _ = oracle_after_store(step)
    _gather_check(step, t["k_cache"], t["v_cache"], kc, vc, step.seq_lens)
