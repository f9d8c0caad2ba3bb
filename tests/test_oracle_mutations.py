"""Planted mistakes: each test swaps one piece of the oracle for a plausibly wrong variant
(on the CPU, inside this process only) and checks that at least one pin then fails.
This shows that the pins in test_oracle_pins.py can see such mistakes at all."""

import numpy as np
import pytest

import oracle
import oracle.paged_attention as pa
import tests.test_oracle_pins as pins


def _expect_pin_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_wrong_gqa_mapping_is_caught(monkeypatch):
    def decode_mod_mapping(q, k_cache, v_cache, block_tables, context_lens, scale,
                           return_weights=False):
        B, Hq, D = q.shape
        Hkv = k_cache.shape[2]
        out = np.zeros((B, Hq, D))
        lse = np.zeros((B, Hq))
        qf = pa.bf16_to_f64(q)
        for b in range(B):
            L = int(context_lens[b])
            keys = pa.bf16_to_f64(pa.gather_kv(k_cache, block_tables[b], L))
            vals = pa.bf16_to_f64(pa.gather_kv(v_cache, block_tables[b], L))
            for h in range(Hq):
                hk = h % Hkv                                   # planted: interleaved groups
                out[b, h], lse[b, h], _ = pa.attend(qf[b, h], keys[:, hk], vals[:, hk], scale)
        return out, lse

    monkeypatch.setattr(oracle, "paged_decode_attention", decode_mod_mapping)
    _expect_pin_failure(pins.test_decode_matches_contiguous_sdpa, [1, 5, 16, 17], 4, 2, 16, 4)


def test_top_left_causal_alignment_is_caught(monkeypatch):
    def top_left(num_q, num_k):
        r = np.arange(num_q)[:, None]
        j = np.arange(num_k)[None, :]
        return j <= r                                          # planted: ignores the prefix

    monkeypatch.setattr(pa, "causal_mask", top_left)
    _expect_pin_failure(pins.test_prefix_cached_prefill_equals_tail_of_full_prefill,
                        [20, 33, 9], [8, 16, 0], 8)


def test_logical_block_id_is_caught(monkeypatch):
    real = pa.gather_kv

    def gather_logical(cache, block_table_row, length):
        ident = np.arange(len(block_table_row))                # planted: table not consulted
        return real(cache, ident, length)

    monkeypatch.setattr(pa, "gather_kv", gather_logical)
    _expect_pin_failure(pins.test_decode_matches_contiguous_sdpa, [33, 7], 8, 2, 32, 16)


def test_dropped_scale_is_caught(monkeypatch):
    real = pa.attend

    def attend_unscaled(q_vec, keys, values, scale):
        return real(q_vec, keys, values, 1.0)                  # planted: scale ignored

    monkeypatch.setattr(pa, "attend", attend_unscaled)
    _expect_pin_failure(pins.test_decode_matches_contiguous_sdpa, [64], 6, 6, 8, 8)


def test_linear_lse_merge_is_caught(monkeypatch):
    def combine_linear(o_parts, lse_parts):
        w = np.asarray(lse_parts, np.float64)                  # planted: no exponential
        w = w / w.sum()
        return w @ np.asarray(o_parts, np.float64), float(np.log(np.exp(lse_parts).sum()))

    monkeypatch.setattr(oracle, "lse_combine", combine_linear)
    _expect_pin_failure(pins.test_lse_split_identity, [0, 5, 17])


def test_store_row_off_by_one_is_caught(monkeypatch):
    def slot_shifted(slot, block_size):
        blk, row = divmod(int(slot), block_size)
        return blk, min(row + 1, block_size - 1)               # planted: row shifted

    monkeypatch.setattr(pa, "slot_to_block_row", slot_shifted)
    _expect_pin_failure(pins.test_worked_example_in_tiny_decode_workload)


def test_last_block_count_slip_is_caught(monkeypatch):
    def blocks_floor(num_tokens, block_size):
        full, rem = divmod(num_tokens, block_size)
        return full, rem, block_size - rem                     # planted: partial block lost

    monkeypatch.setattr(oracle, "blocks_for_tokens", blocks_floor)
    _expect_pin_failure(pins.test_worked_example_700_tokens)


def test_missing_normalisation_is_caught(monkeypatch):
    real = pa.attend

    def attend_unnormalised(q_vec, keys, values, scale):
        o, l, w = real(q_vec, keys, values, scale)
        return o * len(w), l, w * len(w)                       # planted: mean instead of sum

    monkeypatch.setattr(pa, "attend", attend_unnormalised)
    _expect_pin_failure(pins.test_softmax_weights_sum_to_one)
