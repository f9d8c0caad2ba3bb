"""CPU oracle for paged-KV attention: the plain definition, written out slowly.

TEST INFRASTRUCTURE.  Only the tests, the smoke check in __graft_entry__ and the CPU
baseline leg of bench.py may import this module.  It shares no code with the CUDA
library: it has its own bf16 decoding, its own block/offset arithmetic and its own
softmax, and it never reads anything the GPU produced.

Arithmetic is float64 on values decoded exactly from bf16.  Attention is computed the
obvious way: gather the keys and values of one sequence block by block through its
block table, form all scores, subtract the maximum, exponentiate, normalise, multiply by
the values.  None of the GPU path's tiling, splitting or online rescaling appears here.

Sources (page title, then section):
  [P1] Neutree AI, "Nano-vLLM part 1" (Chinese translation on blog.itpub.net):
       section 4.1 "From Sequences to Blocks" (fixed-size blocks, default 256 tokens; a
       700-token sequence fills two blocks and 188 rows of a third), section 4.2
       "Prefix caching through hashing" (one physical block reused by refcount),
       section 4.3 (freed blocks are not zeroed), section 5.2 (cumulative sequence
       lengths for prefill; one token per sequence plus slot mappings for decode).
  [P3] "Nano-vLLM inference engine architecture" (blog.hotdry.top), section
       "PagedAttention's lightweight implementation" (slot_mapping maps each new
       token to a cache slot; the cache is a flat [total_slots, head_dim] array written
       by store_kvcache_kernel) and section "Low-level performance details" (prefill
       uses a varlen attention over cumulative lengths, decode an attention that reads
       the cached keys and values).

Readings where the pages are silent:
  * context_lens counts the token stored in the same step, so decode attends to keys
    0 .. context_len-1 including the newest one;
  * query head h reads KV head h // (Hq / Hkv) (contiguous head groups);
  * causal prefill with a cached prefix is bottom-right aligned: suffix query r of a
    sequence with Lq queries and Lk keys sits at absolute position Lk - Lq + r and sees
    keys 0 .. Lk - Lq + r;
  * slot -1 marks a padding token that is skipped; any other slot outside
    [0, num_blocks * block_size) is invalid, skipped and reported;
  * the flat [total_slots, ...] view of [P3] and the [num_blocks, block_size, Hkv, D]
    view are the same memory: slot = block * block_size + row.

Parity pins (tests/test_oracle_pins.py): the 700-token example of [P1] section 4.1,
brute force against contiguous-cache attention from torch's CPU float64 scaled dot
product attention, invariance under relabelling of physical blocks, shared-vs-duplicated
prefix blocks, softmax weights summing to one, constant-V and single-key closed forms,
zero-query mean, the log-sum-exp split identity, decode equal to the last row of causal
prefill, and prefix-cached prefill equal to the tail of a full prefill.
"""

from __future__ import annotations

import math

import numpy as np

PAD_SLOT = -1


# ---------------------------------------------------------------------------------
# bf16 decoding (the oracle's own; exact: every bf16 value is a float64 value)
# ---------------------------------------------------------------------------------

def _bf16_fields_to_f64(bits) -> np.ndarray:
    """Decode uint16 bf16 bit patterns to float64 exactly, from the bit fields.

    A bf16 value is the upper half of an IEEE binary32 value: sign, 8 exponent bits and
    7 fraction bits.  It is decoded here from its fields, not through a float32 view.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.int64)
    sign = np.where((b >> 15) & 1, -1.0, 1.0)
    exp = (b >> 7) & 0xFF
    frac = (b & 0x7F).astype(np.float64)
    normal = sign * np.ldexp(1.0 + frac / 128.0, exp - 127)
    subnormal = sign * np.ldexp(frac / 128.0, -126)
    out = np.where(exp == 0, subnormal, normal)
    special = exp == 0xFF
    if np.any(special):
        out = np.where(special & (frac == 0), sign * np.inf, out)
        out = np.where(special & (frac != 0), np.nan, out)
    return out


_BF16_TABLE = None


def bf16_to_f64(bits) -> np.ndarray:
    """Decode uint16 bf16 bit patterns to float64 exactly.

    Uses a table of all 65536 patterns, each decoded once by _bf16_fields_to_f64.
    """
    global _BF16_TABLE
    if _BF16_TABLE is None:
        _BF16_TABLE = _bf16_fields_to_f64(np.arange(1 << 16, dtype=np.uint32).astype(np.uint16))
    return _BF16_TABLE[np.asarray(bits, dtype=np.uint16)]


# ---------------------------------------------------------------------------------
# block arithmetic and the cache write ([P1] 4.1, [P3] PagedAttention section)
# ---------------------------------------------------------------------------------

def blocks_for_tokens(num_tokens: int, block_size: int):
    """How a sequence of num_tokens tokens lies in blocks of block_size tokens.

    Returns (number of blocks, tokens in the last block, idle slots in the last block).
    [P1] section 4.1: 700 tokens in blocks of 256 take three blocks, the last one
    holding 188 tokens with 68 slots idle.
    """
    if num_tokens <= 0:
        return 0, 0, 0
    full, rem = divmod(num_tokens, block_size)
    nblocks = full + (1 if rem else 0)
    last = rem if rem else block_size
    return nblocks, last, block_size - last


def slot_to_block_row(slot: int, block_size: int):
    """A flat cache slot as (physical block, row inside the block)."""
    return divmod(int(slot), block_size)


def store_kvcache(k_cache, v_cache, k, v, slot_mapping):
    """Write each token's K and V rows into the cache at its slot ([P3] store_kvcache).

    k_cache, v_cache: indexable by physical block id, each block [block_size, Hkv, D]
    of uint16 bf16 bits; they are modified in place (pass copies).
    k, v: [N, Hkv, D] uint16.  slot_mapping: [N] integers.
    Tokens are written in order.  Slot -1 is a padding token and is skipped.  A slot
    outside [0, num_blocks*block_size) is skipped and its token index returned in the
    list of invalid tokens.
    """
    num_blocks, block_size = k_cache.shape[0], k_cache.shape[1]
    capacity = num_blocks * block_size
    invalid = []
    for t in range(len(slot_mapping)):
        s = int(slot_mapping[t])
        if s == PAD_SLOT:
            continue
        if s < 0 or s >= capacity:
            invalid.append(t)
            continue
        blk, row = slot_to_block_row(s, block_size)
        k_cache[blk][row] = k[t]
        v_cache[blk][row] = v[t]
    return invalid


def gather_kv(cache, block_table_row, length: int) -> np.ndarray:
    """Keys (or values) 0 .. length-1 of one sequence, read block by block.

    Token j lives in logical block j // block_size, whose physical id is
    block_table_row[j // block_size], at row j % block_size.  Only the rows that hold a
    live token are read; table entries past the last block are never looked at.
    Returns [length, Hkv, D] uint16 (bit-exact copy of the cache rows).
    """
    block_size = cache.shape[1]
    nblocks, last, _ = blocks_for_tokens(length, block_size)
    parts = []
    for j in range(nblocks):
        phys = int(block_table_row[j])
        if not 0 <= phys < cache.shape[0]:
            raise IndexError(f"block table entry {phys} outside the pool")
        rows = block_size if j < nblocks - 1 else last
        parts.append(np.asarray(cache[phys][:rows]))
    if not parts:
        return np.zeros((0,) + tuple(cache.shape[2:]), np.uint16)
    return np.concatenate(parts, axis=0)


# ---------------------------------------------------------------------------------
# attention ([P3] low-level section; readings listed in the module docstring)
# ---------------------------------------------------------------------------------

def attend(q_vec, keys, values, scale):
    """Softmax attention of one query over L keys, by definition.

    q_vec [D], keys [L, D], values [L, D] (float64).  Returns (out [D], lse, weights [L])
    where weights = softmax(scale * keys @ q_vec), out = weights @ values and
    lse = log(sum(exp(scale * keys @ q_vec))).  With L = 0 the output is zero and the
    lse is -inf.
    """
    if keys.shape[0] == 0:
        return np.zeros(values.shape[1]), -np.inf, np.zeros(0)
    s = scale * (keys @ q_vec)
    m = np.max(s)
    p = np.exp(s - m)
    denom = np.sum(p)
    w = p / denom
    return w @ values, m + math.log(denom), w


def group_size(num_q_heads: int, num_kv_heads: int) -> int:
    if num_kv_heads <= 0 or num_q_heads % num_kv_heads:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    return num_q_heads // num_kv_heads


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale,
                           return_weights=False):
    """Decode attention: one query token per sequence over its paged context.

    q: [B, Hq, D] uint16 bf16 bits.  k_cache, v_cache: pools indexable by block id,
    [num_blocks, block_size, Hkv, D].  block_tables: [B, max_blocks] int.
    context_lens: [B] int, counting the newest token.  Query head h reads KV head
    h // (Hq / Hkv).
    Returns out [B, Hq, D] float64, lse [B, Hq] float64 and, if asked, the list of
    per-(b, h) softmax weight vectors.
    """
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    g = group_size(Hq, Hkv)
    out = np.zeros((B, Hq, D))
    lse = np.full((B, Hq), -np.inf)
    weights = [[None] * Hq for _ in range(B)]
    qf = bf16_to_f64(q)
    for b in range(B):
        L = int(context_lens[b])
        keys = bf16_to_f64(gather_kv(k_cache, block_tables[b], L))
        vals = bf16_to_f64(gather_kv(v_cache, block_tables[b], L))
        for h in range(Hq):
            hk = h // g
            o, l, w = attend(qf[b, h], keys[:, hk, :], vals[:, hk, :], scale)
            out[b, h] = o
            lse[b, h] = l
            weights[b][h] = w
    if return_weights:
        return out, lse, weights
    return out, lse


def causal_mask(num_q: int, num_k: int) -> np.ndarray:
    """[num_q, num_k] boolean, True where query r may see key j.

    Bottom-right alignment: query r is at absolute position num_k - num_q + r and sees
    keys up to and including that position.
    """
    r = np.arange(num_q)[:, None]
    j = np.arange(num_k)[None, :]
    return j <= (num_k - num_q) + r


def varlen_prefill_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, cu_seqlens_k,
                             scale, causal=True):
    """Varlen prefill attention over paged keys ([P1] 5.2 cumulative lengths).

    q: [total_q, Hq, D] uint16.  Sequence i owns query rows cu_seqlens_q[i] ..
    cu_seqlens_q[i+1]-1 (its uncached suffix) and keys 0 .. Lk-1 with
    Lk = cu_seqlens_k[i+1] - cu_seqlens_k[i], read through block_tables[i] (cached prefix
    plus the suffix written in this step).  Returns out [total_q, Hq, D] and
    lse [total_q, Hq], float64.  A query row that sees no key gets zeros and -inf.
    """
    total_q, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    g = group_size(Hq, Hkv)
    out = np.zeros((total_q, Hq, D))
    lse = np.full((total_q, Hq), -np.inf)
    qf = bf16_to_f64(q)
    B = len(cu_seqlens_q) - 1
    for i in range(B):
        q0, q1 = int(cu_seqlens_q[i]), int(cu_seqlens_q[i + 1])
        Lq = q1 - q0
        Lk = int(cu_seqlens_k[i + 1]) - int(cu_seqlens_k[i])
        if Lq == 0:
            continue
        if Lq > Lk:
            raise ValueError("a sequence has more queries than keys")
        keys = bf16_to_f64(gather_kv(k_cache, block_tables[i], Lk))
        vals = bf16_to_f64(gather_kv(v_cache, block_tables[i], Lk))
        mask = causal_mask(Lq, Lk) if causal else np.ones((Lq, Lk), bool)
        for h in range(Hq):
            hk = h // g
            s = scale * (qf[q0:q1, h, :] @ keys[:, hk, :].T)      # [Lq, Lk]
            s = np.where(mask, s, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            seen = np.isfinite(m[:, 0])
            m = np.where(np.isfinite(m), m, 0.0)
            p = np.where(mask, np.exp(s - m), 0.0)
            denom = np.sum(p, axis=1, keepdims=True)
            w = p / np.where(denom > 0, denom, 1.0)
            out[q0:q1, h, :] = w @ vals[:, hk, :]
            lse[q0:q1, h] = np.where(seen, m[:, 0] + np.log(np.where(denom[:, 0] > 0,
                                                                      denom[:, 0], 1.0)),
                                     -np.inf)
    return out, lse


def lse_combine(o_parts, lse_parts):
    """Merge attention over disjoint key subsets.

    o_parts [P, D]: each part's normalised output; lse_parts [P]: each part's
    log-sum-exp.  The merged lse is log(sum_p exp(lse_p)); the merged output is
    sum_p exp(lse_p - lse) * o_p.  Parts with lse = -inf (no keys) weigh zero.
    """
    lse_parts = np.asarray(lse_parts, np.float64)
    o_parts = np.asarray(o_parts, np.float64)
    finite = np.isfinite(lse_parts)
    if not finite.any():
        return np.zeros(o_parts.shape[1]), -np.inf
    m = np.max(lse_parts[finite])
    e = np.where(finite, np.exp(np.where(finite, lse_parts, m) - m), 0.0)
    total = np.sum(e)
    lse = m + math.log(total)
    return (e / total) @ o_parts, lse
