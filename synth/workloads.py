"""Seeded workload generators (test and benchmark inputs only).

Every array produced here is plain input data: bf16 values are stored as uint16 bit
patterns, indices as int32.  The generators stand in for Nano-vLLM's control plane:

* the block manager cuts each sequence into fixed-size blocks and hands out physical
  block ids (Nano-vLLM part 1, Neutree AI, section 4.1 "From Sequences to Blocks");
* blocks whose content is a shared prefix are referenced by several sequences with a
  refcount above one (same page, section 4.2 "Prefix caching through hashing");
* freed blocks are not cleared, so rows that hold no live token keep old bytes
  (same page, section 4.3).  Here such rows hold a bf16 NaN, so that any read of them
  shows up in an attention output;
* the model runner turns the batch into cumulative sequence lengths (prefill) or one
  token per sequence with its slot mapping (decode) (same page, section 5.2).

The values themselves are N(0, 1) draws from numpy's default_rng(seed), rounded once to
bf16.  The same bytes are fed to the oracle and to the GPU library.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

# Quiet NaN in bf16: the content of every cache row that holds no live token.
POISON_BF16 = 0x7FC0

# Blocks generated per numpy call when filling large pools (bounds float32 temporaries).
_CHUNK_ROWS = 1 << 22


def bf16_bits_from_f32(x) -> np.ndarray:
    """Round float32 values to bf16, nearest-even, and return the uint16 bit patterns.

    Inputs are finite (they are normal draws), so no NaN/Inf special-casing is needed.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def _f32_from_bf16_bits(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """N(0,1) draws rounded to bf16.

    One 63-bit key is taken from `rng`; chunk i of the output (along axis 0) is then drawn
    from default_rng(SeedSequence([key, i])).  Chunks are filled on a thread pool, so
    large pools are generated quickly, and the result depends only on `rng`'s state.
    """
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.uint16)
    key = int(rng.integers(0, 2**63 - 1))
    if out.size == 0:
        return out
    per = max(1, out.size // max(1, shape[0]))
    step = max(1, _CHUNK_ROWS // per)
    starts = list(range(0, shape[0], step))

    def fill(ci):
        i = starts[ci]
        j = min(shape[0], i + step)
        g = np.random.default_rng(np.random.SeedSequence([key, ci]))
        out[i:j] = bf16_bits_from_f32(g.standard_normal((j - i,) + shape[1:], dtype=np.float32))

    if len(starts) == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(len(starts))))
    return out


class PagedPool:
    """One block-paged cache pool, [num_blocks, block_size, num_kv_heads, head_dim] bf16 bits.

    Only blocks handed to some sequence are stored (`ids`, `data`).  Any other block reads
    as all-NaN, the stand-in for a freed block whose old bytes were never cleared.
    Indexing by a physical block id returns that block's [block_size, Hkv, D] array
    (a view, writable), so code written against a dense numpy pool works unchanged.
    """

    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim, ids=None, data=None):
        self.shape = (int(num_blocks), int(block_size), int(num_kv_heads), int(head_dim))
        if ids is None:
            ids = np.zeros(0, np.int64)
            data = np.zeros((0,) + self.shape[1:], np.uint16)
        self.ids = np.asarray(ids, np.int64)
        self.data = data
        self._index = {int(b): i for i, b in enumerate(self.ids)}
        self._extra: dict[int, np.ndarray] = {}

    def __getitem__(self, blk):
        blk = int(blk)
        if not 0 <= blk < self.shape[0]:
            raise IndexError(f"physical block {blk} outside pool of {self.shape[0]}")
        i = self._index.get(blk)
        if i is not None:
            return self.data[i]
        extra = self._extra.get(blk)
        if extra is None:
            extra = np.full(self.shape[1:], POISON_BF16, np.uint16)
            self._extra[blk] = extra
        return extra

    def copy(self) -> "PagedPool":
        p = PagedPool(*self.shape, ids=self.ids.copy(), data=self.data.copy())
        p._extra = {k: v.copy() for k, v in self._extra.items()}
        return p

    def stored_blocks(self):
        """(ids, data) of every block that holds anything other than the NaN fill."""
        if not self._extra:
            return self.ids, self.data
        ex = sorted(self._extra)
        return (np.concatenate([self.ids, np.asarray(ex, np.int64)]),
                np.concatenate([self.data, np.stack([self._extra[k] for k in ex])]))

    def dense(self) -> np.ndarray:
        """The whole pool as one array (small pools only)."""
        full = np.full(self.shape, POISON_BF16, np.uint16)
        ids, data = self.stored_blocks()
        if len(ids):
            full[ids] = data
        return full

    @property
    def nbytes(self) -> int:
        return int(np.prod(self.shape)) * 2


@dataclass
class DecodeStep:
    """One decode step: store each sequence's newest token, then attend over its context."""

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: np.ndarray   # int32 [B]; counts the token stored by this step
    block_tables: np.ndarray   # int32 [B, max_blocks_per_seq]; unused entries are -1
    q: np.ndarray              # bf16 bits [B, Hq, D]
    k_new: np.ndarray          # bf16 bits [N, Hkv, D]
    v_new: np.ndarray          # bf16 bits [N, Hkv, D]
    slot_mapping: np.ndarray   # int32 [N]; -1 marks a padding token
    k_pool: PagedPool          # cache contents before the step
    v_pool: PagedPool
    shared_blocks: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int32))

    @property
    def batch(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.batch else 0


@dataclass
class PrefillStep:
    """One varlen prefill step: store the uncached suffix tokens, then causal attention."""

    name: str
    seed: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    seq_lens: np.ndarray       # int32 [B] total tokens per sequence (cached prefix + suffix)
    cached_blocks: np.ndarray  # int32 [B] leading blocks already in the cache
    cu_seqlens_q: np.ndarray   # int32 [B+1] over the suffix lengths
    cu_seqlens_k: np.ndarray   # int32 [B+1] over the total lengths
    block_tables: np.ndarray   # int32 [B, max_blocks_per_seq]; unused entries are -1
    q: np.ndarray              # bf16 bits [total_q, Hq, D]
    k_new: np.ndarray          # bf16 bits [total_q, Hkv, D]
    v_new: np.ndarray
    slot_mapping: np.ndarray   # int32 [total_q]
    k_pool: PagedPool
    v_pool: PagedPool

    @property
    def batch(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def max_seqlen_q(self) -> int:
        return int(np.diff(self.cu_seqlens_q).max()) if self.batch else 0

    @property
    def max_seqlen_k(self) -> int:
        return int(np.diff(self.cu_seqlens_k).max()) if self.batch else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])


# ----------------------------------------------------------------------------------
# shared helpers: block assignment and pool filling
# ----------------------------------------------------------------------------------

def _assign_blocks(rng, blocks_needed, num_blocks, shared_prefix_blocks=0, share=None):
    """Block tables from a shuffled pool.  Sequences flagged in `share` start with the
    same `shared_prefix_blocks` physical blocks (refcount > 1); all other blocks are
    private and drawn without reuse from one permutation of the pool."""
    B = len(blocks_needed)
    perm = rng.permutation(num_blocks).astype(np.int32)
    cursor = 0
    shared = perm[:shared_prefix_blocks].copy()
    cursor += shared_prefix_blocks
    width = max(1, int(max(blocks_needed))) if B else 1
    bt = np.full((B, width), -1, np.int32)
    for b in range(B):
        n = int(blocks_needed[b])
        start = 0
        if share is not None and share[b]:
            assert n > shared_prefix_blocks
            bt[b, :shared_prefix_blocks] = shared
            start = shared_prefix_blocks
        take = n - start
        if cursor + take > num_blocks:
            raise ValueError("pool too small for the requested sequences")
        bt[b, start:n] = perm[cursor:cursor + take]
        cursor += take
    return bt, shared


def _fill_pools(rng, block_tables, live_rows_fn, shape):
    """K and V pools holding N(0,1) bf16 rows where a live token sits, NaN elsewhere.

    live_rows_fn(b, j) gives how many leading rows of sequence b's j-th block hold a
    token that is already cached before the step.
    """
    num_blocks, bs, hkv, d = shape
    order = []
    live = {}
    for b in range(block_tables.shape[0]):
        for j, blk in enumerate(block_tables[b]):
            if blk < 0:
                continue
            blk = int(blk)
            n = int(live_rows_fn(b, j))
            if blk not in live:
                order.append(blk)
                live[blk] = n
            else:
                live[blk] = max(live[blk], n)
    ids = np.asarray(order, np.int64)
    pools = []
    for _ in range(2):
        data = _normal_bf16(rng, (len(ids), bs, hkv, d))
        for i, blk in enumerate(order):
            data[i, live[blk]:] = POISON_BF16
        pools.append(PagedPool(num_blocks, bs, hkv, d, ids=ids, data=data))
    return pools[0], pools[1]


def _slot(block_tables, b, pos, bs):
    return int(block_tables[b, pos // bs]) * bs + pos % bs


# ----------------------------------------------------------------------------------
# generic builders
# ----------------------------------------------------------------------------------

def _build_decode(rng, name, seed, context_lens, num_q_heads, num_kv_heads, head_dim,
                  block_size, num_blocks, shared_prefix_blocks=0, share=None,
                  pad_positions=(), q_mult=1.0, scale=None):
    ctx = np.asarray(context_lens, np.int64)
    B = len(ctx)
    bs = block_size
    need = np.maximum(1, -(-ctx // bs))
    if num_blocks is None:
        num_blocks = int(need.sum()) + 3
    bt, shared = _assign_blocks(rng, need, num_blocks, shared_prefix_blocks, share)
    q = _normal_bf16(rng, (B, num_q_heads, head_dim))
    if q_mult != 1.0:
        q = bf16_bits_from_f32(_f32_from_bf16_bits(q) * np.float32(q_mult))
    n_tok = B + len(pad_positions)
    k_new = _normal_bf16(rng, (n_tok, num_kv_heads, head_dim))
    v_new = _normal_bf16(rng, (n_tok, num_kv_heads, head_dim))
    # The newest token of sequence b sits at position ctx[b]-1; padding tokens get -1.
    real_slots = [(_slot(bt, b, int(ctx[b]) - 1, bs) if ctx[b] > 0 else -1) for b in range(B)]
    slots = []
    it = iter(real_slots)
    pads = set(int(p) for p in pad_positions)
    for t in range(n_tok):
        slots.append(-1 if t in pads else next(it))
    slot_mapping = np.asarray(slots, np.int32)

    def live(b, j):
        if share is not None and share[b] and j < shared_prefix_blocks:
            return bs
        return int(np.clip(ctx[b] - 1 - j * bs, 0, bs))

    k_pool, v_pool = _fill_pools(rng, bt, live, (num_blocks, bs, num_kv_heads, head_dim))
    return DecodeStep(
        name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=bs, num_blocks=num_blocks,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        context_lens=ctx.astype(np.int32), block_tables=bt, q=q, k_new=k_new, v_new=v_new,
        slot_mapping=slot_mapping, k_pool=k_pool, v_pool=v_pool,
        shared_blocks=np.asarray(shared, np.int32))


def make_decode_step(seed, context_lens, num_q_heads=4, num_kv_heads=2, head_dim=64,
                     block_size=16, num_blocks=None, shared_prefix_blocks=0, share=None,
                     pad_positions=(), q_mult=1.0, scale=None, name="decode"):
    """A decode step with explicit context lengths (small parity and edge cases)."""
    rng = np.random.default_rng(seed)
    return _build_decode(rng, name, seed, context_lens, num_q_heads, num_kv_heads, head_dim,
                         block_size, num_blocks, shared_prefix_blocks, share, pad_positions,
                         q_mult, scale)


def _build_prefill(rng, name, seed, seq_lens, cached_blocks, num_q_heads, num_kv_heads,
                   head_dim, block_size, num_blocks, scale=None):
    lens = np.asarray(seq_lens, np.int64)
    cached = np.asarray(cached_blocks, np.int64)
    bs = block_size
    B = len(lens)
    need = np.maximum(1, -(-lens // bs))
    if num_blocks is None:
        num_blocks = int(need.sum()) + 3
    bt, _ = _assign_blocks(rng, need, num_blocks)
    lq = lens - cached * bs
    assert (lq >= 0).all()
    cu_q = np.zeros(B + 1, np.int32)
    cu_q[1:] = np.cumsum(lq)
    cu_k = np.zeros(B + 1, np.int32)
    cu_k[1:] = np.cumsum(lens)
    total_q = int(cu_q[-1])
    q = _normal_bf16(rng, (total_q, num_q_heads, head_dim))
    k_new = _normal_bf16(rng, (total_q, num_kv_heads, head_dim))
    v_new = _normal_bf16(rng, (total_q, num_kv_heads, head_dim))
    slots = np.empty(total_q, np.int32)
    for i in range(B):
        for t in range(int(lq[i])):
            slots[cu_q[i] + t] = _slot(bt, i, int(cached[i]) * bs + t, bs)

    def live(b, j):
        return bs if j < cached[b] else 0

    k_pool, v_pool = _fill_pools(rng, bt, live, (num_blocks, bs, num_kv_heads, head_dim))
    return PrefillStep(
        name=name, seed=seed, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=bs, num_blocks=num_blocks,
        scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
        seq_lens=lens.astype(np.int32), cached_blocks=cached.astype(np.int32),
        cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, block_tables=bt, q=q, k_new=k_new, v_new=v_new,
        slot_mapping=slots, k_pool=k_pool, v_pool=v_pool)


def make_prefill_step(seed, seq_lens, cached_blocks=None, num_q_heads=4, num_kv_heads=2,
                      head_dim=64, block_size=16, num_blocks=None, scale=None, name="prefill"):
    """A prefill step with explicit lengths and cached-prefix block counts."""
    rng = np.random.default_rng(seed)
    if cached_blocks is None:
        cached_blocks = np.zeros(len(seq_lens), np.int64)
    return _build_prefill(rng, name, seed, seq_lens, cached_blocks, num_q_heads, num_kv_heads,
                          head_dim, block_size, num_blocks, scale)


# ----------------------------------------------------------------------------------
# the five named workloads
# ----------------------------------------------------------------------------------

def decode_tiny() -> DecodeStep:
    """Tiny decode step, seed 0: batch 4 with context lengths 17, 256, 300 and 700,
    block size 256, 4 query heads over 2 KV heads, head_dim 64, a 16-block pool in
    shuffled order, and one padding token (slot -1) after the four real tokens.  The
    700-token sequence is the three-block example of Nano-vLLM part 1, section 4.1."""
    rng = np.random.default_rng(0)
    return _build_decode(rng, "decode_tiny_b4", 0, [17, 256, 300, 700], 4, 2, 64, 256, 16,
                         pad_positions=(4,))


def decode_mid() -> DecodeStep:
    """Mid-size decode step, seed 1: batch 64, context lengths uniform in [512, 4096],
    block size 256, 16 query / 8 KV heads, head_dim 128, 2048-block shuffled pool."""
    rng = np.random.default_rng(1)
    ctx = rng.integers(512, 4097, size=64)
    return _build_decode(rng, "decode_mid_b64", 1, ctx, 16, 8, 128, 256, 2048)


def decode_batch512_shared_prefix() -> DecodeStep:
    """Large-batch decode with prefix sharing, seed 2: batch 512, context lengths
    lognormal (median 1024, sigma 0.75) clipped to [16, 4096]; a random half of the
    sequences start with the same 1024-token prefix held in 4 shared physical blocks
    (those sequences are lengthened to at least 1025 tokens so that their newest token
    lands in a private block); 16 query / 8 KV heads, head_dim 128, block size 256,
    16384-block shuffled pool."""
    rng = np.random.default_rng(2)
    z = rng.standard_normal(512)
    ctx = np.clip(np.rint(np.exp(math.log(1024.0) + 0.75 * z)), 16, 4096).astype(np.int64)
    share = np.zeros(512, bool)
    share[rng.permutation(512)[:256]] = True
    ctx[share] = np.maximum(ctx[share], 1025)
    return _build_decode(rng, "decode_b512_shared_prefix", 2, ctx, 16, 8, 128, 256, 16384,
                         shared_prefix_blocks=4, share=share)


def prefill_varlen_prefix_hits() -> PrefillStep:
    """Varlen causal prefill with prefix-cache hits, seed 3: 32 sequences with total
    lengths uniform in [64, 2048]; a random 16 of them have floor(floor(len/256)/2)
    leading blocks already cached; 16 query / 8 KV heads, head_dim 128, block size 256,
    512-block shuffled pool."""
    rng = np.random.default_rng(3)
    lens = rng.integers(64, 2049, size=32)
    cached = np.zeros(32, np.int64)
    hit = rng.permutation(32)[:16]
    cached[hit] = (lens[hit] // 256) // 2
    return _build_prefill(rng, "prefill_varlen_prefix_hits_b32", 3, lens, cached, 16, 8, 128,
                          256, 512)


def decode_long_fragmented() -> DecodeStep:
    """Long-context fragmented decode, seed 4: batch 8 with 32768 tokens each, block
    size 16 (2048 blocks per sequence taken from a shuffled 20000-block pool), 32 query
    / 8 KV heads (group 4), head_dim 128, Q scaled by 2."""
    rng = np.random.default_rng(4)
    return _build_decode(rng, "decode_long_b8_ctx32k_bs16", 4, [32768] * 8, 32, 8, 128, 16,
                         20000, q_mult=2.0)


def decode_graph_batch(batch: int):
    """Small captured-batch decode shapes (Nano-vLLM part 1, section 5.3 captures decode
    CUDA graphs for batch 1, 2, 4, 8, 16, ...): `batch` sequences of 4096 tokens (the
    largest context of the batch-512 workload), 16 query / 8 KV heads, head_dim 128,
    block size 256, shuffled pool with 16 spare blocks.  Seed 100 + batch.  Used to
    measure how the split-KV partitioning fills the GPU when the batch is small."""
    def make() -> DecodeStep:
        rng = np.random.default_rng(100 + batch)
        return _build_decode(rng, f"decode_graph_b{batch}_ctx4096", 100 + batch, [4096] * batch,
                             16, 8, 128, 256, batch * 16 + 16)
    return make


WORKLOADS = {
    "decode_tiny_b4": decode_tiny,
    "decode_mid_b64": decode_mid,
    "decode_b512_shared_prefix": decode_batch512_shared_prefix,
    "prefill_varlen_prefix_hits_b32": prefill_varlen_prefix_hits,
    "decode_long_b8_ctx32k_bs16": decode_long_fragmented,
    # measurement shapes beyond the five workloads: small captured decode batches
    "decode_graph_b1_ctx4096": decode_graph_batch(1),
    "decode_graph_b4_ctx4096": decode_graph_batch(4),
    "decode_graph_b16_ctx4096": decode_graph_batch(16),
}
