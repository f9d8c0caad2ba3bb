"""torch-tensor front end of the C ABI: argument marshalling only.

Each function checks dtypes/devices/shapes, allocates outputs the caller did not pass
(torch is the allocator), takes the current CUDA stream, and calls the C entry point of
the same name.  Every step of the computation runs in libnvpa's kernels.
"""

from __future__ import annotations

import torch

from ._lib import check, lib

_BF16 = torch.bfloat16
_I32 = torch.int32


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {t.dim()}")


def _contig(t, name):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cache_dims(k_cache, v_cache):
    _need(k_cache, _BF16, "k_cache", 4)
    _need(v_cache, _BF16, "v_cache", 4)
    _contig(k_cache, "k_cache")
    _contig(v_cache, "v_cache")
    if k_cache.shape != v_cache.shape:
        raise ValueError("k_cache and v_cache shapes differ")
    return tuple(int(x) for x in k_cache.shape)


def store_kvcache(k, v, k_cache, v_cache, slot_mapping, err_flag=None, stream=None):
    """Write k[t], v[t] ([N, Hkv, D] bf16, token stride may exceed Hkv*D) into the caches
    at slot_mapping[t]; slot -1 skips the token."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(k, _BF16, "k", 3)
    _need(v, _BF16, "v", 3)
    _need(slot_mapping, _I32, "slot_mapping", 1)
    _contig(slot_mapping, "slot_mapping")
    n = int(slot_mapping.shape[0])
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != (n, hkv, d):
            raise ValueError(f"{name} must be [{n}, {hkv}, {d}], got {tuple(t.shape)}")
        if t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{name}: heads and dims of a token must be contiguous")
    if err_flag is not None:
        _need(err_flag, _I32, "err_flag")
    st = lib().nvpa_store_kvcache(_ptr(k), _ptr(v), k.stride(0), v.stride(0), _ptr(k_cache),
                                  _ptr(v_cache), _ptr(slot_mapping), n, hkv, d, nb, bs,
                                  _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_store_kvcache")


def paged_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                block_size, num_splits=0) -> int:
    return int(lib().nvpa_paged_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                      max_context_len, block_size, num_splits))


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                           softmax_scale, out=None, lse=None, workspace=None, num_splits=0,
                           err_flag=None, stream=None, return_lse=False):
    """Decode attention: q [B, Hq, D] bf16, one query per sequence, keys 0..ctx-1 read
    through block_tables [B, max_blocks] (int32) and context_lens [B] (int32)."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(q, _BF16, "q", 3)
    _contig(q, "q")
    b, hq, dq = (int(x) for x in q.shape)
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    _need(block_tables, _I32, "block_tables", 2)
    _contig(block_tables, "block_tables")
    _need(context_lens, _I32, "context_lens", 1)
    _contig(context_lens, "context_lens")
    if block_tables.shape[0] != b or context_lens.shape[0] != b:
        raise ValueError("block_tables / context_lens batch differs from q's")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, _BF16, "out", 3)
        _contig(out, "out")
    if return_lse and lse is None:
        lse = torch.empty((b, hq), dtype=torch.float32, device=q.device)
    need = paged_decode_workspace_size(b, hq, hkv, d, max_context_len, bs, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().nvpa_paged_decode_attention(
        _ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(context_lens), b, hq, hkv, d, nb, bs,
        int(max_context_len), float(softmax_scale), int(num_splits), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_paged_decode_attention")
    return (out, lse) if return_lse else out


def decode_step(q, k_new, v_new, k_cache, v_cache, slot_mapping, block_tables, context_lens,
                max_context_len, softmax_scale, out=None, lse=None, workspace=None, num_splits=0,
                err_flag=None, stream=None, return_lse=False):
    """Store each sequence's new K/V row (k_new[b] -> slot_mapping[b]) and run decode
    attention over contexts that include it, in one call."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(q, _BF16, "q", 3)
    _contig(q, "q")
    b, hq, dq = (int(x) for x in q.shape)
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _need(t, _BF16, name, 3)
        if tuple(t.shape) != (b, hkv, d) or t.stride(2) != 1 or t.stride(1) != d:
            raise ValueError(f"{name} must be [{b}, {hkv}, {d}] with contiguous heads and dims")
    for name, t in (("slot_mapping", slot_mapping), ("block_tables", block_tables),
                    ("context_lens", context_lens)):
        _need(t, _I32, name)
        _contig(t, name)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((b, hq), dtype=torch.float32, device=q.device)
    need = paged_decode_workspace_size(b, hq, hkv, d, max_context_len, bs, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().nvpa_decode_step(
        _ptr(out), _ptr(lse), _ptr(q), _ptr(k_new), _ptr(v_new), k_new.stride(0), v_new.stride(0),
        _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(context_lens), b, hq, hkv, d, nb, bs,
        int(max_context_len), float(softmax_scale), int(num_splits), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_decode_step")
    return (out, lse) if return_lse else out


def decode_shared_prefix_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                        max_context_len, block_size, num_splits=0,
                                        min_group_size=0) -> int:
    return int(lib().nvpa_decode_shared_prefix_workspace_size(
        batch, num_q_heads, num_kv_heads, head_dim, max_context_len, block_size, num_splits,
        min_group_size))


def decode_step_shared_prefix(q, k_new, v_new, k_cache, v_cache, slot_mapping, block_tables,
                              context_lens, max_context_len, softmax_scale, out=None, lse=None,
                              workspace=None, num_splits=0, min_group_size=0, err_flag=None,
                              stream=None, return_lse=False):
    """decode_step (or, with k_new = v_new = slot_mapping = None, paged_decode_attention)
    with each group of sequences that share leading cache blocks attending its shared
    prefix once, on the tensor cores."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(q, _BF16, "q", 3)
    _contig(q, "q")
    b, hq, dq = (int(x) for x in q.shape)
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    store = k_new is not None
    if store != (v_new is not None) or store != (slot_mapping is not None):
        raise ValueError("k_new, v_new and slot_mapping must be given together")
    if store:
        for name, t in (("k_new", k_new), ("v_new", v_new)):
            _need(t, _BF16, name, 3)
            if tuple(t.shape) != (b, hkv, d) or t.stride(2) != 1 or t.stride(1) != d:
                raise ValueError(f"{name} must be [{b}, {hkv}, {d}] with contiguous heads and dims")
        _need(slot_mapping, _I32, "slot_mapping")
        _contig(slot_mapping, "slot_mapping")
    for name, t in (("block_tables", block_tables), ("context_lens", context_lens)):
        _need(t, _I32, name)
        _contig(t, name)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((b, hq), dtype=torch.float32, device=q.device)
    need = decode_shared_prefix_workspace_size(b, hq, hkv, d, max_context_len, bs, num_splits,
                                               min_group_size)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().nvpa_decode_step_shared_prefix(
        _ptr(out), _ptr(lse), _ptr(q), _ptr(k_new), _ptr(v_new),
        k_new.stride(0) if store else 0, v_new.stride(0) if store else 0,
        _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(context_lens), b, hq, hkv, d, nb, bs,
        int(max_context_len), float(softmax_scale), int(num_splits), int(min_group_size),
        _ptr(workspace), int(workspace.numel() * workspace.element_size()), _ptr(err_flag),
        _stream_handle(stream))
    check(st, "nvpa_decode_step_shared_prefix")
    return (out, lse) if return_lse else out


def varlen_prefill_workspace_size(batch, total_q) -> int:
    return int(lib().nvpa_varlen_prefill_workspace_size(batch, total_q))


def varlen_prefill_attention(q, k_cache, v_cache, block_tables, cu_seqlens_q, cu_seqlens_k,
                             max_seqlen_q, max_seqlen_k, softmax_scale, causal=True, out=None,
                             lse=None, workspace=None, err_flag=None, stream=None,
                             return_lse=False):
    """Varlen (prefix-cached) causal prefill: q [total_q, Hq, D] bf16; keys of sequence i
    are 0..Lk-1 read through block_tables[i]."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(q, _BF16, "q", 3)
    _contig(q, "q")
    total_q, hq, dq = (int(x) for x in q.shape)
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    for name, t in (("block_tables", block_tables), ("cu_seqlens_q", cu_seqlens_q),
                    ("cu_seqlens_k", cu_seqlens_k)):
        _need(t, _I32, name)
        _contig(t, name)
    batch = int(cu_seqlens_q.shape[0]) - 1
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((total_q, hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(varlen_prefill_workspace_size(batch, total_q), dtype=torch.uint8,
                                device=q.device)
    st = lib().nvpa_varlen_prefill_attention(
        _ptr(out), _ptr(lse), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), batch, total_q,
        int(max_seqlen_q), int(max_seqlen_k), hq, hkv, d, nb, bs, float(softmax_scale),
        1 if causal else 0, _ptr(workspace), int(workspace.numel() * workspace.element_size()),
        _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_varlen_prefill_attention")
    return (out, lse) if return_lse else out


def check_bounded_wait(err_flag, stream=None):
    """Run the bounded-wait check kernel (a wait that cannot complete); afterwards
    err_flag holds NVPA_FLAG_TIMEOUT."""
    _need(err_flag, _I32, "err_flag")
    check(lib().nvpa_check_bounded_wait(_ptr(err_flag), _stream_handle(stream)), "nvpa_check_bounded_wait")


def gather_kv(cache, block_tables, cu_seqlens_k, total_k, out=None, err_flag=None, stream=None):
    """Contiguous copy of each sequence's paged rows: [total_k, Hkv, D] bf16."""
    _need(cache, _BF16, "cache", 4)
    _contig(cache, "cache")
    nb, bs, hkv, d = (int(x) for x in cache.shape)
    _need(block_tables, _I32, "block_tables", 2)
    _need(cu_seqlens_k, _I32, "cu_seqlens_k", 1)
    if out is None:
        out = torch.empty((int(total_k), hkv, d), dtype=_BF16, device=cache.device)
    st = lib().nvpa_gather_kv(_ptr(out), _ptr(cache), _ptr(block_tables),
                              int(block_tables.shape[1]), _ptr(cu_seqlens_k),
                              int(cu_seqlens_k.shape[0]) - 1, int(total_k), hkv, d, nb, bs,
                              _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_gather_kv")
    return out


def paged_decode_partial(q, k_cache, v_cache, block_tables, context_lens, max_context_len,
                         softmax_scale, o_part=None, lse_part=None, workspace=None, num_splits=0,
                         err_flag=None, stream=None):
    """Decode attention over the keys this call sees, as a partial for lse_combine:
    (o_part [B, Hq, D] fp32 normalised over these keys, lse_part [B, Hq] fp32)."""
    nb, bs, hkv, d = _cache_dims(k_cache, v_cache)
    _need(q, _BF16, "q", 3)
    _contig(q, "q")
    b, hq, dq = (int(x) for x in q.shape)
    if dq != d:
        raise ValueError("q head_dim differs from the cache's")
    for name, t in (("block_tables", block_tables), ("context_lens", context_lens)):
        _need(t, _I32, name)
        _contig(t, name)
    if o_part is None:
        o_part = torch.empty((b, hq, d), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((b, hq), dtype=torch.float32, device=q.device)
    _need(o_part, torch.float32, "o_part", 3)
    _need(lse_part, torch.float32, "lse_part", 2)
    need = paged_decode_workspace_size(b, hq, hkv, d, max_context_len, bs, num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().nvpa_paged_decode_partial(
        _ptr(o_part), _ptr(lse_part), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(context_lens), b, hq, hkv, d, nb, bs,
        int(max_context_len), float(softmax_scale), int(num_splits), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _ptr(err_flag), _stream_handle(stream))
    check(st, "nvpa_paged_decode_partial")
    return o_part, lse_part


def lse_combine(o_parts, lse_parts, out=None, lse_out=None, stream=None, return_lse=False):
    """Merge partials over disjoint key sets: o_parts [R, B, Hq, D] fp32 and lse_parts
    [R, B, Hq] fp32 -> out [B, Hq, D] bf16 (and lse [B, Hq])."""
    _need(o_parts, torch.float32, "o_parts", 4)
    _need(lse_parts, torch.float32, "lse_parts", 3)
    _contig(o_parts, "o_parts")
    _contig(lse_parts, "lse_parts")
    r, b, hq, d = (int(x) for x in o_parts.shape)
    if tuple(lse_parts.shape) != (r, b, hq):
        raise ValueError(f"lse_parts must be [{r}, {b}, {hq}]")
    if out is None:
        out = torch.empty((b, hq, d), dtype=_BF16, device=o_parts.device)
    if return_lse and lse_out is None:
        lse_out = torch.empty((b, hq), dtype=torch.float32, device=o_parts.device)
    st = lib().nvpa_lse_combine(_ptr(out), _ptr(lse_out), _ptr(o_parts), _ptr(lse_parts), r, b, hq,
                                d, _stream_handle(stream))
    check(st, "nvpa_lse_combine")
    return (out, lse_out) if return_lse else out
