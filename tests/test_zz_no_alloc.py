"""nvpa_paged_decode_attention_static_scratch: decode without any device allocation.

It serves callers that cannot allocate device memory (a plugin whose host runtime owns
all device memory, or code where an allocation is not allowed).  The test calls it
through the C ABI twice in a row, on two different problems, and checks each output
against nvpa_paged_decode_attention with a caller-allocated workspace, within the
attention tolerance used by every parity test, and against the CPU oracle.  The second
call also shows that what the first call left in the shared scratch array does not leak
into the next result.  Once both problems have run (so every kernel of the path is
loaded), repeating both calls must leave the device's free memory unchanged: the entry
point allocates nothing.
This file is collected last so that a failure here cannot hide any other test.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_422_b200 as nvpa
from paged_kv_cache_422_b200 import _lib
from synth import decode_mid, make_decode_step
from synth.device import decode_to_device
from tests.helpers import (TOL_ABS, TOL_REL, assert_attention_close, assert_lse_close,
                           oracle_after_store)

import oracle

pytestmark = pytest.mark.gpu


def _static_scratch_call(step, t, out, lse, stream):
    lib = _lib.lib()
    return lib.nvpa_paged_decode_attention_static_scratch(
        out.data_ptr(), lse.data_ptr(), t["q"].data_ptr(), t["k_cache"].data_ptr(),
        t["v_cache"].data_ptr(), t["block_tables"].data_ptr(), int(t["block_tables"].shape[1]),
        t["context_lens"].data_ptr(), step.batch, step.num_q_heads, step.num_kv_heads,
        step.head_dim, step.num_blocks, step.block_size, step.max_context_len, float(step.scale),
        0, None, int(stream.cuda_stream))


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    return bool(np.all(np.abs(a - b) <= TOL_ABS + TOL_REL * np.abs(b)))


def test_static_scratch_matches_workspace_entry_twice(cuda_device):
    steps = [decode_mid(),
             make_decode_step(77, [5, 3000, 1, 257, 1800], num_q_heads=32, num_kv_heads=8,
                              head_dim=128, block_size=16)]
    stream = torch.cuda.current_stream(cuda_device)
    prepared = []
    for step in steps:
        t = decode_to_device(step, cuda_device)
        nvpa.store_kvcache(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], t["slot_mapping"])
        ref, ref_lse = nvpa.paged_decode_attention(
            t["q"], t["k_cache"], t["v_cache"], t["block_tables"], t["context_lens"],
            step.max_context_len, step.scale, return_lse=True)
        out = torch.full_like(t["q"], float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        st = _static_scratch_call(step, t, out, lse, stream)
        assert st == 0, _lib.lib().nvpa_last_error()
        torch.cuda.synchronize(cuda_device)
        assert _close(out, ref)
        assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), atol=2e-3)
        # and against the oracle itself, on every sequence
        kc, vc, _ = oracle_after_store(step)
        ora, ora_lse = oracle.paged_decode_attention(step.q, kc, vc, step.block_tables,
                                                     step.context_lens, step.scale)
        assert_attention_close(out, ora, "static scratch decode vs oracle")
        assert_lse_close(lse, ora_lse, "static scratch decode lse vs oracle")
        prepared.append((step, t, out, lse, ref))

    # every kernel of both problems is loaded now: repeating both calls allocates nothing
    torch.cuda.synchronize(cuda_device)
    free_before, _ = torch.cuda.mem_get_info(cuda_device)
    for step, t, out, lse, _ in prepared:
        assert _static_scratch_call(step, t, out, lse, stream) == 0, _lib.lib().nvpa_last_error()
    torch.cuda.synchronize(cuda_device)
    free_after, _ = torch.cuda.mem_get_info(cuda_device)
    assert free_after == free_before, f"device free memory changed by {free_before - free_after} B"
    for step, t, out, lse, ref in prepared:
        assert _close(out, ref)


def test_static_scratch_rejects_oversized_problem():
    lib = _lib.lib()
    # batch 1024 at 4096 keys with the default partitioning needs 97 MiB of the 64;
    # the size check happens before any device work, so null pointers are fine here
    assert nvpa.paged_decode_workspace_size(1024, 16, 8, 128, 4096, 256, 0) > 64 << 20
    st = lib.nvpa_paged_decode_attention_static_scratch(
        None, None, None, None, None, None, 16, None, 1024, 16, 8, 128, 16384, 256, 4096, 0.1, 0,
        None, None)
    assert st == _lib.NVPA_ERR_WORKSPACE_TOO_SMALL
    assert b"static scratch holds" in lib.nvpa_last_error()
