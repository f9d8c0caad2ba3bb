"""Shared helpers for the GPU parity tests (comparison rules and oracle runs)."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from synth.device import bits_of, pool_to_device

# Attention outputs: bf16 out, fp32 accumulation, against the float64 oracle.
TOL_ABS = 1e-2
TOL_REL = 1e-2
# Log-sum-exp is returned in float32; its error is that of the fp32 score sums.
LSE_TOL = 2e-3


def assert_attention_close(gpu_out: torch.Tensor, ora: np.ndarray, what: str):
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    assert g.shape == ora.shape, f"{what}: shape {g.shape} vs {ora.shape}"
    err = np.abs(g - ora)
    bound = TOL_ABS + TOL_REL * np.abs(ora)
    bad = ~(err <= bound)          # NaN counts as bad
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(np.isnan(err), np.inf, err)), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside "
                             f"{TOL_ABS} + {TOL_REL}|ref|; worst at {i}: gpu {g[i]} ref {ora[i]}")


def assert_lse_close(gpu_lse: torch.Tensor, ora: np.ndarray, what: str):
    g = gpu_lse.detach().cpu().numpy().astype(np.float64)
    both_inf = np.isneginf(g) & np.isneginf(ora)
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(g - ora))
    bad = ~(err <= LSE_TOL * (1 + np.abs(np.where(np.isfinite(ora), ora, 0))))
    assert not bad.any(), f"{what}: lse mismatch at {np.argwhere(bad)[:5].tolist()}"


def oracle_after_store(step):
    """The oracle's pools after the step's store (copies of the step's pools)."""
    kc, vc = step.k_pool.copy(), step.v_pool.copy()
    bad = oracle.store_kvcache(kc, vc, step.k_new, step.v_new, step.slot_mapping)
    return kc, vc, bad


def assert_pool_equal(gpu_pool: torch.Tensor, ora_pool, what: str):
    """Bit-exact comparison of a whole device pool with the oracle's pool contents."""
    expect = pool_to_device(ora_pool, gpu_pool.device)
    a = gpu_pool.view(torch.int16)
    b = expect.view(torch.int16)
    nb = a.shape[0]
    step = 1024
    for i in range(0, nb, step):
        if not torch.equal(a[i:i + step], b[i:i + step]):
            diff = (a[i:i + step] != b[i:i + step]).nonzero()
            raise AssertionError(f"{what}: pool differs, first at {(diff[0] + torch.tensor([i, 0, 0, 0], device=diff.device)).tolist()}")
    del expect


def cu_from_lens(lens) -> np.ndarray:
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    return cu


def gathered_bits(t: torch.Tensor) -> np.ndarray:
    return bits_of(t)
