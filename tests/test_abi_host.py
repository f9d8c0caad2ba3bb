"""The C ABI on the host (no GPU needed): the library loads, exports every function the
headers declare, and rejects bad arguments before touching the device."""

import ctypes
import glob
import os
import re

import pytest

from paged_kv_cache_422_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(nvpa_[a-z0-9_]+)\s*\(", text):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_422_b200.build import build
    build()
    return _lib.lib()


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert {"nvpa_store_kvcache", "nvpa_paged_decode_attention", "nvpa_varlen_prefill_attention",
            "nvpa_paged_decode_workspace_size", "nvpa_gather_kv"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(_lib.SIGNATURES), "binding signatures out of step with the header"


def test_status_strings(lib):
    assert lib.nvpa_status_string(0) == b"NVPA_OK"
    assert lib.nvpa_status_string(4) == b"NVPA_ERR_WORKSPACE_TOO_SMALL"
    assert lib.nvpa_version() >= 100


def test_workspace_size_is_host_only_and_monotone(lib):
    f = lib.nvpa_paged_decode_workspace_size
    small = f(64, 16, 8, 128, 256, 256, 0)
    big = f(64, 16, 8, 128, 4096, 256, 0)
    assert 0 < small < big
    assert f(512, 16, 8, 128, 4096, 256, 1) < big      # one split: no partials
    assert f(-1, 16, 8, 128, 4096, 256, 0) == 0


FAKE = 0x10000  # 256-byte aligned fake device address; never dereferenced by these calls


def _decode(lib, **kw):
    a = dict(out=FAKE, lse=None, q=FAKE, k=FAKE, v=FAKE, bt=FAKE, maxblk=4, ctx=FAKE, batch=2,
             hq=8, hkv=2, d=128, nb=16, bs=16, maxctx=64, scale=0.1, ns=0, ws=FAKE, wsb=1 << 20)
    a.update(kw)
    return lib.nvpa_paged_decode_attention(a["out"], a["lse"], a["q"], a["k"], a["v"], a["bt"],
                                           a["maxblk"], a["ctx"], a["batch"], a["hq"], a["hkv"],
                                           a["d"], a["nb"], a["bs"], a["maxctx"], a["scale"],
                                           a["ns"], a["ws"], a["wsb"], None, None)


def test_decode_host_checks(lib):
    assert _decode(lib, d=96) == _lib.NVPA_ERR_UNSUPPORTED
    assert _decode(lib, bs=8) == _lib.NVPA_ERR_UNSUPPORTED
    assert _decode(lib, hq=6, hkv=4) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, hq=18, hkv=2) == _lib.NVPA_ERR_UNSUPPORTED
    assert _decode(lib, q=None) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, q=FAKE + 8) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, ws=FAKE + 16) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, scale=float("nan")) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, batch=-1) == _lib.NVPA_ERR_INVALID_ARG
    assert _decode(lib, batch=0) == _lib.NVPA_OK
    assert _decode(lib, maxctx=100000, wsb=16) == _lib.NVPA_ERR_WORKSPACE_TOO_SMALL
    assert b"workspace" in lib.nvpa_last_error()


def test_store_host_checks(lib):
    def st(**kw):
        a = dict(k=FAKE, v=FAKE, ks=256, vs=256, kc=FAKE, vc=FAKE, slots=FAKE, n=4, hkv=2, d=128,
                 nb=8, bs=16)
        a.update(kw)
        return lib.nvpa_store_kvcache(a["k"], a["v"], a["ks"], a["vs"], a["kc"], a["vc"],
                                      a["slots"], a["n"], a["hkv"], a["d"], a["nb"], a["bs"],
                                      None, None)
    assert st(n=-1) == _lib.NVPA_ERR_INVALID_ARG
    assert st(n=0, k=None) == _lib.NVPA_OK
    assert st(ks=255) == _lib.NVPA_ERR_INVALID_ARG
    assert st(ks=128) == _lib.NVPA_ERR_INVALID_ARG
    assert st(d=100) == _lib.NVPA_ERR_INVALID_ARG
    assert st(kc=FAKE + 2) == _lib.NVPA_ERR_INVALID_ARG
    assert st(nb=1 << 24, bs=1 << 8) == _lib.NVPA_ERR_UNSUPPORTED


def test_prefill_host_checks(lib):
    def pf(**kw):
        a = dict(batch=2, total_q=10, mq=8, mk=8, hq=4, hkv=2, d=64, nb=8, bs=16, causal=1,
                 q=FAKE, ws=FAKE)
        a.update(kw)
        return lib.nvpa_varlen_prefill_attention(FAKE, None, a["q"], FAKE, FAKE, FAKE, 2, FAKE,
                                                 FAKE, a["batch"], a["total_q"], a["mq"], a["mk"],
                                                 a["hq"], a["hkv"], a["d"], a["nb"], a["bs"], 0.1,
                                                 a["causal"], a["ws"], 1 << 20, None, None)
    assert pf(causal=2) == _lib.NVPA_ERR_INVALID_ARG
    assert pf(d=256) == _lib.NVPA_ERR_UNSUPPORTED
    assert pf(total_q=0) == _lib.NVPA_OK
    assert pf(q=None) == _lib.NVPA_ERR_INVALID_ARG
    assert pf(total_q=-3) == _lib.NVPA_ERR_INVALID_ARG
    assert pf(ws=None) == _lib.NVPA_ERR_INVALID_ARG
    assert pf(ws=FAKE + 64) == _lib.NVPA_ERR_INVALID_ARG
    assert lib.nvpa_varlen_prefill_workspace_size(32, 24594) >= 256 + 16 * (32 + 24594 // 128)


def test_prefill_workspace_holds_every_plan_entry(lib):
    """The prefill plan writes one 16-byte entry per pair of query tiles after a 256-byte
    header; a tile is 128 / P tokens of one sequence (P = 1, 2, 4 or 8 query heads per
    tile).  The size query, which sees only the batch and the query rows, must cover the
    largest pair count any layout of those rows can give."""
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(300):
        batch = int(rng.integers(1, 400))
        kind = rng.integers(0, 3)
        if kind == 0:
            lq = rng.integers(0, 3, size=batch)                 # empty and one-token rows
        elif kind == 1:
            lq = rng.choice([1, 15, 16, 17, 31, 33], size=batch)
        else:
            lq = rng.integers(0, 5000, size=batch)
        total_q = int(lq.sum())
        size = lib.nvpa_varlen_prefill_workspace_size(batch, total_q)
        for tq in (128, 64, 32, 16):
            tiles = -(-lq // tq)
            pairs = int(((tiles + 1) // 2).sum())
            assert size >= 256 + 16 * pairs, (batch, total_q, tq, pairs, size)


def test_gather_host_checks(lib):
    f = lib.nvpa_gather_kv
    assert f(FAKE, FAKE, FAKE, 4, FAKE, 2, 10, 2, 64, 8, 24, None, None) == _lib.NVPA_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 4, FAKE, 2, 0, 2, 64, 8, 16, None, None) == _lib.NVPA_OK
    assert f(None, FAKE, FAKE, 4, FAKE, 2, 10, 2, 64, 8, 16, None, None) == _lib.NVPA_ERR_INVALID_ARG


def test_bounded_wait_check_host_checks(lib):
    # a null error word is refused before anything is launched
    assert lib.nvpa_check_bounded_wait(None, None) == _lib.NVPA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()
