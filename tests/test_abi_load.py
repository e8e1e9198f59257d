"""The C-ABI library builds, loads and exports every symbol include/mla.h
declares (no GPU needed: only host-side entry points are called)."""
import ctypes
import os
import re

import pytest

from head_latent_attention_03_b200 import build, mla
from head_latent_attention_03_b200.inputs import TINY, LITE, V2

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "mla.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("mla_compress_append", "mla_absorb_q", "mla_decode_attn", "mla_prefill_attn", "mla_out_proj",
              "mla_workspace_size", "mla_get_last_error", "mla_status_string"):
        assert f in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_host_only_entry_points(lib):
    assert mla.version() >> 16 == 0
    assert mla.status_string(0) == "ok"
    assert "timed out" in mla.status_string(5)
    for dims in (TINY, LITE, V2):
        d = mla.layer_desc(dims)
        assert mla.workspace_size(d, 64, 64, 8256) > 0


def test_invalid_arguments_are_rejected_without_a_gpu(lib):
    d = mla.layer_desc(V2)
    w = mla.Weights()
    cache = mla.PagedCache()
    # null pointers: host validation returns before any CUDA call
    code = mla.lib().mla_compress_append(ctypes.byref(d), ctypes.byref(w), None, None, None, 4,
                                         ctypes.byref(cache), None, 0, None)
    assert code == 1
    bad = mla.layer_desc(V2)
    bad.d_hr = 63  # odd RoPE width
    assert mla.workspace_size(bad, 1, 1, 64) == 0
    # the wait probe's limit must lie in 1 ns .. 0.1 s; checked before any CUDA call
    assert mla.lib().mla_debug_wait_probe(0, None) == 1
    assert mla.lib().mla_debug_wait_probe(100_000_001, None) == 1


def test_fp8_cache_rows_and_limits_without_a_gpu(lib):
    import dataclasses
    assert mla.cache_row_bytes(mla.layer_desc(LITE)) == 1152
    assert mla.cache_row_bytes(mla.layer_desc(TINY)) == (TINY.d_c + TINY.d_hr) * 4
    fp8 = mla.layer_desc(dataclasses.replace(LITE, cache_dtype="fp8"))
    # 512 code bytes + 128 bytes of bf16 k^R + 4-byte scale, padded to 16 bytes
    assert mla.cache_row_bytes(fp8) == 656
    # FP8 rows need a bf16 layer: an fp32 layer with them is an invalid desc
    assert mla.cache_row_bytes(mla.layer_desc(dataclasses.replace(TINY, cache_dtype="fp8"))) == 0
    # the un-absorbed prefill decompresses bf16 rows only: refused on the
    # host, before any CUDA call (the pointers are never dereferenced)
    v2 = mla.layer_desc(dataclasses.replace(V2, cache_dtype="fp8"))
    cache = mla.PagedCache(16, 1, 16, 1)
    w = mla.Weights(*([16] * 10))
    code = mla.lib().mla_prefill_attn_unabsorbed(ctypes.byref(v2), ctypes.byref(w), 16, 16, ctypes.byref(cache),
                                                 16, 4, 1, 16, 1 << 20, 16, None, None)
    assert code == 2
    # encoding rows into the FP8 format needs a desc with FP8 rows
    assert mla.lib().mla_cache_quantize(ctypes.byref(mla.layer_desc(LITE)), 16, 1, 32, None) == 1


def declared_arity():
    """Number of parameters of every function include/mla.h declares."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(mla_[a-z_]+)\s*\(([^)]*)\)\s*;", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_marshals_every_declared_entry_point_with_its_arity():
    # the ctypes signatures in mla.py are the only marshalling layer: every
    # declared function must be bound, with exactly the header's parameters
    arity = declared_arity()
    assert set(arity) - set(mla._SIGS) == set(), set(arity) - set(mla._SIGS)
    for name, (_, argtypes) in mla._SIGS.items():
        assert name in arity, name
        assert len(argtypes) == arity[name], (name, len(argtypes), arity[name])
