"""ctypes binding of libmla_b200.so (include/mla.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (device memory and streams come
from PyTorch); their data pointers and the current stream are handed to the C
ABI.  A missing library raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmla_b200.so")

MLA_F32, MLA_BF16 = 0, 1
MLA_CACHE_NATIVE, MLA_CACHE_FP8_E4M3 = 0, 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_CAPACITY",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_TIMEOUT"}


class MLAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)}")
        self.code = code


class LayerDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_c", ctypes.c_int),
                ("d_cq", ctypes.c_int), ("d_hr", ctypes.c_int), ("block_size", ctypes.c_int),
                ("dtype", ctypes.c_int), ("rope_base", ctypes.c_double), ("yarn_scale", ctypes.c_double),
                ("yarn_orig_ctx", ctypes.c_int), ("yarn_alpha", ctypes.c_double), ("yarn_beta", ctypes.c_double),
                ("attn_logit_factor", ctypes.c_double), ("latent_norm", ctypes.c_int), ("norm_eps", ctypes.c_double),
                ("scale_kv", ctypes.c_double), ("scale_q", ctypes.c_double), ("cache_dtype", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_dkv", "w_kr", "w_dq", "w_uq", "w_qr", "w_uk", "w_uv", "w_o",
                                                "g_kv", "g_q")]


class PagedCache(ctypes.Structure):
    _fields_ = [("pool", ctypes.c_void_p), ("num_blocks", ctypes.c_int), ("block_table", ctypes.c_void_p),
                ("max_blocks", ctypes.c_int)]


_lib: Optional[ctypes.CDLL] = None

_SIGS = {
    "mla_version": (ctypes.c_int, []),
    "mla_launch_count": (ctypes.c_ulonglong, []),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(LayerDesc), ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "mla_compress_append": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                           ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p]),
    "mla_absorb_q": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights), ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mla_decode_attn": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                       ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p]),
    "mla_decode_attn_noalloc": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "mla_prefill_attn": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p]),
    "mla_decode_attn_partial": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_void_p]),
    "mla_lse_merge": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "mla_out_proj": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights), ctypes.c_void_p,
                                    ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                    ctypes.c_void_p]),
    "mla_get_last_error": (ctypes.c_int, [ctypes.c_void_p]),
    "mla_prefill_unabsorbed_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(LayerDesc), ctypes.c_int,
                                                                ctypes.c_int, ctypes.c_int]),
    "mla_queries": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights), ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_size_t, ctypes.c_void_p]),
    "mla_prefill_attn_unabsorbed": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights),
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(PagedCache),
                                                   ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                                   ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p,
                                                   ctypes.c_void_p]),
    "mla_out_proj_unabsorbed": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights), ctypes.c_void_p,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "mla_cache_row_bytes": (ctypes.c_size_t, [ctypes.POINTER(LayerDesc)]),
    "mla_debug_attention_events": (None, [ctypes.c_void_p, ctypes.c_void_p]),
    "mla_debug_wait_probe": (ctypes.c_int, [ctypes.c_longlong, ctypes.c_void_p]),
    "mla_compress_append_absorb_q": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(Weights),
                                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                                    ctypes.POINTER(PagedCache), ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "mla_cache_quantize": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.c_void_p, ctypes.c_longlong,
                                          ctypes.c_void_p, ctypes.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """Load libmla_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m head_latent_attention_03_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(fn: str, code: int):
    if code != 0:
        raise MLAError(fn, code)


def layer_desc(dims) -> LayerDesc:
    """LayerDesc from any object with the mla_layer_desc field names (e.g. inputs.LayerDims)."""
    return LayerDesc(dims.d, dims.n_h, dims.d_h, dims.d_c, dims.d_cq, dims.d_hr, dims.block_size,
                     MLA_BF16 if dims.dtype == "bf16" else MLA_F32, dims.rope_base, dims.yarn_scale,
                     dims.yarn_orig_ctx, dims.yarn_alpha, dims.yarn_beta, dims.attn_logit_factor,
                     int(getattr(dims, "latent_norm", False)), getattr(dims, "norm_eps", 0.0),
                     getattr(dims, "scale_kv", 1.0), getattr(dims, "scale_q", 1.0),
                     MLA_CACHE_FP8_E4M3 if getattr(dims, "cache_dtype", "bf16") == "fp8" else MLA_CACHE_NATIVE)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def weights(w: dict) -> Weights:
    return Weights(*[_ptr(w.get(n)) for n in ("w_dkv", "w_kr", "w_dq", "w_uq", "w_qr", "w_uk", "w_uv", "w_o",
                                               "g_kv", "g_q")])


def paged_cache(pool, block_table) -> PagedCache:
    return PagedCache(pool.data_ptr(), pool.shape[0], block_table.data_ptr(), block_table.shape[1])


def version() -> int:
    return lib().mla_version()


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return lib().mla_launch_count()


def status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def debug_attention_events(before=None, after=None):
    """Record torch.cuda.Event `before` / `after` around every attention kernel
    from now on (None, None: stop).  The events must have been recorded once
    (so that they exist)."""
    lib().mla_debug_attention_events(before.cuda_event if before is not None else None,
                                     after.cuda_event if after is not None else None)


def debug_wait_probe(limit_ns: int, stream=None) -> int:
    """Run one bounded wait that nothing completes, under a wait limit of
    limit_ns; returns the call's status (the timeout is read with
    get_last_error)."""
    return lib().mla_debug_wait_probe(int(limit_ns), _stream(stream))


def cache_row_bytes(desc: LayerDesc) -> int:
    return lib().mla_cache_row_bytes(ctypes.byref(desc))


def cache_quantize(desc, src, dst, stream=None):
    """bf16 cache rows src [..., d_c + d_hr] -> FP8 rows dst [..., cache_row_bytes] (uint8)."""
    n = src.numel() // (desc.d_c + desc.d_hr)
    _check("mla_cache_quantize", lib().mla_cache_quantize(ctypes.byref(desc), _ptr(src), n, _ptr(dst),
                                                          _stream(stream)))


def workspace_size(desc: LayerDesc, T: int, B: int, max_kv_len: int) -> int:
    return lib().mla_workspace_size(ctypes.byref(desc), T, B, max_kv_len)


def compress_append(desc, w: Weights, h, seq_idx, pos, cache: PagedCache, ws, stream=None):
    _check("mla_compress_append", lib().mla_compress_append(
        ctypes.byref(desc), ctypes.byref(w), _ptr(h), _ptr(seq_idx), _ptr(pos), h.shape[0], ctypes.byref(cache),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def compress_append_absorb_q(desc, w: Weights, h, seq_idx, pos, cache: PagedCache, q_lat, q_rope, ws, stream=None):
    _check("mla_compress_append_absorb_q", lib().mla_compress_append_absorb_q(
        ctypes.byref(desc), ctypes.byref(w), _ptr(h), _ptr(seq_idx), _ptr(pos), h.shape[0], ctypes.byref(cache),
        _ptr(q_lat), _ptr(q_rope), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
        _stream(stream)))


def absorb_q(desc, w: Weights, h, pos, q_lat, q_rope, ws, stream=None):
    _check("mla_absorb_q", lib().mla_absorb_q(
        ctypes.byref(desc), ctypes.byref(w), _ptr(h), _ptr(pos), h.shape[0], _ptr(q_lat), _ptr(q_rope),
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def decode_attn(desc, q_lat, q_rope, cache: PagedCache, kv_len, ws, o_lat, lse=None, num_splits=0, stream=None):
    _check("mla_decode_attn", lib().mla_decode_attn(
        ctypes.byref(desc), _ptr(q_lat), _ptr(q_rope), ctypes.byref(cache), _ptr(kv_len), kv_len.shape[0],
        _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, num_splits, _ptr(o_lat), _ptr(lse),
        _stream(stream)))


def decode_attn_noalloc(desc, q_lat, q_rope, cache: PagedCache, kv_len, o_lat, lse=None, num_splits=0, stream=None):
    """mla_decode_attn with the library's own fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check("mla_decode_attn_noalloc", lib().mla_decode_attn_noalloc(
        ctypes.byref(desc), _ptr(q_lat), _ptr(q_rope), ctypes.byref(cache), _ptr(kv_len), kv_len.shape[0],
        num_splits, _ptr(o_lat), _ptr(lse), _stream(stream)))


def decode_attn_partial(desc, q_lat, q_rope, cache: PagedCache, kv_begin, kv_end, ws, o_part, lse_part,
                        stream=None):
    """Attention over rows [kv_begin, kv_end) of each sequence: fp32 o_part
    (normalised within the range) and lse_part, for a context-parallel merge."""
    _check("mla_decode_attn_partial", lib().mla_decode_attn_partial(
        ctypes.byref(desc), _ptr(q_lat), _ptr(q_rope), ctypes.byref(cache), _ptr(kv_begin), _ptr(kv_end),
        kv_end.shape[0], _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _ptr(o_part),
        _ptr(lse_part), _stream(stream)))


def lse_merge(desc, o_parts, lse_parts, o_lat, lse=None, stream=None):
    """Merge R partials o_parts [R, B, n_h, d_c], lse_parts [R, B, n_h] into o_lat, lse."""
    _check("mla_lse_merge", lib().mla_lse_merge(
        ctypes.byref(desc), _ptr(o_parts), _ptr(lse_parts), o_parts.shape[0], o_parts.shape[1], _ptr(o_lat),
        _ptr(lse), _stream(stream)))


def prefill_attn(desc, q_lat, q_rope, cache: PagedCache, q_start, q_per_seq, ws, o_lat, lse=None, stream=None):
    _check("mla_prefill_attn", lib().mla_prefill_attn(
        ctypes.byref(desc), _ptr(q_lat), _ptr(q_rope), ctypes.byref(cache), _ptr(q_start), q_per_seq,
        q_start.shape[0], _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _ptr(o_lat),
        _ptr(lse), _stream(stream)))


def out_proj(desc, w: Weights, o_lat, u, ws, stream=None):
    _check("mla_out_proj", lib().mla_out_proj(
        ctypes.byref(desc), ctypes.byref(w), _ptr(o_lat), o_lat.shape[0], _ptr(u), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def prefill_unabsorbed_workspace_size(desc: LayerDesc, num_blocks: int, B: int, max_blocks: int) -> int:
    return lib().mla_prefill_unabsorbed_workspace_size(ctypes.byref(desc), num_blocks, B, max_blocks)


def queries(desc, w: Weights, h, pos, q_c, q_rope, ws, stream=None):
    """q^C [T, n_h, d_h] and RoPE'd q^R [T, n_h, d_hr] without the W^UK absorption."""
    _check("mla_queries", lib().mla_queries(
        ctypes.byref(desc), ctypes.byref(w), _ptr(h), _ptr(pos), h.shape[0], _ptr(q_c), _ptr(q_rope), _ptr(ws),
        ws.numel() * ws.element_size() if ws is not None else 0, _stream(stream)))


def prefill_attn_unabsorbed(desc, w: Weights, q_c, q_rope, cache: PagedCache, q_start, q_per_seq, ws, o, lse=None,
                            stream=None):
    """Causal attention of a prefill chunk with decompressed per-head keys and values: o [T, n_h, d_h]."""
    _check("mla_prefill_attn_unabsorbed", lib().mla_prefill_attn_unabsorbed(
        ctypes.byref(desc), ctypes.byref(w), _ptr(q_c), _ptr(q_rope), ctypes.byref(cache), _ptr(q_start), q_per_seq,
        q_start.shape[0], _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0, _ptr(o), _ptr(lse),
        _stream(stream)))


def out_proj_unabsorbed(desc, w: Weights, o, u, stream=None):
    """u = W^O o for per-head outputs o [T, n_h, d_h]."""
    _check("mla_out_proj_unabsorbed", lib().mla_out_proj_unabsorbed(
        ctypes.byref(desc), ctypes.byref(w), _ptr(o), o.shape[0], _ptr(u), _stream(stream)))


def get_last_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status code."""
    return lib().mla_get_last_error(_stream(stream))
