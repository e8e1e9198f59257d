"""One MLA layer on the GPU: device buffers plus the C-ABI calls in step order.

    layer = MLALayer(dims, weights)                  # weights: numpy [out, in]
    state = layer.upload(batch)                      # cache pool, page table, h ...
    u = layer.step(state)    # append + queries -> attention (+ LSE combine) -> out_proj

Everything here is buffer management and argument marshalling; the
arithmetic runs in libmla_b200.so.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np
import torch

from . import mla


def prefill_flops(dims, prior_lens, q_per_seq: int) -> Dict[str, int]:
    """FLOPs of the attention of a prefill chunk in each form.

    Latent (absorbed) form: 2 n_h (2 d_c + d_h^R) per (query, key) pair.
    Un-absorbed form: 2 n_h (2 d_h + d_h^R) per pair, plus the decompression
    of every cached row of the chunk's sequences into per-head keys and values
    (2 * 2 n_h d_h d_c per row).
    """
    pairs = sum(int(L) * q_per_seq + q_per_seq * (q_per_seq + 1) // 2 for L in prior_lens)
    rows = sum(int(L) + q_per_seq for L in prior_lens)
    D = dims
    return {"absorbed": pairs * 2 * D.n_h * (2 * D.d_c + D.d_hr),
            "unabsorbed": pairs * 2 * D.n_h * (2 * D.d_h + D.d_hr) + rows * 4 * D.n_h * D.d_h * D.d_c}


def cheaper_prefill_form(dims, prior_lens, q_per_seq: int) -> str:
    """The form with fewer FLOPs for this chunk (bf16 layers with d_h = 128
    have both; others only the absorbed one)."""
    if dims.dtype != "bf16" or dims.d_h != 128:
        return "absorbed"
    f = prefill_flops(dims, prior_lens, q_per_seq)
    return "unabsorbed" if f["unabsorbed"] < f["absorbed"] else "absorbed"


def torch_dtype(dims) -> torch.dtype:
    return torch.bfloat16 if dims.dtype == "bf16" else torch.float32


def to_device(x: np.ndarray, dtype: torch.dtype, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device, dtype=dtype)


@dataclasses.dataclass
class DecodeState:
    """Device tensors of one decode (or prefill) step."""
    h: torch.Tensor            # [T, d]
    seq_idx: torch.Tensor      # [T] int32
    pos: torch.Tensor          # [T] int32
    kv_len: torch.Tensor       # [B] int32 (decode: prior + 1)
    q_start: torch.Tensor      # [B] int32 (first new position)
    pool: torch.Tensor         # [num_blocks, 64, d_c + d_hr]
    table: torch.Tensor        # [B, max_blocks] int32
    q_lat: torch.Tensor
    q_rope: torch.Tensor
    o_lat: torch.Tensor
    lse: torch.Tensor
    u: torch.Tensor
    ws: torch.Tensor
    new_per_seq: int


class MLALayer:
    def __init__(self, dims, weights: Dict[str, Optional[np.ndarray]], device: str = "cuda"):
        self.dims = dims
        self.device = device
        self.desc = mla.layer_desc(dims)
        dt = torch_dtype(dims)
        self.w = {k: (None if v is None else to_device(v, dt, device)) for k, v in weights.items()}
        self.cw = mla.weights(self.w)

    def alloc(self, T: int, B: int, pool: torch.Tensor, table: torch.Tensor, h: torch.Tensor,
              seq_idx: torch.Tensor, pos: torch.Tensor, kv_len: torch.Tensor, q_start: torch.Tensor,
              new_per_seq: int) -> DecodeState:
        D, dev, dt = self.dims, self.device, torch_dtype(self.dims)
        rows = T
        ws_bytes = mla.workspace_size(self.desc, T, rows, table.shape[1] * D.block_size)
        return DecodeState(
            h=h, seq_idx=seq_idx, pos=pos, kv_len=kv_len, q_start=q_start, pool=pool, table=table,
            q_lat=torch.empty((rows, D.n_h, D.d_c), dtype=dt, device=dev),
            q_rope=torch.empty((rows, D.n_h, D.d_hr), dtype=dt, device=dev),
            o_lat=torch.empty((rows, D.n_h, D.d_c), dtype=dt, device=dev),
            lse=torch.empty((rows, D.n_h), dtype=torch.float32, device=dev),
            u=torch.empty((rows, D.d), dtype=torch.float32, device=dev),
            ws=torch.empty((max(ws_bytes, 256),), dtype=torch.uint8, device=dev),
            new_per_seq=new_per_seq)

    def upload(self, batch) -> DecodeState:
        """Copy a host Batch (inputs.gen_batch) to the device."""
        D, dev, dt = self.dims, self.device, torch_dtype(self.dims)
        new = batch.workload.new_tokens
        pool = to_device(batch.pool, dt, dev)
        if getattr(D, "cache_dtype", "bf16") == "fp8":
            # the drawn rows, encoded on the device into the FP8 row format
            rows = pool
            pool = torch.empty((rows.shape[0], rows.shape[1], mla.cache_row_bytes(self.desc)), dtype=torch.uint8,
                               device=dev)
            mla.cache_quantize(self.desc, rows, pool)
            del rows
        table = torch.from_numpy(batch.block_table).to(dev)
        h = to_device(batch.h, dt, dev)
        seq_idx = torch.from_numpy(batch.seq_idx.astype(np.int32)).to(dev)
        pos = torch.from_numpy(batch.positions.astype(np.int32)).to(dev)
        kv_len = torch.from_numpy((batch.prior_len + 1).astype(np.int32)).to(dev)
        q_start = torch.from_numpy(batch.prior_len.astype(np.int32)).to(dev)
        return self.alloc(h.shape[0], len(batch.prior_len), pool, table, h, seq_idx, pos, kv_len, q_start, new)

    def cache(self, st: DecodeState) -> mla.PagedCache:
        return mla.paged_cache(st.pool, st.table)

    # the four hot-path steps -------------------------------------------------
    def compress_append(self, st: DecodeState, stream=None):
        mla.compress_append(self.desc, self.cw, st.h, st.seq_idx, st.pos, self.cache(st), st.ws, stream)

    def absorb_q(self, st: DecodeState, stream=None):
        mla.absorb_q(self.desc, self.cw, st.h, st.pos, st.q_lat, st.q_rope, st.ws, stream)

    def attend(self, st: DecodeState, num_splits: int = 0, stream=None):
        if st.new_per_seq == 1:
            mla.decode_attn(self.desc, st.q_lat, st.q_rope, self.cache(st), st.kv_len, st.ws, st.o_lat, st.lse,
                            num_splits, stream)
        else:
            mla.prefill_attn(self.desc, st.q_lat, st.q_rope, self.cache(st), st.q_start, st.new_per_seq, st.ws,
                             st.o_lat, st.lse, stream)

    def out_proj(self, st: DecodeState, stream=None):
        mla.out_proj(self.desc, self.cw, st.o_lat, st.u, st.ws, stream)

    def compress_append_absorb_q(self, st: DecodeState, stream=None):
        mla.compress_append_absorb_q(self.desc, self.cw, st.h, st.seq_idx, st.pos, self.cache(st), st.q_lat,
                                     st.q_rope, st.ws, stream)

    def step(self, st: DecodeState, num_splits: int = 0, stream=None) -> torch.Tensor:
        """One whole layer step: append and queries (one call), attention,
        output projection."""
        self.compress_append_absorb_q(st, stream)
        self.attend(st, num_splits, stream)
        self.out_proj(st, stream)
        return st.u

    # un-absorbed chunked prefill ---------------------------------------------
    def prefill_buffers(self, st: DecodeState):
        """q^C, per-head o and the decompression workspace of the un-absorbed form."""
        D, dev = self.dims, self.device
        T = st.h.shape[0]
        if not hasattr(st, "q_c"):
            st.q_c = torch.empty((T, D.n_h, D.d_h), dtype=torch.bfloat16, device=dev)
            st.o = torch.empty((T, D.n_h, D.d_h), dtype=torch.bfloat16, device=dev)
            ws = mla.prefill_unabsorbed_workspace_size(self.desc, st.pool.shape[0], st.table.shape[0],
                                                       st.table.shape[1])
            st.ws_pf = torch.empty((ws,), dtype=torch.uint8, device=dev)
        return st

    def prefill_step_unabsorbed(self, st: DecodeState, stream=None) -> torch.Tensor:
        """Append, queries without absorption, un-absorbed causal attention, W^O."""
        self.prefill_buffers(st)
        self.compress_append(st, stream)
        mla.queries(self.desc, self.cw, st.h, st.pos, st.q_c, st.q_rope, st.ws, stream)
        mla.prefill_attn_unabsorbed(self.desc, self.cw, st.q_c, st.q_rope, self.cache(st), st.q_start,
                                    st.new_per_seq, st.ws_pf, st.o, st.lse, stream)
        mla.out_proj_unabsorbed(self.desc, self.cw, st.o, st.u, stream)
        return st.u
