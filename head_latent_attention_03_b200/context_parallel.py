"""Context parallelism for long decodes: one sequence's cached rows spread
over the ranks of a process group, merged by log-sum-exp.

With 128K-token contexts (the YaRN setting of the DeepSeek-V2 explainer,
section 3.1.3) a single sequence's latent cache can be split across GPUs.
Each rank holds the pages of a contiguous, tile-aligned range of rows and
computes the attention of every head over its rows only
(mla_decode_attn_partial: fp32 output normalised within the range plus its
log-sum-exp).  The ranks exchange these partials — n_h * (d_c + 1) floats
per sequence and rank, one all-gather — and every rank merges them
(mla_lse_merge), which gives exactly the attention over all rows.

Host logic only: the arithmetic runs in libmla_b200.so; torch.distributed
(NCCL between GPUs) carries the exchange.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from . import mla

TILE = 128  # rows per attention tile: range boundaries fall on tiles


def shard_ranges(kv_len: Sequence[int], world: int, align: int = TILE) -> np.ndarray:
    """[world, B, 2] int32: rank r attends rows [begin, end) of sequence b.

    The ranges of a sequence are contiguous, in rank order, cover [0, kv_len),
    start on multiples of `align`, and differ in size by at most one tile
    (trailing ranks may be empty for short sequences).
    """
    kv = np.asarray(kv_len, dtype=np.int64)
    out = np.zeros((world, len(kv), 2), dtype=np.int32)
    for b, L in enumerate(kv):
        tiles = -(-int(L) // align)
        for r in range(world):
            t0, t1 = r * tiles // world, (r + 1) * tiles // world
            out[r, b, 0] = min(t0 * align, int(L))
            out[r, b, 1] = min(t1 * align, int(L))
    return out


def gather_partials(o_part, lse_part, group=None) -> Tuple["object", "object"]:
    """All-gather every rank's (o_part [B, n_h, d_c], lse_part [B, n_h]) into
    rank-major tensors [world, ...] (the layout mla_lse_merge reads)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    os_ = [torch.empty_like(o_part) for _ in range(world)]
    ls_ = [torch.empty_like(lse_part) for _ in range(world)]
    dist.all_gather(os_, o_part.contiguous(), group=group)
    dist.all_gather(ls_, lse_part.contiguous(), group=group)
    return torch.stack(os_), torch.stack(ls_)


def cp_decode_attn(desc, q_lat, q_rope, cache, kv_begin, kv_end, ws, o_lat, lse=None, group=None, stream=None):
    """Decode attention of sequences whose rows are spread over the group:
    this rank's partial over [kv_begin, kv_end), one all-gather of the
    partials, then the log-sum-exp merge into o_lat (and lse)."""
    import torch
    B, n_h, d_c = q_lat.shape[0], q_lat.shape[1], q_lat.shape[2]
    o_part = torch.empty((B, n_h, d_c), dtype=torch.float32, device=q_lat.device)
    lse_part = torch.empty((B, n_h), dtype=torch.float32, device=q_lat.device)
    mla.decode_attn_partial(desc, q_lat, q_rope, cache, kv_begin, kv_end, ws, o_part, lse_part, stream)
    o_parts, lse_parts = gather_partials(o_part, lse_part, group)
    mla.lse_merge(desc, o_parts, lse_parts, o_lat, lse, stream)
    return o_lat
