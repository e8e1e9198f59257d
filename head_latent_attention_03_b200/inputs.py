"""Seeded synthetic inputs for the MLA decode / prefill layer.

This module only draws numbers and lays them out; it holds none of the
method's arithmetic.  Both the fp64 oracle (tests, bench baseline) and the
CUDA path consume what it returns, so the two sides see bit-identical inputs.

Shapes follow the layers described in the DeepSeek-V2 explainer
(adg.csdn.net, section 3.1.1 "model hyperparameters" for the full model and
the DeepSeek-V2-Lite paragraph of part two): d = 5120, n_h = 128, d_h = 128,
d_c = 512, d_c' = 1536, d_h^R = 64 (V2) and d = 2048, n_h = 16, d_h = 128,
d_c = 512, d_h^R = 64, no query compression (V2-Lite).

Seeding: numpy PCG64 streams from SeedSequence([0, cfg_id, tensor_id]).
Draws are N(0, 1) scaled to N(0, 1/fan_in) for weights; bf16 layers round
each value once, round-to-nearest-even, and keep it as an exactly
representable float32 so that an fp64 consumer sees the same value.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

BLOCK = 64  # tokens per cache page


@dataclasses.dataclass(frozen=True)
class LayerDims:
    d: int
    n_h: int
    d_h: int
    d_c: int
    d_cq: int  # 0: no query compression (queries read h directly)
    d_hr: int
    dtype: str  # "f32" or "bf16"
    rope_base: float = 10000.0
    yarn_scale: float = 1.0
    yarn_orig_ctx: int = 4096
    yarn_alpha: float = 1.0
    yarn_beta: float = 32.0
    attn_logit_factor: float = 1.0
    block_size: int = BLOCK
    # RMSNorm after the compressed latents c^KV and c^Q, then a scale factor
    # at each of these width bottlenecks (off in the headline workloads)
    latent_norm: bool = False
    norm_eps: float = 1e-6
    scale_kv: float = 1.0
    scale_q: float = 1.0
    # latent cache storage: "bf16" (the layer's precision) or "fp8" (E4M3
    # codes of c^KV with one power-of-two scale per row; k^R stays bf16)
    cache_dtype: str = "bf16"

    @property
    def row(self) -> int:
        """Values per cached token: [c^KV (d_c) | k^R (d_h^R)]."""
        return self.d_c + self.d_hr


def yarn_logit_factor(s: float) -> float:
    """Logit multiplier used with YaRN scale s: (0.0707 ln s + 1)^2.

    The pages state only that the length-scaling factor was adjusted (the
    formula image is lost); this value is a parameter of both sides.
    """
    return (0.0707 * math.log(s) + 1.0) ** 2 if s > 1.0 else 1.0


TINY = LayerDims(d=64, n_h=4, d_h=16, d_c=32, d_cq=0, d_hr=8, dtype="f32")
LITE = LayerDims(d=2048, n_h=16, d_h=128, d_c=512, d_cq=0, d_hr=64, dtype="bf16")
V2 = LayerDims(d=5120, n_h=128, d_h=128, d_c=512, d_cq=1536, d_hr=64, dtype="bf16")
V2_YARN = dataclasses.replace(V2, yarn_scale=40.0, attn_logit_factor=yarn_logit_factor(40.0))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: a layer plus batch, cache lengths and page order."""
    name: str
    cfg_id: int
    dims: LayerDims
    batch: int
    prior: str  # "fixed:<L>", "uniform:<lo>:<hi>" or "list:<L0>,<L1>,..."
    new_tokens: int = 1  # tokens appended per sequence (1 = decode)
    permute_pages: bool = False
    h_std: str = "unit"  # "unit" -> h ~ N(0,1); "fan_in" -> N(0, 1/d)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, TINY, 1, "fixed:64", h_std="fan_in"),
    "lite": Workload("lite", 2, LITE, 32, "fixed:4096"),
    "v2": Workload("v2", 3, V2, 64, "uniform:1:8192", permute_pages=True),
    "long": Workload("long", 4, V2_YARN, 4, "fixed:131072"),
    "prefill": Workload("prefill", 5, V2, 8, "fixed:4096", new_tokens=4096),
    # the V2-Lite and V2 workloads (same draws) over an FP8 latent cache
    "lite_fp8": Workload("lite_fp8", 2, dataclasses.replace(LITE, cache_dtype="fp8"), 32, "fixed:4096"),
    "v2_fp8": Workload("v2_fp8", 3, dataclasses.replace(V2, cache_dtype="fp8"), 64, "uniform:1:8192",
                       permute_pages=True),
}

# tensor ids inside a workload's seed tree
_T_W = {"w_dkv": 1, "w_kr": 2, "w_dq": 3, "w_uq": 4, "w_qr": 5, "w_uk": 6, "w_uv": 7, "w_o": 8, "g_kv": 9, "g_q": 10}
_T_H, _T_LENS, _T_PRIOR, _T_PERM = 20, 21, 22, 23


def rng_for(cfg_id: int, tensor_id: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([0, cfg_id, tensor_id, sub])))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of values that are already bf16-exact."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _store(x: np.ndarray, dims: LayerDims) -> np.ndarray:
    return round_bf16(x) if dims.dtype == "bf16" else x


def gen_weights(w: Workload) -> Dict[str, Optional[np.ndarray]]:
    """All projection matrices of one MLA layer, [out, in] row-major.

    W^UQ / W^QR act on c^Q (d_c' wide) when queries are compressed, else on h.
    W^UK / W^UV are [n_h*d_h, d_c] with head i in rows [i*d_h, (i+1)*d_h).
    """
    D = w.dims
    q_in = D.d_cq if D.d_cq else D.d
    shapes = {
        "w_dkv": (D.d_c, D.d), "w_kr": (D.d_hr, D.d),
        "w_dq": (D.d_cq, D.d) if D.d_cq else None,
        "w_uq": (D.n_h * D.d_h, q_in), "w_qr": (D.n_h * D.d_hr, q_in),
        "w_uk": (D.n_h * D.d_h, D.d_c), "w_uv": (D.n_h * D.d_h, D.d_c),
        "w_o": (D.d, D.n_h * D.d_h),
    }
    out: Dict[str, Optional[np.ndarray]] = {}
    for name, shp in shapes.items():
        if shp is None:
            out[name] = None
            continue
        out[name] = _store(_normal(rng_for(w.cfg_id, _T_W[name]), shp, 1.0 / math.sqrt(shp[1])), D)
    # RMSNorm gains of the latents: 1 + N(0, 0.1^2) per feature
    out["g_kv"] = out["g_q"] = None
    if D.latent_norm:
        out["g_kv"] = _store(1.0 + _normal(rng_for(w.cfg_id, _T_W["g_kv"]), (D.d_c,), 0.1), D)
        if D.d_cq:
            out["g_q"] = _store(1.0 + _normal(rng_for(w.cfg_id, _T_W["g_q"]), (D.d_cq,), 0.1), D)
    return out


def prior_lengths(w: Workload) -> np.ndarray:
    kind, *args = w.prior.split(":")
    if kind == "list":
        vals = [int(v) for v in args[0].split(",")]
        assert len(vals) == w.batch
        return np.array(vals, dtype=np.int64)
    if kind == "fixed":
        return np.full(w.batch, int(args[0]), dtype=np.int64)
    lo, hi = int(args[0]), int(args[1])
    return rng_for(w.cfg_id, _T_LENS).integers(lo, hi + 1, size=w.batch, dtype=np.int64)


@dataclasses.dataclass
class Batch:
    """Host-side inputs of one decode (or chunked-prefill) step.

    pool[num_blocks, block, d_c+d_hr] holds the prior rows at
    (block_table[b][j // block], j % block) for j < prior_len[b]; every other
    slot is filled with `fill` (NaN by default, so that a kernel reading an
    unwritten slot is caught).  h[b*new_tokens + t] is the hidden state of the
    token at position prior_len[b] + t of sequence b.
    """
    workload: Workload
    h: np.ndarray  # [B*new, d] float32 (bf16-exact for bf16 layers)
    prior_len: np.ndarray  # [B] int64
    positions: np.ndarray  # [B*new] int64
    seq_idx: np.ndarray  # [B*new] int64
    block_table: np.ndarray  # [B, max_blocks] int32, -1 padded
    pool: np.ndarray  # [num_blocks, block, row] float32


def gen_batch(w: Workload, fill: float = float("nan"), seqs: Optional[List[int]] = None) -> Batch:
    """Draw h, the prior cache rows and the page table of workload `w`.

    `seqs` restricts the draw to a subset of sequences (same values as in the
    full draw: each sequence has its own stream), which keeps oracle samples of
    large workloads cheap.
    """
    D = w.dims
    lens_all = prior_lengths(w)
    seqs = list(range(w.batch)) if seqs is None else list(seqs)
    lens = lens_all[seqs]
    new = w.new_tokens
    n_blocks = [(int(L) + new + D.block_size - 1) // D.block_size for L in lens]
    total = int(sum(n_blocks))
    max_blocks = max(n_blocks)
    if w.permute_pages and len(seqs) == w.batch:
        perm = rng_for(w.cfg_id, _T_PERM).permutation(total).astype(np.int32)
    else:
        perm = np.arange(total, dtype=np.int32)
    table = np.full((len(seqs), max_blocks), -1, dtype=np.int32)
    pool = np.full((total, D.block_size, D.row), fill, dtype=np.float32)
    h = np.empty((len(seqs) * new, D.d), dtype=np.float32)
    h_std = 1.0 if w.h_std == "unit" else 1.0 / math.sqrt(D.d)
    cursor = 0
    for i, (b, L) in enumerate(zip(seqs, lens)):
        L = int(L)
        ids = perm[cursor:cursor + n_blocks[i]]
        cursor += n_blocks[i]
        table[i, :len(ids)] = ids
        rows = _store(_normal(rng_for(w.cfg_id, _T_PRIOR, b), (L, D.row), 1.0), D)
        for p in range(0, L, D.block_size):
            blk = ids[p // D.block_size]
            n = min(D.block_size, L - p)
            pool[blk, :n] = rows[p:p + n]
        h[i * new:(i + 1) * new] = _store(_normal(rng_for(w.cfg_id, _T_H, b), (new, D.d), h_std), D)
    positions = np.concatenate([np.arange(int(L), int(L) + new) for L in lens]).astype(np.int64)
    seq_idx = np.repeat(np.arange(len(seqs)), new).astype(np.int64)
    return Batch(w, h, lens.astype(np.int64), positions, seq_idx, table, pool)
