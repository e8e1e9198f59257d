"""fp64 CPU oracle of one Multi-head Latent Attention (MLA) layer.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline leg may import this module.  It shares no code with the CUDA path
(head_latent_attention_03_b200/csrc); both consume the same seeded inputs from
head_latent_attention_03_b200.inputs, which holds no arithmetic of the method.

Sources (the pages this restates; equation numbers are the arXiv paper's, as
printed on the pages):
  [notes]     "DeepSeek-V2" reading notes (irregular6612.github.io), section
              2.1.1 eqs (1)-(8) (standard MHA) and 2.1.2 eqs (9)-(13)
              (low-rank key-value joint compression, query compression).
  [explainer] DeepSeek-V2 explainer (adg.csdn.net), section 2.2.1.1 (KV
              joint compression), 2.2.1.2 (query compression), 2.2.2
              (decoupled RoPE: q^R from the query latent, one shared k^R taken
              directly from h_t, concatenation [q^C; q^R], [k^C; k^R], and the
              absorption of W^UK into the query side and of W^UV into W^O),
              3.1.1 (V2 hyper-parameters) and 3.1.3 (YaRN on the shared k^R).
  [papertrace] DeepSeek-V2 bilingual rendering (PaperTrace), abstract and
              section 2.1.

Readings where the pages are silent or garbled (each is a parameter or an
explicit choice here, shared by the CUDA path only as a convention):
  * softmax scale = attn_logit_factor / sqrt(d_h + d_h^R); eq (7) prints
    1/sqrt(d_h) for plain MHA, the decoupled form adds d_h^R to the dot product.
  * eq (7)'s garbled summation index is read as j = 1..t (all keys up to and
    including the current token).
  * RoPE: interleaved pairs (2k, 2k+1), theta_k = base^(-2k/d_h^R), the same
    rotation for q^R and k^R.
  * YaRN: "NTK-by-parts" frequency blend with s, alpha, beta and the original
    window; the logit factor is a parameter (its formula is lost on the page).
  * q^R = RoPE(W^QR c^Q) with c^Q = W^DQ h when queries are compressed, else
    c^Q := h (V2-Lite does not compress queries).
  * The RMSNorm after the compressed latents and the extra scale factors at
    these width bottlenecks ([explainer] 3.1.1, no formula printed), when a
    layer turns them on: c <- s * g * c / sqrt(mean(c^2) + eps) for c^KV
    (before it is cached) and for c^Q (before W^UQ and W^QR), with per-feature
    gains g and scalar factors s_kv, s_q.  The factor follows the norm (a
    factor in front of it would cancel).  k^R is not a compressed latent and
    is not normalised.
  * The quantised latent cache ([explainer] 3.1.4 serves V2 with the KV
    cache quantised to about 6 bits per element; no format is printed), when
    a layer uses it: each cached c^KV row is stored as FP8 E4M3 codes (OCP
    8-bit float: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
    subnormals, no infinities, largest finite 448) times one power-of-two
    scale 2^e per row, e the smallest integer with max|c| <= 448 * 2^e, codes
    rounded to nearest with ties to even and saturated at +-448.  k^R stays
    in the layer's precision (positions need its bits).  The attention reads
    the dequantised row codes * 2^e.

Every function is fp64 and written for clarity, not speed.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# rotary position embedding (decoupled RoPE carrier), [explainer] 2.2.2, 3.1.3
# ---------------------------------------------------------------------------

def rope_frequencies(d_hr: int, base: float = 10000.0, yarn_scale: float = 1.0,
                     orig_ctx: int = 4096, alpha: float = 1.0, beta: float = 32.0) -> np.ndarray:
    """Rotation frequency theta_k (radians per position) of pair k, k < d_hr/2.

    Plain RoPE: theta_k = base^(-2k/d_hr).  With YaRN scale s > 1 each pair is
    classified by r_k = orig_ctx / wavelength_k = orig_ctx * theta_k / (2 pi):
    r_k < alpha -> interpolated (theta_k / s); r_k > beta -> kept (theta_k);
    in between -> linear blend with gamma = (r_k - alpha) / (beta - alpha).
    """
    k = np.arange(d_hr // 2, dtype=F64)
    theta = base ** (-2.0 * k / d_hr)
    if yarn_scale == 1.0:
        return theta
    r = orig_ctx * theta / (2.0 * math.pi)
    out = np.empty_like(theta)
    for i in range(len(theta)):
        if r[i] < alpha:
            out[i] = theta[i] / yarn_scale
        elif r[i] > beta:
            out[i] = theta[i]
        else:
            g = (r[i] - alpha) / (beta - alpha)
            out[i] = (1.0 - g) * theta[i] / yarn_scale + g * theta[i]
    return out


def rope_rotate(x: np.ndarray, pos: int, theta: np.ndarray) -> np.ndarray:
    """Rotate each interleaved pair (x[2k], x[2k+1]) of the last axis by pos*theta_k."""
    x = np.asarray(x, dtype=F64)
    out = np.empty_like(x)
    ang = pos * theta
    c, s = np.cos(ang), np.sin(ang)
    even, odd = x[..., 0::2], x[..., 1::2]
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


def dims_theta(D) -> np.ndarray:
    return rope_frequencies(D.d_hr, D.rope_base, D.yarn_scale, D.yarn_orig_ctx, D.yarn_alpha, D.yarn_beta)


def softmax_scale(D) -> float:
    return D.attn_logit_factor / math.sqrt(D.d_h + D.d_hr)


# ---------------------------------------------------------------------------
# projections, [notes] eqs (9), (12), (13); [explainer] 2.2.2, 3.1.1
# ---------------------------------------------------------------------------

def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float) -> np.ndarray:
    """gain * x / sqrt(mean(x^2) + eps) over the last axis."""
    x = np.asarray(x, dtype=F64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return np.asarray(gain, dtype=F64) * x / np.sqrt(ms + eps)


def latent_norm(D, W, c: np.ndarray, which: str) -> np.ndarray:
    """The compressed latent as the layer uses it: RMSNorm plus the bottleneck
    scale factor when the layer has them ([explainer] 3.1.1), else c."""
    if not getattr(D, "latent_norm", False):
        return np.asarray(c, dtype=F64)
    gain = W["g_kv"] if which == "kv" else W["g_q"]
    scale = D.scale_kv if which == "kv" else D.scale_q
    return scale * rms_norm(c, gain, D.norm_eps)


# ---------------------------------------------------------------------------
# quantised latent cache, [explainer] 3.1.4 (KV cache quantisation for serving)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0    # largest finite E4M3 value, 1.75 * 2^8
E4M3_MIN_EXP = -6   # exponent of the smallest normal E4M3 value (1 - bias)
E4M3_MANT = 3       # stored mantissa bits


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Nearest FP8 E4M3 value of each element, ties to even, saturated to +-448.

    In the binade [2^k, 2^(k+1)) the representable values are 2^(k-3) apart;
    below 2^-6 (subnormals) they are 2^-9 apart.  Rounding the quotient by
    that spacing to the nearest integer, halves to even, rounds the stored
    mantissa to nearest even; a quotient that reaches 16 is the next binade's
    first value.
    """
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    _, k = np.frexp(a)                          # a = f 2^k with f in [0.5, 1)
    exp = np.maximum(k - 1, E4M3_MIN_EXP)
    step = np.ldexp(1.0, exp - E4M3_MANT)
    q = np.round(a / step) * step               # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, x)


def fp8_scale_exponent(amax: float) -> int:
    """Smallest integer e with amax <= 448 * 2^e (0 for a zero row): the row's
    largest magnitude lands in the top binade of E4M3."""
    if not amax > 0.0:
        return 0
    _, k = math.frexp(amax)                     # amax in [2^(k-1), 2^k)
    e = (k - 1) - 8                             # 448 * 2^e = 1.75 * 2^(k-1)
    if amax > E4M3_MAX * 2.0 ** e:
        e += 1
    return e


def quantize_latent(c: np.ndarray) -> Tuple[np.ndarray, int]:
    """One cached c^KV row as (E4M3 code values, e), c ~ codes * 2^e."""
    c = np.asarray(c, dtype=F64)
    e = fp8_scale_exponent(float(np.max(np.abs(c))))
    return e4m3_round(np.ldexp(c, -e)), e


def cached_row(D, row: np.ndarray) -> np.ndarray:
    """A cache row [c^KV ; k^R] as the attention reads it back: with the FP8
    cache c^KV is dequantised from its codes, k^R is kept."""
    row = np.asarray(row, dtype=F64)
    if getattr(D, "cache_dtype", "bf16") != "fp8":
        return row
    codes, e = quantize_latent(row[:D.d_c])
    return np.concatenate([np.ldexp(codes, e), row[D.d_c:]])


def cached_rows(D, rows: np.ndarray) -> np.ndarray:
    """cached_row of every row of rows [L, d_c + d_hr]."""
    rows = np.asarray(rows, dtype=F64)
    if getattr(D, "cache_dtype", "bf16") != "fp8":
        return rows
    return np.stack([cached_row(D, r) for r in rows]) if len(rows) else rows


def compress_kv(D, W: Dict[str, np.ndarray], h_t: np.ndarray, pos: int) -> np.ndarray:
    """The cached row of token t: [c^KV_t ; k^R_t].

    c^KV_t = W^DKV h_t (eq 9), normalised and scaled when the layer has the
    latent RMSNorm ([explainer] 3.1.1).  k^R_t = RoPE_pos(W^KR h_t): the
    shared RoPE key comes straight from h_t, not from the latent
    ([explainer] 2.2.2).
    """
    h = np.asarray(h_t, dtype=F64)
    c_kv = latent_norm(D, W, W["w_dkv"].astype(F64) @ h, "kv")
    k_r = rope_rotate(W["w_kr"].astype(F64) @ h, pos, dims_theta(D))
    return np.concatenate([c_kv, k_r])


def queries(D, W: Dict[str, np.ndarray], h_t: np.ndarray, pos: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-head queries q^C [n_h, d_h] and rotated q^R [n_h, d_hr] of one token.

    c^Q = W^DQ h (eq 12) when queries are compressed, else c^Q = h;
    q^C = W^UQ c^Q (eq 13); q^R_i = RoPE_pos(W^QR_i c^Q) ([explainer] 2.2.2).
    """
    h = np.asarray(h_t, dtype=F64)
    c_q = latent_norm(D, W, W["w_dq"].astype(F64) @ h, "q") if D.d_cq else h
    q_c = (W["w_uq"].astype(F64) @ c_q).reshape(D.n_h, D.d_h)
    q_r_pre = (W["w_qr"].astype(F64) @ c_q).reshape(D.n_h, D.d_hr)
    q_r = rope_rotate(q_r_pre, pos, dims_theta(D))
    return q_c, q_r


# ---------------------------------------------------------------------------
# attention, un-absorbed (the definition) and absorbed (the inference form)
# ---------------------------------------------------------------------------

def softmax_weights(z: np.ndarray) -> Tuple[np.ndarray, float]:
    """softmax over the last axis with max subtraction; returns (p, logsumexp)."""
    z = np.asarray(z, dtype=F64)
    m = z.max()
    e = np.exp(z - m)
    s = e.sum()
    return e / s, float(m + math.log(s))


def attend_unabsorbed(D, W, q_c: np.ndarray, q_r: np.ndarray, rows: np.ndarray):
    """Attention of one query token over cached rows [L, d_c + d_hr].

    Up-projects every key and value, k^C_{j,i} = W^UK_i c^KV_j (eq 10),
    v^C_{j,i} = W^UV_i c^KV_j (eq 11), then runs eq (7) on the concatenated
    vectors q_{t,i} = [q^C_i; q^R_i], k_{j,i} = [k^C_{j,i}; k^R_j]
    ([explainer] 2.2.2) and applies W^O (eq 8).
    Returns (o [n_h, d_h], lse [n_h], u [d]).
    """
    rows = np.asarray(rows, dtype=F64)
    c_kv, k_r = rows[:, :D.d_c], rows[:, D.d_c:]
    k_c = c_kv @ W["w_uk"].astype(F64).T  # [L, n_h*d_h]
    v_c = c_kv @ W["w_uv"].astype(F64).T
    scale = softmax_scale(D)
    o = np.empty((D.n_h, D.d_h))
    lse = np.empty(D.n_h)
    for i in range(D.n_h):
        hs = slice(i * D.d_h, (i + 1) * D.d_h)
        q_i = np.concatenate([q_c[i], q_r[i]])
        k_i = np.concatenate([k_c[:, hs], k_r], axis=1)  # [L, d_h + d_hr]
        p, lse[i] = softmax_weights(scale * (k_i @ q_i))
        o[i] = p @ v_c[:, hs]
    u = W["w_o"].astype(F64) @ o.reshape(-1)
    return o, lse, u


def absorb_query(D, W, q_c: np.ndarray) -> np.ndarray:
    """q_lat_i = (W^UK_i)^T q^C_i, [n_h, d_c]: W^UK folded into the query."""
    w_uk = W["w_uk"].astype(F64).reshape(D.n_h, D.d_h, D.d_c)
    return np.einsum("ihc,ih->ic", w_uk, q_c)


def attend_absorbed(D, W, q_lat: np.ndarray, q_r: np.ndarray, rows: np.ndarray):
    """Absorbed form ([explainer] 2.2.2): keys and values never materialised.

    z_j = scale (q_lat_i . c^KV_j + q^R_i . k^R_j); o_lat_i = sum_j p_j c^KV_j;
    o_i = W^UV_i o_lat_i; u = W^O [o_1; ...; o_nh].
    Returns (o_lat [n_h, d_c], lse [n_h], u [d]).
    """
    rows = np.asarray(rows, dtype=F64)
    c_kv, k_r = rows[:, :D.d_c], rows[:, D.d_c:]
    scale = softmax_scale(D)
    o_lat = np.empty((D.n_h, D.d_c))
    lse = np.empty(D.n_h)
    for i in range(D.n_h):
        p, lse[i] = softmax_weights(scale * (c_kv @ q_lat[i] + k_r @ q_r[i]))
        o_lat[i] = p @ c_kv
    u = out_project(D, W, o_lat)
    return o_lat, lse, u


def merge_partials(o_parts: Sequence[np.ndarray], lse_parts: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Attention over the union of disjoint row sets from the attentions over
    each set: with Z_r = sum over set r of e^{z_j} = e^{lse_r}, the softmax over
    the union weighs set r by Z_r / sum Z; lse = log sum Z.  An empty set has
    lse = -inf and weight 0.  Arrays [..., d] and [...] per part."""
    lse = np.stack([np.asarray(l, dtype=F64) for l in lse_parts])
    m = np.max(lse, axis=0)
    w = np.exp(lse - m)
    tot = np.sum(w, axis=0)
    out = sum(w[r][..., None] * np.asarray(o_parts[r], dtype=F64) for r in range(len(o_parts))) / tot[..., None]
    return out, m + np.log(tot)


def out_project(D, W, o_lat: np.ndarray) -> np.ndarray:
    """u = W^O [W^UV_1 o_lat_1; ...; W^UV_nh o_lat_nh] (eq 8 with W^UV absorbed)."""
    w_uv = W["w_uv"].astype(F64).reshape(D.n_h, D.d_h, D.d_c)
    o = np.einsum("ihc,ic->ih", w_uv, np.asarray(o_lat, dtype=F64))
    return W["w_o"].astype(F64) @ o.reshape(-1)


# ---------------------------------------------------------------------------
# standard MHA, [notes] eqs (1)-(8) — used to pin the MLA oracle
# ---------------------------------------------------------------------------

def mha_step(W_q: np.ndarray, W_k: np.ndarray, W_v: np.ndarray, W_o: np.ndarray,
             hs: np.ndarray, n_h: int, d_h: int, scale: Optional[float] = None) -> np.ndarray:
    """u_t of the last token of hs [t, d] under eqs (1)-(8)."""
    hs = np.asarray(hs, dtype=F64)
    q = W_q @ hs[-1]
    k = hs @ W_k.T
    v = hs @ W_v.T
    scale = 1.0 / math.sqrt(d_h) if scale is None else scale
    o = np.empty((n_h, d_h))
    for i in range(n_h):
        sl = slice(i * d_h, (i + 1) * d_h)
        p, _ = softmax_weights(scale * (k[:, sl] @ q[sl]))
        o[i] = p @ v[:, sl]
    return W_o @ o.reshape(-1)


def kv_cache_elements_per_token(kind: str, n_layers: int, n_h: int = 0, d_h: int = 0,
                                d_c: int = 0, d_hr: int = 0, n_groups: int = 0) -> int:
    """Cached elements per token: MHA 2 n_h d_h l; GQA 2 n_g d_h l; MLA (d_c + d_h^R) l.

    MHA: [notes] 2.1.1; MLA: [explainer] 2.2.2 (c^KV and k^R are what is cached).
    """
    if kind == "mha":
        return 2 * n_h * d_h * n_layers
    if kind == "gqa":
        return 2 * n_groups * d_h * n_layers
    if kind == "mla":
        return (d_c + d_hr) * n_layers
    raise ValueError(kind)


# ---------------------------------------------------------------------------
# a full decode / prefill step over the paged cache
# ---------------------------------------------------------------------------

def gather_rows(pool: np.ndarray, table_row: np.ndarray, n: int, block: int) -> np.ndarray:
    """Rows 0..n-1 of one sequence from the page pool."""
    out = np.empty((n, pool.shape[2]), dtype=F64)
    for j in range(n):
        out[j] = pool[table_row[j // block], j % block]
    return out


def decode_token(D, W, h_t: np.ndarray, pos: int, prior_rows: np.ndarray, absorbed: bool = False) -> Dict[str, np.ndarray]:
    """One new token at position `pos` attending over prior rows + itself.

    Returns the new cache row (and as the attention reads it back from the
    cache: "row_cached"), q^C, q^R, (absorbed only) q_lat and o_lat, lse and
    u.  With the FP8 cache every row, prior and new, is read back dequantised.
    """
    row = compress_kv(D, W, h_t, pos)
    rows = cached_rows(D, np.concatenate([np.asarray(prior_rows, dtype=F64), row[None, :]], axis=0))
    q_c, q_r = queries(D, W, h_t, pos)
    out = {"row": row, "row_cached": rows[-1], "q_c": q_c, "q_r": q_r}
    if absorbed:
        q_lat = absorb_query(D, W, q_c)
        o_lat, lse, u = attend_absorbed(D, W, q_lat, q_r, rows)
        out.update(q_lat=q_lat, o_lat=o_lat, lse=lse, u=u)
    else:
        o, lse, u = attend_unabsorbed(D, W, q_c, q_r, rows)
        out.update(o=o, lse=lse, u=u)
    return out


def decode_batch(batch, W, seqs: Optional[Sequence[int]] = None, absorbed: bool = False):
    """decode_token for each sequence of a Batch (decode: one new token each)."""
    D = batch.workload.dims
    res = []
    seqs = range(len(batch.prior_len)) if seqs is None else seqs
    for b in seqs:
        L = int(batch.prior_len[b])
        prior = gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
        res.append(decode_token(D, W, batch.h[b], L, prior, absorbed=absorbed))
    return res


def prefill_sequence(D, W, h_new: np.ndarray, start: int, prior_rows: np.ndarray,
                     query_ids: Sequence[int], absorbed: bool = True):
    """Chunked prefill of one sequence: append all new tokens, then causal attention.

    New token q (0-based) sits at position start+q and attends keys 0..start+q
    (eq 7's causal sum).  Returns the new rows and, for each q in query_ids,
    (q_lat, o_lat, lse, u) (absorbed) or (o, lse, u).
    """
    new_rows = np.stack([compress_kv(D, W, h_new[q], start + q) for q in range(len(h_new))])
    rows = cached_rows(D, np.concatenate([np.asarray(prior_rows, dtype=F64), new_rows], axis=0))
    outs = {}
    for q in query_ids:
        pos = start + q
        q_c, q_r = queries(D, W, h_new[q], pos)
        if absorbed:
            q_lat = absorb_query(D, W, q_c)
            o_lat, lse, u = attend_absorbed(D, W, q_lat, q_r, rows[:pos + 1])
            outs[q] = {"q_lat": q_lat, "q_r": q_r, "o_lat": o_lat, "lse": lse, "u": u}
        else:
            o, lse, u = attend_unabsorbed(D, W, q_c, q_r, rows[:pos + 1])
            outs[q] = {"q_r": q_r, "o": o, "lse": lse, "u": u}
    return new_rows, outs
