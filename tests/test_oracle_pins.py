"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test names the identity or closed form it checks and the page passage it
follows.  A plausible slip anywhere in the oracle (a transposed W^UK, a
dropped d_h^R term, a wrong RoPE sign, a missing max subtraction, a causal
off-by-one) breaks at least one of them; test_planted_mistakes.py plants such
slips in a copy of the oracle and checks that they are caught.
"""
import math

import numpy as np
import pytest

from oracle import mla_oracle as O
from head_latent_attention_03_b200.inputs import LayerDims, TINY, LITE, V2


def _rand_weights(D, rng, std=None):
    q_in = D.d_cq if D.d_cq else D.d

    def n(shape):
        return rng.standard_normal(shape) / math.sqrt(shape[1]) if shape[0] and shape[1] else np.zeros(shape)

    W = {"w_dkv": n((D.d_c, D.d)), "w_kr": n((D.d_hr, D.d)),
         "w_dq": n((D.d_cq, D.d)) if D.d_cq else None,
         "w_uq": n((D.n_h * D.d_h, q_in)), "w_qr": n((D.n_h * D.d_hr, q_in)),
         "w_uk": n((D.n_h * D.d_h, D.d_c)), "w_uv": n((D.n_h * D.d_h, D.d_c)),
         "w_o": n((D.d, D.n_h * D.d_h))}
    return W


SMALL = [
    TINY,
    LayerDims(d=48, n_h=3, d_h=8, d_c=24, d_cq=20, d_hr=6, dtype="f32"),
    LayerDims(d=40, n_h=2, d_h=12, d_c=16, d_cq=0, d_hr=4, dtype="f32", yarn_scale=8.0, yarn_orig_ctx=64,
              attn_logit_factor=1.3),
]


# 1. absorption identity ([explainer] 2.2.2: W^UK folds into the query side and
#    W^UV into W^O by associativity): absorbed == un-absorbed to 1e-12.
@pytest.mark.parametrize("D", SMALL)
def test_absorption_identity(D):
    rng = np.random.default_rng(1)
    W = _rand_weights(D, rng)
    L = 37
    prior = rng.standard_normal((L, D.row))
    h = rng.standard_normal(D.d)
    un = O.decode_token(D, W, h, L, prior, absorbed=False)
    ab = O.decode_token(D, W, h, L, prior, absorbed=True)
    assert np.max(np.abs(un["u"] - ab["u"])) <= 1e-12 * np.max(np.abs(un["u"]))
    assert np.max(np.abs(un["lse"] - ab["lse"])) <= 1e-12 * np.max(np.abs(un["lse"]))
    w_uv = W["w_uv"].reshape(D.n_h, D.d_h, D.d_c)
    o_from_lat = np.einsum("ihc,ic->ih", w_uv, ab["o_lat"])
    assert np.max(np.abs(o_from_lat - un["o"])) <= 1e-12 * np.max(np.abs(un["o"]))


# 2. MHA equivalence ([notes] eqs 1-8 vs 9-11): when the factors compose to
#    W^K, W^V exactly, MLA with d_h^R = 0 is standard MHA.
def _mla_vs_mha(D, W, W_q, W_k, W_v, W_o, T=9, seed=2):
    rng = np.random.default_rng(seed)
    hs = rng.standard_normal((T, D.d))
    prior = np.stack([O.compress_kv(D, W, hs[j], j) for j in range(T - 1)])
    mla = O.decode_token(D, W, hs[-1], T - 1, prior)["u"]
    mha = O.mha_step(W_q, W_k, W_v, W_o, hs, D.n_h, D.d_h)
    return mla, mha


def test_mha_equivalence_identity_down_projection():
    # d_c = d: W^DKV = I, W^UK = W^K, W^UV = W^V, W^UQ = W^Q (no q compression).
    D = LayerDims(d=32, n_h=2, d_h=16, d_c=32, d_cq=0, d_hr=0, dtype="f32")
    rng = np.random.default_rng(3)
    W_q, W_k, W_v = (rng.standard_normal((32, 32)) / math.sqrt(32) for _ in range(3))
    W_o = rng.standard_normal((32, 32)) / math.sqrt(32)
    W = {"w_dkv": np.eye(32), "w_kr": np.zeros((0, 32)), "w_dq": None, "w_uq": W_q,
         "w_qr": np.zeros((0, 32)), "w_uk": W_k, "w_uv": W_v, "w_o": W_o}
    mla, mha = _mla_vs_mha(D, W, W_q, W_k, W_v, W_o)
    assert np.max(np.abs(mla - mha)) <= 1e-13 * max(1.0, np.max(np.abs(mha)))


def test_mha_equivalence_stacked_factorisation():
    # d_c = 2 n_h d_h: W^DKV = [W^K; W^V], W^UK = [I 0], W^UV = [0 I]; with
    # query compression W^DQ = I, W^UQ = W^Q.  d_c >= n_h d_h as the target asks.
    n_h, d_h, d = 2, 8, 24
    D = LayerDims(d=d, n_h=n_h, d_h=d_h, d_c=2 * n_h * d_h, d_cq=d, d_hr=0, dtype="f32")
    rng = np.random.default_rng(4)
    W_q, W_k, W_v = (rng.standard_normal((n_h * d_h, d)) / math.sqrt(d) for _ in range(3))
    W_o = rng.standard_normal((d, n_h * d_h)) / math.sqrt(n_h * d_h)
    eye, zero = np.eye(n_h * d_h), np.zeros((n_h * d_h, n_h * d_h))
    W = {"w_dkv": np.vstack([W_k, W_v]), "w_kr": np.zeros((0, d)), "w_dq": np.eye(d), "w_uq": W_q,
         "w_qr": np.zeros((0, d)), "w_uk": np.hstack([eye, zero]), "w_uv": np.hstack([zero, eye]), "w_o": W_o}
    mla, mha = _mla_vs_mha(D, W, W_q, W_k, W_v, W_o)
    assert np.max(np.abs(mla - mha)) <= 1e-13 * max(1.0, np.max(np.abs(mha)))


def test_mha_equivalence_padded_latent():
    # d_c > d: W^DKV = [I; 0], W^UK = [W^K, 0] (the case d_c >= n_h d_h).
    n_h, d_h, d, d_c = 2, 8, 16, 24
    D = LayerDims(d=d, n_h=n_h, d_h=d_h, d_c=d_c, d_cq=0, d_hr=0, dtype="f32")
    rng = np.random.default_rng(5)
    W_q, W_k, W_v = (rng.standard_normal((n_h * d_h, d)) / math.sqrt(d) for _ in range(3))
    W_o = rng.standard_normal((d, n_h * d_h)) / math.sqrt(n_h * d_h)
    pad = np.zeros((n_h * d_h, d_c - d))
    W = {"w_dkv": np.vstack([np.eye(d), np.zeros((d_c - d, d))]), "w_kr": np.zeros((0, d)), "w_dq": None,
         "w_uq": W_q, "w_qr": np.zeros((0, d)), "w_uk": np.hstack([W_k, pad]),
         "w_uv": np.hstack([W_v, pad]), "w_o": W_o}
    mla, mha = _mla_vs_mha(D, W, W_q, W_k, W_v, W_o)
    assert np.max(np.abs(mla - mha)) <= 1e-13 * max(1.0, np.max(np.abs(mha)))


def test_zero_rope_part_uses_joint_scale():
    # With W^KR = W^QR = 0 the decoupled part adds nothing to the dot product,
    # so MLA equals MHA run with scale 1/sqrt(d_h + d_h^R): the reading of the
    # scale that reduces to eq (7)'s 1/sqrt(d_h) when d_h^R = 0.
    n_h, d_h, d, d_hr = 2, 8, 16, 4
    D = LayerDims(d=d, n_h=n_h, d_h=d_h, d_c=d, d_cq=0, d_hr=d_hr, dtype="f32")
    rng = np.random.default_rng(6)
    W_q, W_k, W_v = (rng.standard_normal((n_h * d_h, d)) / math.sqrt(d) for _ in range(3))
    W_o = rng.standard_normal((d, n_h * d_h)) / math.sqrt(n_h * d_h)
    W = {"w_dkv": np.eye(d), "w_kr": np.zeros((d_hr, d)), "w_dq": None, "w_uq": W_q,
         "w_qr": np.zeros((n_h * d_hr, d)), "w_uk": W_k, "w_uv": W_v, "w_o": W_o}
    T = 7
    hs = rng.standard_normal((T, d))
    prior = np.stack([O.compress_kv(D, W, hs[j], j) for j in range(T - 1)])
    mla = O.decode_token(D, W, hs[-1], T - 1, prior)["u"]
    mha = O.mha_step(W_q, W_k, W_v, W_o, hs, n_h, d_h, scale=1.0 / math.sqrt(d_h + d_hr))
    assert np.max(np.abs(mla - mha)) <= 1e-13 * np.max(np.abs(mha))


# 3. cache-size formula ([explainer] 2.2.2, [notes] 2.1.1): MLA caches
#    (d_c + d_h^R) l elements per token, MHA 2 n_h d_h l; V2 equals GQA with
#    2.25 groups, i.e. (9/2) d_h l when d_c = 4 d_h and d_h^R = d_h / 2.
def test_cache_size_formula():
    rng = np.random.default_rng(7)
    for D in (TINY, LITE, V2):
        small = LayerDims(d=16, n_h=D.n_h, d_h=D.d_h, d_c=D.d_c, d_cq=0, d_hr=D.d_hr, dtype="f32")
        W = {"w_dkv": rng.standard_normal((D.d_c, 16)), "w_kr": rng.standard_normal((D.d_hr, 16))}
        row = O.compress_kv(small, W, rng.standard_normal(16), 3)
        assert row.size == O.kv_cache_elements_per_token("mla", 1, d_c=D.d_c, d_hr=D.d_hr)
    layers = 60  # V2 layer count ([explainer] 3.1.1)
    mla = O.kv_cache_elements_per_token("mla", layers, d_c=512, d_hr=64)
    mha = O.kv_cache_elements_per_token("mha", layers, n_h=128, d_h=128)
    assert mla == 576 * 60 and mha == 32768 * 60
    assert mla == O.kv_cache_elements_per_token("gqa", layers, n_groups=1, d_h=128) * 9 // 4
    assert mla * 2 == 9 * 128 * layers  # (9/2) d_h l
    assert 1 - mla / mha == pytest.approx(1 - 576 / 32768)


# 4. brute-force softmax and its special cases.
def test_softmax_brute_force_long_double():
    rng = np.random.default_rng(8)
    for L in (1, 2, 5, 40):
        z = rng.standard_normal(L) * 3
        p, lse = O.softmax_weights(z)
        zl = z.astype(np.longdouble)
        e = np.exp(zl)
        ref = e / e.sum()
        assert np.max(np.abs(p - ref.astype(np.float64))) < 1e-15
        assert abs(lse - float(np.log(e.sum()))) < 1e-13
    # max subtraction keeps huge logits finite
    p, lse = O.softmax_weights(np.array([1000.0, 999.0]))
    assert np.isfinite(p).all() and p[0] == pytest.approx(1 / (1 + math.exp(-1)))


def test_single_row_returns_its_latent():
    # L + 1 = 1: softmax over one key is 1, so o_lat = c^KV_t and
    # u = W^O blockdiag(W^UV) c^KV exactly.
    D = SMALL[1]
    rng = np.random.default_rng(9)
    W = _rand_weights(D, rng)
    h = rng.standard_normal(D.d)
    res = O.decode_token(D, W, h, 0, np.zeros((0, D.row)), absorbed=True)
    c_kv = W["w_dkv"] @ h
    assert np.allclose(res["o_lat"], np.broadcast_to(c_kv, res["o_lat"].shape), rtol=0, atol=1e-14)
    u_ref = W["w_o"] @ (W["w_uv"].reshape(D.n_h, D.d_h, D.d_c) @ c_kv).reshape(-1)
    assert np.max(np.abs(res["u"] - u_ref)) <= 1e-13 * np.max(np.abs(u_ref))


def test_identical_keys_average_values():
    D = SMALL[0]
    rng = np.random.default_rng(10)
    W = _rand_weights(D, rng)
    q_lat, q_r = rng.standard_normal((D.n_h, D.d_c)), rng.standard_normal((D.n_h, D.d_hr))
    rows = rng.standard_normal((6, D.row))
    rows[:, D.d_c:] = rows[0, D.d_c:]  # same rope key
    base = rows[0, :D.d_c].copy()
    # keys identical in the latent too, values differ only along a direction
    # orthogonal to every head's query: scores tie, p is uniform
    rows[:, :D.d_c] = base
    o_lat, _, _ = O.attend_absorbed(D, W, q_lat, q_r, rows)
    assert np.allclose(o_lat, base[None, :], atol=1e-14)
    # uniform scores by zero queries: o_lat is the plain mean of the latents
    rows2 = rng.standard_normal((6, D.row))
    o_lat2, lse2, _ = O.attend_absorbed(D, W, np.zeros_like(q_lat), np.zeros_like(q_r), rows2)
    assert np.allclose(o_lat2, rows2[:, :D.d_c].mean(0)[None, :], atol=1e-14)
    assert np.allclose(lse2, math.log(6), atol=1e-14)


def test_dominant_key_selects_its_value():
    D = SMALL[0]
    rng = np.random.default_rng(11)
    W = _rand_weights(D, rng)
    rows = rng.standard_normal((5, D.row)) * 1e-3
    q_lat = np.zeros((D.n_h, D.d_c))
    q_lat[:, 0] = 1e5
    rows[3, 0] = 1.0
    o_lat, _, _ = O.attend_absorbed(D, W, q_lat, np.zeros((D.n_h, D.d_hr)), rows)
    assert np.allclose(o_lat, rows[3, :D.d_c][None, :], atol=1e-12)


# 5. RoPE invariants ([explainer] 2.2.2: R_m^T R_n depends only on n - m).
def test_rope_invariants():
    rng = np.random.default_rng(12)
    theta = O.rope_frequencies(16, 10000.0)
    q, k = rng.standard_normal(16), rng.standard_normal(16)
    for m, n, delta in [(0, 5, 7), (100, 3, 1000), (131072, 17, 4096)]:
        a = O.rope_rotate(q, m, theta) @ O.rope_rotate(k, n, theta)
        b = O.rope_rotate(q, m + delta, theta) @ O.rope_rotate(k, n + delta, theta)
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)
        assert np.linalg.norm(O.rope_rotate(q, m, theta)) == pytest.approx(np.linalg.norm(q), rel=1e-14)
    assert np.array_equal(O.rope_rotate(q, 0, theta), q)
    # composition: rotating by a then b is rotating by a + b
    r = O.rope_rotate(O.rope_rotate(q, 11, theta), 29, theta)
    assert np.allclose(r, O.rope_rotate(q, 40, theta), atol=1e-13)
    # pair 0 has theta_0 = 1 (base^0): a quarter turn at pos pi/2 is not an
    # integer position, so check the closed form at pos 1 instead
    x = np.zeros(16)
    x[0] = 1.0
    r1 = O.rope_rotate(x, 1, theta)
    assert r1[0] == pytest.approx(math.cos(1.0)) and r1[1] == pytest.approx(math.sin(1.0))
    # the last pair turns by base^(-(d-2)/d)
    x = np.zeros(16)
    x[14] = 1.0
    r2 = O.rope_rotate(x, 1000, theta)
    ang = 1000 * 10000.0 ** (-14 / 16)
    assert r2[14] == pytest.approx(math.cos(ang)) and r2[15] == pytest.approx(math.sin(ang))


def test_yarn_reductions_and_bounds():
    plain = O.rope_frequencies(64, 10000.0)
    assert np.array_equal(O.rope_frequencies(64, 10000.0, yarn_scale=1.0), plain)
    s = 40.0
    y = O.rope_frequencies(64, 10000.0, yarn_scale=s, orig_ctx=4096, alpha=1.0, beta=32.0)
    # every frequency lies between the fully interpolated and the original one
    assert np.all(y <= plain * (1 + 1e-15)) and np.all(y >= plain / s * (1 - 1e-15))
    # pair 0 turns ~652 times over 4096 positions (> beta): kept as is;
    # the last pair turns < 1 time (< alpha): divided by s
    assert y[0] == plain[0] and y[-1] == pytest.approx(plain[-1] / s, rel=1e-15)
    # the ratio y/plain is non-decreasing with frequency (monotone blend)
    ratio = (y / plain)[::-1]
    assert np.all(np.diff(ratio) >= -1e-15)


def test_decode_shift_invariance_of_the_whole_layer():
    # Shifting every position by the same offset leaves u unchanged: the
    # decoupled RoPE carries relative position only ([explainer] 2.2.2).
    D = SMALL[1]
    rng = np.random.default_rng(13)
    W = _rand_weights(D, rng)
    T = 11
    hs = rng.standard_normal((T, D.d))
    outs = []
    for off in (0, 517):
        prior = np.stack([O.compress_kv(D, W, hs[j], j + off) for j in range(T - 1)])
        outs.append(O.decode_token(D, W, hs[-1], T - 1 + off, prior)["u"])
    assert np.max(np.abs(outs[0] - outs[1])) <= 1e-10 * np.max(np.abs(outs[0]))
    # ... while a position mismatch between query and keys changes it
    prior = np.stack([O.compress_kv(D, W, hs[j], j) for j in range(T - 1)])
    wrong = O.decode_token(D, W, hs[-1], T + 3, prior)["u"]
    assert np.max(np.abs(wrong - outs[0])) > 1e-6


def test_prefill_is_causal_decode():
    # Query q of a prefill chunk equals a decode step at position start+q over
    # rows 0..start+q (eq 7's causal sum j <= t).
    D = SMALL[2]
    rng = np.random.default_rng(14)
    W = _rand_weights(D, rng)
    start, n_new = 5, 6
    prior = rng.standard_normal((start, D.row))
    h_new = rng.standard_normal((n_new, D.d))
    new_rows, outs = O.prefill_sequence(D, W, h_new, start, prior, [0, 3, 5], absorbed=False)
    rows = np.concatenate([prior, new_rows])
    for q in (0, 3, 5):
        dec = O.decode_token(D, W, h_new[q], start + q, rows[:start + q], absorbed=False)
        assert np.allclose(dec["row"], new_rows[q], atol=1e-14)
        assert np.max(np.abs(dec["u"] - outs[q]["u"])) <= 1e-13 * np.max(np.abs(dec["u"]))


def test_self_score_is_unrotated_dot():
    # A token attending to its own key sits at relative offset 0, so its RoPE
    # score is the plain dot (W^QR_i c^Q) . (W^KR h): with W^UK = 0 and L zero
    # prior rows, lse_i = log(L + exp(scale * that dot)) in closed form.
    D = SMALL[2]
    rng = np.random.default_rng(15)
    W = _rand_weights(D, rng)
    W["w_uk"] = np.zeros_like(W["w_uk"])
    h = rng.standard_normal(D.d)
    L, pos = 4, 1234
    res = O.decode_token(D, W, h, pos, np.zeros((L, D.row)))
    qr = (W["w_qr"] @ h).reshape(D.n_h, D.d_hr)
    kr = W["w_kr"] @ h
    scale = D.attn_logit_factor / math.sqrt(D.d_h + D.d_hr)
    ref = np.log(L + np.exp(scale * (qr @ kr)))
    assert np.max(np.abs(res["lse"] - ref)) < 1e-12


# Paged cache ([explainer] 2.2.2: one cached row [c^KV | k^R] per token, here
# in 64-token pages reached through a page table).  The generator draws each
# sequence's prior rows in token order from its own seeded stream before
# scattering them over permuted pages; the oracle's gather must return exactly
# that order (a swapped page/slot index or a shifted slot reads other rows).
def test_gather_rows_returns_rows_in_token_order():
    import dataclasses
    from head_latent_attention_03_b200 import inputs as I
    D = dataclasses.replace(TINY, block_size=8)
    w = I.Workload("gather_pin", 7, D, 3, "list:5,17,30", permute_pages=True)
    batch = I.gen_batch(w)
    assert not np.array_equal(batch.block_table[:, 0], np.arange(3))  # pages really permuted
    for b, L in enumerate(batch.prior_len):
        want = I._store(I._normal(I.rng_for(w.cfg_id, I._T_PRIOR, b), (int(L), D.row), 1.0), D)
        got = O.gather_rows(batch.pool, batch.block_table[b], int(L), D.block_size)
        assert np.array_equal(got, want.astype(np.float64)), b


def test_gather_rows_hand_computed_lookup():
    # a fixed 3-page pool of 4-slot pages whose row values encode (page,
    # slot); the table sends token j of the sequence to page [2, 0, 1][j // 4],
    # slot j % 4.  Token 5 sits on page 0 slot 1, token 9 on page 1 slot 1,
    # token 2 on page 2 slot 2 (worked out by hand from that table).
    pool = np.array([[[10 * p + s, -(10 * p + s)] for s in range(4)] for p in range(3)], dtype=np.float64)
    table = np.array([2, 0, 1], dtype=np.int32)
    rows = O.gather_rows(pool, table, 10, 4)
    assert rows.shape == (10, 2)
    assert rows[5].tolist() == [1.0, -1.0]
    assert rows[9].tolist() == [11.0, -11.0]
    assert rows[2].tolist() == [22.0, -22.0]
    assert rows[0].tolist() == [20.0, -20.0] and rows[4].tolist() == [0.0, 0.0]


# Data flow of the decoupled RoPE parts ([explainer] 2.2.2): the shared key
# k^R is computed from h_t itself, not from the latent c^KV, and both query
# parts come from the query latent c^Q.  Zeroing W^DKV must leave k^R intact;
# zeroing W^DQ must silence q^C and q^R.
def test_key_rope_comes_from_h_and_query_parts_from_the_query_latent():
    D = SMALL[1]  # query compression on (d_cq > 0)
    rng = np.random.default_rng(11)
    W = _rand_weights(D, rng)
    h = rng.standard_normal(D.d)
    W0 = dict(W, w_dkv=np.zeros_like(W["w_dkv"]))
    row = O.compress_kv(D, W0, h, 5)
    assert np.all(row[:D.d_c] == 0)
    assert np.linalg.norm(row[D.d_c:]) > 0.1 * np.linalg.norm(O.compress_kv(D, W, h, 5)[D.d_c:])
    W1 = dict(W, w_dq=np.zeros_like(W["w_dq"]))
    q_c, q_r = O.queries(D, W1, h, 5)
    assert np.all(q_c == 0) and np.all(q_r == 0)
    q_c, q_r = O.queries(D, W, h, 5)
    assert np.linalg.norm(q_c) > 0 and np.linalg.norm(q_r) > 0


# Vanishing queries (eq 7 with every logit zero): the softmax is uniform over
# the L + 1 visible rows (prior rows and the new token), so each head's o_lat
# is the plain mean of their c^KV parts, the new row included, and the lse is
# log(L + 1).
def test_vanishing_queries_attend_uniformly_over_all_visible_rows():
    for D in SMALL:
        rng = np.random.default_rng(13)
        W = _rand_weights(D, rng)
        W = dict(W, w_uq=np.zeros_like(W["w_uq"]), w_qr=np.zeros_like(W["w_qr"]))
        L = 9
        prior = rng.standard_normal((L, D.d_c + D.d_hr))
        h = rng.standard_normal(D.d)
        out = O.decode_token(D, W, h, L, prior, absorbed=True)
        rows = np.concatenate([prior, out["row"][None, :]], axis=0)
        want = rows[:, :D.d_c].mean(axis=0)
        for i in range(D.n_h):
            np.testing.assert_allclose(out["o_lat"][i], want, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out["lse"], math.log(L + 1), rtol=1e-12)


# RMSNorm after the compressed latents and the bottleneck scale factors
# ([explainer] 3.1.1, no formula printed; the reading: c <- s * g * c / rms(c)).
NORM_DIMS = LayerDims(d=40, n_h=2, d_h=8, d_c=24, d_cq=20, d_hr=6, dtype="f32", latent_norm=True, norm_eps=0.0,
                      scale_kv=1.7, scale_q=0.6)


def _norm_weights(D, rng, gains=True):
    W = _rand_weights(D, rng)
    W["g_kv"] = 1.0 + 0.1 * rng.standard_normal(D.d_c) if gains else np.ones(D.d_c)
    W["g_q"] = 1.0 + 0.1 * rng.standard_normal(D.d_cq) if gains else np.ones(D.d_cq)
    return W


def test_latent_norm_gives_the_scale_as_rms():
    # unit gains, eps = 0: the cached latent's root mean square is exactly the
    # bottleneck scale factor, whatever h is; the factor acts after the norm,
    # so doubling it doubles the latent
    rng = np.random.default_rng(31)
    D = NORM_DIMS
    W = _norm_weights(D, rng, gains=False)
    for _ in range(3):
        h = rng.standard_normal(D.d) * rng.uniform(0.1, 10.0)
        c = O.compress_kv(D, W, h, 5)[:D.d_c]
        assert abs(math.sqrt(np.mean(c * c)) - D.scale_kv) < 1e-12
        D2 = LayerDims(**{**D.__dict__, "scale_kv": 2 * D.scale_kv})
        assert np.allclose(O.compress_kv(D2, W, h, 5)[:D.d_c], 2 * c, rtol=1e-13, atol=0)


def test_latent_norm_removes_the_scale_of_h_but_not_from_k_rope():
    # c^KV and c^Q are linear in h; after the norm (eps = 0) they no longer
    # depend on h's scale, so neither do q^C and q^R.  k^R comes from h
    # directly and scales with it.
    rng = np.random.default_rng(32)
    D = NORM_DIMS
    W = _norm_weights(D, rng)
    h = rng.standard_normal(D.d)
    a = 3.25
    r1, r2 = O.compress_kv(D, W, h, 9), O.compress_kv(D, W, a * h, 9)
    assert np.allclose(r2[:D.d_c], r1[:D.d_c], rtol=1e-12, atol=0)
    assert np.allclose(r2[D.d_c:], a * r1[D.d_c:], rtol=1e-12, atol=0)
    (qc1, qr1), (qc2, qr2) = O.queries(D, W, h, 9), O.queries(D, W, a * h, 9)
    assert np.allclose(qc2, qc1, rtol=1e-12, atol=1e-14) and np.allclose(qr2, qr1, rtol=1e-12, atol=1e-14)
    # without the norm the queries scale with h
    D0 = LayerDims(**{**D.__dict__, "latent_norm": False})
    qc0a, _ = O.queries(D0, W, h, 9)
    qc0b, _ = O.queries(D0, W, a * h, 9)
    assert np.allclose(qc0b, a * qc0a, rtol=1e-12, atol=1e-14)


def test_latent_norm_gain_is_per_feature():
    # eps = 0: the latent with gains g, divided feature by feature by the
    # latent with unit gains, is g itself
    rng = np.random.default_rng(33)
    D = NORM_DIMS
    W = _norm_weights(D, rng)
    W1 = dict(W, g_kv=np.ones(D.d_c), g_q=np.ones(D.d_cq))
    h = rng.standard_normal(D.d)
    assert np.allclose(O.compress_kv(D, W, h, 2)[:D.d_c] / O.compress_kv(D, W1, h, 2)[:D.d_c], W["g_kv"],
                       rtol=1e-12, atol=0)


def test_latent_norm_epsilon_closed_form():
    # unit gains and factors: mean(y^2) = m / (m + eps), m = mean(c^2) of the
    # raw latent W^DKV h
    rng = np.random.default_rng(34)
    D = LayerDims(**{**NORM_DIMS.__dict__, "norm_eps": 0.05, "scale_kv": 1.0})
    W = _norm_weights(D, rng, gains=False)
    h = 0.2 * rng.standard_normal(D.d)
    raw = W["w_dkv"] @ h
    m = float(np.mean(raw * raw))
    y = O.compress_kv(D, W, h, 0)[:D.d_c]
    assert abs(float(np.mean(y * y)) - m / (m + D.norm_eps)) < 1e-13


# Context parallelism (the attention over a sequence's rows split between
# ranks): the softmax over a union of disjoint row sets is the sets' softmaxes
# weighted by their partition sums, so the merged partial attentions are the
# attention over all rows (1e-12), an empty set included.
def test_merged_partials_equal_attention_over_all_rows():
    rng = np.random.default_rng(41)
    D = SMALL[1]
    W = _rand_weights(D, rng)
    rows = rng.standard_normal((70, D.row)) * 1.5
    q_lat = rng.standard_normal((D.n_h, D.d_c))
    q_r = rng.standard_normal((D.n_h, D.d_hr))
    full_o, full_lse, _ = O.attend_absorbed(D, W, q_lat, q_r, rows)
    cuts = [(0, 0), (0, 23), (23, 64), (64, 70)]  # the first rank holds no rows
    parts_o, parts_l = [], []
    for a, b in cuts:
        if a == b:
            parts_o.append(np.zeros((D.n_h, D.d_c)))
            parts_l.append(np.full(D.n_h, -np.inf))
        else:
            o, l, _ = O.attend_absorbed(D, W, q_lat, q_r, rows[a:b])
            parts_o.append(o)
            parts_l.append(l)
    o, lse = O.merge_partials(parts_o, parts_l)
    assert np.max(np.abs(o - full_o)) <= 1e-12 * np.max(np.abs(full_o))
    assert np.max(np.abs(lse - full_lse)) <= 1e-12 * np.max(np.abs(full_lse))


# 13. the quantised latent cache ([explainer] 3.1.4: the KV cache is
# quantised for serving).  The format (FP8 E4M3 codes of c^KV, one
# power-of-two scale per row, k^R kept) is a reading; the pins below fix the
# arithmetic of that reading from the format's bit-level definition, not from
# the oracle's own formula.

def _e4m3_table():
    """Every finite E4M3 value from its bit fields (sign, 4-bit exponent with
    bias 7, 3-bit mantissa; exponent field 0 = subnormal; S.1111.111 = NaN),
    with the mantissa field of each."""
    vals, mants = [], []
    for bits in range(256):
        s, E, m = bits >> 7, (bits >> 3) & 15, bits & 7
        if E == 15 and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if E == 0 else (1.0 + m / 8.0) * 2.0 ** (E - 7)
        vals.append(-v if s else v)
        mants.append(m)
    return np.array(vals), np.array(mants)


def _e4m3_brute(x):
    """Nearest finite E4M3 value by search; a tie goes to the even mantissa
    field; magnitudes past the largest value saturate to it."""
    vals, mants = _e4m3_table()
    out = np.empty_like(x)
    top = np.max(vals)
    for i, v in enumerate(x):
        if abs(v) >= top:
            out[i] = math.copysign(top, v)
            continue
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            best = [b for b in best if mants[b] % 2 == 0 and (vals[b] != 0 or math.copysign(1, vals[b]) == math.copysign(1, v))] or best
        out[i] = vals[best[0]]
    return out


def test_e4m3_rounding_matches_search_over_all_codes():
    vals, _ = _e4m3_table()
    assert np.max(vals) == 448.0 and len(np.unique(vals)) == 253  # 254 finite codes, +0 and -0 equal
    pos = np.unique(vals[vals > 0])
    mids = (pos[:-1] + pos[1:]) / 2  # every tie between neighbours
    rng = np.random.default_rng(13)
    mags = np.ldexp(rng.uniform(1.0, 2.0, 3000), rng.integers(-12, 10, 3000))
    x = np.concatenate([mids, -mids, pos, mags, -mags, [0.0, 2.0 ** -10, 460.0, 464.0, 500.0, 1e4]])
    got = O.e4m3_round(x)
    want = _e4m3_brute(x)
    assert np.array_equal(got, want), x[got != want][:5]


def test_e4m3_worked_values():
    # hand-computed: 1.0625 lies halfway between 1 (mantissa 000) and 1.125
    # (001) -> 1; 1.1875 between 1.125 (001) and 1.25 (010) -> 1.25; 3 * 2^-10
    # between the subnormals 2^-9 (001) and 2^-8 (010) -> 2^-8; 2^-10 between
    # 0 and 2^-9 -> 0; 464 between 448 and the missing 480 -> 448 (saturated)
    x = np.array([1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, 464.0, 1000.0, -1.0625, 240.0, 0.3, 2.0 ** -9])
    want = np.array([1.0, 1.25, 2.0 ** -8, 0.0, 448.0, 448.0, -1.0, 240.0, 0.3125, 2.0 ** -9])
    assert np.array_equal(O.e4m3_round(x), want)


def test_fp8_row_scale_uses_the_top_binade():
    rng = np.random.default_rng(14)
    for _ in range(200):
        c = rng.standard_normal(512) * 2.0 ** rng.uniform(-20, 20)
        amax = np.max(np.abs(c))
        codes, e = O.quantize_latent(c)
        assert 224.0 < amax * 2.0 ** -e <= 448.0
        # largest code in the top binade, nothing saturated beyond rounding
        assert 224.0 <= np.max(np.abs(codes)) <= 448.0
        back = codes * 2.0 ** e
        normal = np.abs(c) * 2.0 ** -e >= 2.0 ** -6
        # normal values: half a spacing of 2^-3 relative; subnormals: 2^-10 * 2^e
        assert np.all(np.abs(back - c)[normal] <= 2.0 ** -4 * np.abs(c)[normal])
        assert np.all(np.abs(back - c)[~normal] <= 2.0 ** (e - 10))
    assert O.fp8_scale_exponent(448.0) == 0 and O.fp8_scale_exponent(448.5) == 1
    assert O.fp8_scale_exponent(1.75) == -8 and O.fp8_scale_exponent(0.0) == 0


def test_fp8_cached_row_keeps_k_rope_and_is_a_fixed_point():
    import dataclasses
    D = dataclasses.replace(LITE, cache_dtype="fp8")
    rng = np.random.default_rng(15)
    row = rng.standard_normal(D.row)
    once = O.cached_row(D, row)
    assert np.array_equal(once[D.d_c:], row[D.d_c:])
    assert not np.array_equal(once[:D.d_c], row[:D.d_c])
    # read back at the row's own magnitude: within half an E4M3 spacing
    # (2^-4 relative) of the largest element
    assert np.max(np.abs(once[:D.d_c] - row[:D.d_c])) <= 2.0 ** -4 * np.max(np.abs(row[:D.d_c]))
    assert np.array_equal(O.cached_row(D, once), once)
    # the bf16 cache reads rows back unchanged
    assert np.array_equal(O.cached_row(LITE, row), row)
