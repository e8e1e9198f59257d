"""CUDA path vs the fp64 oracle, through the C ABI, on seeded synthetic inputs.

Each case runs the whole layer step on the GPU (compress_append -> absorb_q
-> decode/prefill attention -> out_proj) and compares every stage with the
oracle's own intermediates computed from the same generator inputs:
the appended cache row, q_lat / q_rope, o_lat / lse and u.  Tolerances:
fp32 layers max relative error 1e-4; bf16 layers RMS-relative 5e-3 and max
absolute 2e-2 (tests/metrics.py).
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from head_latent_attention_03_b200 import inputs as I
from head_latent_attention_03_b200 import mla
from head_latent_attention_03_b200.layer import MLALayer
from oracle import mla_oracle as O
from tests.metrics import assert_bf16, assert_fp32, rms_rel, max_abs, check_fp8_row, decode_fp8_rows

pytestmark = pytest.mark.gpu

W_CACHE = {}


def weights_for(w):
    key = (w.cfg_id, w.dims)
    if key not in W_CACHE:
        W_CACHE[key] = I.gen_weights(w)
    return W_CACHE[key]


def run_gpu(w, batch, num_splits=0):
    weights = weights_for(w)
    layer = MLALayer(w.dims, weights)
    st = layer.upload(batch)
    layer.step(st, num_splits=num_splits)
    torch.cuda.synchronize()
    code = mla.get_last_error()
    assert code == 0, mla.status_string(code)
    return layer, st


def np32(t):
    return t.float().cpu().numpy()


def new_rows(st, batch):
    """The rows the step appended, as stored (FP8 cache: the raw bytes)."""
    D = batch.workload.dims
    pool = st.pool.cpu().numpy() if st.pool.dtype == torch.uint8 else np32(st.pool)
    out = []
    for b, L in enumerate(batch.prior_len):
        for t in range(batch.workload.new_tokens):
            p = int(L) + t
            out.append(pool[batch.block_table[b, p // D.block_size], p % D.block_size])
    return np.stack(out)


def compare(name, g, r, dims):
    if dims.dtype == "f32":
        assert_fp32(g, r, name)
    else:
        assert_bf16(g, r, name)


def check_decode(w, seqs=None, num_splits=0, batch=None):
    batch = batch or I.gen_batch(w)
    layer, st = run_gpu(w, batch, num_splits)
    D = w.dims
    seqs = list(range(len(batch.prior_len))) if seqs is None else seqs
    ref = O.decode_batch(batch, weights_for(w), seqs=seqs, absorbed=True)
    ref_un = O.decode_batch(batch, weights_for(w), seqs=seqs, absorbed=False)
    rows = new_rows(st, batch)[seqs]
    if D.cache_dtype == "fp8":
        for i, r in enumerate(ref):
            check_fp8_row(rows[i], r["row"], D.d_c, D.d_hr, O.e4m3_round, O.fp8_scale_exponent, f"cache row {i}")
    else:
        compare("cache row", rows, np.stack([r["row"] for r in ref]), D)
    compare("q_lat", np32(st.q_lat)[seqs], np.stack([r["q_lat"] for r in ref]), D)
    compare("q_rope", np32(st.q_rope)[seqs], np.stack([r["q_r"] for r in ref]), D)
    compare("o_lat", np32(st.o_lat)[seqs], np.stack([r["o_lat"] for r in ref]), D)
    lse_g, lse_r = np32(st.lse)[seqs], np.stack([r["lse"] for r in ref])
    assert np.max(np.abs(lse_g - lse_r)) < (1e-4 if D.dtype == "f32" else 2e-2), np.max(np.abs(lse_g - lse_r))
    compare("u", np32(st.u)[seqs], np.stack([r["u"] for r in ref_un]), D)
    return batch, st


# ----------------------------------------------------------------------------
# small cases: every sequence checked, several tiles and a ragged tail
# ----------------------------------------------------------------------------
def test_tiny_fp32_step():
    check_decode(I.WORKLOADS["tiny"])


def test_tiny_fp32_prefill_chunk():
    w = dataclasses.replace(I.WORKLOADS["tiny"], batch=2, prior="list:5,64", new_tokens=9)
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    D = w.dims
    W = weights_for(w)
    rows_g = new_rows(st, batch)
    for b in range(2):
        L = int(batch.prior_len[b])
        prior = O.gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
        new_r, outs = O.prefill_sequence(D, W, batch.h[b * 9:(b + 1) * 9], L, prior, range(9), absorbed=True)
        assert_fp32(rows_g[b * 9:(b + 1) * 9], new_r, "rows")
        for q in range(9):
            r = b * 9 + q
            assert_fp32(np32(st.o_lat)[r], outs[q]["o_lat"], f"o_lat {b},{q}")
            assert_fp32(np32(st.u)[r], outs[q]["u"], f"u {b},{q}")


LITE_SMALL = dataclasses.replace(I.WORKLOADS["lite"], name="lite_small", batch=4, prior="list:0,63,200,700")
V2_SMALL = dataclasses.replace(I.WORKLOADS["v2"], name="v2_small", batch=3, prior="list:127,128,1000")
YARN_SMALL = dataclasses.replace(I.WORKLOADS["long"], name="yarn_small", batch=2, prior="list:129,3000")


@pytest.mark.parametrize("w", [LITE_SMALL, V2_SMALL, YARN_SMALL], ids=lambda w: w.name)
def test_bf16_small(w):
    check_decode(w)


def _with_norm(w, name):
    # RMSNorm after c^KV and c^Q with gains 1 + N(0, 0.1^2) and bottleneck
    # scale factors away from 1
    return dataclasses.replace(w, name=name, dims=dataclasses.replace(w.dims, latent_norm=True, norm_eps=1e-6,
                                                                      scale_kv=1.5, scale_q=0.75))


@pytest.mark.parametrize("w", [_with_norm(I.WORKLOADS["tiny"], "tiny_norm"), _with_norm(LITE_SMALL, "lite_norm"),
                               _with_norm(V2_SMALL, "v2_norm")], ids=lambda w: w.name)
def test_latent_norm(w):
    # the cached c^KV row, q_lat (from the normalised c^Q) and the whole
    # layer against the oracle with the same norm
    check_decode(w)


@pytest.mark.parametrize("n_h,splits", [(32, 0), (32, 3), (64, 0), (64, 3)])
def test_bf16_other_head_counts(n_h, splits):
    # 32 and 64 heads: the one-CTA kernel with one or two 32-head groups per
    # row (the groups of a segment run side by side), automatic and explicit
    # splits.
    w = dataclasses.replace(LITE_SMALL, name=f"heads{n_h}", dims=dataclasses.replace(I.LITE, n_h=n_h))
    check_decode(w, num_splits=splits)


@pytest.mark.parametrize("splits", [1, 2, 4, 5])
def test_split_count_invariance(splits):
    w = dataclasses.replace(LITE_SMALL, prior="list:300,1500,900,64")
    check_decode(w, num_splits=splits)


def test_page_order_invariance():
    # the same sequences on a permuted page table give bit-identical results
    w = dataclasses.replace(LITE_SMALL, prior="list:300,1500,900,64")
    b1 = I.gen_batch(w)
    _, st1 = run_gpu(w, b1, 3)
    u1, o1 = np32(st1.u), np32(st1.o_lat)
    b2 = I.gen_batch(dataclasses.replace(w, permute_pages=True))
    perm = np.random.default_rng(5).permutation(b1.pool.shape[0])
    pool2 = np.full_like(b1.pool, np.nan)
    table2 = b1.block_table.copy()
    for b in range(table2.shape[0]):
        for j in range(table2.shape[1]):
            if table2[b, j] >= 0:
                pool2[perm[b1.block_table[b, j]]] = b1.pool[b1.block_table[b, j]]
                table2[b, j] = perm[b1.block_table[b, j]]
    b2 = dataclasses.replace(b1, pool=pool2, block_table=table2)
    _, st2 = run_gpu(w, b2, 3)
    assert np.array_equal(np32(st2.o_lat), o1)
    assert np.array_equal(np32(st2.u), u1)


def test_single_row_returns_new_latent():
    # kv_len = 1: softmax over one key is exactly 1, o_lat = the appended c^KV
    w = dataclasses.replace(LITE_SMALL, batch=2, prior="list:0,0")
    batch = I.gen_batch(w)
    _, st = run_gpu(w, batch)
    rows = new_rows(st, batch)
    assert np.array_equal(np32(st.o_lat), np.broadcast_to(rows[:, None, :512], (2, 16, 512)))


def test_bad_page_id_reports_capacity_error():
    w = dataclasses.replace(LITE_SMALL, batch=2, prior="list:100,300")
    batch = I.gen_batch(w)
    batch.block_table[1, 2] = batch.pool.shape[0] + 7
    layer = MLALayer(w.dims, weights_for(w))
    st = layer.upload(batch)
    layer.attend(st)
    assert mla.get_last_error() == 3  # MLA_ERR_CAPACITY, no fault
    assert mla.get_last_error() == 0  # cleared


@pytest.mark.parametrize("w", [LITE_SMALL, V2_SMALL], ids=lambda w: w.name)
def test_out_of_range_kv_len_reports_capacity_error(w):
    # kv_len beyond the page table (max_blocks * 64) and kv_len = 0: the plan
    # clamps the rows it deals out and the kernels skip the segment, so no
    # page outside the table is read; the call reports MLA_ERR_CAPACITY
    batch = I.gen_batch(w)
    layer = MLALayer(w.dims, weights_for(w))
    st = layer.upload(batch)
    layer.compress_append(st)
    layer.absorb_q(st)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0
    for bad in (st.table.shape[1] * 64 + 5, 0):
        kv = st.kv_len.clone()
        kv[1] = bad
        mla.decode_attn(layer.desc, st.q_lat, st.q_rope, layer.cache(st), kv, st.ws, st.o_lat, st.lse)
        assert mla.get_last_error() == 3  # MLA_ERR_CAPACITY, no fault
        assert mla.get_last_error() == 0  # cleared
    # the next valid call is unaffected
    layer.attend(st)
    layer.out_proj(st)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0


# ----------------------------------------------------------------------------
# full-size workloads, in the launch configuration bench.py times; the oracle
# checks a sample of sequences
# ----------------------------------------------------------------------------
def test_plan_over_many_rows():
    # More decode rows than the plan kernel's 1024 threads: its scans run in
    # two chunks whose carries decide every later row's segments and slots.
    # Short ragged caches cut most rows across CTAs (combine on).  Rows on
    # both sides of the chunk boundary are checked.
    w = dataclasses.replace(I.WORKLOADS["lite"], name="lite_many", batch=1100, prior="uniform:0:200")
    check_decode(w, seqs=[0, 1, 511, 1022, 1023, 1024, 1025, 1099])


@pytest.mark.parametrize("name,seqs", [("lite", [0, 31]), ("v2", None)])
def test_full_size_sampled(name, seqs):
    w = I.WORKLOADS[name]
    if seqs is None:
        lens = I.prior_lengths(w)
        seqs = [int(np.argmin(lens)), int(np.argmax(lens))]
    check_decode(w, seqs=seqs)


def test_long_context_sampled():
    # 4 x 131072 prior tokens, YaRN s = 40: the appended row (k^R rotated at
    # position 131072 with the blended frequencies) and the queries of every
    # sequence, and the whole attention of one sequence.
    w = I.WORKLOADS["long"]
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    D, W = w.dims, weights_for(w)
    rows = new_rows(st, batch)
    for b in range(w.batch):
        pos = int(batch.positions[b])
        assert pos == 131072
        ref_row = O.compress_kv(D, W, batch.h[b], pos)
        assert_bf16(rows[b], ref_row, f"cache row {b}")
        assert_bf16(rows[b][D.d_c:], ref_row[D.d_c:], f"rotated k^R {b}")
        q_c, q_r = O.queries(D, W, batch.h[b], pos)
        assert_bf16(np32(st.q_rope)[b], q_r, f"q_rope {b}")
        assert_bf16(np32(st.q_lat)[b], O.absorb_query(D, W, q_c), f"q_lat {b}")
    ref = O.decode_batch(batch, W, seqs=[3], absorbed=True)[0]
    assert_bf16(np32(st.o_lat)[3], ref["o_lat"], "o_lat")
    assert np.max(np.abs(np32(st.lse)[3] - ref["lse"])) < 2e-2
    assert_bf16(np32(st.u)[3], ref["u"], "u")


@pytest.mark.parametrize("b,qs", [(5, [0, 1, 63, 64, 1000, 4095]), (0, [62, 63, 2047, 4094])])
def test_prefill_sampled(b, qs):
    # Queries of two of the eight sequences.  With 4096 prior tokens the query
    # at chunk offset q attends rows 0 .. 4096 + q: q = 63 ends on the last slot
    # of a page, q = 64 on the first slot of the next, q = 4095 in the last page.
    w = I.WORKLOADS["prefill"]
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    D, W = w.dims, weights_for(w)
    n = w.new_tokens
    L = int(batch.prior_len[b])
    prior = O.gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
    new_r, outs = O.prefill_sequence(D, W, batch.h[b * n:(b + 1) * n], L, prior, qs, absorbed=True)
    assert_bf16(new_rows(st, batch)[b * n:(b + 1) * n], new_r, "rows")
    for q in qs:
        assert_bf16(np32(st.o_lat)[b * n + q], outs[q]["o_lat"], f"o_lat q={q}")
        assert np.max(np.abs(np32(st.lse)[b * n + q] - outs[q]["lse"])) < 2e-2
        assert_bf16(np32(st.u)[b * n + q], outs[q]["u"], f"u q={q}")


# ----------------------------------------------------------------------------
# context parallelism: each rank's partial over its shard of the rows (the
# ranks run one after another on this GPU; each reads only its rows), merged
# by log-sum-exp
# ----------------------------------------------------------------------------
def _cp_merge(layer, st, batch, world):
    from head_latent_attention_03_b200.context_parallel import shard_ranges
    D = batch.workload.dims
    B = len(batch.prior_len)
    ranges = shard_ranges(batch.prior_len + 1, world)
    o_parts = torch.empty((world, B, D.n_h, D.d_c), dtype=torch.float32, device="cuda")
    l_parts = torch.empty((world, B, D.n_h), dtype=torch.float32, device="cuda")
    cache = layer.cache(st)
    for r in range(world):
        kb = torch.from_numpy(ranges[r, :, 0].copy()).cuda()
        ke = torch.from_numpy(ranges[r, :, 1].copy()).cuda()
        mla.decode_attn_partial(layer.desc, st.q_lat, st.q_rope, cache, kb, ke, st.ws, o_parts[r], l_parts[r])
    o = torch.empty_like(st.o_lat)
    l = torch.empty_like(st.lse)
    mla.lse_merge(layer.desc, o_parts, l_parts, o, l)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0
    return ranges, o_parts, l_parts, o, l


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_merge(world):
    w = dataclasses.replace(I.WORKLOADS["v2"], name="v2_cp", batch=3, prior="list:1000,3000,129")
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    D, W = w.dims, weights_for(w)
    ranges, o_parts, l_parts, o, l = _cp_merge(layer, st, batch, world)
    # one rank's partial against the oracle over that rank's rows
    ref = O.decode_batch(batch, W, absorbed=True)
    r = world - 1
    for b in range(3):
        lo, hi = ranges[r, b]
        rows = O.gather_rows(batch.pool, batch.block_table[b], int(batch.prior_len[b]), D.block_size)
        rows = np.concatenate([rows, ref[b]["row"][None]], axis=0)
        if hi > lo:
            po, pl, _ = O.attend_absorbed(D, W, ref[b]["q_lat"], ref[b]["q_r"], rows[lo:hi])
            assert_bf16(np32(o_parts[r, b]), po, f"partial o rank {r} seq {b}")
            assert np.max(np.abs(np32(l_parts[r, b]) - pl)) < 2e-2
        else:
            assert np.all(np32(o_parts[r, b]) == 0) and np.all(np.isneginf(np32(l_parts[r, b])))
    # the merge against the oracle over all rows and against mla_decode_attn
    assert_bf16(np32(o), np.stack([x["o_lat"] for x in ref]), "merged o_lat")
    assert np.max(np.abs(np32(l) - np.stack([x["lse"] for x in ref]))) < 2e-2
    assert_bf16(np32(o), np32(st.o_lat), "merged vs one-GPU decode")


def test_context_parallel_long_context():
    # 4 x 131073 rows over 4 ranks: the merged result is the one-GPU decode
    w = I.WORKLOADS["long"]
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    _, _, _, o, l = _cp_merge(layer, st, batch, 4)
    assert_bf16(np32(o), np32(st.o_lat), "merged vs one-GPU decode")
    assert np.max(np.abs(np32(l) - np32(st.lse))) < 2e-2


# ----------------------------------------------------------------------------
# un-absorbed chunked prefill: decompressed per-head keys and values, causal
# flash attention, W^O; against the oracle's un-absorbed form (eqs 10-11)
# ----------------------------------------------------------------------------
def _unabsorbed(w, batch):
    layer = MLALayer(w.dims, weights_for(w))
    st = layer.upload(batch)
    layer.prefill_step_unabsorbed(st)
    torch.cuda.synchronize()
    code = mla.get_last_error()
    assert code == 0, mla.status_string(code)
    return layer, st


def _check_unabsorbed(w, batch, st, seqs_queries):
    D, W = w.dims, weights_for(w)
    n = w.new_tokens
    for b, qs in seqs_queries:
        L = int(batch.prior_len[b])
        prior = O.gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
        new_r, outs = O.prefill_sequence(D, W, batch.h[b * n:(b + 1) * n], L, prior, qs, absorbed=False)
        assert_bf16(new_rows(st, batch)[b * n:(b + 1) * n], new_r, "rows")
        for q in qs:
            r = b * n + q
            assert_bf16(np32(st.o)[r], outs[q]["o"], f"o b={b} q={q}")
            assert np.max(np.abs(np32(st.lse)[r] - outs[q]["lse"])) < 2e-2
            assert_bf16(np32(st.u)[r], outs[q]["u"], f"u b={b} q={q}")


def test_unabsorbed_prefill_small():
    # 200 new queries (two query blocks, the second partial) over 100 and 300
    # prior rows; the last page of each sequence is partly unwritten (NaN)
    w = dataclasses.replace(I.WORKLOADS["prefill"], name="pf_small", batch=2, prior="list:100,300", new_tokens=200)
    batch = I.gen_batch(w)
    layer, st = _unabsorbed(w, batch)
    _check_unabsorbed(w, batch, st, [(0, list(range(0, 200, 7)) + [199]), (1, [0, 27, 63, 64, 127, 128, 199])])
    # the latent form of the same chunk gives the same layer output
    _, st2 = run_gpu(w, batch)
    assert_bf16(np32(st.u), np32(st2.u), "un-absorbed vs absorbed u")


def test_unabsorbed_prefill_full_size_sampled():
    w = I.WORKLOADS["prefill"]
    batch = I.gen_batch(w)
    layer, st = _unabsorbed(w, batch)
    _check_unabsorbed(w, batch, st, [(5, [0, 1, 127, 128, 2047, 4095]), (0, [63, 64, 4094])])


# ----------------------------------------------------------------------------
# FP8 latent cache (E4M3 codes of c^KV, one power-of-two scale per row, bf16
# k^R): the encoding of the drawn rows is exact, the new row's codes follow
# the oracle's rounding, and the attention over the dequantised rows matches
# the oracle's attention over its own dequantised rows.
# ----------------------------------------------------------------------------
LITE_FP8_SMALL = dataclasses.replace(I.WORKLOADS["lite_fp8"], name="lite_fp8_small", batch=4,
                                     prior="list:63,200,700,1500")


def test_fp8_encoding_of_the_drawn_rows_is_exact():
    w = LITE_FP8_SMALL
    D = w.dims
    batch = I.gen_batch(w)
    layer = MLALayer(D, weights_for(w))
    st = layer.upload(batch)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0
    assert st.pool.shape[2] == mla.cache_row_bytes(layer.desc) == 656
    raw = st.pool.cpu().numpy()
    for b in range(w.batch):
        L = int(batch.prior_len[b])
        rows = O.gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
        got = np.stack([raw[batch.block_table[b, j // 64], j % 64] for j in range(L)])
        codes, scale, k_r, pad = decode_fp8_rows(got, D.d_c, D.d_hr)
        for j in range(L):
            want, e = O.quantize_latent(rows[j, :D.d_c])
            assert scale[j] == 2.0 ** e, (b, j)
            assert np.array_equal(codes[j], want), (b, j)
        assert np.array_equal(k_r, rows[:, D.d_c:])
        assert not pad.any()


@pytest.mark.parametrize("splits", [0, 3])
def test_fp8_decode_small(splits):
    check_decode(LITE_FP8_SMALL, num_splits=splits)


@pytest.mark.parametrize("n_h", [32, 64])
def test_fp8_decode_other_head_counts(n_h):
    w = dataclasses.replace(LITE_FP8_SMALL, name=f"fp8_heads{n_h}",
                            dims=dataclasses.replace(LITE_FP8_SMALL.dims, n_h=n_h))
    check_decode(w)


def test_fp8_decode_with_latent_norm():
    # the normalised and scaled c^KV is what gets encoded
    w = _with_norm(LITE_FP8_SMALL, "lite_fp8_norm")
    check_decode(w)


def test_fp8_decode_v2_small():
    # 128 heads over FP8 rows: the CTA-pair kernel with its converter warps
    w = dataclasses.replace(I.WORKLOADS["v2_fp8"], name="v2_fp8_small", batch=3, prior="list:127,128,1000")
    check_decode(w)


@pytest.mark.parametrize("splits", [0, 1, 3])
def test_fp8_decode_v2_page_edges(splits):
    # kv_len 1, 64, 65, 192 and 1001 on a permuted page table: a tile whose
    # second page lies past the row, one whose second page holds one row, a
    # full page followed by an empty one; automatic, one-per-row and explicit
    # splits
    w = dataclasses.replace(I.WORKLOADS["v2_fp8"], name="v2_fp8_edges", batch=5, prior="list:0,63,64,191,1000")
    check_decode(w, num_splits=splits)


def test_fp8_decode_v2_with_latent_norm():
    w = _with_norm(dataclasses.replace(I.WORKLOADS["v2_fp8"], name="v2_fp8_norm", batch=2, prior="list:300,65"),
                   "v2_fp8_norm")
    check_decode(w)


def test_fp8_v2_full_size_sampled():
    # the V2 workload over an FP8 cache: two sequences through the oracle
    w = I.WORKLOADS["v2_fp8"]
    lens = I.prior_lengths(w)
    check_decode(w, seqs=[int(np.argmin(lens)), int(np.argmax(lens))])


def test_fp8_full_size_sampled():
    # 32 x 4096 prior tokens (the V2-Lite workload over an FP8 cache): two
    # sequences through the oracle
    w = I.WORKLOADS["lite_fp8"]
    check_decode(w, seqs=[0, 31])


def test_fp8_prefill_chunk():
    # latent-form causal prefill over FP8 rows: 9 new tokens per sequence
    w = dataclasses.replace(LITE_FP8_SMALL, name="lite_fp8_prefill", batch=2, prior="list:63,200", new_tokens=9)
    batch = I.gen_batch(w)
    layer, st = run_gpu(w, batch)
    D, W = w.dims, weights_for(w)
    rows_g = new_rows(st, batch)
    for b in range(2):
        L = int(batch.prior_len[b])
        prior = O.gather_rows(batch.pool, batch.block_table[b], L, D.block_size)
        new_r, outs = O.prefill_sequence(D, W, batch.h[b * 9:(b + 1) * 9], L, prior, [0, 4, 8], absorbed=True)
        for q in range(9):
            check_fp8_row(rows_g[b * 9 + q], new_r[q], D.d_c, D.d_hr, O.e4m3_round, O.fp8_scale_exponent,
                          f"row {b},{q}")
        for q in (0, 4, 8):
            r = b * 9 + q
            assert_bf16(np32(st.o_lat)[r], outs[q]["o_lat"], f"o_lat {b},{q}")
            assert_bf16(np32(st.u)[r], outs[q]["u"], f"u {b},{q}")


@pytest.mark.parametrize("w", [V2_SMALL, _with_norm(V2_SMALL, "v2_norm_fused"), LITE_SMALL], ids=lambda w: w.name)
def test_fused_append_and_queries_equal_the_two_calls(w):
    # mla_compress_append_absorb_q shares one GEMM between [W^DKV; W^KR] and
    # W^DQ; each tile's K split and reduction order are those of the separate
    # launches, so cache rows and queries are bit-identical
    batch = I.gen_batch(w)
    layer = MLALayer(w.dims, weights_for(w))
    a, b = layer.upload(batch), layer.upload(batch)
    layer.compress_append(a)
    layer.absorb_q(a)
    layer.compress_append_absorb_q(b)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0
    # bit patterns: unwritten slots hold NaN, which never equals itself
    assert torch.equal(a.pool.view(torch.int16), b.pool.view(torch.int16))
    assert torch.equal(a.q_lat.view(torch.int16), b.q_lat.view(torch.int16))
    assert torch.equal(a.q_rope.view(torch.int16), b.q_rope.view(torch.int16))
