"""mla_decode_attn_noalloc, the decode attention for callers that cannot
allocate device memory at call time (code running where allocation is
forbidden, such as a captured command stream or a serving loop whose memory
was fixed at start-up, with no buffer to lend as workspace).

Instead of a caller workspace it keeps its split-KV partials in a fixed,
library-owned device array.  Its results must match mla_decode_attn's (the
workspace entry point) within the parity tolerances, on two calls in a row:
the array keeps the previous call's contents, which must not leak into the
next result.  The file is named to be collected last, and each test builds
its own inputs, so it passes alone in a fresh process or after the others.
"""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from head_latent_attention_03_b200 import inputs as I
from head_latent_attention_03_b200 import mla
from head_latent_attention_03_b200.layer import MLALayer
from tests.metrics import assert_bf16, assert_fp32

pytestmark = pytest.mark.gpu

LITE = I.WORKLOADS["lite"]
CASES = [
    (dataclasses.replace(LITE, name="lite_splits3", batch=4, prior="list:300,1500,900,64"), 3),
    (dataclasses.replace(LITE, name="lite_auto", batch=4, prior="list:300,1500,900,64"), 0),
    (dataclasses.replace(I.WORKLOADS["v2"], name="v2_splits2", batch=3, prior="list:127,128,3000"), 2),
    (I.WORKLOADS["tiny"], 0),
    # 128 heads, batch 64, ragged lengths, automatic plan: the plan of a full
    # wave (74 CTA pairs) needs more than the 32 MiB array, so the entry point
    # plans for fewer pairs (test_v2_batch64_plan_exceeds_the_array)
    (dataclasses.replace(I.WORKLOADS["v2"], name="v2_b64_auto"), 0),
    # FP8 cache rows, automatic and explicit splits
    (dataclasses.replace(I.WORKLOADS["lite_fp8"], name="lite_fp8_auto", batch=4, prior="list:300,1500,900,64"), 0),
    (dataclasses.replace(I.WORKLOADS["lite_fp8"], name="lite_fp8_splits2", batch=4, prior="list:300,1500,900,64"), 2),
    (dataclasses.replace(I.WORKLOADS["v2_fp8"], name="v2_fp8_auto", batch=3, prior="list:127,128,3000"), 0),
]


def plan_bytes(rows, workers, n_h):
    """Scratch of an automatic decode plan, carved as the library does: segment
    list, row table, CTA table, count word, fp32 partials of at
    most min(rows + workers, 2 * workers) cut segments (each piece 256-byte
    aligned)."""
    def take(used, b):
        return ((used + 255) & ~255) + b
    units = rows + workers
    slots = min(units, 2 * workers)
    u = 0
    for b in (units * 16, rows * 16, (workers + 1) * 4, 16, slots * n_h * 512 * 4, slots * n_h * 4):
        u = take(u, b)
    return u


def test_v2_batch64_plan_exceeds_the_array():
    # one wave of CTA pairs on a 148-SM B200 is 74 pairs; its plan does not fit
    # 32 MiB, the largest plan that fits has 63 pairs
    cap = (32 << 20) - 256
    assert plan_bytes(64, 74, 128) > cap
    assert max(w for w in range(1, 75) if plan_bytes(64, w, 128) <= cap) == 63


@pytest.mark.parametrize("w,splits", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_noalloc_matches_workspace_entry_point(w, splits):
    batch = I.gen_batch(w)
    layer = MLALayer(w.dims, I.gen_weights(w))
    st = layer.upload(batch)
    layer.compress_append(st)
    layer.absorb_q(st)
    cache = layer.cache(st)
    mla.decode_attn(layer.desc, st.q_lat, st.q_rope, cache, st.kv_len, st.ws, st.o_lat, st.lse, num_splits=splits)
    torch.cuda.synchronize()
    assert mla.get_last_error() == 0
    ref_o, ref_l = st.o_lat.float().cpu().numpy(), st.lse.cpu().numpy()
    for call in range(2):
        o = torch.full_like(st.o_lat, float("nan"))
        l = torch.full_like(st.lse, float("nan"))
        mla.decode_attn_noalloc(layer.desc, st.q_lat, st.q_rope, cache, st.kv_len, o, l, num_splits=splits)
        torch.cuda.synchronize()
        assert mla.get_last_error() == 0
        got_o, got_l = o.float().cpu().numpy(), l.cpu().numpy()
        if splits > 0:
            # explicit split counts: both entry points run the same plan
            assert np.array_equal(got_o, ref_o), f"o_lat call {call}"
            assert np.array_equal(got_l, ref_l), f"lse call {call}"
        elif w.dims.dtype == "f32":
            assert_fp32(got_o, ref_o, f"o_lat call {call}")
            assert_fp32(got_l, ref_l, f"lse call {call}")
        else:
            assert_bf16(got_o, ref_o, f"o_lat call {call}")
            assert np.max(np.abs(got_l - ref_l)) < 2e-2


def test_noalloc_rejects_partials_beyond_its_array():
    # 16 splits x 64 rows x 128 heads x 2052 bytes = 269 MB > 32 MiB: refused
    # on the host before any launch.
    D = I.V2
    desc = mla.layer_desc(D)
    dev = "cuda"
    q_lat = torch.zeros((64, D.n_h, D.d_c), dtype=torch.bfloat16, device=dev)
    q_rope = torch.zeros((64, D.n_h, D.d_hr), dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q_lat)
    pool = torch.zeros((1, 64, D.row), dtype=torch.bfloat16, device=dev)
    table = torch.zeros((64, 40), dtype=torch.int32, device=dev)
    kv_len = torch.ones((64,), dtype=torch.int32, device=dev)
    with pytest.raises(mla.MLAError) as e:
        mla.decode_attn_noalloc(desc, q_lat, q_rope, mla.paged_cache(pool, table), kv_len, o, None, num_splits=16)
    assert e.value.code == 3  # MLA_ERR_CAPACITY
