"""Choice between the latent (absorbed) and the un-absorbed prefill form by
FLOP count (the reading notes' eqs 10-11 against the explainer's absorbed
form, section 2.2.2)."""
import pytest

pytest.importorskip("torch")

from head_latent_attention_03_b200 import inputs as I
from head_latent_attention_03_b200.layer import cheaper_prefill_form, prefill_flops


def test_per_pair_costs_of_the_two_forms():
    D = I.V2
    # one query over one key, decompression not counted: 278,528 vs 81,920
    f = prefill_flops(D, [0], 1)
    assert f["absorbed"] == 278528
    assert f["unabsorbed"] - 4 * D.n_h * D.d_h * D.d_c == 81920


def test_decode_keeps_the_latent_form_and_long_chunks_decompress():
    D = I.V2
    assert cheaper_prefill_form(D, [8000] * 64, 1) == "absorbed"       # decode
    assert cheaper_prefill_form(D, [4096] * 8, 4096) == "unabsorbed"   # the chunked-prefill workload
    assert cheaper_prefill_form(I.TINY, [4096], 4096) == "absorbed"    # fp32 layers: latent form only
