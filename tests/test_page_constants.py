"""The layer shapes and cache-size facts printed on the pages (tests/golden)
against the workload definitions and the oracle's cache-size formula."""
import os

import pytest

from oracle import mla_oracle as O
from head_latent_attention_03_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.txt")


def _load():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            vals[k] = float(v)
    return vals


def test_layer_shapes_match_pages():
    g = _load()
    for key, D in (("v2", I.V2), ("lite", I.LITE)):
        for f in ("d", "n_h", "d_h", "d_c", "d_cq", "d_hr"):
            assert getattr(D, f) == g[f"{key}.{f}"], (key, f)
    assert I.V2_YARN.yarn_scale == g["yarn.s"]
    assert I.V2_YARN.yarn_alpha == g["yarn.alpha"] and I.V2_YARN.yarn_beta == g["yarn.beta"]
    assert I.V2_YARN.yarn_orig_ctx == g["yarn.orig_ctx"]


def test_cache_per_token_matches_pages():
    g = _load()
    for key in ("v2", "lite"):
        l = int(g[f"{key}.layers"])
        mla = O.kv_cache_elements_per_token("mla", l, d_c=int(g[f"{key}.d_c"]), d_hr=int(g[f"{key}.d_hr"]))
        assert mla / (g[f"{key}.d_h"] * l) == pytest.approx(g["mla.cache_per_token_over_d_h_l"])
        gqa_group = O.kv_cache_elements_per_token("gqa", l, n_groups=1, d_h=int(g[f"{key}.d_h"]))
        assert mla / gqa_group == pytest.approx(g["mla.gqa_equivalent_groups"])
