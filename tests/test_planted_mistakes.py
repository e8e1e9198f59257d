"""Plant plausible slips in a copy of the oracle and check the pins catch each.

The copy is built from the oracle's source text with one substitution and run
on the CPU only; the real oracle is untouched.
"""
import importlib.util
import inspect
import sys
import types

import pytest

import tests.test_oracle_pins as pins
from oracle import mla_oracle

MUTATIONS = {
    # transposed / wrong head slice in the up-projection (eq 10)
    "uk_transposed": ("k_c = c_kv @ W[\"w_uk\"].astype(F64).T", "k_c = c_kv @ W[\"w_uv\"].astype(F64).T"),
    # dropped d_h^R from the softmax scale
    "scale_drops_rope_dim": ("math.sqrt(D.d_h + D.d_hr)", "math.sqrt(D.d_h)"),
    # wrong sign in one RoPE component
    "rope_sign": ("out[..., 1::2] = even * s + odd * c", "out[..., 1::2] = even * s - odd * c"),
    # RoPE position not applied to the key
    "rope_key_unrotated": ("k_r = rope_rotate(W[\"w_kr\"].astype(F64) @ h, pos, dims_theta(D))",
                           "k_r = W[\"w_kr\"].astype(F64) @ h"),
    # query RoPE taken at a shifted position
    "rope_query_pos": ("q_r = rope_rotate(q_r_pre, pos, dims_theta(D))",
                       "q_r = rope_rotate(q_r_pre, pos + 1, dims_theta(D))"),
    # current token left out of its own attention (eq 7 sums j <= t)
    "causal_off_by_one": ("rows[:pos + 1])", "rows[:pos])"),
    # absorbed query with the wrong contraction index
    "absorb_wrong_axis": ("np.einsum(\"ihc,ih->ic\", w_uk, q_c)",
                          "np.einsum(\"ihc,ih->ic\", w_uk, q_c[:, ::-1])"),
    # softmax normaliser dropped
    "softmax_unnormalised": ("return e / s, float(m + math.log(s))", "return e, float(m + math.log(s))"),
    # log-sum-exp missing the max
    "lse_missing_max": ("float(m + math.log(s))", "float(math.log(s))"),
    # YaRN blend with the wrong end points
    "yarn_blend_swapped": ("out[i] = (1.0 - g) * theta[i] / yarn_scale + g * theta[i]",
                           "out[i] = g * theta[i] / yarn_scale + (1.0 - g) * theta[i]"),
    # paged-cache gather reading the neighbouring slot of each page
    "gather_slot_shift": ("out[j] = pool[table_row[j // block], j % block]",
                          "out[j] = pool[table_row[j // block], (j + 1) % block]"),
    # latent RMSNorm dividing by the sum of squares instead of their mean
    "norm_sum_not_mean": ("ms = np.mean(x * x, axis=-1, keepdims=True)", "ms = np.sum(x * x, axis=-1, keepdims=True)"),
    # latent RMSNorm without its gains
    "norm_gain_dropped": ("return np.asarray(gain, dtype=F64) * x / np.sqrt(ms + eps)",
                          "return x / np.sqrt(ms + eps)"),
    # epsilon added outside the square root
    "norm_eps_outside": ("x / np.sqrt(ms + eps)", "x / (np.sqrt(ms) + eps)"),
    # bottleneck scale factor dropped
    "norm_scale_dropped": ("return scale * rms_norm(c, gain, D.norm_eps)", "return rms_norm(c, gain, D.norm_eps)"),
    # query latent left un-normalised
    "norm_query_skipped": ("c_q = latent_norm(D, W, W[\"w_dq\"].astype(F64) @ h, \"q\") if D.d_cq else h",
                           "c_q = W[\"w_dq\"].astype(F64) @ h if D.d_cq else h"),
    # merge of partial attentions without the normaliser
    "merge_unnormalised": ("/ tot[..., None]", ""),
    # merge weighing the parts equally
    "merge_equal_weights": ("w = np.exp(lse - m)", "w = np.ones_like(lse)"),
    # FP8 cache: halves rounded away from zero instead of to even
    "e4m3_ties_away": ("q = np.round(a / step) * step", "q = np.floor(a / step + 0.5) * step"),
    # FP8 cache: no subnormal range (the spacing keeps shrinking below 2^-6)
    "e4m3_no_subnormals": ("exp = np.maximum(k - 1, E4M3_MIN_EXP)", "exp = k - 1"),
    # FP8 cache: the largest value of a format with exponent bias 8
    "e4m3_wrong_bias": ("E4M3_MAX = 448.0 ", "E4M3_MAX = 240.0 "),
    # FP8 cache: scale exponent rounded down (the row maximum saturates)
    "fp8_scale_rounded_down": ("    if amax > E4M3_MAX * 2.0 ** e:\n        e += 1\n", ""),
    # FP8 cache: k^R quantised with the latent
    "fp8_quantises_rope": ("codes, e = quantize_latent(row[:D.d_c])\n    return np.concatenate([np.ldexp(codes, e), row[D.d_c:]])",
                           "codes, e = quantize_latent(row)\n    return np.ldexp(codes, e)"),
    # FP8 cache: codes read back without their scale
    "fp8_scale_not_applied": ("return np.concatenate([np.ldexp(codes, e), row[D.d_c:]])",
                              "return np.concatenate([codes, row[D.d_c:]])"),
    # W^O applied before W^UV's head split is undone
    "out_proj_heads": ("o = np.einsum(\"ihc,ic->ih\", w_uv, np.asarray(o_lat, dtype=F64))",
                       "o = np.einsum(\"ihc,ic->ih\", w_uv, np.asarray(o_lat, dtype=F64)[::-1])"),
}


def _mutated(name):
    src = inspect.getsource(mla_oracle)
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation {name} does not match the oracle source"
    mod = types.ModuleType(f"mla_oracle_mut_{name}")
    exec(compile(src.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    return mod


def _pin_tests():
    out = []
    for n, f in inspect.getmembers(pins, inspect.isfunction):
        if n.startswith("test_"):
            params = getattr(f, "pytestmark", [])
            argsets = [()]
            for m in params:
                if m.name == "parametrize":
                    argsets = [(v,) for v in m.args[1]]
            out.extend((n, f, a) for a in argsets)
    return out


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    monkeypatch.setattr(pins, "O", _mutated(name))
    caught = []
    for n, f, args in _pin_tests():
        try:
            f(*args)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(n)
    assert caught, f"no pin caught mutation {name}"
