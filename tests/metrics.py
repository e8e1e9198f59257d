"""Parity metrics and tolerances (fp32: max relative error 1e-4 with a floor of
1e-3 * max|ref|; bf16: RMS-relative 5e-3 and max absolute 2e-2)."""
import numpy as np

FP32_MAX_REL = 1e-4
BF16_RMS_REL = 5e-3
BF16_MAX_ABS = 2e-2


def max_rel(g, r):
    g, r = np.asarray(g, np.float64), np.asarray(r, np.float64)
    floor = 1e-3 * np.max(np.abs(r))
    return float(np.max(np.abs(g - r) / np.maximum(np.abs(r), floor)))


def rms_rel(g, r):
    g, r = np.asarray(g, np.float64), np.asarray(r, np.float64)
    return float(np.linalg.norm(g - r) / np.linalg.norm(r))


def max_abs(g, r):
    return float(np.max(np.abs(np.asarray(g, np.float64) - np.asarray(r, np.float64))))


def assert_fp32(g, r, what=""):
    e = max_rel(g, r)
    assert e <= FP32_MAX_REL, f"{what}: max rel err {e:.3e} > {FP32_MAX_REL}"


def assert_bf16(g, r, what=""):
    e1, e2 = rms_rel(g, r), max_abs(g, r)
    assert e1 <= BF16_RMS_REL and e2 <= BF16_MAX_ABS, f"{what}: rms rel {e1:.3e}, max abs {e2:.3e}"


# ----------------------------------------------------------------------------
# FP8 cache rows read back from the device: E4M3 codes of c^KV (d_c bytes),
# k^R as bf16 (2 d_hr bytes), an fp32 scale, zero padding.  Decoded from the
# bit fields (sign, 4-bit exponent with bias 7, 3-bit mantissa, exponent 0 =
# subnormal, S.1111.111 = NaN).
# ----------------------------------------------------------------------------
def e4m3_decode_table():
    t = np.empty(256)
    for bits in range(256):
        s, E, m = bits >> 7, (bits >> 3) & 15, bits & 7
        if E == 15 and m == 7:
            t[bits] = np.nan
            continue
        v = (m / 8.0) * 2.0 ** -6 if E == 0 else (1.0 + m / 8.0) * 2.0 ** (E - 7)
        t[bits] = -v if s else v
    return t


def decode_fp8_rows(raw, d_c, d_hr):
    """raw uint8 [..., row_bytes] -> (code values [..., d_c], scale [...], k^R [..., d_hr], padding bytes)."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    codes = e4m3_decode_table()[raw[..., :d_c]]
    kr_bits = raw[..., d_c:d_c + 2 * d_hr].copy().view(np.uint16)
    k_r = (kr_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    off = d_c + 2 * d_hr
    scale = raw[..., off:off + 4].copy().view(np.float32)[..., 0].astype(np.float64)
    return codes, scale, k_r, raw[..., off + 4:]


def check_fp8_row(raw, ref_row, d_c, d_hr, e4m3_round, scale_exponent, what=""):
    """A device-encoded FP8 cache row against the oracle's encoding of the
    exact row: the scale exponent and every code whose rounding the inputs
    decide must match; a code whose value lies within the device's fp32
    arithmetic error (1e-5 relative) of a rounding midpoint may take either
    neighbour, and a row maximum within that error of a scale boundary may
    take either exponent.  k^R is checked at the bf16 tolerance."""
    codes, scale, k_r, pad = decode_fp8_rows(raw, d_c, d_hr)
    c = np.asarray(ref_row[:d_c], np.float64)
    e_g = int(np.log2(scale))
    assert scale == 2.0 ** e_g, f"{what}: scale {scale} is not a power of two"
    amax = float(np.max(np.abs(c)))
    e_o = scale_exponent(amax)
    if e_g != e_o:
        lo = min(e_g, e_o)
        assert abs(amax - 448.0 * 2.0 ** lo) <= 1e-5 * amax, f"{what}: exponent {e_g} vs {e_o}"
    x = c * 2.0 ** -e_g
    want = e4m3_round(x)
    down, up = e4m3_round(x * (1 - 1e-5)), e4m3_round(x * (1 + 1e-5))
    ok = (codes == want) | ((codes == down) | (codes == up))
    unique = down == up
    assert np.all(codes[unique] == want[unique]), f"{what}: {int(np.sum(codes[unique] != want[unique]))} codes differ"
    assert np.all(ok), f"{what}: codes off by more than one rounding step"
    assert np.all(pad == 0), f"{what}: padding not zero"
    assert_bf16(k_r, ref_row[d_c:], f"{what} k^R")
