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
