"""Comparison rules between the CUDA path and the oracle (test infrastructure).

Tolerances, from the stated parity contract and the arithmetic:
  * codes and sign bits: bit-exact, except coordinates whose oracle value lies
    within 1e-6 of a decision boundary (|y_i - t_k| < 1e-6 in the rotated,
    unit-normalised domain for codes; |p_j| < 1e-6 for signs).  Those
    mismatches are counted and must stay below 1e-5 of all coordinates.  A row
    with an exempt code mismatch has a different residual, so its signs and
    rnorm are not compared (the row is counted instead).
  * norm: relative (d / 2 + 4) 2^-24, the worst-case bound of an fp32 sum of
    d squares plus the square root.
  * rnorm: |diff| <= 1e-5 * norm (the fp32 rotation error of y is below 1e-6 in
    unit-normalised units).
  * logits: |diff| <= 1e-4 |q| |k|.
  * dequant fp32: |diff_i| <= 1e-3 (|x_i| + |x| / sqrt(d)); bf16: the oracle
    value rounded to bf16, or one bf16 step away, or -- for elements that
    cancel to near zero, where one bf16 step is smaller than the fp32
    arithmetic noise of the row -- within 2^-16 |x| / sqrt(d) of the oracle.
"""

from __future__ import annotations

import math

import numpy as np

from oracle import turboquant as ot

BAND = 1e-6


def compare_quantize(P, got: dict, want: dict):
    """got: packed numpy dict from the GPU; want: oracle.quantize(..., keep_intermediates=True)."""
    d, m = P.d, P.m
    N = want["y"].shape[0]
    cg = ot.unpack_codes(got["codes"], d, P.B)
    co = want["code"]
    cmis = cg != co
    near = np.min(np.abs(want["y"][..., None] - P.thresholds[None, None, :]), axis=-1) < BAND
    bad_codes = int(np.sum(cmis & ~(near & (np.abs(cg - co) == 1))))
    exempt_codes = int(np.sum(cmis & near))
    row_cmis = np.any(cmis, axis=1)
    bg = ot.unpack_signs(got["signs"], m)
    bo = want["bits"]
    smis = (bg != bo) & ~row_cmis[:, None]
    nearp = np.abs(want["p"]) < BAND
    bad_signs = int(np.sum(smis & ~nearp))
    exempt_signs = int(np.sum(smis & nearp))
    n_o = want["norm"].astype(np.float64)
    n_g = got["norm"].astype(np.float64)
    tol_n = (d / 2 + 4) * 2.0 ** -24 * n_o + 1e-30
    bad_norm = int(np.sum(np.abs(n_g - n_o) > tol_n))
    rn_o = want["rnorm"].astype(np.float64)
    rn_g = got["rnorm"].astype(np.float64)
    bad_rnorm = int(np.sum((np.abs(rn_g - rn_o) > 1e-5 * n_o + 1e-30) & ~row_cmis))
    return {
        "rows": N, "coords": N * d, "projections": N * m,
        "bad_codes": bad_codes, "exempt_codes": exempt_codes,
        "bad_signs": bad_signs, "exempt_signs": exempt_signs,
        "rows_with_exempt_code": int(np.sum(row_cmis)),
        "bad_norm": bad_norm, "bad_rnorm": bad_rnorm,
    }


def assert_quantize_ok(rep: dict):
    assert rep["bad_codes"] == 0, rep
    assert rep["bad_signs"] == 0, rep
    assert rep["bad_norm"] == 0, rep
    assert rep["bad_rnorm"] == 0, rep
    assert rep["exempt_codes"] <= max(1e-5 * rep["coords"], 1), rep
    assert rep["exempt_signs"] <= max(1e-5 * rep["projections"], 1), rep


def logit_tolerance(q: np.ndarray, k_norm: np.ndarray, n_sets: int, g: int, n_keys: int) -> np.ndarray:
    qn = np.linalg.norm(q.astype(np.float64), axis=1).reshape(n_sets, g, 1)
    kn = k_norm.astype(np.float64).reshape(n_sets, 1, n_keys)
    return 1e-4 * qn * kn


def bf16_round(x: np.ndarray) -> np.ndarray:
    from kv_cache_vector_15_b200.inputs import bf16_bits, bf16_to_f32
    return bf16_to_f32(bf16_bits(x.astype(np.float32))).astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_dequant_ok(got: np.ndarray, want: np.ndarray, bf16: bool):
    got = got.astype(np.float64)
    if bf16:
        r = bf16_round(want)
        d = want.shape[1]
        floor = 2.0 ** -16 * np.linalg.norm(want, axis=1, keepdims=True) / math.sqrt(d)
        ok = (got == r) | (np.abs(got - r) <= bf16_ulp(r) * 1.0001) | (np.abs(got - want) <= floor)
        assert ok.all(), f"{int((~ok).sum())} bf16 elements off by more than one step"
    else:
        d = want.shape[1]
        scale = np.linalg.norm(want, axis=1, keepdims=True) / math.sqrt(d)
        err = np.abs(got - want)
        ok = err <= 1e-3 * (np.abs(want) + scale) + 1e-30
        assert ok.all(), f"max rel err {np.max(err / (np.abs(want) + scale + 1e-30))}"
