"""CPU check of the wide-row tensor-core design's arithmetic (no GPU).

The wide-row kernels feed the tensor cores binary16 halves of fp32 operands
(hi = rn16(v), lo = rn16(v - hi)) and accumulate exact products in fp32.  This
test emulates those operands in fp64 (numpy float16 rounding) and pins the two
claims the kernels rest on against the oracle:

  * the projection P = (r_hi + r_lo) S^T differs from the oracle's S r by less
    than the split part of the sign bound, 2 * 2^-22 ||S_j|| ||r|| s +
    2^-24 ||S_j||_1 (the kernel's bound adds d/8 accumulation steps on top);
  * the estimates from [c_hi | c_lo | z] x [q_hi | q_lo | sq_hi | sq_lo] with
    the three MSE products c_hi q_hi + c_lo q_hi + c_hi q_lo stay far inside
    the 1e-4 |q| |k| logit tolerance.
A third check covers the d = 128 logits kernel's centroid byte planes for
3-bit codes (16-bit fixed point, high and low byte).
The emulation is independent of the CUDA sources: it restates the operand
construction from its definition, not from the kernels.
"""

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot
from tests import parity


def f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def pow2_ceil_sqrt(d):
    k = 0
    while (1 << (2 * k)) < d:
        k += 1
    return float(1 << k)


@pytest.mark.parametrize("d,b,m", [(256, 3, 256), (1024, 4, 1024), (512, 2, 128)])
def test_projection_split_within_the_sign_bound(d, b, m):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d + b)
    x = rng.standard_normal((300, d)) * rng.uniform(0.1, 10, size=(300, 1))
    q = ot.quantize(x, P, keep_intermediates=True)
    r = (q["y"] - P.centroids[q["code"]]).astype(np.float32).astype(np.float64)
    s = 8.0 * pow2_ceil_sqrt(d)
    hi = f16(r * s)
    lo = f16(r * s - hi)
    p = hi @ P.S.T + lo @ P.S.T                       # exact products, summed in fp64
    snorm = np.linalg.norm(P.S, axis=1)
    s1 = np.abs(P.S).sum(axis=1).max()
    rn = s * np.linalg.norm(r, axis=1)
    split_bound = 2 * 2.0 ** -22 * snorm[None, :] * rn[:, None] + 2.0 ** -24 * s1
    assert np.all(np.abs(p - s * (r @ P.S.T)) <= split_bound)
    # the kernel's full bound leaves room for d/8 fp32 accumulation steps
    full = (d / 8 + 2) * 2.0 ** -22 * snorm[None, :] * rn[:, None] + 2.0 ** -24 * s1
    assert np.all(split_bound < full)
    # and the share of projections the fix-up recomputes stays small
    assert np.mean(np.abs(p) <= full) < 0.01


@pytest.mark.parametrize("d,b,m", [(256, 3, 256), (1024, 4, 1024)])
def test_estimate_decomposition_within_the_logit_tolerance(d, b, m):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(7 * d + b)
    k = rng.standard_normal((200, d)) * rng.uniform(0.1, 10, size=(200, 1))
    pk = ot.quantize(k, P)
    qq = rng.standard_normal((40, d)).astype(np.float32).astype(np.float64)
    sc = pow2_ceil_sqrt(d)
    c = P.centroids
    c_hi = f16(c * sc)
    c_lo = f16(c * sc - c_hi)
    code = ot.unpack_codes(pk["codes"], d, P.B)
    z = 1.0 - 2.0 * ot.unpack_signs(pk["signs"], m)
    q_rot, sq = ot.query_prep(qq, P)
    q_rot = q_rot.astype(np.float32).astype(np.float64)
    sq = sq.astype(np.float32).astype(np.float64)

    def split(v):                                    # power-of-two scale: largest magnitude in [1, 2)
        e = np.frexp(np.abs(v).max(axis=1))[1]
        s = np.ldexp(1.0, 1 - e)
        h = f16(v * s[:, None])
        return h, f16(v * s[:, None] - h), s

    qh, ql, s_q = split(q_rot)
    sh, sl, s_s = split(sq)
    acc0 = c_hi[code] @ qh.T + c_lo[code] @ qh.T + c_hi[code] @ ql.T
    acc1 = z @ sh.T + z @ sl.T
    qjl = float(np.float32(np.sqrt(np.pi / 2) / m))
    est = (pk["norm"][:, None] * acc0 / (sc * s_q[None, :]) + pk["rnorm"][:, None] * acc1 * (qjl / s_s[None, :])).T
    want = ot.logits(qq, pk, P, 1, 40, 200)[0]
    tol = parity.logit_tolerance(qq, np.linalg.norm(k, axis=1), 1, 40, 200)[0]
    assert np.all(np.abs(est - want) <= 1e-2 * tol)


def test_centroid_byte_planes_within_the_logit_tolerance():
    """The d = 128 warp-specialized logits kernel takes 3-bit codes' centroids as
    the high and low byte of round(c s), s = 32767 / max |c| (a signed high byte
    and an unsigned low byte).  Restated from that definition: the two bytes
    recompose the fixed-point value exactly, each centroid moves by at most
    max |c| / 65534, and the MSE term of the estimator moves by far less than
    the 1e-4 |q| |k| logit tolerance -- also in the worst case, max |delta| times
    ||q||_1 <= max |delta| sqrt(d) |q|."""
    d, b, m = 128, 4, 128
    P = op.Params(d, b, m, seed=0)
    c = P.centroids
    s = 32767.0 / np.abs(c).max()
    fx = np.clip(np.rint(c * s), -32767, 32767).astype(np.int64)
    hi, lo = fx >> 8, fx & 0xFF
    assert np.all((-128 <= hi) & (hi <= 127)) and np.all((0 <= lo) & (lo <= 255))
    assert np.array_equal(256 * hi + lo, fx)
    delta = fx / s - c
    assert np.abs(delta).max() <= np.abs(c).max() / 65534 * (1 + 1e-12)
    worst = np.abs(delta).max() * np.sqrt(d)          # per unit |q| |k| (unit-norm rotated keys)
    assert worst < 3.4e-5 < 1e-4
    rng = np.random.default_rng(11)
    k = rng.standard_normal((500, d)) * rng.uniform(0.1, 10, size=(500, 1))
    pk = ot.quantize(k, P)
    code = ot.unpack_codes(pk["codes"], d, P.B)
    qq = rng.standard_normal((64, d))
    q_rot, _ = ot.query_prep(qq, P)
    moved = (q_rot @ delta[code].T) * pk["norm"][None, :]    # change of the MSE term
    tol = 1e-4 * np.linalg.norm(qq, axis=1)[:, None] * np.linalg.norm(k, axis=1)[None, :]
    assert np.all(np.abs(moved) <= 0.34 * tol)
