"""Oracle: the TurboQuant hot path in plain fp64 NumPy (test infrastructure only).

Write half (``quantize``), per row x in R^d:
  1. n = ||x||; a row with n < 1e-10 is stored as all zeros
     [0h-n0.github.io "ICLR 2026論文解説: TurboQuant", section "Step 1:
     PolarQuant" (normalise onto the unit sphere, keep the norm) and section
     "実装のポイント" (norm storage); the 1e-10 zero rule is the one in that
     page's encoder sketch];
  2. y = R (x / n), R = H_d D / sqrt(d)   [same page, "Step 1: PolarQuant"];
  3. code_i = #{k : t_k < y_i}, yhat = c[code]   [Qiita TurboQuant explainer
     (qiita.com/kai_kou), "Stage 1: PolarQuant", step 3 Lloyd-Max];
  4. r = y - yhat, rho = ||r||; p = S r; bit_j = 1 iff p_j < 0  [Qiita
     explainer, "Stage 2: QJL"; ai.spot.hk "Google TurboQuant", section
     "無偏內積估計" (b-1 bits of MSE quantizer, then 1-bit QJL on the residual)];
  5. store codes, sign bits, norm = n and rnorm = n * rho (fp32).

Read half:
  logit(q, k) = norm * <R q, yhat> + rnorm * sqrt(pi/2) / m * <S R q, z>,
  z_j = +1 - 2 bit_j   [Qiita explainer, "Stage 2: QJL", the estimator
  <q,k> ~ <q,k_mse> + ||residual|| sqrt(pi/2)/m <S q, sign(S residual)>];
  dequant (PROD) x~ = R^T (norm * yhat + sqrt(pi/2)/m * rnorm * S^T z)
  [ai.spot.hk, "無偏內積估計": E<y, Q^-1(Q(x))> = <y, x>];
  dequant (MSE)  x~ = norm * R^T yhat  [Qiita explainer, "APIの構成"
  (values compressed by the MSE stage alone)];
  attention: softmax over keys of scale * logit, times the dequantized values.

Readings taken where the pages are silent:
  * the residual lives in the rotated, unit-normalised domain, and rnorm is
    stored in the original units (n * rho);
  * y_i exactly on a threshold goes to the lower cell; p_j = 0 counts as
    positive (bit 0); bit 1 means negative, as in the 0h-n0 encoder sketch;
  * codes are an LSB-first bitstream per row, code i in bits [B i, B i + B);
    sign j is bit (j mod 8) of byte j // 8;
  * the logit carries no 1/sqrt(d) softmax scale;
  * a row length d that is not a power of two is zero-padded to the next
    power of two (``padded_dim``, ``pad_rows``); every parameter and the
    packed format are those of the padded length, and reconstructed rows are
    read back in their first d coordinates.
"""

from __future__ import annotations

import math

import numpy as np

SQRT_HALF_PI = math.sqrt(math.pi / 2.0)
ZERO_NORM = 1e-10


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------
def sylvester_hadamard(d: int) -> np.ndarray:
    """H_1 = [1], H_2d = [[H_d, H_d], [H_d, -H_d]]  [0h-n0 explainer,
    "Step 1: PolarQuant", recursive Hadamard definition]."""
    H = np.ones((1, 1))
    base = np.array([[1.0, 1.0], [1.0, -1.0]])
    while H.shape[0] < d:
        H = np.kron(base, H)
    return H


def rotation_matrix(D: np.ndarray) -> np.ndarray:
    """Dense R = H_d diag(D) / sqrt(d)."""
    d = D.shape[0]
    return sylvester_hadamard(d) * D.astype(np.float64)[None, :] / math.sqrt(d)


def fwht(v: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform along the last axis, the
    butterfly (a, b) -> (a + b, a - b) at strides 1, 2, 4, ...  [0h-n0
    explainer, "実装のポイント" (butterfly structure, O(d log d))].
    Equal to v @ H_d (H_d symmetric)."""
    v = np.array(v, dtype=np.float64, copy=True)
    d = v.shape[-1]
    h = 1
    while h < d:
        w = v.reshape(v.shape[:-1] + (d // (2 * h), 2, h))
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b
        w[..., 1, :] = a - b
        h *= 2
    return v


def rotate(v: np.ndarray, P) -> np.ndarray:
    """Row-wise R v = H_d (D v) / sqrt(d) (v has rows of length d), by the
    butterfly; equal to the dense P.R @ v (pinned in the tests)."""
    return fwht(np.asarray(v, dtype=np.float64) * P.D) / math.sqrt(P.d)


def rotate_inverse(v: np.ndarray, P) -> np.ndarray:
    """Row-wise R^T v = D (H_d v) / sqrt(d)."""
    return fwht(np.asarray(v, dtype=np.float64)) * P.D / math.sqrt(P.d)


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------
def padded_dim(d: int) -> int:
    """The power of two a row of length d is zero-padded to before the
    rotation [0h-n0 "ICLR 2026論文解説: TurboQuant", "実装のポイント": RHT needs
    a power-of-two dimension; pad with zeros up to the nearest one above]."""
    p = 1
    while p < d:
        p *= 2
    return p


def pad_rows(x: np.ndarray, d_pad: int) -> np.ndarray:
    """Rows of x (..., d) with d_pad - d zero coordinates appended."""
    x = np.asarray(x, dtype=np.float64)
    return np.concatenate([x, np.zeros(x.shape[:-1] + (d_pad - x.shape[-1],))], axis=-1)


def packed_sizes(d: int, b: int, m: int):
    """Bytes per row: codes d (b-1) / 8, signs m / 8, plus two fp32 norms."""
    return d * (b - 1) // 8, m // 8


def pack_codes(codes: np.ndarray, B: int) -> np.ndarray:
    """LSB-first bitstream: bit B*i + j of the row is bit j of code i."""
    codes = np.asarray(codes, dtype=np.int64)
    N, d = codes.shape
    bits = ((codes[:, :, None] >> np.arange(B)[None, None, :]) & 1).astype(np.uint8)
    return np.packbits(bits.reshape(N, d * B), axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, d: int, B: int) -> np.ndarray:
    bits = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, bitorder="little")
    bits = bits[:, : d * B].reshape(-1, d, B).astype(np.int64)
    return np.sum(bits << np.arange(B)[None, None, :], axis=2)


def pack_signs(bits: np.ndarray) -> np.ndarray:
    """Sign j is bit (j mod 8) of byte j // 8; bit 1 means negative."""
    return np.packbits(np.asarray(bits, dtype=np.uint8), axis=1, bitorder="little")


def unpack_signs(packed: np.ndarray, m: int) -> np.ndarray:
    bits = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, bitorder="little")
    return bits[:, :m].astype(np.int64)


# --------------------------------------------------------------------------
# Write half
# --------------------------------------------------------------------------
def bucketize(y: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """code = number of thresholds strictly below y (ties go to the lower cell)."""
    return np.sum(y[..., None] > thresholds, axis=-1)


def quantize(x: np.ndarray, P, *, keep_intermediates: bool = False, codes_override=None):
    """TurboQuant_prod write half for rows x (N, d), values exactly as the
    kernel reads them (bf16 or fp32 inputs widened to fp64).

    Returns a dict with packed ``codes`` (N, d B / 8) u8, ``signs`` (N, m / 8)
    u8, ``norm`` and ``rnorm`` (N,) fp32; with ``keep_intermediates`` also the
    fp64 ``y``, ``code``, ``p``, ``bits``, ``n`` and ``rho``.

    ``codes_override`` lets a test fix the codes of some rows (values chosen
    by the test, e.g. the other side of a threshold within the tie band) to
    see what the residual stage gives for them; it is never fed kernel output.
    """
    x = np.asarray(x, dtype=np.float64)
    N = x.shape[0]
    n = np.sqrt(np.sum(x * x, axis=1))
    zero = n < ZERO_NORM
    safe = np.where(zero, 1.0, n)
    u = x / safe[:, None]
    y = rotate(u, P)
    code = bucketize(y, P.thresholds) if codes_override is None else np.asarray(codes_override)
    yhat = P.centroids[code]
    r = y - yhat
    rho = np.sqrt(np.sum(r * r, axis=1))
    p = r @ P.S.T
    bits = (p < 0).astype(np.int64)
    code = np.where(zero[:, None], 0, code)
    bits = np.where(zero[:, None], 0, bits)
    out = {
        "codes": pack_codes(code, P.B),
        "signs": pack_signs(bits),
        "norm": np.where(zero, 0.0, n).astype(np.float32),
        "rnorm": np.where(zero, 0.0, n * rho).astype(np.float32),
    }
    if keep_intermediates:
        out.update(y=y, code=code, p=p, bits=bits, n=n, rho=rho, zero=zero)
    return out


# --------------------------------------------------------------------------
# Read half
# --------------------------------------------------------------------------
def decode(packed: dict, P):
    """yhat (N, d) from the codes and z (N, m) in {+1, -1} from the signs."""
    code = unpack_codes(packed["codes"], P.d, P.B)
    yhat = P.centroids[code]
    z = 1.0 - 2.0 * unpack_signs(packed["signs"], P.m)
    return yhat, z


def qjl_correction(sq: np.ndarray, z: np.ndarray, rnorm, m: int) -> np.ndarray:
    """||residual|| * sqrt(pi/2) / m * <S q, sign(S residual)>, for every
    (query row of ``sq``, key row of ``z``) pair; z_j = +-1."""
    return (np.asarray(rnorm, dtype=np.float64) * (SQRT_HALF_PI / m)) * (sq @ z.T)


def query_prep(q: np.ndarray, P):
    """q_rot = R q and sq = S q_rot, once per query."""
    q_rot = rotate(q, P)
    return q_rot, q_rot @ P.S.T


def logits(q: np.ndarray, packed: dict, P, n_sets: int, g: int, n_keys: int) -> np.ndarray:
    """Estimated <q, k> for every query of a set against every key of that set.

    q: (n_sets * g, d) rows, query j of set s at row s * g + j.
    packed: rows of set s at [s * n_keys, (s + 1) * n_keys).
    Returns (n_sets, g, n_keys) fp64."""
    yhat, z = decode(packed, P)
    norm = np.asarray(packed["norm"], dtype=np.float64)
    rnorm = np.asarray(packed["rnorm"], dtype=np.float64)
    q_rot, sq = query_prep(np.asarray(q, dtype=np.float64).reshape(n_sets * g, P.d), P)
    out = np.empty((n_sets, g, n_keys))
    for s in range(n_sets):
        ks = slice(s * n_keys, (s + 1) * n_keys)
        qs = slice(s * g, (s + 1) * g)
        mse = q_rot[qs] @ yhat[ks].T
        out[s] = norm[ks][None, :] * mse + qjl_correction(sq[qs], z[ks], rnorm[ks], P.m)
    return out


DEQUANT_PROD = 0
DEQUANT_MSE = 1


def dequant(packed: dict, P, mode: int = DEQUANT_PROD) -> np.ndarray:
    """Reconstructed rows (N, d) fp64.
    PROD: R^T (norm * yhat + sqrt(pi/2)/m * rnorm * S^T z).
    MSE:  R^T (norm * yhat)."""
    yhat, z = decode(packed, P)
    norm = np.asarray(packed["norm"], dtype=np.float64)
    rnorm = np.asarray(packed["rnorm"], dtype=np.float64)
    v = norm[:, None] * yhat
    if mode == DEQUANT_PROD:
        v = v + (SQRT_HALF_PI / P.m) * rnorm[:, None] * (z @ P.S)
    return rotate_inverse(v, P)


def attention(q: np.ndarray, keys: dict, values: dict, P, n_sets: int, g: int, n_keys: int, scale: float,
              mode: int = DEQUANT_PROD, logits_in=None) -> np.ndarray:
    """Decode attention read from packed keys and values: for query j of set s,
    softmax over the set's keys of scale * logit, times the dequantized values
    of the same keys.  [Qiita explainer, "APIの構成": attention scores taken
    from the compressed keys (asymmetric_attention_scores) and values kept in
    compressed form; the weighted sum of values is ordinary attention.]

    logits_in: (n_sets, g, n_keys) logits to use instead of the estimator's
    own (so a caller can evaluate the softmax and the value sum on given
    scores).  Returns (n_sets, g, d) fp64."""
    s = logits(q, keys, P, n_sets, g, n_keys) if logits_in is None else np.asarray(logits_in, dtype=np.float64)
    z = scale * s.reshape(n_sets, g, n_keys)
    z = z - z.max(axis=-1, keepdims=True)
    w = np.exp(z)
    w /= w.sum(axis=-1, keepdims=True)
    xv = dequant(values, P, mode).reshape(n_sets, n_keys, P.d)
    out = np.empty((n_sets, g, P.d))
    for st in range(n_sets):
        out[st] = w[st] @ xv[st]
    return out


def topk(scores: np.ndarray, k: int):
    """Per row, the k largest scores, larger first, equal scores by lower
    index first.  Returns (idx int32, val)."""
    scores = np.asarray(scores)
    order = np.argsort(-scores, axis=1, kind="stable")[:, :k]
    return order.astype(np.int32), np.take_along_axis(scores, order, axis=1)


# --------------------------------------------------------------------------
# Fractional bit widths by a channel split.  The pages report 2.5- and 3.5-bit
# results without the split rule [inlevel9 "TurboQuantのメモリ圧縮と半導体需要",
# section "TurboQuantが実際に行っていること"]; the reading followed here (and by
# the library): channels [0, d_hi) of every row are one instance with b_hi bits
# per coordinate and channels [d_hi, d) another with b_lo bits, each with its
# own D, S and codebook, m = the part's channel count, seeds seed and seed + 1;
# a part whose channel count is not a power of two is zero-padded like any
# row.  Inner products add over disjoint channel sets, so the estimate of
# <q, k> is the sum of the parts' estimates.

def split_parts(d: int, d_hi: int, b_hi: int, b_lo: int, seed: int, params_cls):
    """[(first channel, channel count, Params of the padded part)] for the two parts."""
    parts = []
    for p, (c0, dc, b) in enumerate(((0, d_hi, b_hi), (d_hi, d - d_hi, b_lo))):
        parts.append((c0, dc, params_cls(padded_dim(dc), b, dc, seed=seed + p)))
    return parts


def split_bits_per_coordinate(parts) -> float:
    """Stored bits per coordinate of the caller's row, norms aside: b - 1 code
    bits per (padded) channel plus one sign per projection."""
    d = sum(dc for _, dc, _ in parts)
    return sum(P.d * P.B + P.m for _, _, P in parts) / d


def split_quantize(x: np.ndarray, parts, **kw):
    """(packed part 0, packed part 1) of rows x [N, d]."""
    x = np.asarray(x, dtype=np.float64)
    return tuple(quantize(pad_rows(x[:, c0:c0 + dc], P.d), P, **kw) for c0, dc, P in parts)


def split_logits(q: np.ndarray, packed, parts, n_sets: int, g: int, n_keys: int) -> np.ndarray:
    """The sum of the two parts' estimates, (n_sets, g, n_keys)."""
    q = np.asarray(q, dtype=np.float64)
    return sum(logits(pad_rows(q[:, c0:c0 + dc], P.d), pk, P, n_sets, g, n_keys)
               for (c0, dc, P), pk in zip(parts, packed))


def split_dequant(packed, parts, mode: int = DEQUANT_PROD) -> np.ndarray:
    """Reconstructed rows [N, d]: each part's channels from its packed rows."""
    return np.concatenate([dequant(pk, P, mode)[:, :dc] for (_, dc, P), pk in zip(parts, packed)], axis=1)
