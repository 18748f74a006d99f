"""Pins for the oracle's rotation, write half and read half.

Independent anchors only: the closed-form entries of Sylvester's Hadamard
matrix, orthogonality, brute-force nearest-centroid and projection loops on
tiny inputs, a hand-derived packing fixture, Gaussian identities (QJL
unbiasedness and variance), the quadrature distortion, and the exact
orthogonality of the MSE reconstruction error.
"""

import math
import os

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Rotation
# --------------------------------------------------------------------------
def hadamard_entry(i, j):
    """Sylvester H_d[i, j] = (-1)^popcount(i & j)."""
    return -1.0 if bin(i & j).count("1") % 2 else 1.0


@pytest.mark.parametrize("d", [2, 4, 8, 16, 64])
def test_sylvester_matrix_closed_form(d):
    H = ot.sylvester_hadamard(d)
    want = np.array([[hadamard_entry(i, j) for j in range(d)] for i in range(d)])
    assert np.array_equal(H, want)


@pytest.mark.parametrize("d", [2, 4, 8, 16])
def test_fwht_equals_brute_force_matvec(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((5, d))
    brute = np.array([[sum(hadamard_entry(i, j) * row[j] for j in range(d)) for i in range(d)] for row in x])
    assert np.allclose(ot.fwht(x), brute, rtol=0, atol=1e-13)


@pytest.mark.parametrize("d", [16, 128, 1024])
def test_rotation_is_orthogonal_and_oriented(d):
    P = op.Params(d, 3, 32, seed=5)
    R = P.R
    assert np.max(np.abs(R @ R.T - np.eye(d))) < 1e-12
    # R e_j = D_j H[:, j] / sqrt(d): D multiplies a whole column, so every
    # entry of column j has the same sign pattern as H[:, j] times D_j.
    j = 3
    col = R[:, j]
    H = ot.sylvester_hadamard(d)
    assert np.allclose(col, P.D[j] * H[:, j] / math.sqrt(d), rtol=0, atol=1e-15)
    # and the butterfly agrees with the dense matrix: R x = H (D x) / sqrt(d)
    x = np.random.default_rng(1).standard_normal((3, d))
    assert np.allclose(ot.rotate(x, P), ot.fwht(x * P.D) / math.sqrt(d), rtol=0, atol=1e-12)
    assert np.allclose(ot.rotate_inverse(ot.rotate(x, P), P), x, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------
def _golden_packing():
    vals = {}
    for line in open(os.path.join(GOLDEN, "packing.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *rest = line.split()
        vals[key] = rest
    return vals


def test_packing_matches_hand_derived_fixture():
    g = _golden_packing()
    B = int(g["codes_B"][0])
    codes = np.array([[int(v) for v in g["codes"]]])
    want = np.array([[int(v, 16) for v in g["codes_bytes"]]], dtype=np.uint8)
    got = ot.pack_codes(codes, B)
    assert np.array_equal(got, want)
    assert np.array_equal(ot.unpack_codes(got, codes.shape[1], B), codes)
    proj = np.array([[float(v) for v in g["projections"]]])
    bits = (proj < 0).astype(np.int64)
    want_s = np.array([[int(v, 16) for v in g["signs_bytes"]]], dtype=np.uint8)
    assert np.array_equal(ot.pack_signs(bits), want_s)
    assert np.array_equal(ot.unpack_signs(want_s, 16), bits)


@pytest.mark.parametrize("d,B,m", [(16, 1, 32), (128, 2, 128), (128, 3, 128), (1024, 3, 1024), (64, 4, 96)])
def test_pack_roundtrip_and_sizes(d, B, m):
    rng = np.random.default_rng(d + B)
    codes = rng.integers(0, 1 << B, size=(7, d))
    pk = ot.pack_codes(codes, B)
    assert pk.shape == (7, d * B // 8)
    assert np.array_equal(ot.unpack_codes(pk, d, B), codes)
    bits = rng.integers(0, 2, size=(7, m))
    ps = ot.pack_signs(bits)
    assert ps.shape == (7, m // 8)
    assert np.array_equal(ot.unpack_signs(ps, m), bits)
    assert ot.packed_sizes(d, B + 1, m) == (d * B // 8, m // 8)


# --------------------------------------------------------------------------
# Write half, brute force on tiny inputs
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b", [2, 3, 4, 5])
def test_quantize_brute_force_tiny(b):
    d, m = 16, 32
    P = op.Params(d, b, m, seed=2)
    rng = np.random.default_rng(b)
    x = rng.standard_normal((40, d)) * rng.uniform(0.1, 10, size=(40, 1))
    q = ot.quantize(x, P, keep_intermediates=True)
    c = P.centroids
    for r in range(x.shape[0]):
        n = math.sqrt(sum(v * v for v in x[r]))
        u = [v / n for v in x[r]]
        # y_i = sum_j H[i, j] D_j u_j / sqrt(d)
        y = [sum(hadamard_entry(i, j) * P.D[j] * u[j] for j in range(d)) / math.sqrt(d) for i in range(d)]
        for i in range(d):
            # nearest centroid; midpoint thresholds make it the Lloyd-Max cell
            dist = [abs(y[i] - ck) for ck in c]
            k = int(np.argmin(dist))
            if abs(y[i] - P.thresholds64[min(max(k - 1, 0), P.L - 2)]) > 1e-7 and \
               abs(y[i] - P.thresholds64[min(k, P.L - 2)]) > 1e-7:
                assert q["code"][r, i] == k
        res = [y[i] - c[q["code"][r, i]] for i in range(d)]
        assert abs(q["rho"][r] - math.sqrt(sum(v * v for v in res))) < 1e-12
        for j in range(m):
            pj = sum(P.S[j, i] * res[i] for i in range(d))
            assert abs(pj - q["p"][r, j]) < 1e-12
            assert q["bits"][r, j] == (1 if pj < 0 else 0)
        assert abs(q["norm"][r] - np.float32(n)) == 0
        assert q["rnorm"][r] == np.float32(n * q["rho"][r])


def test_quantize_zero_and_tie_rows():
    P = op.Params(16, 3, 32, seed=0)
    x = np.zeros((3, 16))
    x[1, 0] = 1e-12                     # below the zero-norm rule: stored as zero
    x[2, :2] = 1.0                      # y has exact zeros (ties at t = 0)
    q = ot.quantize(x, P, keep_intermediates=True)
    for r in (0, 1):
        assert not q["codes"][r].any() and not q["signs"][r].any()
        assert q["norm"][r] == 0 and q["rnorm"][r] == 0
    y = q["y"][2]
    zeros = np.abs(y) < 1e-15
    assert zeros.any()
    # exactly zero sits on the middle threshold and goes to the lower cell
    assert np.all(q["code"][2][zeros] == P.L // 2 - 1)


# --------------------------------------------------------------------------
# Gaussian identities behind QJL (Qiita explainer "Stage 2: QJL";
# ai.spot.hk "無偏內積估計")
# --------------------------------------------------------------------------
def test_qjl_unbiased_over_1e5_seeds():
    d, m = 16, 32
    rng = np.random.default_rng(11)
    q = rng.standard_normal(d)
    r = rng.standard_normal(d) * 0.3
    want = float(q @ r)
    ests = []
    for chunk in range(10):
        seeds = np.arange(chunk * 10000, (chunk + 1) * 10000, dtype=np.uint64) + np.uint64(1000)
        S = op.gaussian_projection(m, d, seeds)                  # (n, m, d)
        sq = S @ q                                               # (n, m)
        p = S @ r
        z = np.where(p < 0, -1.0, 1.0)                           # bit 1 = negative
        rn = np.linalg.norm(r)
        ests.append(np.array([ot.qjl_correction(sq[i][None], z[i][None], rn, m)[0, 0] for i in range(len(seeds))]))
    e = np.concatenate(ests)
    se = e.std(ddof=1) / math.sqrt(e.size)
    assert abs(e.mean() - want) < 3 * se
    # variance of the m-sample average: ((pi/2) |q|^2 |r|^2 - <q, r>^2) / m
    var_want = (math.pi / 2 * (q @ q) * (r @ r) - want ** 2) / m
    assert abs(e.var(ddof=1) / var_want - 1) < 0.03


def test_full_estimator_unbiased_over_seeds():
    """E over (D, S) of the logit equals <q, k>: the MSE part is fixed given D
    and the QJL part is unbiased for the residual, so any dropped term, sign
    flip, wrong scale or transposed rotation shows up as a bias."""
    d, b, m = 16, 3, 32
    rng = np.random.default_rng(21)
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((1, d)) * 3.0
    want = float(q[0] @ k[0])
    vals = []
    for seed in range(4000):
        P = op.Params(d, b, m, seed=seed)
        pk = ot.quantize(k, P)
        vals.append(ot.logits(q, pk, P, 1, 1, 1)[0, 0, 0])
    v = np.array(vals)
    se = v.std(ddof=1) / math.sqrt(v.size)
    assert abs(v.mean() - want) < 3 * se
    # the estimator is not trivially exact: its spread is non-zero
    assert se > 1e-4


def test_dequant_prod_matches_logit_and_is_unbiased():
    d, b, m = 16, 3, 32
    rng = np.random.default_rng(31)
    y_probe = rng.standard_normal((1, d))
    x = rng.standard_normal((1, d)) * 2.0
    vals = []
    for seed in range(3000):
        P = op.Params(d, b, m, seed=seed)
        pk = ot.quantize(x, P)
        xt = ot.dequant(pk, P, ot.DEQUANT_PROD)
        lg = ot.logits(y_probe, pk, P, 1, 1, 1)[0, 0, 0]
        # <y, x~_PROD> equals the logit estimator exactly (same linear form)
        assert abs(float(y_probe[0] @ xt[0]) - lg) < 1e-10 * (1 + abs(lg))
        vals.append(lg)
    v = np.array(vals)
    assert abs(v.mean() - float(y_probe[0] @ x[0])) < 3 * v.std(ddof=1) / math.sqrt(v.size)


def test_dequant_mse_error_is_the_stored_residual():
    # x - x~_MSE = n R^T y - norm R^T yhat.  With the fp64 norm this is
    # n R^T (y - yhat), whose length is exactly n * rho; the stored fp32 norm
    # moves it by at most |n - norm| * |yhat| (about 1e-7 relative).
    P = op.Params(128, 3, 128, seed=4)
    x = np.random.default_rng(4).standard_normal((50, 128)) * 5
    q = ot.quantize(x, P, keep_intermediates=True)
    exact = dict(q, norm=q["n"])
    err = np.linalg.norm(x - ot.dequant(exact, P, ot.DEQUANT_MSE), axis=1)
    assert np.allclose(err, q["n"] * q["rho"], rtol=1e-12)
    err32 = np.linalg.norm(x - ot.dequant(q, P, ot.DEQUANT_MSE), axis=1)
    assert np.allclose(err32, q["rnorm"], rtol=2e-6)


@pytest.mark.parametrize("B", [1, 2, 3, 4])
def test_empirical_distortion_matches_quadrature(B):
    # Isotropic Gaussian rows are uniform on the sphere after any fixed
    # orthogonal R, so E[rho^2] equals the codebook's quadrature distortion.
    d = 128
    P = op.Params(d, B + 1, 32, seed=9)
    x = np.random.default_rng(100 + B).standard_normal((20000, d))
    q = ot.quantize(x, P, keep_intermediates=True)
    r2 = q["rho"] ** 2
    D = op.mse_distortion(d, P.centroids64)
    assert abs(r2.mean() - D) < 3 * r2.std(ddof=1) / math.sqrt(r2.size)


def test_logit_cosine_agrees_with_closed_form_prediction():
    """Cosine between estimated and exact logits over many keys: for
    independent Gaussian q, k the estimator error has variance
    |q|^2 |r|^2 (pi/2 - 1/d) / m against a signal variance |q|^2 |k|^2 / d,
    so cos = (1 + d D_B (pi/2 - 1/d) / m)^-1/2  (about 0.92 at d = m = 128,
    b = 3: the literal "> 0.99" for Gaussian keys is out of the method's reach)."""
    d, b, m = 128, 3, 128
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(77)
    k = rng.standard_normal((4096, d))
    qs = rng.standard_normal((32, d))
    pk = ot.quantize(k, P)
    est = ot.logits(qs, pk, P, 1, 32, 4096)[0]
    exact = qs @ k.T
    cos = np.sum(est * exact, axis=1) / (np.linalg.norm(est, axis=1) * np.linalg.norm(exact, axis=1))
    D = op.mse_distortion(d, P.centroids64)
    pred = (1 + d * D * (math.pi / 2 - 1 / d) / m) ** -0.5
    se = cos.std(ddof=1) / math.sqrt(cos.size)
    assert abs(cos.mean() - pred) < max(3 * se, 0.005)
    assert 0.90 < cos.mean() < 0.94


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(5)
    s = rng.integers(0, 6, size=(9, 40)).astype(np.float64)   # many ties
    idx, val = ot.topk(s, 10)
    for r in range(s.shape[0]):
        want = sorted(range(s.shape[1]), key=lambda j: (-s[r, j], j))[:10]
        assert list(idx[r]) == want
        assert np.array_equal(val[r], s[r, want])


# ---------------------------------------------------------------------------
# attention from packed keys and values: pinned by what softmax-weighted
# averaging must do, independent of the formula's own arithmetic
# ---------------------------------------------------------------------------
def _packed_pair(d=32, b=3, m=32, n=7, seed=3):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n, d)) * 2.0
    v = rng.standard_normal((n, d))
    return P, ot.quantize(k, P), ot.quantize(v, P), rng


def test_attention_single_key_returns_that_value():
    P, pk, pv, rng = _packed_pair(n=1)
    q = rng.standard_normal((3, P.d))
    out = ot.attention(q, pk, pv, P, 1, 3, 1, scale=0.7)
    xv = ot.dequant(pv, P)
    assert np.allclose(out[0], np.repeat(xv, 3, axis=0), rtol=0, atol=1e-12)


def test_attention_equal_scores_average_the_values():
    P, pk, pv, rng = _packed_pair(n=9)
    q = rng.standard_normal((2, P.d))
    out = ot.attention(q, pk, pv, P, 1, 2, 9, scale=1.0, logits_in=np.zeros((1, 2, 9)))
    for mode in (ot.DEQUANT_PROD, ot.DEQUANT_MSE):
        o = ot.attention(q, pk, pv, P, 1, 2, 9, scale=1.0, mode=mode, logits_in=np.full((1, 2, 9), 3.5))
        assert np.allclose(o[0], ot.dequant(pv, P, mode).mean(axis=0)[None, :], atol=1e-12)
    assert np.allclose(out[0][0], out[0][1])


def test_attention_large_scale_selects_the_top_key():
    P, pk, pv, rng = _packed_pair(n=6)
    s = np.array([[[0.1, 2.0, -1.0, 1.9, 0.0, 0.5]]])
    o = ot.attention(rng.standard_normal((1, P.d)), pk, pv, P, 1, 1, 6, scale=1e4, logits_in=s)
    assert np.allclose(o[0, 0], ot.dequant(pv, P)[1], atol=1e-9)


def test_attention_is_invariant_to_key_order_and_weights_sum_to_one():
    P, pk, pv, rng = _packed_pair(n=8)
    q = rng.standard_normal((1, P.d))
    perm = rng.permutation(8)
    pk2 = {k: v[perm] for k, v in pk.items()}
    pv2 = {k: v[perm] for k, v in pv.items()}
    a = ot.attention(q, pk, pv, P, 1, 1, 8, scale=0.3)
    b = ot.attention(q, pk2, pv2, P, 1, 1, 8, scale=0.3)
    assert np.allclose(a, b, atol=1e-12)
    # against softmax weights built by hand from the estimator's logits
    s = ot.logits(q, pk, P, 1, 1, 8)[0, 0]
    w = np.exp(0.3 * (s - s.max()))
    w /= w.sum()
    assert abs(w.sum() - 1.0) < 1e-15
    assert np.allclose(a[0, 0], w @ ot.dequant(pv, P), atol=1e-12)


def test_padding_to_a_power_of_two():
    """Zero padding changes neither the norm nor any inner product, and the
    padded rotation keeps the padded vector's length: the padded quantizer sees
    the same geometry as the original row."""
    assert [ot.padded_dim(d) for d in (32, 33, 96, 100, 128, 3072, 4096)] == [32, 64, 128, 128, 128, 4096, 4096]
    rng = np.random.default_rng(1)
    x, y = rng.standard_normal((2, 100))
    px, py = ot.pad_rows(x, 128), ot.pad_rows(y, 128)
    assert px.shape == (128,) and np.all(px[100:] == 0) and np.array_equal(px[:100], x)
    assert np.isclose(px @ py, x @ y, rtol=1e-14)
    P = op.Params(128, 3, 128, seed=0)
    assert np.isclose(np.linalg.norm(ot.rotate(px[None, :], P)), np.linalg.norm(x), rtol=1e-13)


# ---------------------------------------------------------------------------
# fractional bit widths by a channel split (the library's reading; see
# oracle.turboquant.split_parts)

def test_split_bit_budgets():
    """64 + 64 channels at b = 3 / 2 store 2.5 bits per coordinate, at 4 / 3
    3.5 bits (codes b - 1 per channel plus one sign per channel, m = d_part)."""
    p25 = ot.split_parts(128, 64, 3, 2, 0, op.Params)
    p35 = ot.split_parts(128, 64, 4, 3, 0, op.Params)
    assert ot.split_bits_per_coordinate(p25) == 2.5
    assert ot.split_bits_per_coordinate(p35) == 3.5
    # packed bytes per row: codes + signs of both parts, plus two fp32 norms each
    assert sum(sum(ot.packed_sizes(P.d, P.b, P.m)[:2]) for _, _, P in p25) == 128 * 2.5 / 8
    assert [P.seed for _, _, P in p25] == [0, 1] and [c0 for c0, _, _ in p25] == [0, 64]


def test_split_query_on_one_part_is_that_parts_estimate():
    """A query that is zero on one part's channels gets exactly the other
    part's estimate: catches swapped parts and wrong column offsets."""
    parts = ot.split_parts(96, 64, 4, 2, 3, op.Params)      # 64 + 32 channels
    rng = np.random.default_rng(5)
    k = rng.standard_normal((7, 96)) * 2.0
    pk = ot.split_quantize(k, parts)
    q = rng.standard_normal((1, 96))
    q_hi, q_lo = q.copy(), q.copy()
    q_hi[:, 64:] = 0.0
    q_lo[:, :64] = 0.0
    (c0, dc, P0), (c1, dc1, P1) = parts
    own_hi = ot.logits(q[:, :64], pk[0], P0, 1, 1, 7)
    own_lo = ot.logits(ot.pad_rows(q[:, 64:], P1.d), pk[1], P1, 1, 1, 7)
    assert np.array_equal(ot.split_logits(q_hi, pk, parts, 1, 1, 7), own_hi)
    assert np.array_equal(ot.split_logits(q_lo, pk, parts, 1, 1, 7), own_lo)
    assert np.allclose(ot.split_logits(q, pk, parts, 1, 1, 7), own_hi + own_lo, rtol=1e-14, atol=1e-14)


def test_split_estimator_unbiased_over_seeds():
    """E over the two parts' (D, S) of the split estimate equals <q, k>."""
    rng = np.random.default_rng(41)
    q = rng.standard_normal((1, 32))
    k = rng.standard_normal((1, 32)) * 2.0
    want = float(q[0] @ k[0])
    vals = []
    for seed in range(0, 6000, 2):
        parts = ot.split_parts(32, 16, 3, 2, seed, op.Params)
        vals.append(ot.split_logits(q, ot.split_quantize(k, parts), parts, 1, 1, 1)[0, 0, 0])
    v = np.array(vals)
    se = v.std(ddof=1) / math.sqrt(v.size)
    assert abs(v.mean() - want) < 3 * se and se > 1e-4


def test_split_mse_error_per_part_and_distortion():
    """On each part's channels, x - x~_MSE has length n_p rho_p (that part's
    stored residual norm, as for one instance), and E[rho_p^2] is that part's
    codebook distortion: the higher-width part about 4x below the lower."""
    parts = ot.split_parts(128, 64, 4, 3, 9, op.Params)
    x = np.random.default_rng(77).standard_normal((6000, 128))
    pk = ot.split_quantize(x, parts, keep_intermediates=True)
    xt = ot.split_dequant(pk, parts, ot.DEQUANT_MSE)
    dist = []
    for (c0, dc, P), p in zip(parts, pk):
        err = np.linalg.norm(x[:, c0:c0 + dc] - xt[:, c0:c0 + dc], axis=1)
        assert np.allclose(err, p["rnorm"], rtol=2e-6)
        r2 = p["rho"] ** 2
        D = op.mse_distortion(P.d, P.centroids64)
        assert abs(r2.mean() - D) < 3 * r2.std(ddof=1) / math.sqrt(r2.size)
        dist.append(D)
    assert 3.0 < dist[1] / dist[0] < 4.5
