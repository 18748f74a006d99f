"""GPU parity of the wide-row tensor-core paths (d >= 256, many rows): the
QJL projection of the write half as an fp16 GEMM with a listed fp64 fix-up of
the projections inside its error bound, and the all-pairs estimates as an
fp16 GEMM over decoded keys and split queries.

Row counts span more than one write-half chunk (296 tiles of 128 rows) and end
in a ragged tile; query counts end in a ragged 256-column tile.  Codes, signs,
norms and estimates follow the oracle rules of tests/parity.py.
"""

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot
from tests import parity
from tests.test_gpu_parity import edge_rows, make_ctx, make_rows

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CHUNK = 148 * 128


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_15_b200 import tq as _tq
    return _tq


@pytest.mark.parametrize("d,b,m,dtype,n", [
    (256, 3, 256, "f32", 2 * CHUNK + 1001),     # two write-half chunks (37888 rows each)
    (256, 2, 96, "bf16", CHUNK + 77),
    (512, 4, 128, "bf16", 4096),
    (1024, 4, 1024, "f32", CHUNK + 777),
    (2048, 3, 64, "bf16", 5000),
])
def test_wide_quantize_parity(tq, d, b, m, dtype, n):
    xt, x = make_rows(d, n, dtype, seed=d + 7 * b + m)
    P = op.Params(d, b, m, seed=0)
    T = make_ctx(tq, d, b, m)
    got = T.quantize(xt.cuda()).to_numpy()
    T.sync_status()
    rep = parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True))
    parity.assert_quantize_ok(rep)


@pytest.mark.parametrize("d,b,m,n_sets,g,n_keys,qdtype", [
    (256, 3, 256, 2, 300, CHUNK + 513, "f32"),
    (512, 2, 128, 3, 64, 5000, "bf16"),
    (1024, 4, 1024, 1, 1024, 4500, "f32"),
    (256, 5, 64, 1, 257, 4096, "bf16"),
])
def test_wide_logits_parity(tq, d, b, m, n_sets, g, n_keys, qdtype):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d + g + b)
    k = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1))
    k[:3] = edge_rows(d, rng)[:3]
    pk = ot.quantize(k, P)
    qt, q = make_rows(d, n_sets * g, qdtype, seed=3 * g + b)
    T = make_ctx(tq, d, b, m)
    got = T.logits(qt.cuda(), tq.Packed.from_numpy(pk), n_sets, g, n_keys).cpu().numpy()
    T.sync_status()
    want = ot.logits(q, pk, P, n_sets, g, n_keys)
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    err = np.abs(got - want)
    assert np.all(err <= tol + 1e-30), float(np.max(err / (tol + 1e-30)))


def test_wide_quantize_then_logits_end_to_end(tq):
    """GPU quantize -> GPU estimates on the wide paths against the oracle's
    quantize -> estimates; keys whose packed bytes differ (boundary band) are
    counted, not compared."""
    d, b, m, g, n_keys = 1024, 4, 1024, 300, 6000
    P = op.Params(d, b, m, seed=0)
    kt, k = make_rows(d, n_keys, "f32", seed=21)
    qt, q = make_rows(d, g, "f32", seed=22)
    T = make_ctx(tq, d, b, m)
    pg = T.quantize(kt.cuda())
    got = T.logits(qt.cuda(), pg, 1, g, n_keys).cpu().numpy()
    T.sync_status()
    po = ot.quantize(k, P)
    want = ot.logits(q, po, P, 1, g, n_keys)
    png = pg.to_numpy()
    same = np.all(png["codes"] == po["codes"], axis=1) & np.all(png["signs"] == po["signs"], axis=1)
    assert np.mean(~same) <= 1e-2
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), 1, g, n_keys)
    ok = (np.abs(got - want) <= tol + 1e-30) | ~same.reshape(1, 1, n_keys)
    assert ok.all()


@pytest.mark.parametrize("d,b,m,n_q,n_keys,k,qdtype", [
    (256, 3, 256, 300, CHUNK + 513, 10, "f32"),     # fused: ragged key and query tiles
    (256, 3, 256, 64, 80000, 10, "f32"),             # fused: lists carried across two key chunks
    (1024, 4, 1024, 64, 5000, 16, "bf16"),           # fused, k = 16
    (512, 2, 128, 100, 4096, 1, "f32"),              # fused, k = 1
    (128, 3, 128, 37, 3000, 10, "bf16"),             # through the scores (d = 128)
    (256, 3, 256, 10, 5000, 5, "f32"),               # through the scores (fewer than 64 queries)
])
def test_search_equals_topk_of_logits(tq, d, b, m, n_q, n_keys, k, qdtype):
    """tq_search picks the k best rows by the same estimates tq_logits writes
    (its own tensor-core pass: values equal to the scores within fp32
    accumulation-order noise, every pick within that noise of the k-th best,
    larger first, no repeats), and its choices agree with the oracle's
    estimates."""
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d + n_q + k)
    kk = rng.standard_normal((n_keys, d)) * rng.uniform(0.1, 10, size=(n_keys, 1))
    kk[:3] = edge_rows(d, rng)[:3]
    pk = ot.quantize(kk, P)
    qt, q = make_rows(d, n_q, qdtype, seed=5 * n_q + b)
    T = make_ctx(tq, d, b, m)
    dpk = tq.Packed.from_numpy(pk)
    scores = T.logits(qt.cuda(), dpk, 1, n_q, n_keys)
    i_ref, v_ref = tq.topk(scores[0], k)
    i_got, v_got = T.search(qt.cuda(), dpk, n_keys, k)
    T.sync_status()
    sc = scores[0].cpu().numpy().astype(np.float64)
    ig64 = i_got.cpu().numpy().astype(np.int64)
    vg64 = v_got.cpu().numpy().astype(np.float64)
    r_ = np.arange(n_q)[:, None]
    eps = 1e-5 * np.abs(sc).max(axis=1, keepdims=True)
    assert np.all(np.abs(vg64 - sc[r_, ig64]) <= eps)
    assert np.all(sc[r_, ig64] >= -np.sort(-sc, axis=1)[:, k - 1:k] - eps)
    assert np.all(np.diff(vg64, axis=1) <= 0)
    assert all(len(set(row)) == k for row in ig64.tolist())
    assert np.mean(ig64 == i_ref.cpu().numpy()) >= 0.98
    want = ot.logits(q, pk, P, 1, n_q, n_keys)[0]
    tol = parity.logit_tolerance(q, np.linalg.norm(kk, axis=1), 1, n_q, n_keys)[0]
    ig = i_got.cpu().numpy().astype(np.int64)
    vg = v_got.cpu().numpy().astype(np.float64)
    rows = np.arange(n_q)[:, None]
    assert np.all(np.abs(vg - want[rows, ig]) <= tol[rows, ig] + 1e-30)
    # every chosen row is within the estimate tolerance of the oracle's k-th best
    kth = -np.sort(-want, axis=1)[:, k - 1]
    assert np.all(want[rows, ig] >= kth[:, None] - 2 * tol.max(axis=1, keepdims=True))


def test_search_argument_errors(tq):
    d, b, m, n_keys = 256, 3, 256, 4096
    P = op.Params(d, b, m, seed=0)
    pk = tq.Packed.from_numpy(ot.quantize(np.random.default_rng(0).standard_normal((n_keys, d)), P))
    T = make_ctx(tq, d, b, m)
    q = torch.randn(64, d, device="cuda")
    for bad in (0, 17):
        with pytest.raises(tq.TQError):
            T.search(q, pk, n_keys, bad)
    with pytest.raises(tq.TQError):
        T.search(q, pk, 3, 4)                                    # k > n_keys
    with pytest.raises(tq.TQError):
        T.search(q, pk, n_keys, 10, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    T.sync_status()
