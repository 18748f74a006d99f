"""GPU parity: every entry point of the C ABI against the fp64 oracle, on the
same seeded inputs, element by element.  Sizes span several tiles and a
ragged tail; edge rows (zero, tiny, huge, one-hot, constant) are mixed in.

The read-half kernels are fed packed rows produced by the oracle, so both
sides compute on byte-identical inputs; the write half is compared with the
boundary-band rule in tests/parity.py.
"""

import math

import numpy as np
import pytest

from kv_cache_vector_15_b200 import inputs
from oracle import params as op
from oracle import turboquant as ot
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_15_b200 import tq as _tq
    return _tq


def make_ctx(tq, d, b, m, kernels="auto"):
    """A context whose compute calls use the hot-path kernels ("auto") or the
    general CUDA-core kernels ("generic"); the choice is fixed at creation."""
    import os
    old = os.environ.pop("TQ_KERNELS", None)
    if kernels == "generic":
        os.environ["TQ_KERNELS"] = "generic"
    try:
        return tq.TurboQuant(d, b, m, seed=0)
    finally:
        os.environ.pop("TQ_KERNELS", None)
        if old is not None:
            os.environ["TQ_KERNELS"] = old


def edge_rows(d, rng):
    rows = [np.zeros(d), np.full(d, 0.5), np.eye(1, d, 3)[0] * 7.0, rng.standard_normal(d) * 1e-8,
            rng.standard_normal(d) * 3e3, np.concatenate([np.ones(2), np.zeros(d - 2)])]
    return np.stack(rows)


def make_rows(d, n, dtype, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) * rng.uniform(0.1, 10, size=(n, 1))
    e = edge_rows(d, rng)
    x[: min(6, n)] = e[: min(6, n)]
    x = x.astype(np.float32)
    if dtype == "bf16":
        bits = inputs.bf16_bits(x)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16), inputs.bf16_to_f32(bits)
    return torch.from_numpy(x), x


CASES = [(32, 2, 32), (64, 3, 64), (128, 2, 128), (128, 3, 128), (128, 4, 128), (128, 5, 128),
         (256, 3, 96), (512, 4, 256), (1024, 4, 1024), (2048, 2, 64), (4096, 3, 128)]


@pytest.mark.parametrize("b", [2, 3, 4, 5])
def test_quantize_d128_tensor_core_small_first(tq, b):
    """The tcgen05 write half on a handful of rows (one partial tile)."""
    d, m = 128, 128
    xt, x = make_rows(d, 37, "bf16", seed=b)
    P = op.Params(d, b, m, seed=0)
    T = make_ctx(tq, d, b, m)
    got = T.quantize(xt.cuda()).to_numpy()
    T.sync_status()
    parity.assert_quantize_ok(parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True)))


@pytest.mark.parametrize("b", [2, 3, 4, 5])
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 128), ("bf16", 64)])
def test_quantize_d128_many_tiles(tq, b, dtype, d):
    """Enough rows that every CTA loops over several tiles (phase flips of
    every barrier), with a ragged last tile; d = 64 bf16 rows take the same
    tensor-core kernel at half width (two CTAs per SM)."""
    m, n = d, 100003
    xt, x = make_rows(d, n, dtype, seed=100 + b)
    P = op.Params(d, b, m, seed=0)
    T = make_ctx(tq, d, b, m)
    got = T.quantize(xt.cuda()).to_numpy()
    T.sync_status()
    rep = parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True))
    parity.assert_quantize_ok(rep)


@pytest.mark.parametrize("d,b,m", CASES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("kernels", ["auto", "generic"])
def test_quantize_parity(tq, d, b, m, dtype, kernels):
    if kernels == "generic" and d != 128:
        pytest.skip("shapes other than d = 128 always use the general kernels")
    n = 1531 if d <= 1024 else 301
    xt, x = make_rows(d, n, dtype, seed=d * 10 + b)
    P = op.Params(d, b, m, seed=0)
    T = make_ctx(tq, d, b, m, kernels)
    got = T.quantize(xt.cuda()).to_numpy()
    T.sync_status()
    want = ot.quantize(x, P, keep_intermediates=True)
    rep = parity.compare_quantize(P, got, want)
    parity.assert_quantize_ok(rep)


def test_quantize_strided_rows(tq):
    d, b, m = 128, 3, 128
    xt, x = make_rows(d, 777, "bf16", seed=5)
    wide = torch.zeros((777, 200), dtype=torch.bfloat16)
    wide[:, :d] = xt
    P = op.Params(d, b, m, seed=0)
    T = tq.TurboQuant(d, b, m, seed=0)
    got = T.quantize(wide.cuda()[:, :d]).to_numpy()
    parity.assert_quantize_ok(parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True)))


@pytest.mark.parametrize("d,b,m,n_sets,g,n_keys", [
    (128, 3, 128, 3, 4, 1000), (128, 4, 128, 2, 1, 4097), (128, 2, 128, 5, 8, 333), (64, 5, 64, 2, 3, 700),
    (128, 3, 128, 2, 16, 1500), (256, 3, 128, 1, 40, 900), (1024, 4, 1024, 1, 37, 600), (32, 2, 32, 4, 5, 129)])
@pytest.mark.parametrize("qdtype", ["bf16", "f32"])
def test_logits_parity_on_oracle_packed_keys(tq, d, b, m, n_sets, g, n_keys, qdtype):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d + g)
    k = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1))
    k[:3] = edge_rows(d, rng)[:3]
    pk = ot.quantize(k, P)
    qt, q = make_rows(d, n_sets * g, qdtype, seed=7 + g)
    T = tq.TurboQuant(d, b, m, seed=0)
    got = T.logits(qt.cuda(), tq.Packed.from_numpy(pk), n_sets, g, n_keys).cpu().numpy()
    want = ot.logits(q, pk, P, n_sets, g, n_keys)
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    err = np.abs(got - want)
    assert np.all(err <= tol + 1e-30), float(np.max(err / (tol + 1e-30)))


@pytest.mark.parametrize("b,g", [(3, 4), (2, 8), (3, 5), (3, 1), (4, 4), (4, 8), (4, 1)])
@pytest.mark.parametrize("kernels", ["auto", "generic"])
def test_logits_d128_many_tiles_and_sets(tq, b, g, kernels):
    """Several 128-key tiles per warpgroup, sets changing inside a warpgroup's
    tile range, ragged last tile of every set."""
    d, m, n_sets, n_keys = 128, 128, 7, 20001
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(b * 10 + g)
    k = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1))
    pk = ot.quantize(k, P)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=3 + g)
    T = make_ctx(tq, d, b, m, kernels)
    got = T.logits(qt.cuda(), tq.Packed.from_numpy(pk), n_sets, g, n_keys).cpu().numpy()
    T.sync_status()
    want = ot.logits(q, pk, P, n_sets, g, n_keys)
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    err = np.abs(got - want)
    assert np.all(err <= tol + 1e-30), float(np.max(err / (tol + 1e-30)))


@pytest.mark.parametrize("d,b,m", [(128, 3, 128), (128, 4, 128), (64, 2, 96), (1024, 4, 1024)])
def test_end_to_end_quantize_then_logits(tq, d, b, m):
    """GPU quantize -> GPU logits against oracle quantize -> oracle logits.
    Keys whose packed bytes differ (boundary-band cases) are counted, not compared."""
    n_sets, g, n_keys = 2, 4, 1200
    P = op.Params(d, b, m, seed=0)
    kt, k = make_rows(d, n_sets * n_keys, "bf16", seed=11)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=12)
    T = tq.TurboQuant(d, b, m, seed=0)
    pg = T.quantize(kt.cuda())
    got = T.logits(qt.cuda(), pg, n_sets, g, n_keys).cpu().numpy()
    po = ot.quantize(k, P)
    want = ot.logits(q, po, P, n_sets, g, n_keys)
    png = pg.to_numpy()
    same = (np.all(png["codes"] == po["codes"], axis=1) & np.all(png["signs"] == po["signs"], axis=1))
    assert np.mean(~same) <= 1e-3
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    ok = (np.abs(got - want) <= tol + 1e-30) | ~same.reshape(n_sets, 1, n_keys)
    assert ok.all()


@pytest.mark.parametrize("d,b,m,n", [(128, 3, 128, 1029), (128, 4, 128, 1029), (128, 2, 128, 1029),
                                     (64, 5, 32, 1029), (1024, 4, 1024, 1029), (4096, 3, 64, 130),
                                     (128, 3, 128, 77777), (128, 5, 128, 40001),
                                     (64, 2, 64, 1029), (64, 3, 64, 40001), (64, 4, 64, 40001),
                                     (64, 5, 64, 1029)])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_dequant_parity_on_oracle_packed_rows(tq, d, b, m, n, mode, out):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d * 3 + b)
    x = rng.standard_normal((n, d)) * rng.uniform(0.1, 10, size=(n, 1))
    x[:6] = edge_rows(d, rng)
    pk = ot.quantize(x, P)
    T = tq.TurboQuant(d, b, m, seed=0)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    got = T.dequant(tq.Packed.from_numpy(pk), out_dtype=dt, mode=mode).float().cpu().numpy()
    want = ot.dequant(pk, P, mode)
    parity.assert_dequant_ok(got, want, out == "bf16")


@pytest.mark.parametrize("rows,cols,k", [(7, 1000, 10), (3, 5, 5), (64, 100003, 10), (5, 4096, 64), (2, 77, 1)])
def test_topk_parity_with_ties(tq, rows, cols, k):
    rng = np.random.default_rng(rows * cols + k)
    s = rng.standard_normal((rows, cols)).astype(np.float32)
    s[:, ::7] = np.round(s[:, ::7] * 2) / 2          # many exact ties
    s[0, :] = 1.0                                   # an all-equal row
    idx, val = tq.topk(torch.from_numpy(s).cuda(), k)
    wi, wv = ot.topk(s, k)
    assert np.array_equal(idx.cpu().numpy(), wi)
    assert np.array_equal(val.cpu().numpy(), wv)


@pytest.mark.parametrize("d,g,n_sets,n_keys", [(128, 4, 3, 2049), (64, 1, 3, 2049), (256, 8, 3, 2049),
                                               (128, 3, 3, 2049), (128, 2, 700, 5), (64, 8, 50, 3001),
                                               (256, 5, 9, 77), (128, 4, 1, 1)])
def test_bf16_baseline_logits(tq, d, g, n_sets, n_keys):
    """Ragged key chunks: n_keys below one chunk (set boundaries inside one warp's range), one key."""
    kt, k = make_rows(d, n_sets * n_keys, "bf16", seed=d + g)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=d * g)
    got = tq.logits_bf16(qt.cuda(), kt.cuda(), n_sets, g, n_keys).cpu().numpy()
    want = np.einsum("sgd,snd->sgn", q.reshape(n_sets, g, d).astype(np.float64),
                     k.reshape(n_sets, n_keys, d).astype(np.float64))
    bound = np.einsum("sgd,snd->sgn", np.abs(q.reshape(n_sets, g, d)), np.abs(k.reshape(n_sets, n_keys, d)))
    assert np.all(np.abs(got - want) <= d * 2.0 ** -24 * bound + 1e-30)


def test_gpu_api_errors_and_empty_calls(tq):
    T = tq.TurboQuant(128, 3, 128)
    x = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
    p = T.quantize(x)                              # n = 0: no-op
    assert p.n_rows == 0
    xb = torch.zeros((10, 129), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tq.TQError) as e:
        T.quantize(xb[:, 1:])                      # misaligned base pointer
    assert e.value.status == tq.TQ_ERR_INVALID_ARG
    with pytest.raises(tq.TQError):
        T.quantize(torch.zeros((10, 100), dtype=torch.float32, device="cuda"))   # ld < d is caught below
    with pytest.raises(tq.TQError):
        T.logits(torch.zeros((4, 128), device="cuda"), T.empty_packed(8), 1, 0, 8)  # g = 0
    before = tq.launch_count()
    with pytest.raises(tq.TQError):
        T.logits(torch.zeros((4, 128), device="cuda"), T.empty_packed(8), 1, 4, 8,
                 workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert tq.launch_count() == before


@pytest.mark.parametrize("d,b,m,n_sets,g,n_keys", [
    (128, 3, 128, 3, 4, 5000), (128, 4, 128, 2, 8, 2049), (128, 2, 128, 2, 1, 77), (64, 3, 96, 2, 3, 4100),
    (128, 3, 128, 2, 3, 4099), (128, 4, 128, 1, 5, 2100),
    (256, 4, 128, 1, 5, 1500), (1024, 4, 1024, 1, 2, 300)])
@pytest.mark.parametrize("mode", [0, 1])
def test_attention_parity(tq, d, b, m, n_sets, g, n_keys, mode):
    """Attention from packed keys and values against the oracle's softmax and
    dequantized value sum, driven by the kernel's own logits (the logits have
    their own parity test): what is compared is the softmax, the weighted sum
    in the rotated domain, the QJL term and the rotation back."""
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(d + b + g)
    k = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.5, 2, size=(n_sets * n_keys, 1))
    v = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1))
    v[:4] = edge_rows(d, rng)[:4]
    pk, pv = ot.quantize(k, P), ot.quantize(v, P)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=9)
    T = tq.TurboQuant(d, b, m, seed=0)
    keys, vals = tq.Packed.from_numpy(pk), tq.Packed.from_numpy(pv)
    scale = 1.0 / np.sqrt(d)
    got = T.attention(qt.cuda(), keys, vals, n_sets, g, n_keys, scale=scale, mode=mode).cpu().numpy()
    lg = T.logits(qt.cuda(), keys, n_sets, g, n_keys).cpu().numpy()
    T.sync_status()
    want = ot.attention(q, pk, pv, P, n_sets, g, n_keys, scale, mode=mode, logits_in=lg).reshape(n_sets * g, d)
    # per element: 1e-4 of the element plus 1e-4 of the row's rms scale, where
    # the scale also covers cancellation in the weighted sum (the rms of the
    # weighted sum of |dequantized row|, which bounds what fp32 accumulation
    # of the terms can lose)
    xv = ot.dequant(pv, P, mode).reshape(n_sets, n_keys, d)
    z = scale * lg.astype(np.float64).reshape(n_sets, g, n_keys)
    w = np.exp(z - z.max(axis=2, keepdims=True))
    w /= w.sum(axis=2, keepdims=True)
    absum = np.einsum("sgk,skd->sgd", w, np.abs(xv)).reshape(n_sets * g, d)
    rms = lambda a: np.linalg.norm(a, axis=1, keepdims=True) / np.sqrt(d)  # noqa: E731
    tol = 1e-4 * (np.abs(want) + rms(want) + rms(absum))
    err = np.abs(got - want)
    assert np.all(err <= tol + 1e-30), float(np.max(err / tol))


def test_attention_matches_logits_softmax_on_full_oracle(tq):
    """End to end against the oracle's own logits: agreement within what the
    logit tolerance lets the softmax move."""
    d, b, m, n_sets, g, n_keys = 128, 3, 128, 2, 4, 3000
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(21)
    k = rng.standard_normal((n_sets * n_keys, d)) * 0.3
    v = rng.standard_normal((n_sets * n_keys, d))
    pk, pv = ot.quantize(k, P), ot.quantize(v, P)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=22)
    T = tq.TurboQuant(d, b, m, seed=0)
    got = T.attention(qt.cuda(), tq.Packed.from_numpy(pk), tq.Packed.from_numpy(pv), n_sets, g, n_keys).cpu().numpy()
    want = ot.attention(q, pk, pv, P, n_sets, g, n_keys, 1.0 / np.sqrt(d)).reshape(n_sets * g, d)
    vmax = np.abs(ot.dequant(pv, P)).max()
    assert np.max(np.abs(got - want)) <= 1e-3 * vmax


def test_attention_argument_errors(tq):
    T = tq.TurboQuant(128, 3, 128, seed=0)
    q = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    pk = T.empty_packed(10, "cuda")
    with pytest.raises(tq.TQError):
        T.attention(q, pk, pk, 1, 9, 10)                 # g > 8
    with pytest.raises(tq.TQError):
        T.attention(q, pk, pk, 1, 4, 0)                  # no keys
    out = torch.empty((0, 128), dtype=torch.float32, device="cuda")
    T.attention(q, pk, pk, 0, 4, 10, out=out)            # no sets: no-op


@pytest.mark.parametrize("d,b,m,n", [(128, 3, 128, 256), (128, 4, 128, 32), (64, 2, 96, 77), (1024, 4, 1024, 9)])
def test_quantize_scatter_into_paged_cache(tq, d, b, m, n):
    """Append n new rows into a 1000-row packed cache at scattered slots: the
    slots hold what the oracle packs for those rows, every other slot keeps
    its previous contents byte for byte."""
    P = op.Params(d, b, m, seed=0)
    xt, x = make_rows(d, n, "bf16", seed=d + n)
    T = tq.TurboQuant(d, b, m, seed=0)
    cache = T.empty_packed(1000, "cuda")
    for f in ("codes", "signs"):
        getattr(cache, f).fill_(0xA5)
    cache.norm.fill_(-1.0)
    cache.rnorm.fill_(-2.0)
    before = cache.to_numpy()
    slots = np.random.default_rng(n).choice(1000, size=n, replace=False)
    T.quantize_scatter(xt.cuda(), torch.from_numpy(slots.astype(np.int64)).cuda(), cache)
    T.sync_status()
    after = cache.to_numpy()
    want = ot.quantize(x, P, keep_intermediates=True)
    got = {k: after[k][slots] for k in ("codes", "signs", "norm", "rnorm")}
    parity.assert_quantize_ok(parity.compare_quantize(P, got, want))
    untouched = np.setdiff1d(np.arange(1000), slots)
    for k in ("codes", "signs", "norm", "rnorm"):
        assert np.array_equal(after[k][untouched], before[k][untouched]), k


def test_quantize_scatter_rejects_out_of_range_slot(tq):
    T = tq.TurboQuant(128, 3, 128, seed=0)
    cache = T.empty_packed(10, "cuda")
    cache.norm.fill_(-1.0)
    x = torch.ones((2, 128), dtype=torch.bfloat16, device="cuda")
    T.quantize_scatter(x, torch.tensor([3, 10], dtype=torch.int64, device="cuda"), cache)
    with pytest.raises(tq.TQError):
        T.sync_status()
    norm = cache.norm.cpu().numpy()
    assert norm[3] > 0 and np.all(np.delete(norm, 3) == -1.0)
    T.sync_status()                                      # the record was cleared


@pytest.mark.parametrize("d,b,m", [(96, 3, 128), (100, 4, 128), (200, 3, 64), (3072, 4, 128)])
def test_padded_dimension_end_to_end(tq, d, b, m):
    """A row length that is not a power of two: the library pads rows and
    queries with zeros to the next power of two, and dequant / attention give
    back the first d coordinates -- compared with the oracle on explicitly
    padded inputs."""
    dp = ot.padded_dim(d)
    P = op.Params(dp, b, m, seed=0)
    n_sets, g, n_keys = 2, 3, 700
    # random rows only: the structured edge rows put whole groups of rotated
    # coordinates within 1e-6 of a threshold once padded (exempt, but counted)
    rng = np.random.default_rng(d)
    xs = (rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1)))
    bits = inputs.bf16_bits(xs.astype(np.float32))
    xt = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    x = inputs.bf16_to_f32(bits)
    qt, q = make_rows(d, n_sets * g, "bf16", seed=d + 1)
    T = tq.TurboQuant(d, b, m, seed=0)
    pk = T.quantize(xt.cuda())
    got = pk.to_numpy()
    T.sync_status()
    want = ot.quantize(ot.pad_rows(x, dp), P, keep_intermediates=True)
    parity.assert_quantize_ok(parity.compare_quantize(P, got, want))
    po = {k: want[k] for k in ("codes", "signs", "norm", "rnorm")}
    keys = tq.Packed.from_numpy(po)
    lg = T.logits(qt.cuda(), keys, n_sets, g, n_keys).cpu().numpy()
    lw = ot.logits(ot.pad_rows(q, dp), po, P, n_sets, g, n_keys)
    tol = parity.logit_tolerance(q, np.linalg.norm(x, axis=1), n_sets, g, n_keys)
    assert np.all(np.abs(lg - lw) <= tol + 1e-30)
    dq = T.dequant(keys, out_dtype=torch.float32).cpu().numpy()
    assert dq.shape == (n_sets * n_keys, d)
    parity.assert_dequant_ok(dq, ot.dequant(po, P)[:, :d], bf16=False)
    if dp + m > 2048:                                    # beyond tq_attention's shapes
        with pytest.raises(tq.TQError):
            T.attention(qt.cuda(), keys, keys, n_sets, g, n_keys)
        return
    att = T.attention(qt.cuda(), keys, keys, n_sets, g, n_keys).cpu().numpy()
    aw = ot.attention(ot.pad_rows(q, dp), po, po, P, n_sets, g, n_keys, 1.0 / np.sqrt(d), logits_in=lg)
    aw = aw.reshape(n_sets * g, dp)[:, :d]
    vscale = np.abs(ot.dequant(po, P)).max()
    assert att.shape == (n_sets * g, d)
    assert np.max(np.abs(att - aw)) <= 1e-4 * vscale


@pytest.mark.parametrize("d,b,m,dtype", [(256, 3, 128, "bf16"), (64, 4, 96, "f32"), (1024, 2, 64, "bf16")])
def test_quantize_general_kernel_many_rows(tq, d, b, m, dtype):
    """The general write half with four rows per warp (taken from 65536 rows
    on): every row of a ragged last group, and the edge rows.  (With the
    hot-path kernels on, these shapes take the wide-row tensor-core path.)"""
    n = 70001
    xt, x = make_rows(d, n, dtype, seed=d + b)
    P = op.Params(d, b, m, seed=0)
    T = make_ctx(tq, d, b, m, "generic")
    got = T.quantize(xt.cuda()).to_numpy()
    T.sync_status()
    parity.assert_quantize_ok(parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True)))
