"""Parity on the named workloads at their full sizes (GPU).

The CUDA path runs on the whole workload, in the same calls bench.py makes;
the oracle checks sampled rows / keys / queries, which it can recompute one
by one from the seeded generators (inputs.RowTensor.take re-draws any row).
Small workloads (single head, 8K decode) are compared in full.
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


def to_dev(rt: inputs.RowTensor):
    """Whole tensor on the device (bf16 bits as torch.bfloat16, or fp32)."""
    if rt.dtype == "bf16":
        h = torch.empty((rt.n_rows, rt.d), dtype=torch.int16)
        rt.fill(h.numpy().view(np.uint16))
        return h.view(torch.bfloat16).cuda()
    h = torch.empty((rt.n_rows, rt.d), dtype=torch.float32)
    rt.fill(h.numpy())
    return h.cuda()


def sampled_quantize_check(P, rt, packed, idx):
    x = rt.as_f32(rt.take(idx)).astype(np.float64)
    got = {k: getattr(packed, k)[torch.from_numpy(idx).cuda()].cpu().numpy()
           for k in ("codes", "signs", "norm", "rnorm")}
    want = ot.quantize(x, P, keep_intermediates=True)
    rep = parity.compare_quantize(P, got, want)
    parity.assert_quantize_ok(rep)
    return rep, want


def test_single_head_full(tq):
    """4096 fp32 keys with 4 outlier channels, 16 queries, d = 128, b = 3: all of it."""
    K, Q = inputs.single_head()
    P = op.Params(128, 3, 128, seed=0)
    T = tq.TurboQuant(128, 3, 128, seed=0)
    k, q = K.all(), Q.all()
    pk = T.quantize(torch.from_numpy(k).cuda())
    T.sync_status()
    want = ot.quantize(k, P, keep_intermediates=True)
    parity.assert_quantize_ok(parity.compare_quantize(P, pk.to_numpy(), want))
    # logits of all 16 queries against all keys, from the oracle's packed keys
    po = {x: want[x] for x in ("codes", "signs", "norm", "rnorm")}
    got = T.logits(torch.from_numpy(q).cuda(), tq.Packed.from_numpy(po), 1, 16, 4096).cpu().numpy()
    lw = ot.logits(q, po, P, 1, 16, 4096)
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), 1, 16, 4096)
    assert np.all(np.abs(got - lw) <= tol + 1e-30)


@pytest.mark.parametrize("b", [3, 4])
def test_llama_8k_decode_full(tq, b):
    """Llama-3.1-8B-shaped decode: quantize K and V, logits for 32 heads (GQA 4), dequant V."""
    batch, ctx, g = 1, 8192, 4
    K, V, Q = inputs.decode(batch, ctx)
    P = op.Params(128, b, 128, seed=0)
    T = tq.TurboQuant(128, b, 128, seed=0)
    dK, dV = to_dev(K), to_dev(V)
    qb = Q.all()
    pk, pv = T.quantize(dK), T.quantize(dV)
    T.sync_status()
    k = K.as_f32(K.all()).astype(np.float64)
    v = V.as_f32(V.all()).astype(np.float64)
    wk = ot.quantize(k, P, keep_intermediates=True)
    wv = ot.quantize(v, P, keep_intermediates=True)
    parity.assert_quantize_ok(parity.compare_quantize(P, pk.to_numpy(), wk))
    parity.assert_quantize_ok(parity.compare_quantize(P, pv.to_numpy(), wv))
    n_sets = batch * 8
    po = {x: wk[x] for x in ("codes", "signs", "norm", "rnorm")}
    qt = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    got = T.logits(qt, tq.Packed.from_numpy(po), n_sets, g, ctx).cpu().numpy()
    q = Q.as_f32(qb)
    lw = ot.logits(q, po, P, n_sets, g, ctx)
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, ctx)
    assert np.all(np.abs(got - lw) <= tol + 1e-30)
    pvo = {x: wv[x] for x in ("codes", "signs", "norm", "rnorm")}
    dq = T.dequant(tq.Packed.from_numpy(pvo), out_dtype=torch.bfloat16).float().cpu().numpy()
    parity.assert_dequant_ok(dq, ot.dequant(pvo, P, ot.DEQUANT_PROD), bf16=True)


@pytest.mark.parametrize("b", [3, 4])
def test_long_context_decode_sampled(tq, b):
    """The benchmark's shapes (8 x 8 x 131072 keys and values): quantize and
    logits run in full on the GPU, checked on sampled keys and queries; the
    logits beat the bf16-key kernel's output in no way but agree with the
    oracle where the packed bytes agree."""
    batch, ctx, g = 8, 131072, 4
    K, V, Q = inputs.decode(batch, ctx)
    P = op.Params(128, b, 128, seed=0)
    T = tq.TurboQuant(128, b, 128, seed=0)
    dK = to_dev(K)
    pk = T.quantize(dK)
    n_sets = batch * 8
    qb = Q.all()
    qt = torch.from_numpy(qb.view(np.int16)).view(torch.bfloat16).cuda()
    lg = T.logits(qt, pk, n_sets, g, ctx)
    T.sync_status()
    rng = np.random.default_rng(b)
    idx = np.sort(rng.choice(K.n_rows, size=20000, replace=False))
    rep, want = sampled_quantize_check(P, K, pk, idx)
    # logits at the sampled keys, all 4 queries of their set
    got_codes = pk.codes[torch.from_numpy(idx).cuda()].cpu().numpy()
    got_signs = pk.signs[torch.from_numpy(idx).cuda()].cpu().numpy()
    same = np.all(got_codes == want["codes"], axis=1) & np.all(got_signs == want["signs"], axis=1)
    assert np.mean(~same) <= 1e-3
    sets, keys = idx // ctx, idx % ctx
    q = Q.as_f32(qb).astype(np.float64)
    yhat, z = ot.decode(want, P)
    q_rot, sq = ot.query_prep(q, P)
    lgn = lg.cpu().numpy()
    kn = np.linalg.norm(K.as_f32(K.take(idx)).astype(np.float64), axis=1)
    for j in range(g):
        qi = sets * g + j
        est = want["norm"] * np.sum(q_rot[qi] * yhat, axis=1) + \
            want["rnorm"] * (ot.SQRT_HALF_PI / P.m) * np.sum(sq[qi] * z, axis=1)
        gotj = lgn[sets, j, keys]
        tol = 1e-4 * np.linalg.norm(q[qi], axis=1) * kn
        ok = (np.abs(gotj - est) <= tol) | ~same
        assert ok.all()


@pytest.fixture(scope="module")
def prefill_keys():
    """The prefill workload's K (32 x 8 x 32768 bf16 rows), drawn once and kept
    on the device for the three bit widths."""
    K, _ = inputs.prefill()
    dK = to_dev(K)
    yield K, dK
    del dK
    torch.cuda.empty_cache()


@pytest.mark.parametrize("b", [2, 3, 4])
def test_prefill_write_path_sampled(tq, prefill_keys, b):
    """32 layers x 8 heads x 32768 tokens of bf16 keys with 1% of tokens x20,
    b in {2, 3, 4}: quantize all 8.4M rows of K, check 20000 sampled rows (a
    thousand of them from the x20 tokens)."""
    K, dK = prefill_keys
    P = op.Params(128, b, 128, seed=0)
    T = tq.TurboQuant(128, b, 128, seed=0)
    pk = T.quantize(dK)
    T.sync_status()
    rng = np.random.default_rng(4 + b)
    ctx = K.token_mask().size                     # the mask is per token, shared by every (layer, head)
    scaled = rng.choice(np.nonzero(K.token_mask())[0], size=1000) + ctx * rng.integers(0, K.n_rows // ctx, 1000)
    idx = np.sort(np.concatenate([rng.choice(K.n_rows, size=19000, replace=False), scaled]))
    sampled_quantize_check(P, K, pk, np.unique(idx))
    del pk
    T.close()


def test_vector_search_sampled(tq):
    """1e6 x 1024 fp32 unit rows, 1024 queries, b = 4, m = 1024: quantize the
    database, all-pairs estimates, top-10 per query.  Checked on sampled rows,
    sampled (query, key) pairs and the top-k kernel on sampled score rows."""
    db, qs = inputs.vector_search()
    d, b, m = 1024, 4, 1024
    P = op.Params(d, b, m, seed=0)
    T = tq.TurboQuant(d, b, m, seed=0)
    ddb = to_dev(db)
    pk = T.quantize(ddb)
    qf = qs.all()
    dq = torch.from_numpy(qf).cuda()
    scores = T.logits(dq, pk, 1, qs.n_rows, db.n_rows)
    idx_g, val_g = tq.topk(scores[0], 10)
    idx_s, val_s = T.search(dq, pk, db.n_rows, 10)     # top-10 fused into the estimates
    T.sync_status()
    # the fused search agrees with the top-10 of the written scores (its own
    # tensor-core pass: equal up to fp32 accumulation-order noise)
    sv, gv = val_s.cpu().numpy(), val_g.cpu().numpy()
    assert np.allclose(sv, gv, rtol=1e-5, atol=1e-6 * np.abs(gv).max())
    assert np.mean(idx_s.cpu().numpy() == idx_g.cpu().numpy()) >= 0.98
    rng = np.random.default_rng(5)
    ridx = np.sort(rng.choice(db.n_rows, size=1500, replace=False))
    rep, want = sampled_quantize_check(P, db, pk, ridx)
    got_codes = pk.codes[torch.from_numpy(ridx).cuda()].cpu().numpy()
    got_signs = pk.signs[torch.from_numpy(ridx).cuda()].cpu().numpy()
    same = np.all(got_codes == want["codes"], axis=1) & np.all(got_signs == want["signs"], axis=1)
    qsel = rng.choice(qs.n_rows, size=16, replace=False)
    est = ot.logits(qf[qsel].astype(np.float64), want, P, 1, 16, len(ridx))[0]
    gotq = scores[0][torch.from_numpy(qsel).cuda()][:, torch.from_numpy(ridx).cuda()].cpu().numpy()
    tol = 1e-4 * np.linalg.norm(qf[qsel], axis=1)[:, None] * np.linalg.norm(db.take(ridx), axis=1)[None, :]
    assert np.all((np.abs(gotq - est) <= tol) | ~same[None, :])
    # top-k: the kernel's answer on sampled score rows equals the oracle's top-k of those rows
    rows = scores[0][torch.from_numpy(qsel).cuda()].cpu().numpy()
    wi, wv = ot.topk(rows, 10)
    assert np.array_equal(idx_g[torch.from_numpy(qsel).cuda()].cpu().numpy(), wi)
    assert np.array_equal(val_g[torch.from_numpy(qsel).cuda()].cpu().numpy(), wv)
