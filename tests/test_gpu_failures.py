"""Failure paths, provoked on the host (no GPU fault, no hang):

* a bounded device-side wait that runs out: a test setting shortens the wait
  limit of the d = 128 quantize kernel's tile loop to 100 SM clocks, so its
  first wait gives up; the kernel must wind down (drain its own MMAs and stage
  loads, free its tensor memory), write no results and leave an error that
  tq_sync_status reports; the next launch with the normal limit must run (it
  allocates all of the SM's tensor memory, so a leak would show) and match
  the oracle;
* the same for the warp-specialized logits kernel (every role gives up and
  winds down; the next launches reproduce the logits exactly);
* an injected device-allocation failure in tq_init (TQ_ERR_NOMEM, then a
  normal tq_init works);
* an injected launch failure (TQ_ERR_CUDA before anything is launched).
"""

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot
from tests import parity
from tests.test_gpu_parity import make_rows

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_15_b200 import tq as _tq
    yield _tq
    _tq.test_set(_tq.TQ_TEST_WAIT_LIMIT, 0)
    _tq.test_set(_tq.TQ_TEST_FAIL_ALLOC, 0)
    _tq.test_set(_tq.TQ_TEST_FAIL_LAUNCH, 0)
    _tq.test_set(_tq.TQ_TEST_FIXUP_CAP, 0)


@pytest.mark.parametrize("b", [3, 4])
def test_quantize_wait_runs_out_then_recovers(tq, b):
    d, m, n = 128, 128, 40000                       # 313 tiles: every CTA has several
    P = op.Params(d, b, m, seed=0)
    xt, x = make_rows(d, n, "bf16", seed=31)
    T = tq.TurboQuant(d, b, m, seed=0)
    xd = xt.cuda()
    out = T.empty_packed(n, "cuda")
    out.norm.fill_(-1.0)
    tq.test_set(tq.TQ_TEST_WAIT_LIMIT, 100)
    try:
        T.quantize(xd, out)
        with pytest.raises(tq.TQError) as e:
            T.sync_status()
        assert e.value.status == tq.TQ_ERR_CUDA
    finally:
        tq.test_set(tq.TQ_TEST_WAIT_LIMIT, 0)
    assert bool(torch.all(out.norm == -1.0)), "a CTA that gave up wrote results"
    T.sync_status()                                  # the error was reported once and cleared
    for _ in range(2):                               # normal limit: runs, frees and allocates TMEM again
        got = T.quantize(xd).to_numpy()
        T.sync_status()
    parity.assert_quantize_ok(parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True)))
    T.close()


@pytest.mark.parametrize("b", [3, 4])
def test_logits_wait_runs_out_then_recovers(tq, b):
    """The warp-specialized logits kernel (2 sets x 313 key tiles: every CTA's
    range within two sets) under the 100-clock limit: every role gives up,
    drains its own MMAs and copies, and the kernel frees its tensor memory; the
    error is reported once, and the next launches reproduce the logits bit for
    bit."""
    d, m, n_sets, g, n_keys = 128, 128, 2, 4, 40000
    T = tq.TurboQuant(d, b, m, seed=0)
    kt, _ = make_rows(d, n_sets * n_keys, "bf16", seed=41)
    qt, _ = make_rows(d, n_sets * g, "bf16", seed=42)
    keys = T.quantize(kt.cuda())
    qd = qt.cuda()
    want = T.logits(qd, keys, n_sets, g, n_keys).clone()
    T.sync_status()
    tq.test_set(tq.TQ_TEST_WAIT_LIMIT, 100)
    try:
        T.logits(qd, keys, n_sets, g, n_keys)
        with pytest.raises(tq.TQError) as e:
            T.sync_status()
        assert e.value.status == tq.TQ_ERR_CUDA
    finally:
        tq.test_set(tq.TQ_TEST_WAIT_LIMIT, 0)
    T.sync_status()
    for _ in range(2):
        got = T.logits(qd, keys, n_sets, g, n_keys)
        T.sync_status()
        assert torch.equal(got, want)
    T.close()


def test_injected_allocation_failure(tq):
    tq.test_set(tq.TQ_TEST_FAIL_ALLOC, 1)
    with pytest.raises(tq.TQError) as e:
        tq.TurboQuant(128, 3, 128, seed=0)
    assert e.value.status == tq.TQ_ERR_NOMEM
    T = tq.TurboQuant(128, 3, 128, seed=0)           # the injection was used up
    T.close()


def test_injected_launch_failure(tq):
    T = tq.TurboQuant(128, 3, 128, seed=0)
    xt, x = make_rows(128, 300, "bf16", seed=3)
    xd = xt.cuda()
    tq.test_set(tq.TQ_TEST_FAIL_LAUNCH, 1)
    before = tq.launch_count()
    with pytest.raises(tq.TQError) as e:
        T.quantize(xd)
    assert e.value.status == tq.TQ_ERR_CUDA
    assert tq.launch_count() == before
    P = op.Params(128, 3, 128, seed=0)
    got = T.quantize(xd).to_numpy()
    T.sync_status()
    parity.assert_quantize_ok(parity.compare_quantize(P, got, ot.quantize(x, P, keep_intermediates=True)))
    T.close()


@pytest.mark.parametrize("b", [3, 4])
def test_quantize_fixup_overflow_path(tq, b):
    """The d = 128 quantize kernel lists projections inside its tensor-core
    error bound for an exact fp64 fix-up; with the list capped at one entry
    almost every such row takes the overflow path (all its signs recomputed).
    Both paths must give the oracle's signs."""
    d, m, n = 128, 128, 60000
    P = op.Params(d, b, m, seed=0)
    xt, x = make_rows(d, n, "bf16", seed=41 + b)
    T = tq.TurboQuant(d, b, m, seed=0)
    xd = xt.cuda()
    want = ot.quantize(x, P, keep_intermediates=True)
    tq.test_set(tq.TQ_TEST_FIXUP_CAP, 1)
    try:
        got = T.quantize(xd).to_numpy()
        T.sync_status()
    finally:
        tq.test_set(tq.TQ_TEST_FIXUP_CAP, 0)
    parity.assert_quantize_ok(parity.compare_quantize(P, got, want))
    got2 = T.quantize(xd).to_numpy()
    T.sync_status()
    parity.assert_quantize_ok(parity.compare_quantize(P, got2, want))
    assert all(np.array_equal(got[k], got2[k]) for k in ("codes", "signs"))
    T.close()
