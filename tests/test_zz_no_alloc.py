"""The allocation-free logit entry point (tq_logits_noalloc).

It serves callers that cannot allocate device memory where they call: the
per-query operands go to a scratch array built into the library instead of a
caller workspace.  This file is collected last, so a run that stops at the
first failure has already run every other test; it also passes on its own in a
fresh process.
"""

import numpy as np
import pytest

from kv_cache_vector_15_b200 import inputs
from oracle import params as op
from oracle import turboquant as ot
from tests import parity

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _case(d, b, m, n_sets, g, n_keys, seed):
    P = op.Params(d, b, m, seed=0)
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((n_sets * n_keys, d)) * rng.uniform(0.1, 10, size=(n_sets * n_keys, 1))
    qbits = inputs.bf16_bits(rng.standard_normal((n_sets * g, d)).astype(np.float32))
    return P, k, ot.quantize(k, P), qbits, inputs.bf16_to_f32(qbits)


@pytest.mark.parametrize("d,b,m,n_sets,g,n_keys", [(128, 3, 128, 6, 4, 3001), (128, 4, 128, 2, 16, 999),
                                                   (256, 3, 64, 3, 2, 1500)])
def test_noalloc_matches_workspace_call_twice(d, b, m, n_sets, g, n_keys):
    from kv_cache_vector_15_b200 import tq
    P, k, pk, qbits, q = _case(d, b, m, n_sets, g, n_keys, seed=d + g)
    T = tq.TurboQuant(d, b, m, seed=0)
    keys = tq.Packed.from_numpy(pk)
    qt = torch.from_numpy(qbits.view(np.int16)).view(torch.bfloat16).cuda()
    ref = T.logits(qt, keys, n_sets, g, n_keys).cpu().numpy()      # caller-provided workspace
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    for _ in range(2):                                              # the scratch keeps old contents
        out = torch.full((n_sets, g, n_keys), float("nan"), device="cuda")
        T.logits_noalloc(qt, keys, n_sets, g, n_keys, out)
        T.sync_status()
        got = out.cpu().numpy()
        assert np.all(np.abs(got - ref) <= tol + 1e-30)
    want = ot.logits(q, pk, P, n_sets, g, n_keys)
    assert np.all(np.abs(got - want) <= tol + 1e-30)


def test_noalloc_on_wide_rows_allocates_nothing():
    """d = m = 256, g = 64, 4096 keys: tq_logits takes the wide-row GEMM path
    (keys decoded into a workspace operand); the allocation-free call runs the
    general kernels on the packed keys instead.  Its results agree with
    tq_logits' within the logit tolerance, and the device's free memory does not
    move across the call (the first call loads the kernels' code, so the second
    one is measured)."""
    from kv_cache_vector_15_b200 import tq
    d, b, m, n_sets, g, n_keys = 256, 3, 256, 1, 64, 4096
    P, k, pk, qbits, q = _case(d, b, m, n_sets, g, n_keys, seed=5)
    T = tq.TurboQuant(d, b, m, seed=0)
    assert T.workspace_bytes(n_sets, g, n_keys) > n_sets * g * (d + m) * 4      # the GEMM operands
    keys = tq.Packed.from_numpy(pk)
    qt = torch.from_numpy(qbits.view(np.int16)).view(torch.bfloat16).cuda()
    ref = T.logits(qt, keys, n_sets, g, n_keys).cpu().numpy()
    tol = parity.logit_tolerance(q, np.linalg.norm(k, axis=1), n_sets, g, n_keys)
    out = torch.full((n_sets, g, n_keys), float("nan"), device="cuda")
    T.logits_noalloc(qt, keys, n_sets, g, n_keys, out)
    T.sync_status()
    out.fill_(float("nan"))
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    T.logits_noalloc(qt, keys, n_sets, g, n_keys, out)
    T.sync_status()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    got = out.cpu().numpy()
    assert np.all(np.abs(got - ref) <= 2 * tol + 1e-30)
    want = ot.logits(q, pk, P, n_sets, g, n_keys)
    assert np.all(np.abs(got - want) <= tol + 1e-30)
    T.close()


def test_noalloc_checks_like_tq_logits():
    """An empty call is a no-op even when n_sets * g would not fit the array;
    a NULL context is refused before anything else."""
    from kv_cache_vector_15_b200 import tq
    T = tq.TurboQuant(1024, 4, 1024, seed=0)
    keys = T.empty_packed(8)
    q = torch.zeros((600, 1024), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, 600, 8), device="cuda")
    before = tq.launch_count()
    T.logits_noalloc(q, keys, 1, 600, 0, out)                      # n_keys = 0: TQ_OK, nothing launched
    assert tq.launch_count() == before
    st = tq.call_status("tq_logits_noalloc", None, q.data_ptr(), tq.TQ_BF16, 1, 600, keys.c(), 8, out.data_ptr(),
                        None)
    assert st == tq.TQ_ERR_INVALID_ARG
    T.close()


def test_noalloc_rejects_oversized_requests_without_launching():
    from kv_cache_vector_15_b200 import tq
    T = tq.TurboQuant(1024, 4, 1024, seed=0)
    keys = T.empty_packed(8)
    q = torch.zeros((600, 1024), dtype=torch.bfloat16, device="cuda")   # 600 * 2048 * 4 B > 4 MiB
    out = torch.empty((1, 600, 8), device="cuda")
    before = tq.launch_count()
    with pytest.raises(tq.TQError) as e:
        T.logits_noalloc(q, keys, 1, 600, 8, out)
    assert e.value.status == tq.TQ_ERR_UNSUPPORTED
    assert tq.launch_count() == before
