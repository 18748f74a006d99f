"""GPU parity of fractional bit widths by a channel split (tq_split_*):
channels [0, d_hi) as one instance at b_hi bits, [d_hi, d) as another at
b_lo bits, against the oracle's split (oracle.turboquant.split_*).  The
parts run on the instances' own kernels (d = 128 tensor-core, wide-row and
general), reading and writing their columns of the caller's rows."""

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot
from tests import parity
from kv_cache_vector_15_b200 import inputs
from tests.test_gpu_parity import edge_rows, make_rows

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module")
def tq():
    from kv_cache_vector_15_b200 import tq as _tq
    return _tq


def split_rows(d, d_hi, n, dtype, seed, edge):
    """Random rows of mixed scale; row 0 is zero on part 0's channels only,
    row 1 on part 1's only; with ``edge`` the structured edge rows follow
    (left out where a part is zero-padded: padding puts whole groups of their
    rotated coordinates within the tie band, which the count rule flags)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) * rng.uniform(0.1, 10, size=(n, 1))
    x[0, :d_hi] = 0.0
    x[1, d_hi:] = 0.0
    if edge:
        x[2:8] = edge_rows(d, rng)
    x = x.astype(np.float32)
    if dtype == "bf16":
        bits = inputs.bf16_bits(x)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16), inputs.bf16_to_f32(bits)
    return torch.from_numpy(x), x


@pytest.mark.parametrize("d,d_hi,b_hi,b_lo,dtype,n", [
    (128, 64, 3, 2, "bf16", 2000),      # 2.5 bits per coordinate
    (128, 64, 4, 3, "f32", 2000),       # 3.5 bits
    (256, 128, 4, 3, "bf16", 3000),     # both parts on the d = 128 tensor-core kernels
    (96, 64, 3, 2, "f32", 778),         # 64 + 32 channels
    (160, 96, 3, 2, "bf16", 700),       # a part of 96 channels, zero-padded to 128
    (512, 256, 3, 2, "f32", 5000),      # parts on the wide-row write path, strided rows
])
def test_split_end_to_end(tq, d, d_hi, b_hi, b_lo, dtype, n):
    parts = ot.split_parts(d, d_hi, b_hi, b_lo, 0, op.Params)
    T = tq.TurboQuantSplit(d, d_hi, b_hi, b_lo, seed=0)
    assert T.bits_per_coordinate == (d_hi * b_hi + (d - d_hi) * b_lo) / d
    padded = any(P.d != dc for _, dc, P in parts)
    xt, x = split_rows(d, d_hi, n, dtype, seed=d + d_hi + b_hi, edge=not padded)
    got = T.quantize(xt.cuda())
    T.sync_status()
    want = ot.split_quantize(x, parts, keep_intermediates=True)
    for (_, _, P), g_p, w_p in zip(parts, got, want):
        parity.assert_quantize_ok(parity.compare_quantize(P, g_p.to_numpy(), w_p))
    # read half on the oracle's packed rows (byte-identical inputs on both sides)
    n_sets, g, n_keys = 2, 3, n // 2
    po = tuple({k: w_p[k] for k in ("codes", "signs", "norm", "rnorm")} for w_p in want)
    keys = tuple(tq.Packed.from_numpy(p) for p in po)
    qt, q = make_rows(d, n_sets * g, dtype, seed=d + 3)
    lg = T.logits(qt.cuda(), keys, n_sets, g, n_keys).cpu().numpy()
    T.sync_status()
    lw = ot.split_logits(q, po, parts, n_sets, g, n_keys)
    tol = parity.logit_tolerance(q, np.linalg.norm(x[:n_sets * n_keys], axis=1), n_sets, g, n_keys)
    assert np.all(np.abs(lg - lw) <= tol + 1e-30), float(np.max(np.abs(lg - lw) / (tol + 1e-30)))
    for mode in (tq.TQ_DEQUANT_PROD, tq.TQ_DEQUANT_MSE):
        want_dq = ot.split_dequant(po, parts, mode)
        dq = T.dequant(keys, out_dtype=torch.float32, mode=mode).cpu().numpy()
        assert dq.shape == (n_sets * n_keys, d)
        parity.assert_dequant_ok(dq, want_dq, bf16=False)
        # bf16 rows: 64-channel parts go through the tensor-core kernel, each
        # storing into its columns of the full rows
        dqb = T.dequant(keys, out_dtype=torch.bfloat16, mode=mode).float().cpu().numpy()
        parity.assert_dequant_ok(dqb, want_dq, bf16=True)


def test_split_argument_errors(tq):
    for bad in ((128, 48, 3, 2), (128, 128, 3, 2), (64, 16, 3, 2), (128, 64, 6, 2)):
        with pytest.raises(tq.TQError):
            tq.TurboQuantSplit(*bad)
