"""Multi-rank host logic on the CPU (gloo, world size 2).

The data-parallel split has no collective on the data path, so what needs
checking is the bookkeeping: the shards are disjoint, cover the global batch,
and each rank draws exactly the rows the single-process job would; the per-rank
results (here from the oracle, standing in for the kernels) put together equal
the single-process result; and the timing reductions (max of device times, sum
of units) combine the ranks as the bench reports them.
"""

import os
import socket

import numpy as np
import pytest

from kv_cache_vector_15_b200 import dist as du
from kv_cache_vector_15_b200 import inputs

torch = pytest.importorskip("torch")


def test_shard_covers_and_balances():
    for n in (0, 1, 7, 64, 1001):
        for ws in (1, 2, 3, 8):
            parts = [du.shard(n, ws, r) for r in range(ws)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(ws - 1))
            sizes = [hi - lo for lo, hi in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        du.shard(10, 2, 2)
    with pytest.raises(ValueError):
        du.shard(-1, 2, 0)


def test_decode_shard_rows():
    sh = du.decode_shard(3, 4, 2, kv_heads=8, q_heads=32, ctx=1000)
    assert sh.global_batch == 12 and (sh.seq_lo, sh.seq_hi) == (6, 9)
    assert sh.kv_rows == (6 * 8 * 1000, 9 * 8 * 1000)
    assert sh.q_rows == (6 * 32, 9 * 32)
    assert sh.n_sets == 24
    with pytest.raises(ValueError):
        du.decode_shard(1, 2, 0, kv_heads=3, q_heads=4, ctx=10)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# small decode: 2 sequences x 2 kv heads x 96 tokens, 4 query heads (g = 2), d = 32
KV, QH, CTX, D, BITS, M = 2, 4, 96, 32, 3, 32


def _oracle_step(k_bits, v_bits, q_bits, n_sets, g):
    from oracle import params as op
    from oracle import turboquant as ot
    P = op.Params(D, BITS, M, seed=0)
    f = inputs.bf16_to_f32
    pk = ot.quantize(f(k_bits).astype(np.float64), P)
    pv = ot.quantize(f(v_bits).astype(np.float64), P)
    lg = ot.logits(f(q_bits).astype(np.float64), pk, P, n_sets, g, CTX)
    dq = ot.dequant(pv, P, ot.DEQUANT_PROD)
    return pk, lg, dq


def _rank_main(rank, ws, port, out_path):
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sh = du.decode_shard(1, ws, rank, kv_heads=KV, q_heads=QH, ctx=CTX)
        K, V, Q = inputs.decode(sh.global_batch, CTX, kv_heads=KV, q_heads=QH, d=D)
        g = QH // KV
        k = np.empty((sh.kv_rows[1] - sh.kv_rows[0], D), np.uint16)
        v = np.empty_like(k)
        q = np.empty((sh.q_rows[1] - sh.q_rows[0], D), np.uint16)
        K.fill(k, start=sh.kv_rows[0])
        V.fill(v, start=sh.kv_rows[0])
        Q.fill(q, start=sh.q_rows[0])
        pk, lg, dq = _oracle_step(k, v, q, sh.n_sets, g)
        du.barrier(ws)
        t_max = du.max_over_ranks(ws, 1.0 + rank)
        units = du.sum_over_ranks(ws, sh.n_sets * g * CTX)
        parts = [None] * ws
        dist.all_gather_object(parts, (rank, k, q, pk, lg, dq))
        if rank == 0:
            # the single-process job over the whole global batch
            kw, vw, qw = K.all(), V.all(), Q.all()
            n_sets_w = sh.global_batch * KV
            pkw, lgw, dqw = _oracle_step(kw, vw, qw, n_sets_w, g)
            parts.sort(key=lambda p: p[0])
            assert np.array_equal(np.concatenate([p[1] for p in parts]), kw)
            assert np.array_equal(np.concatenate([p[2] for p in parts]), qw)
            for key in ("codes", "signs", "norm", "rnorm"):
                assert np.array_equal(np.concatenate([p[3][key] for p in parts]), pkw[key]), key
            assert np.array_equal(np.concatenate([p[4] for p in parts]), lgw)
            assert np.array_equal(np.concatenate([p[5] for p in parts]), dqw)
            assert t_max == float(ws)
            assert units == n_sets_w * g * CTX
            with open(out_path, "w") as f:
                f.write("ok")
        du.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_single_process(tmp_path):
    import torch.multiprocessing as mp
    out = tmp_path / "result.txt"
    mp.start_processes(_rank_main, args=(2, _free_port(), str(out)), nprocs=2, join=True,
                       start_method="spawn")
    assert out.read_text() == "ok"
