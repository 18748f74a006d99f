"""Seeded synthetic workloads (no arithmetic of the method lives here).

This module only draws inputs.  Both the kernel tests and the oracle tests
read their inputs from here, so the two sides see byte-identical data.  Every
tensor is generated in blocks of ``BLOCK`` rows, block k of tensor t from
``numpy.random.default_rng([seed, t, k])``, so that any row range can be
re-drawn on its own (the full-size parity tests sample rows this way).

bf16 tensors are returned as their uint16 bit patterns (numpy has no bf16);
``bf16_to_f32`` widens them exactly.

Workloads (d = 128 unless stated):

* ``single_head``  -- 4096 fp32 keys N(0,1), 4 outlier channels (picked by
  the generator) scaled x10; 16 fp32 queries N(0,1).
* ``decode``       -- bf16 K and V [batch, 8 kv heads, ctx, 128], entries
  N(0,1) times a per-(kv head, channel) scale drawn log-uniform in [0.1, 10]
  (separately for K and V); bf16 queries [batch, 32 heads, 128] N(0,1).
  Llama-3.1-8B-shaped decode is batch 1, ctx 8192; the long-context case is
  batch 8, ctx 131072.
* ``prefill``      -- bf16 K and V [32 layers, 8 heads, 32768 tokens, 128]
  N(0,1), with one shared mask of 1% of tokens scaled x20.
* ``vector_search``-- 1,000,000 fp32 unit-norm rows in d = 1024: a mixture of
  256 clusters, centres N(0, I/d) normalised, points centre + 0.3 N(0, I/d)
  normalised; 1024 queries from the same mixture.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

BLOCK = 65536


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u                      # finite inputs: no wrap below the NaN range
    r >>= np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _block_normal(seed: int, tensor: int, k: int, d: int) -> np.ndarray:
    return np.random.default_rng([seed, tensor, k]).standard_normal((BLOCK, d), dtype=np.float32)


@dataclass(frozen=True)
class RowTensor:
    """A seeded [n_rows, d] tensor of normal rows with optional structure.

    kind: "normal" | "scaled" (per head/channel scale) | "tokmask" (token
    mask x scale) | "mixture" (unit-norm cluster mixture)."""

    seed: int
    tensor: int
    n_rows: int
    d: int
    dtype: str = "bf16"            # "bf16" or "f32"
    kind: str = "normal"
    heads: int = 1
    ctx: int = 1
    mask_frac: float = 0.0
    mask_scale: float = 1.0
    n_clusters: int = 0
    cluster_std: float = 0.0
    outlier_channels: int = 0
    outlier_scale: float = 1.0

    # -- structure parameters, each from its own generator ----------------
    def channel_scales(self) -> np.ndarray:
        rng = np.random.default_rng([self.seed, self.tensor, 1 << 31])
        return np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(self.heads, self.d))).astype(np.float32)

    def token_mask(self) -> np.ndarray:
        rng = np.random.default_rng([self.seed, 1 << 20, 1 << 31])   # shared by K, V, layers, heads
        n = int(round(self.mask_frac * self.ctx))
        mask = np.zeros(self.ctx, dtype=bool)
        mask[rng.choice(self.ctx, size=n, replace=False)] = True
        return mask

    def centres(self) -> np.ndarray:
        rng = np.random.default_rng([self.seed, 1 << 21, 1 << 31])   # shared by database and queries
        c = rng.standard_normal((self.n_clusters, self.d)) / np.sqrt(self.d)
        return (c / np.linalg.norm(c, axis=1, keepdims=True)).astype(np.float32)

    def outliers(self) -> np.ndarray:
        rng = np.random.default_rng([self.seed, self.tensor, (1 << 31) + 2])
        return np.sort(rng.choice(self.d, size=self.outlier_channels, replace=False))

    # -- rows --------------------------------------------------------------
    def _block(self, k: int) -> np.ndarray:
        x = _block_normal(self.seed, self.tensor, k, self.d)
        r0 = k * BLOCK
        rows = np.arange(r0, r0 + BLOCK)
        if self.kind == "scaled":
            head = (rows // self.ctx) % self.heads
            x *= self.channel_scales()[head]
        elif self.kind == "tokmask":
            x[self.token_mask()[rows % self.ctx]] *= np.float32(self.mask_scale)
        elif self.kind == "mixture":
            rng = np.random.default_rng([self.seed, self.tensor, k, 7])
            cid = rng.integers(0, self.n_clusters, size=BLOCK)
            x = self.centres()[cid] + np.float32(self.cluster_std / np.sqrt(self.d)) * x
            x /= np.linalg.norm(x, axis=1, keepdims=True)
        if self.outlier_channels:
            x[:, self.outliers()] *= np.float32(self.outlier_scale)
        return x

    def rows(self, start: int, stop: int) -> np.ndarray:
        """Rows [start, stop) as uint16 bf16 bits or fp32."""
        stop = min(stop, self.n_rows)
        out = []
        k0, k1 = start // BLOCK, (stop - 1) // BLOCK
        for k in range(k0, k1 + 1):
            blk = self._block(k)
            lo = max(start, k * BLOCK) - k * BLOCK
            hi = min(stop, (k + 1) * BLOCK) - k * BLOCK
            out.append(blk[lo:hi])
        x = np.concatenate(out, axis=0) if out else np.zeros((0, self.d), np.float32)
        return bf16_bits(x) if self.dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)

    def take(self, idx) -> np.ndarray:
        """Rows at arbitrary indices (re-drawing only the blocks they fall in)."""
        idx = np.asarray(idx, dtype=np.int64)
        out = np.empty((idx.size, self.d), dtype=np.uint16 if self.dtype == "bf16" else np.float32)
        for k in np.unique(idx // BLOCK):
            sel = np.nonzero(idx // BLOCK == k)[0]
            blk = self.rows(int(k) * BLOCK, int(k + 1) * BLOCK)
            out[sel] = blk[idx[sel] - int(k) * BLOCK]
        return out

    def all(self) -> np.ndarray:
        return self.rows(0, self.n_rows)

    def fill(self, out: np.ndarray, threads: int = 0, start: int = 0) -> np.ndarray:
        """Write rows [start, start + len(out)) into ``out`` (uint16 for bf16,
        fp32 otherwise) block by block on a thread pool; the same values as
        rows(start, start + len(out)).  With start = 0 and len(out) = n_rows
        this is all()."""
        import concurrent.futures as cf
        import os
        stop = start + out.shape[0]
        if start < 0 or stop > self.n_rows:
            raise ValueError(f"rows [{start}, {stop}) outside [0, {self.n_rows})")
        threads = threads or min(32, os.cpu_count() or 1)
        cuts = list(range(start, stop, BLOCK)) if start % BLOCK == 0 else \
            [start] + list(range((start // BLOCK + 1) * BLOCK, stop, BLOCK))

        def one(lo):
            hi = min(stop, (lo // BLOCK + 1) * BLOCK)
            out[lo - start:hi - start] = self.rows(lo, hi)

        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, cuts))
        return out

    def as_f32(self, rows: np.ndarray) -> np.ndarray:
        return bf16_to_f32(rows) if self.dtype == "bf16" else rows


# ------------------------------------------------------------------------
# Named workloads
# ------------------------------------------------------------------------
def single_head(seed: int = 0):
    keys = RowTensor(seed, 10, 4096, 128, dtype="f32", outlier_channels=4, outlier_scale=10.0)
    queries = RowTensor(seed, 11, 16, 128, dtype="f32")
    return keys, queries


def decode(batch: int, ctx: int, seed: int = 0, kv_heads: int = 8, q_heads: int = 32, d: int = 128):
    n = batch * kv_heads * ctx
    K = RowTensor(seed, 20, n, d, kind="scaled", heads=kv_heads, ctx=ctx)
    V = RowTensor(seed, 21, n, d, kind="scaled", heads=kv_heads, ctx=ctx)
    Q = RowTensor(seed, 22, batch * q_heads, d)
    return K, V, Q


def prefill(seed: int = 0, layers: int = 32, heads: int = 8, ctx: int = 32768, d: int = 128):
    n = layers * heads * ctx
    K = RowTensor(seed, 40, n, d, kind="tokmask", ctx=ctx, mask_frac=0.01, mask_scale=20.0)
    V = RowTensor(seed, 41, n, d, kind="tokmask", ctx=ctx, mask_frac=0.01, mask_scale=20.0)
    return K, V


def vector_search(seed: int = 0, n: int = 1_000_000, n_queries: int = 1024, d: int = 1024):
    db = RowTensor(seed, 50, n, d, dtype="f32", kind="mixture", n_clusters=256, cluster_std=0.3)
    q = RowTensor(seed, 51, n_queries, d, dtype="f32", kind="mixture", n_clusters=256, cluster_std=0.3)
    return db, q
