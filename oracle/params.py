"""Oracle: the method's fixed parameters (test infrastructure only).

Three things are drawn or fitted once per ``(d, b, m, seed)``:

* D -- the Rademacher diagonal of the randomized Hadamard rotation
  R = H_d * D / sqrt(d)  [0h-n0.github.io "ICLR 2026論文解説: TurboQuant",
  section "Step 1: PolarQuant" (RHT definition: D has independent +-1 entries
  with equal probability)];
* S -- the m x d Gaussian projection of QJL  [Qiita TurboQuant explainer
  (qiita.com/kai_kou), section "Stage 2: QJL": a random projection matrix S,
  m projections];
* the (b-1)-bit Lloyd-Max codebook (centroids and thresholds) fitted to the
  law of one rotated coordinate  [Qiita explainer, "Stage 1: PolarQuant",
  step 3 "Lloyd-Max quantization"; ai.spot.hk "Google TurboQuant: LLM KV Cache
  壓縮 6 倍", section "隨機旋轉與Beta分佈" (each rotated coordinate follows a
  concentrated Beta law and one scalar quantizer serves all coordinates)].

Readings taken where the pages are silent:

* Random numbers come from SplitMix64 (Steele, Lea & Flood 2014; Vigna's
  public-domain definition) used counter-style: output(seed, stream, i) is the
  SplitMix64 finalizer applied to seed + (stream * 2**40 + i + 1) * GOLDEN.
  Stream 0 feeds D (D_i = +1 if bit 0 of output i is 0, else -1), stream 1
  feeds S.
* S_{j,i} is one Box-Muller normal sqrt(-2 ln u1) * cos(2 pi u2) from the
  53-bit uniforms of counters 2(j d + i) and 2(j d + i) + 1, u1 taken in
  (0, 1].  The fp64 draw is rounded once, round-to-nearest-even, to IEEE
  binary16; that binary16 value *is* S, on both sides.
* The coordinate law is the exact one for a uniformly random unit vector in
  R^d: f_d(x) = C_d (1 - x^2)^((d-3)/2) on (-1, 1), i.e. (1 + X)/2 ~
  Beta((d-1)/2, (d-1)/2).  Its large-d limit is N(0, 1/d)  [0h-n0 explainer,
  "Step 1: PolarQuant" (Beta law tending to N(0, 1/d))].
* Thresholds are the midpoints of adjacent fp64 centroids; both are then
  rounded to fp32, which is the precision the kernels compare and look up in.
"""

from __future__ import annotations

import functools
import math

import numpy as np
from scipy.special import betaincc, gammaln

GOLDEN = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
STREAM_SHIFT = 40
STREAM_D = 0
STREAM_S = 1


# --------------------------------------------------------------------------
# SplitMix64, counter style
# --------------------------------------------------------------------------
def splitmix64(seed: int, counters) -> np.ndarray:
    """SplitMix64 output for each counter value: the generator's state after
    ``counter + 1`` increments by the golden gamma, passed through its
    finalizer (xor-shift 30, multiply, xor-shift 27, multiply, xor-shift 31).
    All arithmetic is modulo 2**64 (numpy uint64 wraps)."""
    c = np.asarray(counters, dtype=np.uint64)
    if np.ndim(seed) == 0:
        s = np.uint64(int(seed) & 0xFFFFFFFFFFFFFFFF)
    else:                                   # an array of seeds broadcasts against the counters
        s = np.asarray(seed, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = s + (c + np.uint64(1)) * np.uint64(GOLDEN)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(_MIX1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(_MIX2)
        z = z ^ (z >> np.uint64(31))
    return z


def stream_counters(stream: int, n: int) -> np.ndarray:
    return (np.uint64(stream) << np.uint64(STREAM_SHIFT)) + np.arange(n, dtype=np.uint64)


def uniform53(bits: np.ndarray) -> np.ndarray:
    """Top 53 bits of each word scaled by 2**-53: a uniform in [0, 1)."""
    return (bits >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


# --------------------------------------------------------------------------
# D and S
# --------------------------------------------------------------------------
def rademacher_diagonal(d: int, seed) -> np.ndarray:
    """D_i in {+1, -1}: +1 when bit 0 of stream-0 output i is clear.
    ``seed`` may be a 1-D array of seeds (result shape (n_seeds, d))."""
    ctr = stream_counters(STREAM_D, d)
    if np.ndim(seed) == 0:
        words = splitmix64(seed, ctr)
    else:
        words = splitmix64(np.asarray(seed, dtype=np.uint64)[:, None], ctr[None, :])
    bits = words & np.uint64(1)
    return np.where(bits == 0, 1, -1).astype(np.int8)


def round_to_binary16(v: np.ndarray) -> np.ndarray:
    """Round fp64 values once, to nearest with ties to even, onto the IEEE
    binary16 grid; returns the rounded values as fp64.

    Normal range: spacing 2**(e - 10) for |v| in [2**e, 2**(e+1)), e >= -14.
    Subnormal range (|v| < 2**-14): fixed spacing 2**-24.  Values are far
    inside the finite range here (|S| < 40), so overflow is not handled."""
    v = np.asarray(v, dtype=np.float64)
    mant, ex = np.frexp(np.abs(v))          # |v| = mant * 2**ex, mant in [0.5, 1)
    e = ex.astype(np.int64) - 1             # |v| in [2**e, 2**(e+1))
    e = np.maximum(e, -14)                  # subnormals share the 2**-24 spacing
    spacing = np.ldexp(1.0, (e - 10).astype(np.int64))
    return np.round(v / spacing) * spacing  # v / spacing is exact; np.round is half-to-even


def gaussian_projection(m: int, d: int, seed) -> np.ndarray:
    """S in R^{m x d}: Box-Muller normals from stream 1, rounded to binary16.
    Returned as fp64 holding the exact binary16 values.  ``seed`` may be a
    1-D array of seeds, giving one S per seed, shape (n_seeds, m, d)."""
    n = m * d
    ctr = stream_counters(STREAM_S, 2 * n)
    if np.ndim(seed) == 0:
        words = splitmix64(seed, ctr)
    else:
        words = splitmix64(np.asarray(seed, dtype=np.uint64)[:, None], ctr[None, :])
    u = uniform53(words)
    u1 = 1.0 - u[..., 0::2]                 # in (0, 1]
    u2 = u[..., 1::2]
    g = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return round_to_binary16(g).reshape(np.shape(g)[:-1] + (m, d))


# --------------------------------------------------------------------------
# Lloyd-Max codebook for the rotated-coordinate law
# --------------------------------------------------------------------------
def coordinate_density(x, d: int):
    """f_d(x) = C_d (1 - x^2)^((d-3)/2), C_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    k = (d - 3) / 2.0
    logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    x = np.asarray(x, dtype=np.float64)
    return np.exp(logc + k * np.log1p(-x * x))


def upper_tail(x, d: int):
    """P(X > x) for X ~ f_d, via (1 + X)/2 ~ Beta((d-1)/2, (d-1)/2)."""
    a = (d - 1) / 2.0
    return betaincc(a, a, (1.0 + np.asarray(x, dtype=np.float64)) / 2.0)


def partial_first_moment(lo, hi, d: int):
    """Integral of x f_d(x) over (lo, hi), in closed form:
    C_d [(1 - lo^2)^(k+1) - (1 - hi^2)^(k+1)] / (2 (k + 1)),  k = (d-3)/2."""
    k = (d - 3) / 2.0
    logc = gammaln(d / 2.0) - 0.5 * math.log(math.pi) - gammaln((d - 1) / 2.0)
    lo = np.asarray(lo, dtype=np.float64)
    hi = np.asarray(hi, dtype=np.float64)
    return np.exp(logc) * (np.power(1.0 - lo * lo, k + 1) - np.power(1.0 - hi * hi, k + 1)) / (2.0 * (k + 1))


@functools.lru_cache(maxsize=None)
def lloyd_max_cached(d: int, bits_mse: int):
    c, t, it = lloyd_max(d, bits_mse)
    c.setflags(write=False)
    t.setflags(write=False)
    return c, t, it


def lloyd_max(d: int, bits_mse: int, tol: float = 1e-15, max_iter: int = 200000, patience: int = 200):
    """Lloyd-Max quantizer with L = 2**bits_mse levels for X ~ f_d.

    Lloyd's two conditions, iterated: thresholds are midpoints of adjacent
    centroids, centroids are conditional means E[X | cell].  f_d is symmetric
    and log-concave, so the fixed point is unique and symmetric; the
    iteration runs on the positive half (cells (0, t_1], ..., (t_{h-1}, 1))
    and mirrors.  It stops when a step moves no centroid by more than
    ``tol`` relative to the outermost one, or when the step size has not
    reached a new minimum for ``patience`` iterations (the rounding floor of
    the incomplete-beta evaluation, about 1e-13 relative at d >= 1024).
    Returns fp64 (centroids ascending, thresholds ascending, iterations)."""
    L = 1 << bits_mse
    h = L // 2
    # initial positive centroids spread over about 3 standard deviations
    p = (np.arange(h) + 0.5) * (3.0 / h) / math.sqrt(d)
    it = 0
    best, since_best = np.inf, 0
    while True:
        edges = np.concatenate([[0.0], 0.5 * (p[:-1] + p[1:]), [1.0]])
        tail = upper_tail(edges, d)
        mass = tail[:-1] - tail[1:]
        newp = partial_first_moment(edges[:-1], edges[1:], d) / mass
        it += 1
        delta = np.max(np.abs(newp - p))
        p = newp
        if delta < best:
            best, since_best = delta, 0
        else:
            since_best += 1
        if delta <= tol * p[-1] or since_best >= patience or it >= max_iter:
            break
    centroids = np.concatenate([-p[::-1], p])
    thresholds = 0.5 * (centroids[:-1] + centroids[1:])
    thresholds[h - 1] = 0.0                      # exact by symmetry
    return centroids, thresholds, it


def mse_distortion(d: int, centroids: np.ndarray) -> float:
    """Total distortion D_B = E||u - Q(u)||^2 = d E[(X - Q(X))^2] for the
    given (symmetric, Lloyd-optimal) codebook, with midpoint cells:
    E[(X - Q(X))^2] = E[X^2] - sum_cells P(cell) c^2 and E[X^2] = 1/d."""
    c = np.asarray(centroids, dtype=np.float64)
    edges = np.concatenate([[-1.0], 0.5 * (c[:-1] + c[1:]), [1.0]])
    tail = upper_tail(edges, d)
    mass = tail[:-1] - tail[1:]
    return float(d * (1.0 / d - np.sum(mass * c * c)))


class Params:
    """All fixed parameters of one (d, b, m, seed) instance.

    Attributes (fp64 arrays holding exactly the values the kernels use):
      D            (d,)    int8 +-1
      S            (m, d)  binary16 values
      centroids    (L,)    fp32 values, ascending
      thresholds   (L-1,)  fp32 values, ascending
      R            (d, d)  dense H_d diag(D) / sqrt(d), fp64
    """

    def __init__(self, d: int, b: int, m: int, seed: int = 0):
        if d < 2 or d & (d - 1):
            raise ValueError("d must be a power of two")
        if not 2 <= b <= 5:
            raise ValueError("b must be in [2, 5]")
        self.d, self.b, self.m, self.seed = d, b, m, seed
        self.B = b - 1
        self.L = 1 << self.B
        self.D = rademacher_diagonal(d, seed)
        self.S = gaussian_projection(m, d, seed)
        c64, t64, self.lloyd_iterations = lloyd_max_cached(d, self.B)
        self.centroids64, self.thresholds64 = c64, t64
        self.centroids = c64.astype(np.float32).astype(np.float64)
        self.thresholds = t64.astype(np.float32).astype(np.float64)
        from .turboquant import rotation_matrix
        self.R = rotation_matrix(self.D)
