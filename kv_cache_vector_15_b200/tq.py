"""Thin ctypes binding of libtq (include/tq.h).

Argument marshalling only: every step of the method runs inside libtq's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.  If
libtq.so is missing or cannot be loaded this module raises at import time;
there is no fallback path.
"""

from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("TQ_LIB", os.path.join(_HERE, "libtq.so"))

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtq.so not found at {LIB_PATH}; build it with `python -m kv_cache_vector_15_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_NOMEM, TQ_ERR_CUDA = range(5)
TQ_BF16, TQ_F32 = 0, 1
TQ_DEQUANT_PROD, TQ_DEQUANT_MSE = 0, 1
TQ_TEST_WAIT_LIMIT, TQ_TEST_FAIL_ALLOC, TQ_TEST_FAIL_LAUNCH, TQ_TEST_FIXUP_CAP = 0, 1, 2, 3

# exported symbols, in header order
SYMBOLS = [
    "tq_host_params", "tq_init", "tq_destroy", "tq_packed_sizes", "tq_get_params", "tq_quantize_workspace_bytes",
    "tq_quantize", "tq_logits_workspace_bytes", "tq_logits", "tq_logits_noalloc", "tq_dequant", "tq_topk", "tq_logits_bf16",
    "tq_status_str", "tq_sync_status", "tq_last_error", "tq_launch_count", "tq_attention_workspace_bytes",
    "tq_attention", "tq_quantize_scatter", "tq_search_workspace_bytes", "tq_search", "tq_split_init",
    "tq_split_destroy", "tq_split_part", "tq_split_quantize_workspace_bytes", "tq_split_quantize",
    "tq_split_logits_workspace_bytes", "tq_split_logits",
    "tq_split_dequant", "tq_test_set",
]


class _Packed(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("signs", ctypes.c_void_p), ("norm", ctypes.c_void_p),
                ("rnorm", ctypes.c_void_p)]


_vp, _i32, _i64, _u64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
_sig = {
    "tq_host_params": (_i32, [_i32, _i32, _i32, _u64, _vp, _vp, _vp, _vp]),
    "tq_init": (_i32, [_i32, _i32, _i32, _u64, ctypes.POINTER(_vp)]),
    "tq_destroy": (_i32, [_vp]),
    "tq_packed_sizes": (_i32, [_vp, _i64, ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "tq_get_params": (_i32, [_vp, _vp, _vp, _vp, _vp]),
    "tq_quantize_workspace_bytes": (_sz, [_vp, _i64]),
    "tq_quantize": (_i32, [_vp, _vp, _i32, _i64, _i64, _Packed, _vp, _sz, _vp]),
    "tq_quantize_scatter": (_i32, [_vp, _vp, _i32, _i64, _i64, _vp, _i64, _Packed, _vp]),
    "tq_logits_workspace_bytes": (_sz, [_vp, _i64, _i32, _i64]),
    "tq_logits": (_i32, [_vp, _vp, _i32, _i64, _i32, _Packed, _i64, _vp, _vp, _sz, _vp]),
    "tq_logits_noalloc": (_i32, [_vp, _vp, _i32, _i64, _i32, _Packed, _i64, _vp, _vp]),
    "tq_dequant": (_i32, [_vp, _Packed, _i64, _vp, _i32, _i32, _vp]),
    "tq_attention_workspace_bytes": (_sz, [_vp, _i64, _i32, _i64]),
    "tq_attention": (_i32, [_vp, _vp, _i32, _i64, _i32, _Packed, _Packed, _i64, ctypes.c_float, _i32, _vp, _vp, _sz,
                            _vp]),
    "tq_search_workspace_bytes": (_sz, [_vp, _i64, _i64, _i32]),
    "tq_search": (_i32, [_vp, _vp, _i32, _i64, _Packed, _i64, _i32, _vp, _vp, _vp, _sz, _vp]),
    "tq_split_init": (_i32, [_i32, _i32, _i32, _i32, _u64, ctypes.POINTER(_vp)]),
    "tq_split_destroy": (_i32, [_vp]),
    "tq_split_part": (_i32, [_vp, _i32, ctypes.POINTER(_vp)]),
    "tq_split_quantize_workspace_bytes": (_sz, [_vp, _i64]),
    "tq_split_quantize": (_i32, [_vp, _vp, _i32, _i64, _i64, _Packed, _Packed, _vp, _sz, _vp]),
    "tq_split_logits_workspace_bytes": (_sz, [_vp, _i64, _i32, _i64]),
    "tq_split_logits": (_i32, [_vp, _vp, _i32, _i64, _i32, _Packed, _Packed, _i64, _vp, _vp, _sz, _vp]),
    "tq_split_dequant": (_i32, [_vp, _Packed, _Packed, _i64, _vp, _i32, _i32, _vp]),
    "tq_topk": (_i32, [_vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "tq_logits_bf16": (_i32, [_vp, _vp, _i64, _i32, _i64, _i32, _vp, _vp]),
    "tq_status_str": (ctypes.c_char_p, [_i32]),
    "tq_sync_status": (_i32, [_vp, _vp]),
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_launch_count": (_u64, []),
    "tq_test_set": (_i32, [_i32, _i64]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.tq_last_error().decode(errors="replace")
        super().__init__(f"{where}: {_lib.tq_status_str(status).decode()} ({msg})")


def _check(status: int, where: str):
    if status != TQ_OK:
        raise TQError(status, where)


def test_set(knob: int, value: int):
    """Process-wide test setting (tq_test_set): wait limit of the d = 128
    quantize kernel, or injected host-side allocation / launch failures."""
    _check(_lib.tq_test_set(knob, value), "tq_test_set")


def launch_count() -> int:
    """Kernel launches libtq has issued in this process."""
    return int(_lib.tq_launch_count())


def host_params(d: int, b: int, m: int, seed: int = 0):
    """Parameters derived on the host (no CUDA): centroids, thresholds (fp32),
    D (int8), S (binary16 as numpy float16, [m, d']), where d' is d padded to
    the next power of two."""
    L = 1 << (b - 1)
    dp = 1 << (d - 1).bit_length() if d > 0 else 0
    c = np.zeros(L, np.float32)
    t = np.zeros(L - 1, np.float32)
    D = np.zeros(max(dp, 1), np.int8)
    S = np.zeros(max(m * dp, 1), np.uint16)
    _check(_lib.tq_host_params(d, b, m, seed & (2**64 - 1), c.ctypes.data, t.ctypes.data, D.ctypes.data,
                               S.ctypes.data), "tq_host_params")
    return c, t, D, S.view(np.float16).reshape(m, dp)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    if t.dtype == torch.float32:
        return TQ_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


@dataclass
class Packed:
    """Packed rows: codes [N, d(b-1)/8] u8, signs [N, m/8] u8, norm [N], rnorm [N] f32."""

    codes: "object"
    signs: "object"
    norm: "object"
    rnorm: "object"

    @property
    def n_rows(self) -> int:
        return int(self.norm.shape[0])

    def c(self) -> _Packed:
        return _Packed(_ptr(self.codes), _ptr(self.signs), _ptr(self.norm), _ptr(self.rnorm))

    def nbytes(self) -> int:
        return sum(int(t.numel() * t.element_size()) for t in (self.codes, self.signs, self.norm, self.rnorm))

    def rows(self, start: int, stop: int) -> "Packed":
        """Rows [start, stop) as views of the same storage."""
        return Packed(self.codes[start:stop], self.signs[start:stop], self.norm[start:stop], self.rnorm[start:stop])

    def to_numpy(self) -> dict:
        return {k: getattr(self, k).cpu().numpy() for k in ("codes", "signs", "norm", "rnorm")}

    @staticmethod
    def from_numpy(p: dict, device="cuda") -> "Packed":
        import torch
        return Packed(*(torch.from_numpy(np.ascontiguousarray(p[k])).to(device)
                        for k in ("codes", "signs", "norm", "rnorm")))


class TurboQuant:
    """One parameter set (d, b, m, seed) on the current CUDA device."""

    def __init__(self, d: int, b: int, m: int, seed: int = 0):
        self.d, self.b, self.m, self.seed = d, b, m, seed
        # rows of a length that is not a power of two are zero-padded to the next one
        self.d_pad = 1 << (d - 1).bit_length()
        h = _vp()
        _check(_lib.tq_init(d, b, m, seed & (2**64 - 1), ctypes.byref(h)), "tq_init")
        self._h = h
        cb, sb = _sz(), _sz()
        _check(_lib.tq_packed_sizes(h, 1, ctypes.byref(cb), ctypes.byref(sb)), "tq_packed_sizes")
        self.codes_bytes, self.signs_bytes = cb.value, sb.value

    def close(self):
        if getattr(self, "_h", None):
            _lib.tq_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def handle(self):
        return self._h

    @property
    def row_bytes(self) -> int:
        return self.codes_bytes + self.signs_bytes + 8

    def params(self):
        L = 1 << (self.b - 1)
        c = np.zeros(L, np.float32)
        t = np.zeros(L - 1, np.float32)
        D = np.zeros(self.d_pad, np.int8)
        S = np.zeros(self.m * self.d_pad, np.uint16)
        _check(_lib.tq_get_params(self._h, c.ctypes.data, t.ctypes.data, D.ctypes.data, S.ctypes.data),
               "tq_get_params")
        return c, t, D, S.view(np.float16).reshape(self.m, self.d_pad)

    def empty_packed(self, n_rows: int, device="cuda") -> Packed:
        import torch
        return Packed(torch.empty((n_rows, self.codes_bytes), dtype=torch.uint8, device=device),
                      torch.empty((n_rows, self.signs_bytes), dtype=torch.uint8, device=device),
                      torch.empty((n_rows,), dtype=torch.float32, device=device),
                      torch.empty((n_rows,), dtype=torch.float32, device=device))

    def quantize_workspace_bytes(self, n_rows: int) -> int:
        return int(_lib.tq_quantize_workspace_bytes(self._h, n_rows))

    def quantize(self, x, out: Packed | None = None, workspace=None, stream=None) -> Packed:
        """x: [N, d] (or [N, ld] with ld >= d) bf16/fp32 CUDA tensor, unit stride in the last dim."""
        import torch
        assert x.dim() == 2 and x.stride(1) == 1
        n = x.shape[0]
        if out is None:
            out = self.empty_packed(n, x.device)
        need = self.quantize_workspace_bytes(n)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_quantize(self._h, _ptr(x), _dtype_code(x), n, x.stride(0), out.c(), _ptr(workspace), wbytes,
                                _stream(stream)), "tq_quantize")
        return out

    def sync_status(self, stream=None):
        """Wait for the stream and raise if a kernel's bounded wait ran out."""
        _check(_lib.tq_sync_status(self._h, _stream(stream)), "tq_sync_status")

    def workspace_bytes(self, n_sets: int, g: int, n_keys: int) -> int:
        return int(_lib.tq_logits_workspace_bytes(self._h, n_sets, g, n_keys))

    def logits(self, q, keys: Packed, n_sets: int, g: int, n_keys: int, out=None, workspace=None,
               stream=None):
        """q: [n_sets*g, d] bf16/fp32; keys: n_sets*n_keys packed rows; returns [n_sets, g, n_keys] fp32."""
        import torch
        if out is None:
            out = torch.empty((n_sets, g, n_keys), dtype=torch.float32, device=q.device)
        need = self.workspace_bytes(n_sets, g, n_keys)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_logits(self._h, _ptr(q), _dtype_code(q), n_sets, g, keys.c(), n_keys, _ptr(out),
                              _ptr(workspace), wbytes, _stream(stream)), "tq_logits")
        return out

    def logits_noalloc(self, q, keys: Packed, n_sets: int, g: int, n_keys: int, out, stream=None):
        """tq_logits with the library's built-in scratch instead of a workspace;
        allocates nothing on the device (``out`` must be provided)."""
        _check(_lib.tq_logits_noalloc(self._h, _ptr(q), _dtype_code(q), n_sets, g, keys.c(), n_keys, _ptr(out),
                                      _stream(stream)), "tq_logits_noalloc")
        return out

    def dequant(self, packed: Packed, n_rows: int | None = None, out_dtype=None, mode: int = TQ_DEQUANT_PROD,
                out=None, stream=None):
        import torch
        n = packed.n_rows if n_rows is None else n_rows
        if out is None:
            out = torch.empty((n, self.d), dtype=out_dtype or torch.bfloat16, device=packed.norm.device)
        _check(_lib.tq_dequant(self._h, packed.c(), n, _ptr(out), _dtype_code(out), mode, _stream(stream)),
               "tq_dequant")
        return out


    def quantize_scatter(self, x, dest_rows, cache: Packed, stream=None) -> Packed:
        """Append: row i of x [N, d] (bf16/fp32 CUDA tensor) goes to packed row
        dest_rows[i] (int64 CUDA tensor) of ``cache``."""
        import torch
        assert x.dim() == 2 and x.stride(1) == 1
        assert dest_rows.dtype == torch.int64 and dest_rows.is_contiguous() and dest_rows.numel() == x.shape[0]
        _check(_lib.tq_quantize_scatter(self._h, _ptr(x), _dtype_code(x), x.shape[0], x.stride(0), _ptr(dest_rows),
                                        cache.n_rows, cache.c(), _stream(stream)), "tq_quantize_scatter")
        return cache

    def search_workspace_bytes(self, n_q: int, n_keys: int, k: int) -> int:
        return int(_lib.tq_search_workspace_bytes(self._h, n_q, n_keys, k))

    def search(self, q, keys: Packed, n_keys: int, k: int, idx=None, val=None, workspace=None, stream=None):
        """Vector search: per query of q [n_q, d], the k packed rows with the
        largest estimate (larger first, ties to the lower row); returns
        (idx [n_q, k] int32, val [n_q, k] fp32)."""
        import torch
        n_q = q.shape[0]
        if idx is None:
            idx = torch.empty((n_q, k), dtype=torch.int32, device=q.device)
        if val is None:
            val = torch.empty((n_q, k), dtype=torch.float32, device=q.device)
        need = self.search_workspace_bytes(n_q, n_keys, k)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_search(self._h, _ptr(q), _dtype_code(q), n_q, keys.c(), n_keys, k, _ptr(idx), _ptr(val),
                              _ptr(workspace), wbytes, _stream(stream)), "tq_search")
        return idx, val

    def attention_workspace_bytes(self, n_sets: int, g: int, n_keys: int) -> int:
        return int(_lib.tq_attention_workspace_bytes(self._h, n_sets, g, n_keys))

    def attention(self, q, keys: Packed, values: Packed, n_sets: int, g: int, n_keys: int, scale: float | None = None,
                  mode: int = TQ_DEQUANT_PROD, out=None, workspace=None, stream=None):
        """Decode attention from packed keys and values: [n_sets*g, d] fp32
        (softmax over each set's keys of scale * logit, times the dequantized
        values; scale defaults to 1/sqrt(d))."""
        import torch
        if scale is None:
            scale = 1.0 / math.sqrt(self.d)
        if out is None:
            out = torch.empty((n_sets * g, self.d), dtype=torch.float32, device=q.device)
        need = self.attention_workspace_bytes(n_sets, g, n_keys)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_attention(self._h, _ptr(q), _dtype_code(q), n_sets, g, keys.c(), values.c(), n_keys,
                                 float(scale), mode, _ptr(out), _ptr(workspace), wbytes, _stream(stream)),
               "tq_attention")
        return out


class TurboQuantSplit:
    """Fractional bit widths: channels [0, d_hi) as one instance with b_hi
    bits per coordinate, channels [d_hi, d) as another with b_lo bits (seeds
    seed and seed + 1); packed rows come in pairs (part 0, part 1)."""

    def __init__(self, d: int, d_hi: int, b_hi: int, b_lo: int, seed: int = 0):
        self.d, self.d_hi, self.b_hi, self.b_lo, self.seed = d, d_hi, b_hi, b_lo, seed
        h = _vp()
        _check(_lib.tq_split_init(d, d_hi, b_hi, b_lo, seed & (2**64 - 1), ctypes.byref(h)), "tq_split_init")
        self._h = h
        self._sizes, self._parts = [], []
        for p in (0, 1):
            ph = _vp()
            _check(_lib.tq_split_part(h, p, ctypes.byref(ph)), "tq_split_part")
            cb, sb = _sz(), _sz()
            _check(_lib.tq_packed_sizes(ph, 1, ctypes.byref(cb), ctypes.byref(sb)), "tq_packed_sizes")
            self._sizes.append((cb.value, sb.value))
            self._parts.append(ph)

    def sync_status(self, stream=None):
        """Wait for the stream and raise if a kernel of either part reported an error."""
        for ph in self._parts:
            _check(_lib.tq_sync_status(ph, _stream(stream)), "tq_sync_status")

    @property
    def row_bytes(self) -> int:
        """Packed bytes per row over both parts (codes, signs, two fp32 norms each)."""
        return sum(cb + sb + 8 for cb, sb in self._sizes)

    def logits_workspace_bytes(self, n_sets: int, g: int, n_keys: int) -> int:
        return int(_lib.tq_split_logits_workspace_bytes(self._h, n_sets, g, n_keys))

    @property
    def bits_per_coordinate(self) -> float:
        return (self.d_hi * self.b_hi + (self.d - self.d_hi) * self.b_lo) / self.d

    def close(self):
        if getattr(self, "_h", None):
            _lib.tq_split_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def empty_packed(self, n_rows: int, device="cuda"):
        import torch
        return tuple(Packed(torch.empty((n_rows, cb), dtype=torch.uint8, device=device),
                            torch.empty((n_rows, sb), dtype=torch.uint8, device=device),
                            torch.empty((n_rows,), dtype=torch.float32, device=device),
                            torch.empty((n_rows,), dtype=torch.float32, device=device)) for cb, sb in self._sizes)

    def quantize_workspace_bytes(self, n_rows: int) -> int:
        return int(_lib.tq_split_quantize_workspace_bytes(self._h, n_rows))

    def quantize(self, x, out=None, workspace=None, stream=None):
        import torch
        assert x.dim() == 2 and x.stride(1) == 1
        n = x.shape[0]
        if out is None:
            out = self.empty_packed(n, x.device)
        need = self.quantize_workspace_bytes(n)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_split_quantize(self._h, _ptr(x), _dtype_code(x), n, x.stride(0), out[0].c(), out[1].c(),
                                      _ptr(workspace), wbytes, _stream(stream)), "tq_split_quantize")
        return out

    def logits(self, q, keys, n_sets: int, g: int, n_keys: int, out=None, workspace=None, stream=None):
        import torch
        if out is None:
            out = torch.empty((n_sets, g, n_keys), dtype=torch.float32, device=q.device)
        need = self.logits_workspace_bytes(n_sets, g, n_keys)
        if need and workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
        wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        _check(_lib.tq_split_logits(self._h, _ptr(q), _dtype_code(q), n_sets, g, keys[0].c(), keys[1].c(), n_keys,
                                    _ptr(out), _ptr(workspace), wbytes, _stream(stream)), "tq_split_logits")
        return out

    def dequant(self, packed, n_rows: int | None = None, out_dtype=None, mode: int = TQ_DEQUANT_PROD, out=None,
                stream=None):
        import torch
        n = packed[0].n_rows if n_rows is None else n_rows
        if out is None:
            out = torch.empty((n, self.d), dtype=out_dtype or torch.bfloat16, device=packed[0].norm.device)
        _check(_lib.tq_split_dequant(self._h, packed[0].c(), packed[1].c(), n, _ptr(out), _dtype_code(out), mode,
                                     _stream(stream)), "tq_split_dequant")
        return out


def topk(scores, k: int, stream=None):
    import torch
    rows, cols = scores.shape
    idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    val = torch.empty((rows, k), dtype=torch.float32, device=scores.device)
    _check(_lib.tq_topk(_ptr(scores), rows, cols, k, _ptr(idx), _ptr(val), _stream(stream)), "tq_topk")
    return idx, val


def logits_bf16(q, keys, n_sets: int, g: int, n_keys: int, out=None, stream=None):
    """Plain bf16-key logits: q [n_sets*g, d], keys [n_sets*n_keys, d] bf16."""
    import torch
    d = q.shape[-1]
    if out is None:
        out = torch.empty((n_sets, g, n_keys), dtype=torch.float32, device=q.device)
    _check(_lib.tq_logits_bf16(_ptr(q), _ptr(keys), n_sets, g, n_keys, d, _ptr(out), _stream(stream)),
           "tq_logits_bf16")
    return out


def call_status(name: str, *args) -> int:
    """Raw call of an entry point (for API tests)."""
    return getattr(_lib, name)(*args)


def last_error() -> str:
    return _lib.tq_last_error().decode(errors="replace")
