"""C ABI checks that need no GPU: the library loads, exports every entry point
that include/tq.h declares, derives the same parameters as the oracle (two
independent implementations), and rejects bad arguments on the host."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import params as op
from oracle import turboquant as ot

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lib():
    from kv_cache_vector_15_b200 import tq
    return tq


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_symbols():
    tq = _lib()
    assert declared_symbols() == sorted(tq.SYMBOLS)


def test_library_exports_every_declared_symbol():
    tq = _lib()
    lib = ctypes.CDLL(tq.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


@pytest.mark.parametrize("d,b,m,seed", [(32, 2, 32, 0), (128, 2, 128, 0), (128, 3, 128, 0), (128, 4, 128, 7),
                                        (256, 5, 96, 3), (1024, 4, 1024, 0), (4096, 3, 64, 11), (100, 3, 128, 0),
                                        (3072, 4, 128, 5)])
def test_host_params_equal_oracle(d, b, m, seed):
    """A d that is not a power of two gets the parameters of the padded length."""
    tq = _lib()
    c, t, D, S = tq.host_params(d, b, m, seed)
    d = ot.padded_dim(d)
    P = op.Params(d, b, m, seed)
    assert np.array_equal(D, P.D)
    assert np.array_equal(S.astype(np.float64), P.S)           # binary16 bit-exact
    assert np.array_equal(c.astype(np.float64), P.centroids)   # fp32 bit-exact
    assert np.array_equal(t.astype(np.float64), P.thresholds)
    assert np.max(np.abs(c.astype(np.float64) - P.centroids64)) < 1e-7 / np.sqrt(d) * 4


@pytest.mark.parametrize("d,b,m", [(16, 3, 128), (31, 3, 128), (8192, 3, 128), (128, 1, 128), (128, 6, 128),
                                   (128, 3, 100), (128, 3, 0), (128, 3, 8192)])
def test_bad_dims_rejected(d, b, m):
    tq = _lib()
    st = tq.call_status("tq_host_params", d, b, m, 0, None, None, None, None)
    assert st == tq.TQ_ERR_INVALID_ARG
    assert tq.last_error()


def test_host_calls_validate_before_any_launch():
    tq = _lib()
    P = tq._Packed(0, 0, 0, 0)
    before = tq.launch_count()
    assert tq.call_status("tq_quantize", None, None, 0, 10, 128, P, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert tq._lib.tq_quantize_workspace_bytes(None, 10) == 0
    assert tq._lib.tq_logits_workspace_bytes(None, 1, 4, 10) == 0
    assert tq.call_status("tq_dequant", None, P, 10, None, 0, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_logits", None, None, 0, 1, 4, P, 10, None, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_topk", None, 4, 100, 0, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_topk", None, 4, 100, 65, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_topk", None, 4, 5, 10, None, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_topk", None, 0, 5, 10, None, None, None) == tq.TQ_OK   # empty: no-op
    assert tq.call_status("tq_logits_bf16", None, None, 1, 9, 10, 128, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_logits_bf16", None, None, 1, 4, 10, 96, None, None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_logits_bf16", None, None, 0, 4, 10, 128, None, None) == tq.TQ_OK
    assert tq.call_status("tq_attention", None, None, 0, 1, 4, P, P, 10, ctypes.c_float(0.1), 0, None, None, 0,
                          None) == tq.TQ_ERR_INVALID_ARG
    assert tq._lib.tq_attention_workspace_bytes(None, 1, 4, 10) == 0
    # vector search and the channel split: a NULL context is refused before any launch
    assert tq.call_status("tq_search", None, None, 0, 64, P, 4096, 10, None, None, None, 0,
                          None) == tq.TQ_ERR_INVALID_ARG
    assert tq._lib.tq_search_workspace_bytes(None, 64, 4096, 10) == 0
    assert tq.call_status("tq_split_quantize", None, None, 0, 10, 128, P, P, None, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert tq._lib.tq_split_quantize_workspace_bytes(None, 10) == 0
    assert tq.call_status("tq_split_logits", None, None, 0, 1, 4, P, P, 10, None, None, 0,
                          None) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_split_dequant", None, P, P, 10, None, 0, 0, None) == tq.TQ_ERR_INVALID_ARG
    assert tq._lib.tq_split_logits_workspace_bytes(None, 1, 4, 10) == 0
    assert tq.call_status("tq_split_destroy", None) == tq.TQ_OK
    assert tq.call_status("tq_test_set", 0, -1) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_test_set", 7, 0) == tq.TQ_ERR_INVALID_ARG
    assert tq.call_status("tq_test_set", tq.TQ_TEST_FAIL_LAUNCH, 0) == tq.TQ_OK
    assert tq.launch_count() == before


@pytest.mark.parametrize("d,d_hi", [(128, 48), (128, 128), (64, 16), (128, 0), (96, 100)])
def test_split_rejects_bad_channel_splits_on_the_host(d, d_hi):
    """Both parts need a multiple of 32 channels, at least 32: checked before
    any device call, so it holds without a GPU."""
    tq = _lib()
    h = ctypes.c_void_p()
    assert tq.call_status("tq_split_init", d, d_hi, 3, 2, 0, ctypes.byref(h)) == tq.TQ_ERR_INVALID_ARG
    assert not h.value


def test_init_without_device_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    tq = _lib()
    h = ctypes.c_void_p()
    st = tq.call_status("tq_init", 128, 3, 128, 0, ctypes.byref(h))
    assert st in (tq.TQ_ERR_CUDA, tq.TQ_ERR_UNSUPPORTED)
    assert not h.value
    assert tq.call_status("tq_destroy", None) == tq.TQ_OK


def test_status_strings():
    tq = _lib()
    for s, name in enumerate(["TQ_OK", "TQ_ERR_INVALID_ARG", "TQ_ERR_UNSUPPORTED", "TQ_ERR_NOMEM", "TQ_ERR_CUDA"]):
        assert tq._lib.tq_status_str(s).decode() == name
