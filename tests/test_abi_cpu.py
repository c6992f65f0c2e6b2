"""CPU-side checks of the C ABI: the library loads, exports every declared entry
point, its host-only routines agree with the oracle, and argument validation
returns the documented status codes before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import workloads as W

T = pytest.importorskip("kv_cache_vector_05_b200")
from kv_cache_vector_05_b200 import _lib  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "tq.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("tq_codebook_load", "tq_compress_kv", "tq_decode_attention", "tq_decompress"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) == set(_lib.EXPORTED)


@pytest.mark.parametrize("d,bits", [(d, b) for d in (64, 128, 256) for b in (1, 2, 3, 4)]
                         + [(64, 7), (128, 5), (128, 6), (128, 7)])
def test_native_codebook_equals_oracle_fp32(d, bits):
    """The library's fp64 solver (Lloyd iteration up to 4 bits, Newton's method beyond)
    against the oracle's, after rounding both to fp32."""
    c, t = T.tq_lloyd_max_codebook(d, bits)
    oc, ot = O.device_codebook(d, bits)
    np.testing.assert_array_equal(c.astype(np.float64), oc)
    np.testing.assert_array_equal(t.astype(np.float64), ot)


@pytest.mark.parametrize("d", [8, 64, 128, 256])
def test_native_haar_matches_oracle(d):
    g = W.method_draws(d, d)["haar_gaussian"]
    pi = T.tq_haar_from_gaussian(g)
    assert np.max(np.abs(pi.T @ pi - np.eye(d))) < 1e-12
    np.testing.assert_allclose(pi, O.haar_rotation(g), rtol=0, atol=1e-12)


def test_status_strings():
    assert T.tq_status_string(0) == "TQ_OK"
    for s in range(1, 5):
        assert T.tq_status_string(s).startswith("TQ_E")


def test_validation_without_gpu():
    lib = _lib.lib
    assert lib.tq_compress_kv(None, None, None, 0, 1, None, None, None, None, None, None) == _lib.TQ_EINVAL
    assert lib.tq_decompress(None, None, None, None, None, None, 1, None, None, None) == _lib.TQ_EINVAL
    assert lib.tq_decode_workspace_bytes(None, 1, 8, 1, 128) == 0
    assert lib.tq_decode_attention(None, None, 0, 1, 8, 1, None, 16, None, None, None, None, None,
                                   0.0, None, None, None, 0, None) == _lib.TQ_EINVAL
    assert lib.tq_codebook_load(None, None, None) == _lib.TQ_EINVAL
    fp = ctypes.POINTER(ctypes.c_float)
    c = np.zeros(4, np.float32)
    assert lib.tq_lloyd_max_codebook(2, 2, c.ctypes.data_as(fp), c.ctypes.data_as(fp)) == _lib.TQ_EINVAL
    assert lib.tq_lloyd_max_codebook(128, 2, None, None) == _lib.TQ_EINVAL


def test_decode_kernel_selection_validates_without_gpu():
    """Selecting a decode kernel family needs a context; the query of a NULL context or of
    head counts that do not divide reports no family."""
    lib = _lib.lib
    assert lib.tq_set_decode_kernel(None, _lib.TQ_DECODE_MMA) == _lib.TQ_EINVAL
    assert lib.tq_decode_kernel_for(None, 32, 8) == -1
    assert (_lib.TQ_DECODE_AUTO, _lib.TQ_DECODE_TCGEN05, _lib.TQ_DECODE_MMA, _lib.TQ_DECODE_CUDA_CORE) == (0, 1, 2, 3)


def test_split_sequence_entry_points_validate_without_gpu():
    """The partial decode and the merge reject bad sizes and pointers before any launch;
    a merge of zero rows is a no-op."""
    lib, E = _lib.lib, _lib.TQ_EINVAL
    assert lib.tq_decode_attention_partial(None, None, 0, 1, 8, 1, None, 16, None, None, None, None, None,
                                           0.0, None, None, None, None, 0, None) == E
    buf = np.zeros(64, np.float32)
    p = buf.ctypes.data
    odd = ctypes.c_void_p(p + 2)                              # not float-aligned
    ok = ctypes.c_void_p(p)
    assert lib.tq_merge_attention(ok, 8, ok, 2, 0, 2, 4, ok, None, None) == E       # no parts
    assert lib.tq_merge_attention(ok, 8, ok, 2, 2, 2, 0, ok, None, None) == E       # d = 0
    assert lib.tq_merge_attention(ok, 8, ok, 2, 2, -1, 4, ok, None, None) == E      # rows < 0
    assert lib.tq_merge_attention(ok, 7, ok, 2, 2, 2, 4, ok, None, None) == E       # outs stride < rows*d
    assert lib.tq_merge_attention(ok, 8, ok, 1, 2, 2, 4, ok, None, None) == E       # lses stride < rows
    assert lib.tq_merge_attention(None, 8, ok, 2, 2, 2, 4, ok, None, None) == E     # NULL outs
    assert lib.tq_merge_attention(ok, 8, ok, 2, 2, 2, 4, None, None, None) == E     # NULL out
    assert lib.tq_merge_attention(odd, 8, ok, 2, 2, 2, 4, ok, None, None) == E
    assert lib.tq_merge_attention(ok, 8, ok, 2, 2, 2, 4, ok, odd, None) == E
    assert lib.tq_merge_attention(None, 0, None, 0, 3, 0, 4, None, None, None) == _lib.TQ_OK


@pytest.mark.parametrize("field,value,status", [
    ("d", 96, _lib.TQ_EUNSUPPORTED), ("k_lm_bits", 8, _lib.TQ_EUNSUPPORTED),
    ("qjl_m", 48, _lib.TQ_EUNSUPPORTED), ("v_bits", 5, _lib.TQ_EUNSUPPORTED),
    ("v_group", 16, _lib.TQ_EUNSUPPORTED), ("rot", 7, _lib.TQ_EINVAL),
])
def test_codebook_load_rejects_bad_params(field, value, status):
    d = 128
    c, t = T.tq_lloyd_max_codebook(d, 2)
    S = np.ones((d, d), np.float32)
    sg = np.ones(d, np.int8)
    p = _lib.tq_params()
    p.d, p.k_lm_bits, p.qjl_m, p.v_bits, p.v_group, p.rot = d, 2, d, 2, 32, 0
    p.centroids = c.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
    p.boundaries = t.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
    p.qjl_S = S.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
    p.hadamard_signs = sg.ctypes.data_as(ctypes.POINTER(ctypes.c_byte))
    setattr(p, field, value)
    out = ctypes.c_void_p()
    assert _lib.lib.tq_codebook_load(ctypes.byref(p), None, ctypes.byref(out)) == status
    assert not out.value


def test_codebook_load_rejects_unsorted_codebook_and_bad_signs():
    d = 64
    c, t = T.tq_lloyd_max_codebook(d, 2)
    S = np.ones((d, d), np.float32)
    for cc, sg in ((c[::-1].copy(), np.ones(d, np.int8)), (c, np.zeros(d, np.int8))):
        p = _lib.tq_params()
        p.d, p.k_lm_bits, p.qjl_m, p.v_bits, p.v_group, p.rot = d, 2, d, 2, 32, 0
        p.centroids = cc.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        p.boundaries = t.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        p.qjl_S = S.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        p.hadamard_signs = sg.ctypes.data_as(ctypes.POINTER(ctypes.c_byte))
        out = ctypes.c_void_p()
        assert _lib.lib.tq_codebook_load(ctypes.byref(p), None, ctypes.byref(out)) == _lib.TQ_EINVAL
