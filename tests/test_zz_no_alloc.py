"""The allocation-free decode entry point (tq_decode_attention_static).

It serves callers that cannot allocate device memory (see include/tq.h): it takes
no workspace and uses a fixed scratch array inside the library. This file runs
last so a failure here never hides another test. It checks, through the C ABI,
that two calls in a row (different queries) give the same outputs as
tq_decode_attention with a caller workspace, and that an oversized shape is
refused with a clear error instead of overrunning the array."""
import ctypes

import numpy as np
import pytest

import workloads as W
from _parity import assert_close, make_ctx

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_cache_vector_05_b200 as T  # noqa: E402
from kv_cache_vector_05_b200 import _lib  # noqa: E402

DEV = "cuda:0"


def _packed(n_vec, d, lm_bits, v_bits, seed):
    pk = W.random_packed_cache(n_vec, d, lm_bits, d, v_bits, seed=seed)
    out = {}
    for k, v in pk.items():
        a = np.ascontiguousarray(v)
        out[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(DEV)
    return out


def _call_static(ctx, q, packed, batch, hq, hkv, max_len, lens, scores, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return _lib.lib.tq_decode_attention_static(
        ctx.handle, p(q), _lib.TQ_F32, batch, hq, hkv, p(lens), max_len,
        p(packed["k_codes"]), p(packed["k_signs"]), p(packed["k_norms"]),
        p(packed["v_codes"]), p(packed["v_params"]), 0.0, p(scores), p(out), stream)


@pytest.mark.parametrize("d,lm_bits,v_bits,G", [(128, 2, 2, 8), (64, 1, 4, 4)])
def test_static_scratch_matches_workspace_path_twice(d, lm_bits, v_bits, G):
    batch, hkv, max_len = 2, 2, 1100
    hq = hkv * G
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = _packed(batch * hkv * max_len, d, lm_bits, v_bits, seed=21)
    lens = torch.tensor([1100, 613], dtype=torch.int32, device=DEV)
    for call in range(2):                                     # two calls in a row
        q = torch.from_numpy(W.queries((batch, hq, d), seed=30 + call)).to(DEV)
        out_s = torch.full((batch, hq, d), float("nan"), device=DEV)
        sc_s = torch.full((batch, hq, max_len), float("nan"), device=DEV)
        st = _call_static(ctx, q, packed, batch, hq, hkv, max_len, lens, sc_s, out_s)
        assert st == _lib.TQ_OK, _lib.lib.tq_last_error().decode()
        sc_w = torch.full((batch, hq, max_len), float("nan"), device=DEV)
        out_w, _ = T.tq_decode_attention(ctx, q, packed, batch, hq, hkv, max_len, seq_lens=lens, scores=sc_w)
        torch.cuda.synchronize()
        assert_close(out_s.cpu().numpy(), out_w.cpu().numpy(), what=f"out, call {call}")
        a, b = sc_s.cpu().numpy(), sc_w.cpu().numpy()
        np.testing.assert_array_equal(np.isnan(a), np.isnan(b))
        assert_close(np.nan_to_num(a), np.nan_to_num(b), what=f"scores, call {call}")


def test_static_scratch_rejects_oversized_shape():
    ctx = make_ctx(T, 128, 2, 2)
    cap = T.tq_decode_static_scratch_capacity()
    batch, hq, hkv, max_len = 512, 64, 8, 1 << 15            # workspace far above 32 MiB
    assert T.tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len) > cap
    q = torch.zeros((batch, hq, 128), device=DEV)
    dummy = torch.zeros(16, dtype=torch.uint8, device=DEV)
    packed = {k: dummy for k in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params")}
    out = torch.empty((batch, hq, 128), device=DEV)
    st = _call_static(ctx, q, packed, batch, hq, hkv, max_len, None, None, out)
    assert st == _lib.TQ_EUNSUPPORTED
    assert "static buffer holds" in _lib.lib.tq_last_error().decode()
