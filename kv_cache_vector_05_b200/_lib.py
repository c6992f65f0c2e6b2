"""ctypes binding of ``libtq.so`` (the C ABI declared in ``include/tq.h``).

Argument marshalling only: every step of compression and decode runs in the
library's CUDA kernels. Tensors are torch CUDA tensors (torch supplies device
memory and the current stream); host-only helpers take numpy arrays.
Importing this module fails loudly if the shared library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

# TQ_LIBRARY may name another build of the same library (e.g. a debug build).
LIB_PATH = os.environ.get("TQ_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ECUDA, TQ_ENOMEM = 0, 1, 2, 3, 4
TQ_F32, TQ_BF16 = 0, 1
TQ_ROT_HADAMARD, TQ_ROT_HAAR = 0, 1
TQ_DECODE_AUTO, TQ_DECODE_TCGEN05, TQ_DECODE_MMA, TQ_DECODE_CUDA_CORE = 0, 1, 2, 3
DECODE_KERNEL_NAMES = {TQ_DECODE_TCGEN05: "tcgen05", TQ_DECODE_MMA: "mma", TQ_DECODE_CUDA_CORE: "cuda_core"}

EXPORTED = (
    "tq_codebook_load", "tq_free", "tq_status_string", "tq_last_error",
    "tq_lloyd_max_codebook", "tq_haar_from_gaussian", "tq_compress_kv", "tq_compress_kv_slots",
    "tq_decode_workspace_bytes", "tq_decode_attention", "tq_decode_attention_paged", "tq_decompress",
    "tq_set_profile_events", "tq_check_device", "tq_decode_attention_static", "tq_decode_static_scratch_capacity",
    "tq_decode_attention_partial", "tq_merge_attention", "tq_set_decode_kernel", "tq_decode_kernel_for",
)


class TQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        super().__init__(f"{where}: {_status_string(status)}" + (f" ({detail})" if detail else ""))


class tq_params(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int),
        ("k_lm_bits", ctypes.c_int),
        ("qjl_m", ctypes.c_int),
        ("v_bits", ctypes.c_int),
        ("v_group", ctypes.c_int),
        ("rot", ctypes.c_int),
        ("centroids", ctypes.POINTER(ctypes.c_float)),
        ("boundaries", ctypes.POINTER(ctypes.c_float)),
        ("hadamard_signs", ctypes.POINTER(ctypes.c_byte)),
        ("haar", ctypes.POINTER(ctypes.c_double)),
        ("qjl_S", ctypes.POINTER(ctypes.c_float)),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libtq.so is not built ({LIB_PATH}); run `python kv_cache_vector_05_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, c_int, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int, ctypes.c_size_t
    fp = ctypes.POINTER(ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.tq_codebook_load.argtypes = [ctypes.POINTER(tq_params), vp, ctypes.POINTER(vp)]
    lib.tq_codebook_load.restype = c_int
    lib.tq_free.argtypes = [vp]
    lib.tq_free.restype = None
    lib.tq_status_string.argtypes = [c_int]
    lib.tq_status_string.restype = ctypes.c_char_p
    lib.tq_last_error.argtypes = []
    lib.tq_last_error.restype = ctypes.c_char_p
    lib.tq_lloyd_max_codebook.argtypes = [c_int, c_int, fp, fp]
    lib.tq_lloyd_max_codebook.restype = c_int
    lib.tq_haar_from_gaussian.argtypes = [c_int, dp, dp]
    lib.tq_haar_from_gaussian.restype = c_int
    lib.tq_compress_kv.argtypes = [vp, vp, vp, c_int, i64, vp, vp, vp, vp, vp, vp]
    lib.tq_compress_kv.restype = c_int
    lib.tq_compress_kv_slots.argtypes = [vp, vp, vp, c_int, i64, vp, i64, vp, vp, vp, vp, vp, vp]
    lib.tq_compress_kv_slots.restype = c_int
    lib.tq_decode_workspace_bytes.argtypes = [vp, c_int, c_int, c_int, i64]
    lib.tq_decode_workspace_bytes.restype = sz
    lib.tq_decode_attention.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, i64,
                                        vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, sz, vp]
    lib.tq_decode_attention.restype = c_int
    lib.tq_decode_attention_paged.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, i64, vp, i64, i64, i64,
                                              vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, sz, vp]
    lib.tq_decode_attention_paged.restype = c_int
    lib.tq_decode_attention_partial.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, i64,
                                                vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp, vp, sz, vp]
    lib.tq_decode_attention_partial.restype = c_int
    lib.tq_merge_attention.argtypes = [vp, i64, vp, i64, c_int, i64, c_int, vp, vp, vp]
    lib.tq_merge_attention.restype = c_int
    lib.tq_decompress.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp, vp]
    lib.tq_decompress.restype = c_int
    lib.tq_decode_attention_static.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, i64,
                                               vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp]
    lib.tq_decode_attention_static.restype = c_int
    lib.tq_decode_static_scratch_capacity.argtypes = []
    lib.tq_decode_static_scratch_capacity.restype = sz
    lib.tq_check_device.argtypes = [vp, vp]
    lib.tq_check_device.restype = c_int
    lib.tq_set_profile_events.argtypes = [vp, vp, vp]
    lib.tq_set_profile_events.restype = c_int
    lib.tq_set_decode_kernel.argtypes = [vp, c_int]
    lib.tq_set_decode_kernel.restype = c_int
    lib.tq_decode_kernel_for.argtypes = [vp, c_int, c_int]
    lib.tq_decode_kernel_for.restype = c_int
    return lib


lib = _load()


def _status_string(status: int) -> str:
    return lib.tq_status_string(status).decode()


def _check(status: int, where: str):
    if status != TQ_OK:
        raise TQError(status, where, lib.tq_last_error().decode())


def tq_status_string(status: int) -> str:
    return _status_string(status)


# ------------------------------------------------------------------ host helpers

def tq_lloyd_max_codebook(d: int, bits: int):
    """fp32 (centroids, boundaries) of the rotated-coordinate Lloyd-Max quantizer."""
    c = np.zeros(1 << bits, dtype=np.float32)
    t = np.zeros(max((1 << bits) - 1, 1), dtype=np.float32)
    fp = ctypes.POINTER(ctypes.c_float)
    _check(lib.tq_lloyd_max_codebook(d, bits, c.ctypes.data_as(fp), t.ctypes.data_as(fp)),
           "tq_lloyd_max_codebook")
    return c, t[: (1 << bits) - 1]


def tq_haar_from_gaussian(gaussian: np.ndarray) -> np.ndarray:
    """Haar orthogonal matrix (fp64) from a square matrix of N(0,1) draws."""
    g = np.ascontiguousarray(gaussian, dtype=np.float64)
    d = g.shape[0]
    out = np.empty_like(g)
    dp = ctypes.POINTER(ctypes.c_double)
    _check(lib.tq_haar_from_gaussian(d, g.ctypes.data_as(dp), out.ctypes.data_as(dp)),
           "tq_haar_from_gaussian")
    return out


# ------------------------------------------------------------------ device calls

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Context:
    """Owns a ``tq_ctx`` (codebook, rotation and QJL matrix on the device)."""

    def __init__(self, d: int, k_lm_bits: int, v_bits: int, centroids, boundaries, qjl_S,
                 rotation: str = "hadamard", hadamard_signs=None, haar=None, v_group: int = 32,
                 stream=None):
        self.d, self.lm_bits, self.v_bits, self.v_group = d, k_lm_bits, v_bits, v_group
        # qjl_S None (or an empty [0, d] array): keys without the QJL stage, m = 0
        S = np.zeros((0, d), np.float32) if qjl_S is None else np.ascontiguousarray(qjl_S, dtype=np.float32)
        self.m = S.shape[0]
        c = np.ascontiguousarray(centroids, dtype=np.float32)
        t = np.ascontiguousarray(boundaries, dtype=np.float32)
        keep = [S, c, t]
        p = tq_params()
        p.d, p.k_lm_bits, p.qjl_m, p.v_bits, p.v_group = d, k_lm_bits, self.m, v_bits, v_group
        p.rot = TQ_ROT_HADAMARD if rotation == "hadamard" else TQ_ROT_HAAR
        p.centroids = c.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        p.boundaries = t.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        p.qjl_S = S.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        if hadamard_signs is not None:
            sg = np.ascontiguousarray(hadamard_signs, dtype=np.int8)
            keep.append(sg)
            p.hadamard_signs = sg.ctypes.data_as(ctypes.POINTER(ctypes.c_byte))
        if haar is not None:
            h = np.ascontiguousarray(haar, dtype=np.float64)
            keep.append(h)
            p.haar = h.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
        self.rotation = rotation
        handle = ctypes.c_void_p()
        _check(lib.tq_codebook_load(ctypes.byref(p), _stream(stream), ctypes.byref(handle)), "tq_codebook_load")
        self.handle = handle

    def close(self):
        if getattr(self, "handle", None) is not None and self.handle.value:
            lib.tq_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # record sizes (bytes)
    @property
    def k_code_bytes(self):
        return self.lm_bits * self.d // 8

    @property
    def v_code_bytes(self):
        return self.v_bits * self.d // 8


def tq_codebook_load(d: int, k_lm_bits: int, v_bits: int, centroids, boundaries, qjl_S,
                     rotation: str = "hadamard", hadamard_signs=None, haar=None, v_group: int = 32,
                     stream=None) -> Context:
    """Upload a codebook, rotation and QJL matrix; returns the owning Context."""
    return Context(d, k_lm_bits, v_bits, centroids, boundaries, qjl_S, rotation, hadamard_signs,
                   haar, v_group, stream)


def tq_free(ctx: Context) -> None:
    ctx.close()


def tq_check_device(ctx: Context, stream=None) -> None:
    """Synchronize and raise TQError if a kernel's bounded wait timed out since the last check."""
    _check(lib.tq_check_device(ctx.handle, _stream(stream)), "tq_check_device")


def tq_set_profile_events(ctx: Context, start=None, stop=None) -> None:
    """Bracket the main kernel of later calls with two torch.cuda.Event objects (or None)."""
    _check(lib.tq_set_profile_events(ctx.handle, None if start is None else ctypes.c_void_p(start.cuda_event),
                                     None if stop is None else ctypes.c_void_p(stop.cuda_event)),
           "tq_set_profile_events")


def tq_set_decode_kernel(ctx: Context, kernel: int) -> None:
    """Select the decode kernel family (TQ_DECODE_AUTO, _TCGEN05, _MMA or _CUDA_CORE) of later calls."""
    _check(lib.tq_set_decode_kernel(ctx.handle, int(kernel)), "tq_set_decode_kernel")


def tq_decode_kernel_for(ctx: Context, hq: int, hkv: int) -> int:
    """The decode kernel family a call with these head counts runs on `ctx` (-1: unsupported)."""
    return int(lib.tq_decode_kernel_for(ctx.handle, hq, hkv))


def tq_compress_kv(ctx: Context, k, v, k_codes=None, k_signs=None, k_norms=None,
                   v_codes=None, v_params=None, stream=None):
    """Compress keys and/or values (torch CUDA tensors [n, d], fp32 or bf16)."""
    import torch
    src = k if k is not None else v
    n = src.shape[0]
    dev = src.device
    dtype = TQ_F32 if src.dtype == torch.float32 else TQ_BF16
    for t in (k, v):
        if t is not None:
            assert t.is_contiguous() and t.shape == (n, ctx.d) and t.dtype == src.dtype
    out = {}
    if k is not None:
        k_codes = torch.empty((n, ctx.k_code_bytes), dtype=torch.uint8, device=dev) if k_codes is None else k_codes
        k_signs = torch.empty((n, ctx.m // 8), dtype=torch.uint8, device=dev) if k_signs is None else k_signs
        k_norms = torch.empty((n, 2), dtype=torch.int16, device=dev) if k_norms is None else k_norms
        out.update(k_codes=k_codes, k_signs=k_signs, k_norms=k_norms)
    if v is not None:
        v_codes = torch.empty((n, ctx.v_code_bytes), dtype=torch.uint8, device=dev) if v_codes is None else v_codes
        v_params = (torch.empty((n, ctx.d // ctx.v_group, 2), dtype=torch.int16, device=dev)
                    if v_params is None else v_params)
        out.update(v_codes=v_codes, v_params=v_params)
    _check(lib.tq_compress_kv(ctx.handle, _ptr(k), _ptr(v), dtype, n, _ptr(out.get("k_codes")),
                              _ptr(out.get("k_signs")), _ptr(out.get("k_norms")), _ptr(out.get("v_codes")),
                              _ptr(out.get("v_params")), _stream(stream)), "tq_compress_kv")
    return out


def tq_compress_kv_slots(ctx: Context, k, v, slot, packed: dict, stream=None) -> dict:
    """Compress keys and/or values (torch CUDA tensors [n, d]) into the existing packed arrays
    of `packed` (k_codes ... v_params, each [n_rows, ...]), vector i into row slot[i]
    (int64 CUDA tensor [n]). Returns `packed`."""
    import torch
    src = k if k is not None else v
    n = src.shape[0]
    dtype = TQ_F32 if src.dtype == torch.float32 else TQ_BF16
    for t in (k, v):
        if t is not None:
            assert t.is_contiguous() and t.shape == (n, ctx.d) and t.dtype == src.dtype
    assert slot.is_contiguous() and slot.dtype == torch.int64 and slot.numel() == n
    ref = packed["k_codes"] if k is not None else packed["v_codes"]
    n_rows = ref.shape[0]
    _check(lib.tq_compress_kv_slots(
        ctx.handle, _ptr(k), _ptr(v), dtype, n, _ptr(slot), n_rows,
        _ptr(packed.get("k_codes") if k is not None else None), _ptr(packed.get("k_signs") if k is not None else None),
        _ptr(packed.get("k_norms") if k is not None else None), _ptr(packed.get("v_codes") if v is not None else None),
        _ptr(packed.get("v_params") if v is not None else None), _stream(stream)), "tq_compress_kv_slots")
    return packed


def tq_decode_workspace_bytes(ctx: Context, batch: int, hq: int, hkv: int, max_len: int) -> int:
    return int(lib.tq_decode_workspace_bytes(ctx.handle, batch, hq, hkv, max_len))


def tq_decode_attention(ctx: Context, q, packed: dict, batch: int, hq: int, hkv: int, max_len: int,
                        seq_lens=None, softmax_scale: float = 0.0, scores=None, out=None,
                        workspace=None, stream=None):
    """Decode attention of q [batch, hq, d] over a packed cache laid out
    [batch][hkv][max_len][record]. Returns (out [batch, hq, d] fp32, scores or None)."""
    import torch
    dev = q.device
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    assert q.is_contiguous() and q.numel() == batch * hq * ctx.d
    if out is None:
        out = torch.empty((batch, hq, ctx.d), dtype=torch.float32, device=dev)
    need = tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.tq_decode_attention(
        ctx.handle, _ptr(q), q_dtype, batch, hq, hkv, _ptr(seq_lens), max_len,
        _ptr(packed["k_codes"]), _ptr(packed["k_signs"]), _ptr(packed["k_norms"]),
        _ptr(packed["v_codes"]), _ptr(packed["v_params"]), float(softmax_scale),
        _ptr(scores), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)), "tq_decode_attention")
    return out, scores


def tq_decode_attention_partial(ctx: Context, q, packed: dict, batch: int, hq: int, hkv: int, max_len: int,
                                seq_lens=None, softmax_scale: float = 0.0, scores=None, out=None, lse=None,
                                workspace=None, stream=None):
    """tq_decode_attention over this cache's tokens that also returns each row's
    log-partition (for merging with other token ranges by tq_merge_attention).
    Returns (out [batch, hq, d] fp32, lse [batch, hq] fp32, scores or None)."""
    import torch
    dev = q.device
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    assert q.is_contiguous() and q.numel() == batch * hq * ctx.d
    if out is None:
        out = torch.empty((batch, hq, ctx.d), dtype=torch.float32, device=dev)
    if lse is None:
        lse = torch.empty((batch, hq), dtype=torch.float32, device=dev)
    assert out.is_contiguous() and lse.is_contiguous() and lse.dtype == torch.float32
    need = tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.tq_decode_attention_partial(
        ctx.handle, _ptr(q), q_dtype, batch, hq, hkv, _ptr(seq_lens), max_len,
        _ptr(packed["k_codes"]), _ptr(packed["k_signs"]), _ptr(packed["k_norms"]),
        _ptr(packed["v_codes"]), _ptr(packed["v_params"]), float(softmax_scale),
        _ptr(scores), _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)),
        "tq_decode_attention_partial")
    return out, lse, scores


def tq_merge_attention(outs, lses, out=None, lse=None, stream=None):
    """Merge R attention results over disjoint token ranges: outs [R, rows..., d] and
    lses [R, rows...] fp32 device tensors whose trailing dimensions are contiguous (the
    leading stride may be anything, e.g. views into one gathered buffer). Returns
    (out [rows..., d], lse or None)."""
    import torch
    R, d = outs.shape[0], outs.shape[-1]
    rows = int(np.prod(outs.shape[1:-1])) if outs.dim() > 2 else 1
    assert outs.dtype == torch.float32 and lses.dtype == torch.float32 and lses.shape[0] == R
    assert lses[0].numel() == rows
    assert outs[0].is_contiguous() and lses[0].is_contiguous()
    if out is None:
        out = torch.empty(tuple(outs.shape[1:]), dtype=torch.float32, device=outs.device)
    assert out.is_contiguous() and out.numel() == rows * d
    _check(lib.tq_merge_attention(_ptr(outs), int(outs.stride(0)) if R > 1 else rows * d, _ptr(lses),
                                  int(lses.stride(0)) if R > 1 else rows, R, rows, d, _ptr(out), _ptr(lse),
                                  _stream(stream)), "tq_merge_attention")
    return out, lse


def tq_decode_attention_paged(ctx: Context, q, packed: dict, batch: int, hq: int, hkv: int, max_len: int,
                              block_table, page_size: int, n_pages: int, seq_lens=None,
                              softmax_scale: float = 0.0, scores=None, out=None, workspace=None, stream=None):
    """Decode attention over a paged cache: the packed arrays hold n_pages pages of page_size
    records; block_table (int32 [batch, hkv, max_pages]) names the page of each block of
    page_size tokens. Returns (out [batch, hq, d] fp32, scores or None)."""
    import torch
    dev = q.device
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    assert q.is_contiguous() and q.numel() == batch * hq * ctx.d
    assert block_table.is_contiguous() and block_table.dtype == torch.int32 and block_table.dim() == 3
    if out is None:
        out = torch.empty((batch, hq, ctx.d), dtype=torch.float32, device=dev)
    need = tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.tq_decode_attention_paged(
        ctx.handle, _ptr(q), q_dtype, batch, hq, hkv, _ptr(seq_lens), max_len, _ptr(block_table),
        int(page_size), int(block_table.shape[2]), int(n_pages),
        _ptr(packed["k_codes"]), _ptr(packed["k_signs"]), _ptr(packed["k_norms"]),
        _ptr(packed["v_codes"]), _ptr(packed["v_params"]), float(softmax_scale),
        _ptr(scores), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)), "tq_decode_attention_paged")
    return out, scores


def tq_decode_attention_static(ctx: Context, q, packed: dict, batch: int, hq: int, hkv: int,
                               max_len: int, seq_lens=None, softmax_scale: float = 0.0, scores=None,
                               out=None, stream=None):
    """tq_decode_attention without a workspace: the library's fixed scratch array is
    used instead (for callers that cannot allocate device memory; see include/tq.h)."""
    import torch
    q_dtype = TQ_F32 if q.dtype == torch.float32 else TQ_BF16
    assert q.is_contiguous() and q.numel() == batch * hq * ctx.d
    if out is None:
        out = torch.empty((batch, hq, ctx.d), dtype=torch.float32, device=q.device)
    _check(lib.tq_decode_attention_static(
        ctx.handle, _ptr(q), q_dtype, batch, hq, hkv, _ptr(seq_lens), max_len,
        _ptr(packed["k_codes"]), _ptr(packed["k_signs"]), _ptr(packed["k_norms"]),
        _ptr(packed["v_codes"]), _ptr(packed["v_params"]), float(softmax_scale),
        _ptr(scores), _ptr(out), _stream(stream)), "tq_decode_attention_static")
    return out, scores


def tq_decode_static_scratch_capacity() -> int:
    return int(lib.tq_decode_static_scratch_capacity())


def tq_decompress(ctx: Context, packed: dict, n_vec: int, keys: bool = True, values: bool = True,
                  k_out=None, v_out=None, stream=None):
    import torch
    dev = (packed.get("k_codes") if keys else packed.get("v_codes")).device
    if keys and k_out is None:
        k_out = torch.empty((n_vec, ctx.d), dtype=torch.float32, device=dev)
    if values and v_out is None:
        v_out = torch.empty((n_vec, ctx.d), dtype=torch.float32, device=dev)
    _check(lib.tq_decompress(ctx.handle, _ptr(packed.get("k_codes") if keys else None),
                             _ptr(packed.get("k_signs") if keys else None),
                             _ptr(packed.get("k_norms") if keys else None),
                             _ptr(packed.get("v_codes") if values else None),
                             _ptr(packed.get("v_params") if values else None), n_vec,
                             _ptr(k_out if keys else None), _ptr(v_out if values else None),
                             _stream(stream)), "tq_decompress")
    return (k_out if keys else None), (v_out if values else None)
