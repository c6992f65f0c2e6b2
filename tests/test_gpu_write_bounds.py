"""Guard-byte tests of every output buffer (through the C ABI).

compute-sanitizer is not available for these kernels, so out-of-range writes are looked
for directly: each output array is the middle of a larger device buffer whose first and
last 4 KiB hold a known byte. After the call every guard byte must still hold it, and the
outputs must equal those of the same call on plain buffers. Shapes are ragged (sizes that
are not multiples of any tile) and cover the compression kernels (bf16 pipelined, fp32,
d = 64), both decode paths (tensor cores, CUDA cores) with scores, log-partitions and an
exactly sized workspace, the merge and the decompression."""
import numpy as np
import pytest

import workloads as W
from _parity import make_ctx

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_cache_vector_05_b200 as T  # noqa: E402

DEV = "cuda:0"
GUARD = 4096   # bytes on each side (keeps the inner array 16-byte aligned)
FILL = 0x5A


class Guarded:
    """A device array of `shape` and `dtype` with GUARD bytes of FILL on both sides."""

    def __init__(self, shape, dtype):
        itemsize = torch.empty((), dtype=dtype).element_size()
        self.n = int(np.prod(shape)) * itemsize
        self.buf = torch.full((GUARD + self.n + GUARD,), FILL, dtype=torch.uint8, device=DEV)
        self.t = self.buf[GUARD:GUARD + self.n].view(dtype).view(shape)

    def intact(self) -> bool:
        b = self.buf.cpu().numpy()
        return bool((b[:GUARD] == FILL).all() and (b[GUARD + self.n:] == FILL).all())


def _packed_guards(ctx, n):
    d = ctx.d
    return {"k_codes": Guarded((n, ctx.k_code_bytes), torch.uint8),
            "k_signs": Guarded((n, ctx.m // 8), torch.uint8),
            "k_norms": Guarded((n, 2), torch.int16),
            "v_codes": Guarded((n, ctx.v_code_bytes), torch.uint8),
            "v_params": Guarded((n, d // ctx.v_group, 2), torch.int16)}


@pytest.mark.parametrize("d,lm_bits,v_bits,dtype", [
    (128, 2, 2, "bf16"),   # pipelined tensor-core kernel
    (128, 2, 4, "f32"),    # four lanes per vector, tensor-core projection
    (64, 3, 2, "bf16"),    # warp per vector
])
def test_compression_writes_stay_in_their_arrays(d, lm_bits, v_bits, dtype):
    n = 148 * 128 + 77
    ctx = make_ctx(T, d, lm_bits, v_bits)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    K = W.device_normal((n, d), seed=3, device=DEV).to(tdt)
    V = W.device_normal((n, d), seed=4, device=DEV).to(tdt)
    g = _packed_guards(ctx, n)
    T.tq_compress_kv(ctx, K, V, **{k: v.t for k, v in g.items()})
    plain = T.tq_compress_kv(ctx, K, V)
    T.tq_check_device(ctx)
    for name, gb in g.items():
        assert gb.intact(), f"{name}: a guard byte changed"
        assert torch.equal(gb.t, plain[name]), name


def _random_cache(units, max_len, d, lm_bits, v_bits, seed):
    pk = W.random_packed_cache(units * max_len, d, lm_bits, d, v_bits, seed=seed)
    return {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                                else np.ascontiguousarray(v)).to(DEV) for k, v in pk.items()}


@pytest.mark.parametrize("d,lm_bits,v_bits,G", [
    (128, 2, 2, 4),   # tensor-core decode
    (128, 2, 4, 8),   # tensor-core decode, two n-blocks
    (128, 3, 4, 6),   # CUDA-core decode
    (64, 2, 2, 4),
])
def test_decode_writes_stay_in_their_arrays(d, lm_bits, v_bits, G):
    batch, hkv, max_len = 3, 2, 1337
    hq = hkv * G
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = _random_cache(batch * hkv, max_len, d, lm_bits, v_bits, seed=31)
    q = torch.from_numpy(W.queries((batch, hq, d), dtype="f32")).to(DEV)
    lens = torch.tensor([1337, 600, 0], dtype=torch.int32, device=DEV)
    need = T.tq_decode_workspace_bytes(ctx, batch, hq, hkv, max_len)
    out, scores = Guarded((batch, hq, d), torch.float32), Guarded((batch, hq, max_len), torch.float32)
    lse, ws = Guarded((batch, hq), torch.float32), Guarded((need,), torch.uint8)
    T.tq_decode_attention_partial(ctx, q, packed, batch, hq, hkv, max_len, seq_lens=lens, scores=scores.t,
                                  out=out.t, lse=lse.t, workspace=ws.t)
    ref, _ = T.tq_decode_attention(ctx, q, packed, batch, hq, hkv, max_len, seq_lens=lens)
    T.tq_check_device(ctx)
    for name, gb in (("out", out), ("scores", scores), ("lse", lse), ("workspace", ws)):
        assert gb.intact(), f"{name}: a guard byte changed"
    np.testing.assert_allclose(out.t.cpu().numpy(), ref.cpu().numpy(), rtol=1e-5, atol=1e-7)


def test_merge_and_decompress_writes_stay_in_their_arrays():
    R, rows, d = 3, 37, 128
    parts = torch.randn((R, rows, d), device=DEV)
    lses = torch.randn((R, rows), device=DEV)
    out, lse = Guarded((rows, d), torch.float32), Guarded((rows,), torch.float32)
    T.tq_merge_attention(parts, lses, out=out.t, lse=lse.t)
    torch.cuda.synchronize()
    assert out.intact() and lse.intact()

    n = 1001
    ctx = make_ctx(T, d, 2, 4)
    packed = _random_cache(1, n, d, 2, 4, seed=37)
    kx, vx = Guarded((n, d), torch.float32), Guarded((n, d), torch.float32)
    T.tq_decompress(ctx, packed, n, k_out=kx.t, v_out=vx.t)
    torch.cuda.synchronize()
    assert kx.intact() and vx.intact()
