"""GPU tests of the append / paged-cache calls (through the C ABI).

tq_compress_kv_slots writes each vector's records at a caller-chosen row (appending to a
growing cache, filling pages); tq_decode_attention_paged reads a cache scattered over pages
through a block table. Compression is per vector, so the slot-mapped records must equal the
contiguous ones bit for bit. The decode kernels walk the same tiles under either addressing:
scores and outputs must be bit-identical (every partial sum is added in a fixed order), and
the paged decode is also checked against the oracle."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _parity import assert_close, make_ctx, oracle_setup, to_np

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_cache_vector_05_b200 as T  # noqa: E402

DEV = "cuda:0"
SENTINEL = 0xA5


def _empty_cache(ctx, n_rows):
    """Packed arrays of n_rows records, every byte SENTINEL."""
    def full(shape, dtype):
        t = torch.empty(shape, dtype=torch.uint8, device=DEV).fill_(SENTINEL)
        return t.view(dtype) if dtype != torch.uint8 else t
    return {"k_codes": full((n_rows, ctx.k_code_bytes), torch.uint8),
            "k_signs": full((n_rows, ctx.m // 8), torch.uint8),
            "k_norms": full((n_rows, 4), torch.int16).view(n_rows, 2),
            "v_codes": full((n_rows, ctx.v_code_bytes), torch.uint8),
            "v_params": full((n_rows, (ctx.d // ctx.v_group) * 4), torch.int16).view(n_rows, ctx.d // ctx.v_group, 2)}


def _rows_equal(a: np.ndarray, b: np.ndarray) -> bool:
    return np.array_equal(a.reshape(a.shape[0], -1).view(np.uint8), b.reshape(b.shape[0], -1).view(np.uint8))


@pytest.mark.parametrize("d,lm_bits,v_bits,rotation,dtype", [
    (128, 2, 2, "hadamard", "bf16"),   # pipelined tensor-core kernel
    (128, 1, 4, "hadamard", "bf16"),
    (128, 2, 4, "hadamard", "f32"),    # four lanes per vector, tensor-core projection
    (128, 2, 2, "haar", "bf16"),       # tensor-core Haar rotation
    (128, 3, 2, "haar", "f32"),        # CUDA-core rotation, tensor-core projection
    (64, 2, 4, "hadamard", "bf16"),    # warp per vector
    (256, 1, 2, "haar", "f32"),
])
def test_compress_slots_reproduce_contiguous_rows(d, lm_bits, v_bits, rotation, dtype):
    n = 148 * 128 * 2 + 7 * 128 + 77     # several passes per CTA and a ragged tail
    n_rows = n + 5000
    ctx = make_ctx(T, d, lm_bits, v_bits, rotation=rotation)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    gen = torch.Generator(device=DEV)
    gen.manual_seed(d + lm_bits)
    K = (torch.randn((n, d), generator=gen, device=DEV) * 2.0).to(tdt)
    V = torch.randn((n, d), generator=gen, device=DEV).to(tdt)
    K[[0, 999, n - 1]] = 0
    ref = to_np(T.tq_compress_kv(ctx, K, V))
    perm = np.random.default_rng(d).permutation(n_rows)[:n]
    slot = torch.from_numpy(perm.astype(np.int64)).to(DEV)
    cache = _empty_cache(ctx, n_rows)
    T.tq_compress_kv_slots(ctx, K, V, slot, cache)
    T.tq_check_device(ctx)
    got = to_np(cache)
    untouched = np.setdiff1d(np.arange(n_rows), perm)
    for name in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params"):
        assert _rows_equal(got[name][perm], ref[name]), name
        assert (got[name][untouched].reshape(untouched.size, -1).view(np.uint8) == SENTINEL).all(), name


def test_compress_slots_keys_and_values_separately_and_bad_slot():
    d, n = 128, 3000
    ctx = make_ctx(T, d, 2, 2)
    K = torch.randn((n, d), device=DEV).to(torch.bfloat16)
    V = torch.randn((n, d), device=DEV).to(torch.bfloat16)
    ref = to_np(T.tq_compress_kv(ctx, K, V))
    slot = torch.arange(n - 1, -1, -1, dtype=torch.int64, device=DEV)   # reversed
    cache = _empty_cache(ctx, n)
    T.tq_compress_kv_slots(ctx, K, None, slot, cache)
    T.tq_compress_kv_slots(ctx, None, V, slot, cache)
    T.tq_check_device(ctx)
    got = to_np(cache)
    for name in ref:
        assert _rows_equal(got[name][::-1], ref[name]), name
    bad = slot.clone()
    bad[17] = n                                                           # one row past the end
    cache2 = _empty_cache(ctx, n)
    T.tq_compress_kv_slots(ctx, K, V, bad, cache2)
    with pytest.raises(T.TQError):
        T.tq_check_device(ctx)
    got2 = to_np(cache2)
    keep = np.array([i for i in range(n) if i != 17])
    for name in ref:                                                      # the others are written
        assert _rows_equal(got2[name][n - 1 - keep], ref[name][keep]), name
    with pytest.raises(T.TQError):
        T.tq_compress_kv_slots(ctx, K, V, slot, {k: v[:0] for k, v in cache.items()})  # n_rows = 0


def test_append_in_place_equals_one_shot():
    """A [batch][hkv][max_len] cache filled in two appends (a prefix, then new tokens after
    each sequence's end) holds the same bytes as compressing every token at once."""
    d, batch, hkv, max_len = 128, 3, 2, 4096
    lens0, lens1 = [1000, 2049, 3], [777, 1, 4000]
    ctx = make_ctx(T, d, 2, 2)
    units = batch * hkv
    full = torch.randn((units, max_len, d), device=DEV).to(torch.bfloat16)
    once = to_np(T.tq_compress_kv(ctx, full.view(-1, d), full.view(-1, d)))
    cache = _empty_cache(ctx, units * max_len)

    def append(starts, counts):
        rows, src = [], []
        for u in range(units):
            b = u // hkv
            t = np.arange(starts[b], starts[b] + counts[b])
            rows.append(u * max_len + t)
            src.append(full[u, starts[b]:starts[b] + counts[b]])
        slot = torch.from_numpy(np.concatenate(rows).astype(np.int64)).to(DEV)
        x = torch.cat(src).contiguous()
        T.tq_compress_kv_slots(ctx, x, x, slot, cache)

    append([0] * batch, lens0)
    append(lens0, lens1)
    T.tq_check_device(ctx)
    got = to_np(cache)
    for u in range(units):
        b = u // hkv
        rows = np.arange(u * max_len, u * max_len + lens0[b] + lens1[b])
        for name in once:
            assert _rows_equal(got[name][rows], once[name][rows]), (u, name)


def _paged_copy(packed: dict, units: int, max_len: int, page_size: int, extra_pages: int, seed: int):
    """Scatter a contiguous [units][max_len] cache over shuffled pages; returns the paged
    arrays, the block table [units][max_pages] and the page count."""
    max_pages = (max_len + page_size - 1) // page_size
    n_pages = units * max_pages + extra_pages
    order = np.random.default_rng(seed).permutation(n_pages)[:units * max_pages]
    table = order.reshape(units, max_pages).astype(np.int32)
    paged = {}
    for name, a in packed.items():
        rec = a.reshape(a.shape[0], -1)
        out = np.zeros((n_pages * page_size, rec.shape[1]), dtype=rec.dtype)
        for u in range(units):
            for j in range(max_pages):
                t0 = j * page_size
                n = min(page_size, max_len - t0)
                p = table[u, j]
                out[p * page_size:p * page_size + n] = rec[u * max_len + t0:u * max_len + t0 + n]
        paged[name] = out.reshape((n_pages * page_size,) + a.shape[1:])
    return paged, table, n_pages


def _upload(packed: dict):
    out = {}
    for k, v in packed.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(DEV)
    return out


@pytest.mark.parametrize("d,lm_bits,v_bits,G,page_size", [
    (128, 2, 2, 4, 512),     # tensor-core decode, 512-token tiles
    (128, 2, 4, 8, 1024),    # tensor-core decode, 256-token tiles
    (128, 3, 4, 6, 512),     # generic decode (3-bit Lloyd-Max codes)
    (64, 2, 2, 4, 512),      # generic decode, d = 64
])
def test_paged_decode_equals_contiguous_and_oracle(d, lm_bits, v_bits, G, page_size):
    batch, hkv, max_len = 3, 2, 2600
    lens = [2600, 1537, 0]
    hq, units = hkv * G, batch * hkv
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = W.random_packed_cache(units * max_len, d, lm_bits, d, v_bits, seed=11)
    q = torch.from_numpy(W.queries((batch, hq, d), dtype="f32")).to(DEV)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    sc_c = torch.full((batch, hq, max_len), float("nan"), device=DEV)
    out_c, _ = T.tq_decode_attention(ctx, q, _upload(packed), batch, hq, hkv, max_len, seq_lens=lens_t,
                                     scores=sc_c)
    paged, table, n_pages = _paged_copy(packed, units, max_len, page_size, extra_pages=3, seed=d + G)
    bt = torch.from_numpy(table.reshape(batch, hkv, -1)).to(DEV)
    sc_p = torch.full((batch, hq, max_len), float("nan"), device=DEV)
    out_p, _ = T.tq_decode_attention_paged(ctx, q, _upload(paged), batch, hq, hkv, max_len, bt, page_size,
                                           n_pages, seq_lens=lens_t, scores=sc_p)
    T.tq_check_device(ctx)
    oc, op = out_c.cpu().numpy(), out_p.cpu().numpy()
    np.testing.assert_array_equal(op, oc)                                 # bit for bit
    assert np.array_equal(np.isnan(sc_c.cpu().numpy()), np.isnan(sc_p.cpu().numpy()))
    assert np.array_equal(np.nan_to_num(sc_c.cpu().numpy()), np.nan_to_num(sc_p.cpu().numpy()))
    Pi, c, t, S = oracle_setup(d, lm_bits)
    qn = q.cpu().numpy()
    for u in (0, 3):                                                      # and the oracle
        b, kvh = divmod(u, hkv)
        sl = slice(u * max_len, u * max_len + lens[b])
        pk = {"codes": packed["k_codes"][sl], "signs": packed["k_signs"][sl], "norms": packed["k_norms"][sl]}
        pv = {"codes": packed["v_codes"][sl], "params": packed["v_params"][sl]}
        os_, oo = O.decode_attention(qn[b, kvh * G:(kvh + 1) * G].astype(np.float64), pk, pv, Pi, c, S, d,
                                     v_bits)
        assert_close(op[b, kvh * G:(kvh + 1) * G], oo, what=f"paged out unit {u}")


def test_paged_decode_rejects_bad_arguments_and_flags_bad_pages():
    d, batch, hkv, G, max_len, page_size = 128, 1, 1, 4, 1024, 512
    ctx = make_ctx(T, d, 2, 2)
    packed = _upload(W.random_packed_cache(max_len, d, 2, d, 2, seed=3))
    q = torch.randn((batch, hkv * G, d), device=DEV)
    bt = torch.tensor([[[0, 1]]], dtype=torch.int32, device=DEV)
    with pytest.raises(T.TQError):                                        # not a multiple of 512
        T.tq_decode_attention_paged(ctx, q, packed, batch, hkv * G, hkv, max_len, bt, 256, 4)
    with pytest.raises(T.TQError):                                        # too few table entries
        T.tq_decode_attention_paged(ctx, q, packed, batch, hkv * G, hkv, max_len, bt[:, :, :1].contiguous(),
                                    page_size, 2)
    bad = torch.tensor([[[0, 7]]], dtype=torch.int32, device=DEV)          # page 7 of 2
    T.tq_decode_attention_paged(ctx, q, packed, batch, hkv * G, hkv, max_len, bad, page_size, 2)
    with pytest.raises(T.TQError):
        T.tq_check_device(ctx)
    out, _ = T.tq_decode_attention_paged(ctx, q, packed, batch, hkv * G, hkv, max_len, bt, page_size, 2)
    T.tq_check_device(ctx)                                                # the context is still usable
    ref, _ = T.tq_decode_attention(ctx, q, packed, batch, hkv * G, hkv, max_len)
    np.testing.assert_array_equal(out.cpu().numpy(), ref.cpu().numpy())


@pytest.mark.parametrize("d,lm_bits,v_bits,G", [(128, 2, 2, 4), (128, 2, 4, 8), (128, 3, 4, 6)])
def test_decode_is_bit_reproducible(d, lm_bits, v_bits, G):
    """The same call twice gives the same bits (no order-dependent floating-point sums),
    on a cache long enough that several CTAs share each unit."""
    batch, hkv, max_len = 2, 2, 40000
    hq = hkv * G
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = _upload(W.random_packed_cache(batch * hkv * max_len, d, lm_bits, d, v_bits, seed=17))
    q = torch.from_numpy(W.queries((batch, hq, d), seed=5)).to(DEV)
    outs = []
    for _ in range(3):
        o, _ = T.tq_decode_attention(ctx, q, packed, batch, hq, hkv, max_len)
        outs.append(o.cpu().numpy())
    T.tq_check_device(ctx)
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])
