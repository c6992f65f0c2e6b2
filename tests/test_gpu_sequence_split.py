"""GPU tests of decoding a sequence whose cache is split by token range (through the C ABI).

tq_decode_attention_partial returns, besides the attention output over its own cache,
each row's log-partition; tq_merge_attention combines the parts of disjoint token
ranges. Several ranks are emulated on one GPU by decoding each rank's range in turn
(independent launches: nothing waits on another launch) into one gathered buffer laid
out as the all-gather leaves it; the merge must reproduce the decode over the whole
cache and the oracle's decode, and the log-partitions must match the oracle's."""
import numpy as np
import pytest

import oracle as O
import workloads as W
from _parity import assert_close, make_ctx, oracle_setup

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_cache_vector_05_b200 as T  # noqa: E402
from kv_cache_vector_05_b200.sequence_split import SplitSequenceDecoder, local_lengths, token_range  # noqa: E402

DEV = "cuda:0"


def _upload(packed: dict):
    out = {}
    for k, v in packed.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(DEV)
    return out


def _token_slice(packed: dict, units: int, max_len: int, a: int, b: int) -> dict:
    """Records of tokens [a, b) of every unit, as a cache of b - a slots per unit."""
    out = {}
    for k, v in packed.items():
        per = v.reshape((units, max_len) + v.shape[1:])
        out[k] = np.ascontiguousarray(per[:, a:b].reshape((units * (b - a),) + v.shape[1:]))
    return out


def _oracle_unit(packed, u, max_len, length, qn, Pi, c, S, d, v_bits):
    sl = slice(u * max_len, u * max_len + length)
    pk = {"codes": packed["k_codes"][sl], "signs": packed["k_signs"][sl], "norms": packed["k_norms"][sl]}
    pv = {"codes": packed["v_codes"][sl], "params": packed["v_params"][sl]}
    sc, out = O.decode_attention(qn, pk, pv, Pi, c, S, d, v_bits)
    return out, O.log_partition(sc)


CASES = [
    (128, 2, 2, 4, True),     # tensor-core decode
    (128, 1, 4, 8, True),
    (128, 3, 4, 6, True),     # the long-context shape's codes (generic decode)
    (64, 2, 2, 4, True),      # generic decode at d = 64
    (128, 3, 2, 4, False),    # Lloyd-Max keys without the QJL stage
]


@pytest.mark.parametrize("d,lm_bits,v_bits,G,qjl", CASES)
def test_partial_decode_returns_the_log_partition(d, lm_bits, v_bits, G, qjl):
    batch, hkv, max_len = 3, 2, 1300
    lens = [1300, 517, 0]
    hq, units, m = hkv * G, batch * hkv, d if qjl else 0
    ctx = make_ctx(T, d, lm_bits, v_bits) if qjl else _ctx_no_qjl(d, lm_bits, v_bits)
    packed = W.random_packed_cache(units * max_len, d, lm_bits, m, v_bits, seed=17)
    q = torch.from_numpy(W.queries((batch, hq, d), dtype="f32")).to(DEV)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out, lse, _ = T.tq_decode_attention_partial(ctx, q, _upload(packed), batch, hq, hkv, max_len, seq_lens=lens_t)
    ref, _ = T.tq_decode_attention(ctx, q, _upload(packed), batch, hq, hkv, max_len, seq_lens=lens_t)
    T.tq_check_device(ctx)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    np.testing.assert_allclose(out, ref.cpu().numpy(), rtol=1e-5, atol=1e-7)
    assert np.all(lse[2] == -np.inf) and not out[2].any()               # empty sequence
    Pi, c, t, S = oracle_setup(d, lm_bits)
    if not qjl:
        S = np.zeros((0, d))
    qn = q.cpu().numpy().astype(np.float64)
    for u in (0, 1, 3):
        b, kvh = divmod(u, hkv)
        oo, ol = _oracle_unit(packed, u, max_len, lens[b], qn[b, kvh * G:(kvh + 1) * G], Pi, c, S, d, v_bits)
        assert_close(out[b, kvh * G:(kvh + 1) * G], oo, what=f"out unit {u}")
        assert_close(lse[b, kvh * G:(kvh + 1) * G], ol, what=f"lse unit {u}")


def _ctx_no_qjl(d, lm_bits, v_bits):
    """Lloyd-Max keys only (qjl_m = 0), from the same seeded draws as make_ctx."""
    dr = W.method_draws(d, d, 1234)
    c, t = T.tq_lloyd_max_codebook(d, lm_bits)
    return T.tq_codebook_load(d, lm_bits, v_bits, c, t, np.zeros((0, d)), hadamard_signs=dr["hadamard_signs"])


@pytest.mark.parametrize("d,lm_bits,v_bits,G,qjl", CASES[:3])
@pytest.mark.parametrize("world", [1, 3, 4, 8])
def test_split_over_ranks_equals_whole_decode(d, lm_bits, v_bits, G, qjl, world):
    """The cache of 2 sequences x 2 KV heads x 2600 tokens split into `world` token
    ranges of whole 512-token blocks (the last rank's range ragged, some sequences
    shorter than the later ranges' starts, and at 8 ranks the last two with no tokens);
    each range decoded on its own into a gathered buffer with a padded per-rank stride,
    then merged."""
    batch, hkv, max_len = 2, 2, 2600
    lens = [2600, 700]
    hq, units = hkv * G, batch * hkv
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = W.random_packed_cache(units * max_len, d, lm_bits, d, v_bits, seed=23)
    q = torch.from_numpy(W.queries((batch, hq, d), seed=3, dtype="bf16")).to(DEV).to(torch.bfloat16)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    rows = batch * hq
    stride = rows * d + 4 * (-(-rows // 4)) + 16                         # padded part, 16-byte multiple
    buf = torch.full((world, stride), float("nan"), device=DEV)
    outs = buf[:, : rows * d].view(world, batch, hq, d)
    lses = buf[:, rows * d: rows * d + rows].view(world, batch, hq)
    for r in range(world):
        a, b = token_range(max_len, world, r, 512)
        if b > a:
            part = _upload(_token_slice(packed, units, max_len, a, b))
            T.tq_decode_attention_partial(ctx, q, part, batch, hq, hkv, b - a, seq_lens=local_lengths(lens_t, a, b),
                                          out=outs[r], lse=lses[r])
        else:                                                            # a rank without tokens
            none = {k: None for k in packed}
            T.tq_decode_attention_partial(ctx, q, none, batch, hq, hkv, 0, out=outs[r], lse=lses[r])
    merged, mlse = T.tq_merge_attention(outs, lses, lse=torch.empty((batch, hq), device=DEV))
    whole, _ = T.tq_decode_attention(ctx, q, _upload(packed), batch, hq, hkv, max_len, seq_lens=lens_t)
    T.tq_check_device(ctx)
    mo = merged.cpu().numpy()
    np.testing.assert_allclose(mo, whole.cpu().numpy(), rtol=2e-5, atol=1e-6)
    Pi, c, t, S = oracle_setup(d, lm_bits)
    qn = q.float().cpu().numpy().astype(np.float64)
    ml = mlse.cpu().numpy()
    for u in range(units):
        b, kvh = divmod(u, hkv)
        oo, ol = _oracle_unit(packed, u, max_len, lens[b], qn[b, kvh * G:(kvh + 1) * G], Pi, c, S, d, v_bits)
        assert_close(mo[b, kvh * G:(kvh + 1) * G], oo, what=f"merged out unit {u}")
        assert_close(ml[b, kvh * G:(kvh + 1) * G], ol, what=f"merged lse unit {u}")


def test_merge_kernel_matches_the_oracle():
    """Random parts with empty ranges (-inf), an all-empty row, log-partitions hundreds
    apart, one part alone, and d = 256."""
    rng = np.random.default_rng(5)
    for R, rows, d in [(5, 37, 128), (1, 9, 64), (3, 4, 256)]:
        o = rng.standard_normal((R, rows, d)).astype(np.float32)
        ls = (rng.standard_normal((R, rows)) * 4).astype(np.float32)
        if R > 1:
            ls[1, :] = -np.inf                                           # one rank empty everywhere
            ls[:, 2] = -np.inf                                           # a row empty on every rank
            ls[0, 3], ls[-1, 3] = 300.0, -300.0                          # far apart
        out, lse = T.tq_merge_attention(torch.from_numpy(o).to(DEV), torch.from_numpy(ls).to(DEV),
                                        lse=torch.empty(rows, device=DEV))
        want_o, want_l = O.merge_attention(o.astype(np.float64), ls.astype(np.float64))
        got_o, got_l = out.cpu().numpy(), lse.cpu().numpy()
        np.testing.assert_allclose(got_o, want_o, rtol=1e-5, atol=1e-6)
        finite = np.isfinite(want_l)
        assert np.array_equal(np.isfinite(got_l), finite)
        np.testing.assert_allclose(got_l[finite], want_l[finite], rtol=1e-6, atol=1e-5)
        if R > 1:
            assert not got_o[2].any()


def test_zero_length_cache_gives_zero_output_and_empty_log_partition():
    d, batch, hkv, G = 128, 2, 1, 4
    ctx = make_ctx(T, d, 2, 2)
    q = torch.randn((batch, hkv * G, d), device=DEV)
    none = {k: None for k in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params")}
    out = torch.full((batch, hkv * G, d), float("nan"), device=DEV)
    out, lse, _ = T.tq_decode_attention_partial(ctx, q, none, batch, hkv * G, hkv, 0, out=out)
    T.tq_check_device(ctx)
    assert not out.cpu().numpy().any() and np.all(lse.cpu().numpy() == -np.inf)


def test_split_sequence_decoder_in_one_process():
    """SplitSequenceDecoder without a process group (world 1): its part buffer, the
    (skipped) exchange and the merge give the plain decode."""
    d, lm_bits, v_bits, G, batch, hkv, max_len = 128, 2, 2, 4, 2, 2, 1500
    ctx = make_ctx(T, d, lm_bits, v_bits)
    packed = _upload(W.random_packed_cache(batch * hkv * max_len, d, lm_bits, d, v_bits, seed=29))
    q = torch.from_numpy(W.queries((batch, hkv * G, d), seed=4, dtype="f32")).to(DEV)
    lens = torch.tensor([1500, 333], dtype=torch.int32, device=DEV)
    dec = SplitSequenceDecoder(batch, hkv * G, d, device=DEV)
    got = dec(ctx, q, packed, hkv, max_len, seq_lens=lens)
    want, _ = T.tq_decode_attention(ctx, q, packed, batch, hkv * G, hkv, max_len, seq_lens=lens)
    T.tq_check_device(ctx)
    np.testing.assert_allclose(got.cpu().numpy(), want.cpu().numpy(), rtol=1e-5, atol=1e-7)
