"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs. Packed bytes must match under the exemption rule; scores and
attention outputs from identical packed inputs within |g - o| <= 1e-4 + 1e-3 |o|."""
import math

import numpy as np
import pytest

import oracle as O
import workloads as W
from _parity import (assert_close, assert_key_parity, assert_value_parity, compare_keys,
                     compare_values, make_ctx, oracle_setup, to_np)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_cache_vector_05_b200 as T  # noqa: E402

DEV = "cuda:0"


def _compress_both(K, V, d, lm_bits, v_bits, rotation, dtype, m=None):
    m = m or d
    ctx = make_ctx(T, d, lm_bits, v_bits, m, rotation)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    kt = torch.from_numpy(np.ascontiguousarray(K, np.float32)).to(DEV).to(tdt)
    vt = torch.from_numpy(np.ascontiguousarray(V, np.float32)).to(DEV).to(tdt)
    g = to_np(T.tq_compress_kv(ctx, kt, vt))
    T.tq_check_device(ctx)                                  # no bounded wait gave up
    Pi, c, t, S = oracle_setup(d, lm_bits, m, rotation)
    # the oracle sees exactly the values the device read
    Kx = kt.float().cpu().numpy().astype(np.float64)
    Vx = vt.float().cpu().numpy().astype(np.float64)
    ok = O.compress_keys(Kx, Pi, c, t, S, with_diagnostics=True)
    ov = O.quantize_values(Vx, v_bits, with_diagnostics=True)
    return ctx, g, ok, ov


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("lm_bits", [1, 2, 3])
@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_compress_parity_small(d, lm_bits, rotation, dtype):
    v_bits = 2 if (d + lm_bits) % 2 else 4
    n = 1531                                            # several CTAs plus a ragged tail
    rng = np.random.default_rng([d, lm_bits])
    K = rng.standard_normal((n, d)).astype(np.float32) * rng.lognormal(0, 1, d).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    K[[0, 700, n - 1]] = 0.0                             # zero keys
    V[5, :32] = 0.75                                     # a constant value group
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, dtype)
    ks = compare_keys(g, ok, d, lm_bits, d)
    vs = compare_values(g, ov, d, v_bits)
    assert_key_parity(ks)
    assert_value_parity(vs)


def test_compress_parity_qwen_outlier_keys():
    """One (layer, head) of the Qwen2.5-3B-shaped cache: lognormal channel scales with x20 outliers."""
    K, V = W.qwen_layer_head_kv(layer=17, head=1)
    ctx, g, ok, ov = _compress_both(K, V, 128, 2, 2, "hadamard", "bf16")
    assert_key_parity(compare_keys(g, ok, 128, 2, 128))
    assert_value_parity(compare_values(g, ov, 128, 2))


@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
def test_compress_parity_full_sweep_size_sampled(rotation):
    """1,048,576 bf16 N(0,1) vectors (16384 tokens x 64 heads), d=128, 3-bit keys:
    the whole batch is compressed in one call; the oracle checks a sample."""
    d, lm_bits, v_bits, n = 128, 2, 2, W.SWEEP_VECTORS
    ctx = make_ctx(T, d, lm_bits, v_bits, rotation=rotation)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(0)
    kt = torch.randn((n, d), generator=gen, device=DEV).to(torch.bfloat16)
    vt = torch.randn((n, d), generator=gen, device=DEV).to(torch.bfloat16)
    g = T.tq_compress_kv(ctx, kt, vt)
    torch.cuda.synchronize()
    idx = np.unique(np.concatenate([np.random.default_rng(1).integers(0, n, 12000), [0, n - 1]]))
    it = torch.from_numpy(idx).to(DEV)
    gs = to_np({k: v[it] for k, v in g.items()})
    Pi, c, t, S = oracle_setup(d, lm_bits, d, rotation)
    Kx = kt[it].float().cpu().numpy().astype(np.float64)
    Vx = vt[it].float().cpu().numpy().astype(np.float64)
    ks = compare_keys(gs, O.compress_keys(Kx, Pi, c, t, S, with_diagnostics=True), d, lm_bits, d)
    vs = compare_values(gs, O.quantize_values(Vx, v_bits, with_diagnostics=True), d, v_bits)
    assert_key_parity(ks)
    assert_value_parity(vs)


@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("lm_bits", [1, 2, 3])
def test_compress_parity_several_passes_per_cta(lm_bits, rotation):
    """bf16 keys, d = 128 (Hadamard: H diag(sigma) as one bf16 operand tile; Haar: three
    tiles): enough vectors for two to three passes of 128 on every CTA and a ragged last
    pass, so the double-buffered key tiles, tensor-memory halves and value halves all turn
    over; every vector is compared. Then keys alone and values alone."""
    d, v_bits = 128, (4 if lm_bits == 2 else 2)
    n = 148 * 128 * 2 + 7 * 128 + 77
    rng = np.random.default_rng([7, lm_bits])
    K = rng.standard_normal((n, d)).astype(np.float32) * rng.lognormal(0, 1, d).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32) * 3.0 + 1.0
    K[[0, 128 * 148, n - 1]] = 0.0
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, "bf16")
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    kt = torch.from_numpy(K).to(DEV).to(torch.bfloat16)
    vt = torch.from_numpy(V).to(DEV).to(torch.bfloat16)
    gk = to_np(T.tq_compress_kv(ctx, kt, None))
    gv = to_np(T.tq_compress_kv(ctx, None, vt))
    T.tq_check_device(ctx)
    for name in ("k_codes", "k_signs", "k_norms"):
        assert np.array_equal(gk[name], g[name]), name    # same kernel work, keys only
    for name in ("v_codes", "v_params"):
        assert np.array_equal(gv[name], g[name]), name


@pytest.mark.parametrize("lm_bits,rotation", [(2, "hadamard"), (3, "haar"), (1, "hadamard")])
def test_compress_three_bit_values_pipelined_several_passes(lm_bits, rotation):
    """3-bit value codes (fields straddling 32-bit words, the near-tie redo across a word
    boundary) on the pipelined kernel's value warps, bf16, d = 128, with the QJL stage: two to
    three passes per CTA, every vector against the oracle, values alone and keys alone
    giving the same records as the call with both."""
    d, v_bits = 128, 3
    n = 148 * 128 * 2 + 3 * 128 + 45
    rng = np.random.default_rng([43, lm_bits])
    K = rng.standard_normal((n, d)).astype(np.float32) * rng.lognormal(0, 1, d).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    V[7, :32] = 0.25                                      # a constant value group
    V[9, 32:64] = np.arange(32, dtype=np.float32) / 7.0  # codes on exact half steps
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, "bf16")
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    kt = torch.from_numpy(K).to(DEV).to(torch.bfloat16)
    vt = torch.from_numpy(V).to(DEV).to(torch.bfloat16)
    gk = to_np(T.tq_compress_kv(ctx, kt, None))
    gv = to_np(T.tq_compress_kv(ctx, None, vt))
    T.tq_check_device(ctx)
    for name in ("k_codes", "k_signs", "k_norms"):
        assert np.array_equal(gk[name], g[name]), name
    for name in ("v_codes", "v_params"):
        assert np.array_equal(gv[name], g[name]), name


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("lm_bits", [1, 3])
def test_compress_dense_tensor_core_several_passes(d, rotation, lm_bits):
    """bf16 keys at d = 64 and 256 take the dense tensor-core kernel (rotation and QJL
    projection as tcgen05 MMAs; at d = 256 the operand tiles stream through a ring of three
    shared-memory slots): two to three passes of 128 keys per CTA and a ragged last pass,
    zero keys, every vector compared; values in the same call (warp-per-vector kernel)."""
    v_bits = 2
    n = 148 * 128 * 2 + 333
    rng = np.random.default_rng([d, lm_bits, 5])
    K = rng.standard_normal((n, d)).astype(np.float32) * rng.lognormal(0, 1, d).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    K[[0, 128 * 148 + 5, n - 1]] = 0.0
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, "bf16")
    ks = compare_keys(g, ok, d, lm_bits, d)
    assert_key_parity(ks)
    assert ks["sign_bad"] == 0, ks
    assert_value_parity(compare_values(g, ov, d, v_bits))


@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
def test_compress_parity_asymmetric_codebook(rotation):
    """A codebook that is not symmetric about zero (one outer centroid and boundary moved)
    takes the general bucketize (one pass at a time); bf16 keys, d = 128, several passes per
    CTA."""
    d, lm_bits, v_bits = 128, 2, 2
    dr = W.method_draws(d, d, 1234)
    c32, t32 = T.tq_lloyd_max_codebook(d, lm_bits)
    c32, t32 = c32.copy(), t32.copy()
    c32[0] = np.float32(c32[0] * 1.25)
    t32[0] = np.float32(0.5 * (float(c32[0]) + float(c32[1])))
    haar = T.tq_haar_from_gaussian(dr["haar_gaussian"]) if rotation == "haar" else None
    ctx = T.tq_codebook_load(d, lm_bits, v_bits, c32, t32, dr["qjl_S"], rotation=rotation,
                             hadamard_signs=dr["hadamard_signs"], haar=haar)
    n = 148 * 128 * 2 + 333
    rng = np.random.default_rng(99)
    K = rng.standard_normal((n, d)).astype(np.float32)
    kt = torch.from_numpy(K).to(DEV).to(torch.bfloat16)
    g = to_np(T.tq_compress_kv(ctx, kt, None))
    T.tq_check_device(ctx)
    Pi = (O.hadamard_rotation(dr["hadamard_signs"]) if rotation == "hadamard"
          else O.haar_rotation(dr["haar_gaussian"]))
    ok = O.compress_keys(kt.float().cpu().numpy().astype(np.float64), Pi, c32.astype(np.float64),
                         t32.astype(np.float64), dr["qjl_S"], with_diagnostics=True)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
def test_compress_unrounded_gaussian_S(dtype, rotation):
    """The QJL matrix is a plain fp32 N(0,1) draw (almost none of its entries lie on the
    f16 grid): the tensor-core kernels take it as two f16 terms. d = m = 128, several passes
    per CTA, every vector compared."""
    d, lm_bits, v_bits = 128, 2, 2
    S = W.method_draws(d, d, 1234)["qjl_S"]
    assert np.mean(S.astype(np.float16).astype(np.float64) == S) < 0.01
    n = 148 * 128 + 5 * 128 + 19
    rng = np.random.default_rng([11, d])
    K = rng.standard_normal((n, d)).astype(np.float32) * rng.lognormal(0, 1, d).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, dtype)
    ks = compare_keys(g, ok, d, lm_bits, d)
    assert_key_parity(ks)
    assert ks["sign_bad"] == 0, ks
    assert_value_parity(compare_values(g, ov, d, v_bits))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_compress_S_beyond_f16_range_takes_the_warp_per_vector_kernel(dtype):
    """An S entry beyond the f16 range cannot be an f16 operand term: the call falls back to
    the warp-per-vector kernel (CUDA-core projection), which must agree with the oracle too."""
    d, lm_bits, v_bits = 128, 2, 2
    dr = W.method_draws(d, d, 1234)
    S = dr["qjl_S"].copy()
    S[5, 7] = 1.0e5                                       # exact in fp32, above 65504
    c32, t32 = T.tq_lloyd_max_codebook(d, lm_bits)
    ctx = T.tq_codebook_load(d, lm_bits, v_bits, c32, t32, S, rotation="hadamard",
                             hadamard_signs=dr["hadamard_signs"])
    n = 2 * 148 * 8 + 13
    rng = np.random.default_rng([12, d])
    K = rng.standard_normal((n, d)).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    kt = torch.from_numpy(K).to(DEV).to(tdt)
    vt = torch.from_numpy(V).to(DEV).to(tdt)
    g = to_np(T.tq_compress_kv(ctx, kt, vt))
    T.tq_check_device(ctx)
    Pi = O.hadamard_rotation(dr["hadamard_signs"])
    c, t = O.device_codebook(d, lm_bits)
    ok = O.compress_keys(kt.float().cpu().numpy().astype(np.float64), Pi, c, t, S, with_diagnostics=True)
    ov = O.quantize_values(vt.float().cpu().numpy().astype(np.float64), v_bits, with_diagnostics=True)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))
    assert_value_parity(compare_values(g, ov, d, v_bits))


def test_compress_edge_cases():
    ctx = make_ctx(T, 128, 2, 2)
    empty = torch.empty((0, 128), device=DEV)
    T.tq_compress_kv(ctx, empty, empty)                      # n = 0 is a no-op
    one = torch.randn((1, 128), device=DEV)
    g = to_np(T.tq_compress_kv(ctx, one, None))
    Pi, c, t, S = oracle_setup(128, 2)
    ok = O.compress_keys(one.cpu().numpy().astype(np.float64), Pi, c, t, S, with_diagnostics=True)
    assert_key_parity(compare_keys(g, ok, 128, 2, 128))
    vals = torch.randn((300, 128), device=DEV).to(torch.bfloat16)   # values only, 3 passes
    gv = to_np(T.tq_compress_kv(ctx, None, vals))
    assert "k_codes" not in gv
    ov = O.quantize_values(vals.float().cpu().numpy().astype(np.float64), 2, with_diagnostics=True)
    assert_value_parity(compare_values(gv, ov, 128, 2))
    big = torch.randn((3, 129), device=DEV)
    misaligned = big.view(-1)[1:1 + 256].view(2, 128)       # 4-byte offset
    with pytest.raises(T.TQError):
        T.tq_compress_kv(ctx, misaligned, None)


# ------------------------------------------------------------------ decode

def _upload(packed: dict):
    out = {}
    for k, v in packed.items():
        a = np.ascontiguousarray(v)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[k] = torch.from_numpy(a).to(DEV)
    return out


def _oracle_unit(packed, u, max_len, length, q, Pi, c, S, d, v_bits, scale=None):
    sl = slice(u * max_len, u * max_len + length)
    pk = {"codes": packed["k_codes"][sl], "signs": packed["k_signs"][sl], "norms": packed["k_norms"][sl]}
    pv = {"codes": packed["v_codes"][sl], "params": packed["v_params"][sl]}
    return O.decode_attention(q, pk, pv, Pi, c, S, d, v_bits, scale=scale)


KERNELS = {"tcgen05": T.TQ_DECODE_TCGEN05, "mma": T.TQ_DECODE_MMA, "cuda_core": T.TQ_DECODE_CUDA_CORE}


def _decode_check(d, lm_bits, v_bits, batch, hkv, G, max_len, lens, rotation="hadamard",
                  q_dtype="f32", packed=None, units=None, scale=0.0, with_scores=True, kernel=None):
    m = d
    hq = hkv * G
    ctx = make_ctx(T, d, lm_bits, v_bits, m, rotation)
    if kernel is not None:
        T.tq_set_decode_kernel(ctx, KERNELS[kernel])
        if T.tq_decode_kernel_for(ctx, hq, hkv) != KERNELS[kernel]:
            pytest.skip(f"the {kernel} decode does not take this shape")
    n_vec = batch * hkv * max_len
    if packed is None:
        packed = W.random_packed_cache(n_vec, d, lm_bits, m, v_bits, seed=d + lm_bits)
    q = W.queries((batch, hq, d), dtype=q_dtype)
    qt = torch.from_numpy(q).to(DEV)
    if q_dtype == "bf16":
        qt = qt.to(torch.bfloat16)
    dp = _upload(packed)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    scores = torch.full((batch, hq, max_len), float("nan"), device=DEV) if with_scores else None
    out, _ = T.tq_decode_attention(ctx, qt, dp, batch, hq, hkv, max_len, seq_lens=lens_t,
                                   softmax_scale=scale, scores=scores)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    sc = scores.cpu().numpy() if with_scores else None
    Pi, c, t, S = oracle_setup(d, lm_bits, m, rotation)
    units = range(batch * hkv) if units is None else units
    for u in units:
        b, kvh = divmod(u, hkv)
        L = lens[b]
        qs = q[b, kvh * G:(kvh + 1) * G].astype(np.float64)
        os_, oo = _oracle_unit(packed, u, max_len, L, qs, Pi, c, S, d, v_bits,
                               scale=(scale if scale > 0 else None))
        assert_close(out[b, kvh * G:(kvh + 1) * G], oo, what=f"out unit {u}")
        if with_scores:
            assert_close(sc[b, kvh * G:(kvh + 1) * G, :L], os_, what=f"scores unit {u}")
            assert np.isnan(sc[b, kvh * G:(kvh + 1) * G, L:]).all()
    return out


def test_decode_single_head_fp32_oracle_compressed():
    """4096 fp32 N(0,1) keys/values, 8 queries on one head: 3-bit keys, 4-bit values;
    the packed cache comes from the oracle's own compression."""
    K, V, Q = W.single_head_kvq()
    Pi, c, t, S = oracle_setup(128, 2)
    pk = O.compress_keys(K.astype(np.float64), Pi, c, t, S)
    pv = O.quantize_values(V.astype(np.float64), 4)
    packed = {"k_codes": pk["codes"], "k_signs": pk["signs"], "k_norms": pk["norms"],
              "v_codes": pv["codes"], "v_params": pv["params"]}
    ctx = make_ctx(T, 128, 2, 4)
    qt = torch.from_numpy(Q).to(DEV).view(1, 8, 128)
    scores = torch.empty((1, 8, 4096), device=DEV)
    out, _ = T.tq_decode_attention(ctx, qt, _upload(packed), 1, 8, 1, 4096, scores=scores)
    torch.cuda.synchronize()
    os_, oo = O.decode_attention(Q.astype(np.float64), pk, pv, Pi, c, S, 128, 4)
    assert_close(scores.cpu().numpy()[0], os_, what="scores")
    assert_close(out.cpu().numpy()[0], oo, what="out")


@pytest.mark.parametrize("d,lm_bits,v_bits,G", [
    (128, 2, 2, 4), (128, 2, 2, 8), (128, 3, 4, 6), (128, 1, 4, 1),
    (128, 1, 2, 2), (128, 1, 2, 6), (128, 1, 4, 7), (128, 2, 4, 3), (128, 2, 4, 6), (128, 2, 2, 5),
    (64, 2, 4, 8), (64, 3, 2, 5), (256, 2, 2, 4), (256, 3, 4, 2), (256, 1, 2, 8),
])
def test_decode_parity_random_cache(d, lm_bits, v_bits, G):
    _decode_check(d, lm_bits, v_bits, batch=2, hkv=2, G=G, max_len=1100, lens=[1100, 577])


@pytest.mark.parametrize("kernel", ["tcgen05", "mma", "cuda_core"])
@pytest.mark.parametrize("lm_bits,v_bits,G", [(2, 2, 4), (2, 4, 8), (1, 2, 3), (3, 4, 6), (2, 2, 1), (2, 3, 4),
                                              (3, 3, 8)])
def test_decode_each_kernel_family(kernel, lm_bits, v_bits, G):
    """Every decode kernel family, selected explicitly, on the shapes it takes: the same
    packed cache decodes to the oracle's scores and outputs whichever kernel runs."""
    _decode_check(128, lm_bits, v_bits, batch=2, hkv=2, G=G, max_len=1500, lens=[1500, 701], kernel=kernel)


@pytest.mark.parametrize("lm_bits,v_bits,G", [(2, 2, 4), (2, 4, 8), (3, 4, 6), (2, 3, 4)])
def test_decode_variable_lengths_split_by_tokens(lm_bits, v_bits, G):
    """A batch of empty, one-token, partial and full sequences on the mma.sync decode, which
    splits the tiles that hold tokens (not every sequence's max_len) over its CTAs: fewer
    tiles than CTAs, CTAs whose range crosses several units, lengths that are not a multiple
    of 4 (the last tile's bulk copy rounds up), every row against the oracle."""
    _decode_check(128, lm_bits, v_bits, batch=7, hkv=2, G=G, max_len=2048,
                  lens=[0, 2048, 1, 0, 1501, 513, 7], kernel="mma")


def test_decode_many_sequences_split_scan():
    """1500 sequences of 0 to 300 tokens on the mma.sync decode: each of its 512 threads scans
    three sequences' lengths to find the CTA's first tile, and the combine kernel reads each
    sequence's first tile as the decode grid wrote it; rows on either side of the 512- and
    1024-sequence chunk edges and a seeded sample against the oracle."""
    batch = 1500
    lens = np.random.default_rng(31).integers(0, 301, batch)
    lens[[0, 511, 1024]] = 0
    lens[[1, 512, 1499]] = 300
    pick = sorted(set([0, 1, 2, 510, 511, 512, 513, 1023, 1024, 1025, 1499]
                      + list(np.random.default_rng(32).integers(0, batch, 12))))
    _decode_check(128, 2, 2, batch=batch, hkv=1, G=4, max_len=300, lens=[int(x) for x in lens],
                  kernel="mma", units=pick)


def test_decode_kernel_selection():
    """TQ_DECODE_AUTO takes the mma.sync kernel for 1- to 3-bit codes with the QJL stage
    (2- to 4-bit values),
    the tcgen05 kernel for keys without QJL, and the generic kernels for every other shape;
    an explicitly selected family that does not take the shape refuses the call."""
    ctx = make_ctx(T, 128, 2, 2)
    assert T.tq_decode_kernel_for(ctx, 32, 8) == T.TQ_DECODE_MMA
    assert T.tq_decode_kernel_for(ctx, 64, 2) == T.TQ_DECODE_CUDA_CORE        # G = 32
    ctx3 = make_ctx(T, 128, 3, 4)
    assert T.tq_decode_kernel_for(ctx3, 24, 4) == T.TQ_DECODE_MMA
    T.tq_set_decode_kernel(ctx3, T.TQ_DECODE_TCGEN05)
    assert T.tq_decode_kernel_for(ctx3, 24, 4) == T.TQ_DECODE_TCGEN05
    T.tq_set_decode_kernel(ctx3, T.TQ_DECODE_MMA)
    assert T.tq_decode_kernel_for(ctx3, 72, 4) == -1                          # G = 18
    packed = _upload(W.random_packed_cache(4 * 256, 128, 3, 128, 4))
    q = torch.randn((1, 72, 128), device=DEV)
    with pytest.raises(T.TQError):
        T.tq_decode_attention(ctx3, q, packed, 1, 72, 4, 256)
    T.tq_set_decode_kernel(ctx3, T.TQ_DECODE_AUTO)
    out, _ = T.tq_decode_attention(ctx3, q, packed, 1, 72, 4, 256)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    dr = W.method_draws(128, 128, 1234)
    c2, t2 = T.tq_lloyd_max_codebook(128, 2)
    ctx0 = T.tq_codebook_load(128, 2, 2, c2, t2, np.zeros((0, 128)), hadamard_signs=dr["hadamard_signs"])
    assert T.tq_decode_kernel_for(ctx0, 32, 8) == T.TQ_DECODE_TCGEN05
    ctx64 = make_ctx(T, 64, 2, 2)
    assert T.tq_decode_kernel_for(ctx64, 32, 8) == T.TQ_DECODE_CUDA_CORE
    ctx33 = make_ctx(T, 128, 2, 3)                                            # K = V = 3
    assert T.tq_decode_kernel_for(ctx33, 32, 8) == T.TQ_DECODE_MMA


@pytest.mark.parametrize("G", [4, 8])
def test_decode_ragged_sequences_many_tiles_per_cta(G):
    """Ragged sequence lengths with several tiles per CTA: the work split hands a CTA a
    range that runs from the ragged end of one (sequence, KV head) into the next one
    and wraps around its whole ring of stages, so plain-copied and bulk-copied tiles
    alternate in the same stage."""
    batch, hkv, max_len = 6, 8, 10240
    lens = [max_len - 37, max_len, max_len - 511, max_len - 1, 7000, max_len - 300]
    _decode_check(128, 2, 2, batch=batch, hkv=hkv, G=G, max_len=max_len, lens=lens,
                  units=list(range(0, batch * hkv, 3)) + [batch * hkv - 1])


def test_decode_parity_haar_bf16_queries_custom_scale():
    _decode_check(128, 2, 2, batch=1, hkv=3, G=4, max_len=700, lens=[699], rotation="haar",
                  q_dtype="bf16", scale=0.05)


def test_decode_empty_and_tiny_sequences():
    out = _decode_check(128, 2, 2, batch=3, hkv=1, G=4, max_len=130, lens=[0, 1, 130])
    assert not out[0].any()


@pytest.mark.parametrize("name,units", [
    ("qwen2.5-3b_8k_k3v2", [0, 71]),
    ("llama8b_b32_32k_k3v2", [0, 255]),
    ("long_1m_k4v4", [3]),
])
def test_decode_parity_full_size_sampled(name, units):
    """Full-size caches in the benchmark's launch configuration; the oracle
    recomputes every output of the sampled (sequence, KV head) units."""
    w = W.WORKLOADS[name]
    packed = W.random_packed_cache(w.units * w.tokens, w.d, w.lm_bits, w.m, w.v_bits, seed=11)
    lens = [w.tokens] * w.batch
    _decode_check(w.d, w.lm_bits, w.v_bits, w.batch, w.hkv, w.group, w.tokens, lens,
                  q_dtype=w.dtype, packed=packed, units=units, with_scores=(name != "long_1m_k4v4"))


@pytest.mark.parametrize("kernel", ["tcgen05", "mma", "cuda_core"])
@pytest.mark.parametrize("d,lm_bits,v_bits,G", [(128, 2, 2, 4), (128, 2, 4, 8), (128, 3, 4, 6)])
@pytest.mark.parametrize("k_norm_scale", [10.0, 30.0])
def test_decode_parity_large_key_norms(d, lm_bits, v_bits, G, k_norm_scale, kernel):
    """Key norms 10-30 times those of a unit-variance key (the Qwen-shaped cache's outlier
    channels give such norms): logits reach tens, the softmax is sharply peaked, and the
    online softmax rescales often. Some value groups get scales 100x larger, one a zero
    scale; the tensor-core decode (first two) and the generic decode (3-bit codes)."""
    batch, hkv, max_len = 2, 2, 3000
    n_vec = batch * hkv * max_len
    packed = W.random_packed_cache(n_vec, d, lm_bits, d, v_bits, seed=41, k_norm_scale=k_norm_scale)
    vp = packed["v_params"].view(np.float16).copy()
    rng = np.random.default_rng(42)
    big = rng.random(vp.shape[:2]) < 0.05
    vp[..., 0][big] = (vp[..., 0][big].astype(np.float64) * 100.0).astype(np.float16)
    vp[3, 1, 0] = 0.0                                                     # a constant group
    packed["v_params"] = vp.view(np.uint16)
    _decode_check(d, lm_bits, v_bits, batch, hkv, G, max_len, lens=[3000, 2049], packed=packed, kernel=kernel)


@pytest.mark.parametrize("layers", [(0, 17, 35)])
def test_decode_parity_qwen_shaped_library_compressed(layers):
    """Qwen2.5-3B-shaped keys and values (lognormal channel scales, four x20 outlier
    channels, K norms about 100x V norms) compressed by the library, then decoded at G = 8
    (two query-head blocks of the tensor-core decode) for several layers; scores and outputs
    against the oracle decoding the same packed bytes."""
    d, lm_bits, v_bits, G, tokens = 128, 2, 2, 8, 8192
    ctx = make_ctx(T, d, lm_bits, v_bits)
    Pi, c, t, S = oracle_setup(d, lm_bits)
    for layer in layers:
        K, V = W.qwen_layer_head_kv(layer=layer, head=layer % 2, tokens=tokens)
        kt = torch.from_numpy(K).to(DEV).to(torch.bfloat16)
        vt = torch.from_numpy(V).to(DEV).to(torch.bfloat16)
        gp = T.tq_compress_kv(ctx, kt, vt)
        q = W.queries((1, G, d), seed=100 + layer, dtype="bf16")
        qt = torch.from_numpy(q).to(DEV).to(torch.bfloat16)
        scores = torch.full((1, G, tokens), float("nan"), device=DEV)
        out, _ = T.tq_decode_attention(ctx, qt, gp, 1, G, 1, tokens, scores=scores)
        T.tq_check_device(ctx)
        g = to_np(gp)
        pk = {"codes": g["k_codes"], "signs": g["k_signs"], "norms": g["k_norms"]}
        pv = {"codes": g["v_codes"], "params": g["v_params"]}
        os_, oo = O.decode_attention(q[0].astype(np.float64), pk, pv, Pi, c, S, d, v_bits)
        assert np.max(np.abs(os_)) > 5.0                                  # large logits indeed
        assert_close(scores[0].cpu().numpy(), os_, what=f"scores layer {layer}")
        assert_close(out[0].cpu().numpy(), oo, what=f"out layer {layer}")


def test_decode_rejects_small_workspace():
    ctx = make_ctx(T, 128, 2, 2)
    packed = _upload(W.random_packed_cache(256, 128, 2, 128, 2))
    q = torch.randn((1, 4, 128), device=DEV)
    with pytest.raises(T.TQError):
        T.tq_decode_attention(ctx, q, packed, 1, 4, 1, 256, workspace=torch.empty(256, dtype=torch.uint8, device=DEV))


# ------------------------------------------------------------------ decompress

@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("d,lm_bits,v_bits", [(128, 2, 2), (64, 3, 4), (256, 1, 4)])
def test_decompress_parity(rotation, d, lm_bits, v_bits):
    rng = np.random.default_rng(6)
    K = rng.standard_normal((777, d))
    V = rng.standard_normal((777, d))
    Pi, c, t, S = oracle_setup(d, lm_bits, d, rotation)
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, v_bits)
    packed = _upload({"k_codes": pk["codes"], "k_signs": pk["signs"], "k_norms": pk["norms"],
                      "v_codes": pv["codes"], "v_params": pv["params"]})
    ctx = make_ctx(T, d, lm_bits, v_bits, d, rotation)
    kx, vx = T.tq_decompress(ctx, packed, 777)
    torch.cuda.synchronize()
    assert_close(kx.cpu().numpy(), O.decompress_keys(pk, Pi, c, S, d), rtol=1e-4, atol=1e-5, what="keys")
    assert_close(vx.cpu().numpy(), O.dequantize_values(pv, v_bits, d), rtol=1e-6, atol=1e-6, what="values")


# ------------------------------------------------------------------ compression sweep

@pytest.mark.parametrize("rotation", ["hadamard", "haar"])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("b", [2, 3, 4])
def test_sweep_mse_and_inner_product_distortion_vs_oracle(d, b, rotation):
    """The compression sweep's per-configuration figures: key MSE E||k - k_hat||^2 / ||k||^2
    and inner-product distortion E(<q, k> - <q, k_hat>)^2 with 64 N(0,1) queries, from the
    library's own compression and decompression of 4096 bf16 N(0,1) vectors, against the
    oracle's on the same vectors (b total bits: b - 1 Lloyd-Max bits + 1 QJL bit, m = d)."""
    lm_bits, n = b - 1, 4096
    ctx = make_ctx(T, d, lm_bits, 2, rotation=rotation)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(100 * d + b)
    kt = torch.randn((n, d), generator=gen, device=DEV).to(torch.bfloat16)
    g = T.tq_compress_kv(ctx, kt, None)
    khat, _ = T.tq_decompress(ctx, g, n, keys=True, values=False)
    torch.cuda.synchronize()
    K = kt.float().cpu().numpy().astype(np.float64)
    Kg = khat.cpu().numpy().astype(np.float64)
    Pi, c, t, S = oracle_setup(d, lm_bits, d, rotation)
    pk = O.compress_keys(K, Pi, c, t, S)
    Ko = O.decompress_keys(pk, Pi, c, S, d)
    Q = np.random.default_rng(d * 10 + b).standard_normal((64, d))
    norms2 = (K * K).sum(1)

    def figures(Kh):
        mse = float(np.mean(((K - Kh) ** 2).sum(1) / norms2))
        ip = float(np.mean((Q @ K.T - Q @ Kh.T) ** 2))
        return mse, ip

    mse_g, ip_g = figures(Kg)
    mse_o, ip_o = figures(Ko)
    # the packed codes agree (up to decision-point exemptions), so do the figures
    assert mse_g == pytest.approx(mse_o, rel=1e-3)
    assert ip_g == pytest.approx(ip_o, rel=1e-3)
    # and the reconstruction is informative: well below the MSE of reconstructing zero (1)
    assert mse_g < 0.75


# ------------------------------------------------------------------ keys without the QJL stage

@pytest.mark.parametrize("d,lm_bits,v_bits,rotation,dtype", [
    (128, 2, 2, "hadamard", "bf16"), (128, 1, 4, "haar", "f32"), (64, 3, 4, "hadamard", "bf16"),
    (128, 3, 3, "hadamard", "bf16")])
def test_keys_without_qjl_stage(d, lm_bits, v_bits, rotation, dtype):
    """qjl_m = 0 (Lloyd-Max codes only; no sign bytes): compression, decode attention and
    decompression through the C ABI against the oracle given an empty S."""
    dr = W.method_draws(d, d, 1234)
    c32, t32 = T.tq_lloyd_max_codebook(d, lm_bits)
    haar = T.tq_haar_from_gaussian(dr["haar_gaussian"]) if rotation == "haar" else None
    S0 = np.zeros((0, d))
    ctx = T.tq_codebook_load(d, lm_bits, v_bits, c32, t32, S0, rotation=rotation,
                             hadamard_signs=dr["hadamard_signs"], haar=haar)
    assert ctx.m == 0
    n, G = 3000, 4
    rng = np.random.default_rng([d, lm_bits])
    K = rng.standard_normal((n, d)) * rng.lognormal(0, 1, d)
    V = rng.standard_normal((n, d))
    K[[0, n - 1]] = 0.0
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    kt = torch.from_numpy(K.astype(np.float32)).to(DEV).to(tdt)
    vt = torch.from_numpy(V.astype(np.float32)).to(DEV).to(tdt)
    gp = T.tq_compress_kv(ctx, kt, vt)
    T.tq_check_device(ctx)
    g = to_np(gp)
    assert g["k_signs"].shape == (n, 0)
    Pi, c, t, _ = oracle_setup(d, lm_bits, d, rotation)
    ok = O.compress_keys(kt.float().cpu().numpy().astype(np.float64), Pi, c, t, S0, with_diagnostics=True)
    ov = O.quantize_values(vt.float().cpu().numpy().astype(np.float64), v_bits, with_diagnostics=True)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, 0))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    # decode attention over the compressed cache (one sequence, one KV head)
    q = W.queries((1, G, d), dtype="f32")
    scores = torch.full((1, G, n), float("nan"), device=DEV)
    out, _ = T.tq_decode_attention(ctx, torch.from_numpy(q).to(DEV), gp, 1, G, 1, n, scores=scores)
    T.tq_check_device(ctx)
    pk = {"codes": g["k_codes"], "signs": g["k_signs"], "norms": g["k_norms"]}
    pv = {"codes": g["v_codes"], "params": g["v_params"]}
    os_, oo = O.decode_attention(q[0].astype(np.float64), pk, pv, Pi, c, S0, d, v_bits)
    assert_close(scores[0].cpu().numpy(), os_, what="scores")
    assert_close(out[0].cpu().numpy(), oo, what="out")
    # decompression
    kx, _ = T.tq_decompress(ctx, gp, n)
    torch.cuda.synchronize()
    assert_close(kx.cpu().numpy(), O.decompress_keys(pk, Pi, c, S0, d), rtol=1e-4, atol=1e-5, what="keys")


@pytest.mark.parametrize("lm_bits,v_bits,rotation", [
    (1, 2, "hadamard"), (2, 4, "hadamard"), (3, 3, "hadamard"), (2, 2, "haar"), (3, 4, "haar")])
def test_keys_without_qjl_pipelined_compression(lm_bits, v_bits, rotation):
    """qjl_m = 0, bf16, d = 128: keys on the pipelined tensor-core kernel without its
    projection (values on its value warps at 2 and 4 bits, on the warp-per-vector kernel at
    3); two to three passes per CTA and a ragged last pass, zero keys, every vector against
    the oracle; keys alone and values alone give the same records."""
    d = 128
    dr = W.method_draws(d, d, 1234)
    c32, t32 = T.tq_lloyd_max_codebook(d, lm_bits)
    haar = T.tq_haar_from_gaussian(dr["haar_gaussian"]) if rotation == "haar" else None
    S0 = np.zeros((0, d))
    ctx = T.tq_codebook_load(d, lm_bits, v_bits, c32, t32, S0, rotation=rotation,
                             hadamard_signs=dr["hadamard_signs"], haar=haar)
    n = 148 * 128 * 2 + 5 * 128 + 77
    rng = np.random.default_rng([41, lm_bits, v_bits])
    K = rng.standard_normal((n, d)) * rng.lognormal(0, 1, d)
    V = rng.standard_normal((n, d)) * 2.0 - 0.5
    K[[0, 128 * 148, n - 1]] = 0.0
    kt = torch.from_numpy(K.astype(np.float32)).to(DEV).to(torch.bfloat16)
    vt = torch.from_numpy(V.astype(np.float32)).to(DEV).to(torch.bfloat16)
    g = to_np(T.tq_compress_kv(ctx, kt, vt))
    T.tq_check_device(ctx)
    Pi, c, t, _ = oracle_setup(d, lm_bits, d, rotation)
    ok = O.compress_keys(kt.float().cpu().numpy().astype(np.float64), Pi, c, t, S0, with_diagnostics=True)
    ov = O.quantize_values(vt.float().cpu().numpy().astype(np.float64), v_bits, with_diagnostics=True)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, 0))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    gk = to_np(T.tq_compress_kv(ctx, kt, None))
    gv = to_np(T.tq_compress_kv(ctx, None, vt))
    T.tq_check_device(ctx)
    for name in ("k_codes", "k_norms"):
        assert np.array_equal(gk[name], g[name]), name
    for name in ("v_codes", "v_params"):
        assert np.array_equal(gv[name], g[name]), name


@pytest.mark.parametrize("v_bits", [2, 3, 4])
def test_decode_value_codes_keep_the_low_parts(v_bits):
    """Values N(0.5, 2^2) per coordinate (groups with large minima and spans), Haar keys, fp32
    queries, decoded on the mma.sync kernel: the value codes enter the MMAs as f16 subnormals
    at mantissa bit 3 or higher; at the lowest positions their products with the low parts of
    p * scale lost up to 3e-4 of the output (outside the elementwise bound for small outputs)."""
    d, lm_bits, n, G = 128, 2, 2500, 4
    rng = np.random.default_rng([d, 3])
    K = rng.standard_normal((n, d)) * rng.lognormal(0, 1, d)
    V = rng.standard_normal((n, d)) * 2.0 + 0.5
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, "haar", "f32")
    T.tq_set_decode_kernel(ctx, T.TQ_DECODE_MMA)
    gp = _upload({k: g[k] for k in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params")})
    q = W.queries((1, G, d), dtype="f32")
    out, _ = T.tq_decode_attention(ctx, torch.from_numpy(q).to(DEV), gp, 1, G, 1, n)
    T.tq_check_device(ctx)
    Pi, c, t, S = oracle_setup(d, lm_bits, d, "haar")
    pk = {"codes": g["k_codes"], "signs": g["k_signs"], "norms": g["k_norms"]}
    pv = {"codes": g["v_codes"], "params": g["v_params"]}
    _, oo = O.decode_attention(q[0].astype(np.float64), pk, pv, Pi, c, S, d, v_bits)
    assert_close(out[0].cpu().numpy(), oo, what="out")


# ------------------------------------------------------------------ 3-bit values (K = V = 3)

@pytest.mark.parametrize("d,lm_bits,rotation,dtype", [
    (128, 2, "hadamard", "bf16"), (128, 2, "haar", "f32"), (64, 1, "hadamard", "bf16"), (256, 3, "haar", "bf16")])
def test_three_bit_values(d, lm_bits, rotation, dtype):
    """v_bits = 3 (codes straddle 32-bit words): compression, decode attention and
    decompression of values through the C ABI against the oracle; with 2-bit Lloyd-Max keys
    and their QJL bit this is the symmetric K = V = 3 configuration."""
    v_bits, n, G = 3, 2500, 4
    rng = np.random.default_rng([d, 3])
    K = rng.standard_normal((n, d)) * rng.lognormal(0, 1, d)
    V = rng.standard_normal((n, d)) * 2.0 + 0.5
    V[7, :32] = 1.25                                                      # a constant group
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, dtype)
    assert g["v_codes"].shape == (n, 3 * d // 8)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    gp = _upload({k: g[k] for k in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params")})
    q = W.queries((1, G, d), dtype="f32")
    scores = torch.full((1, G, n), float("nan"), device=DEV)
    out, _ = T.tq_decode_attention(ctx, torch.from_numpy(q).to(DEV), gp, 1, G, 1, n, scores=scores)
    T.tq_check_device(ctx)
    Pi, c, t, S = oracle_setup(d, lm_bits, d, rotation)
    pk = {"codes": g["k_codes"], "signs": g["k_signs"], "norms": g["k_norms"]}
    pv = {"codes": g["v_codes"], "params": g["v_params"]}
    os_, oo = O.decode_attention(q[0].astype(np.float64), pk, pv, Pi, c, S, d, v_bits)
    assert_close(scores[0].cpu().numpy(), os_, what="scores")
    assert_close(out[0].cpu().numpy(), oo, what="out")
    _, vx = T.tq_decompress(ctx, gp, n, keys=False)
    torch.cuda.synchronize()
    assert_close(vx.cpu().numpy(), O.dequantize_values(pv, v_bits, d), rtol=1e-6, atol=1e-6, what="values")


# ------------------------------------------------------------------ 4- to 7-bit Lloyd-Max codes

@pytest.mark.parametrize("d,lm_bits,rotation,dtype,v_bits", [
    (128, 4, "hadamard", "bf16", 4), (64, 4, "haar", "f32", 2), (256, 4, "hadamard", "bf16", 3),
    (128, 7, "hadamard", "bf16", 4),   # 8-bit keys (7-bit Lloyd-Max + the QJL sign), 4-bit values
    (64, 5, "haar", "bf16", 2), (128, 6, "haar", "f32", 3)])
def test_wide_lloyd_max_keys(d, lm_bits, rotation, dtype, v_bits):
    """k_lm_bits = 4..7 (16- to 128-level sphere codebooks, Lloyd iteration or Newton's
    method): compression, decode attention and decompression through the C ABI against the
    oracle."""
    n, G = 2000, 6
    rng = np.random.default_rng([d, lm_bits])
    K = rng.standard_normal((n, d)) * rng.lognormal(0, 1, d)
    V = rng.standard_normal((n, d))
    K[[3, n - 2]] = 0.0
    ctx, g, ok, ov = _compress_both(K, V, d, lm_bits, v_bits, rotation, dtype)
    assert g["k_codes"].shape == (n, lm_bits * d // 8)
    assert_key_parity(compare_keys(g, ok, d, lm_bits, d))
    assert_value_parity(compare_values(g, ov, d, v_bits))
    gp = _upload({k: g[k] for k in ("k_codes", "k_signs", "k_norms", "v_codes", "v_params")})
    q = W.queries((1, G, d), dtype="f32")
    scores = torch.full((1, G, n), float("nan"), device=DEV)
    out, _ = T.tq_decode_attention(ctx, torch.from_numpy(q).to(DEV), gp, 1, G, 1, n, scores=scores)
    T.tq_check_device(ctx)
    Pi, c, t, S = oracle_setup(d, lm_bits, d, rotation)
    pk = {"codes": g["k_codes"], "signs": g["k_signs"], "norms": g["k_norms"]}
    pv = {"codes": g["v_codes"], "params": g["v_params"]}
    os_, oo = O.decode_attention(q[0].astype(np.float64), pk, pv, Pi, c, S, d, v_bits)
    assert_close(scores[0].cpu().numpy(), os_, what="scores")
    assert_close(out[0].cpu().numpy(), oo, what="out")
    kx, _ = T.tq_decompress(ctx, gp, n, values=False)
    torch.cuda.synchronize()
    assert_close(kx.cpu().numpy(), O.decompress_keys(pk, Pi, c, S, d), rtol=1e-4, atol=1e-5, what="keys")
