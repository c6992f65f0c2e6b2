"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle by a route other than the oracle's own code: printed
table values, closed forms, brute force, Monte Carlo, or invariants. A plausible
slip (a dropped term, a sign, a transposed operand, a wrong exponent in the
density) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
from scipy import special

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


# ---------------------------------------------------------------- rotations

def test_hadamard_matches_hand_written_sylvester():
    rows = _read_rows("hadamard_sylvester.txt")
    mats, cur = {}, None
    for r in rows:
        if r.startswith("d="):
            cur = int(r[2:])
            mats[cur] = []
        else:
            mats[cur].append([float(x) for x in r.split()])
    for d, m in mats.items():
        np.testing.assert_array_equal(O.hadamard_matrix(d), np.array(m))


@pytest.mark.parametrize("d", [2, 4, 8, 64, 128, 256])
def test_hadamard_rotation_orthogonal(d):
    H = O.hadamard_matrix(d)
    np.testing.assert_array_equal(H @ H.T, d * np.eye(d))      # exact in fp64
    sig = W.method_draws(d, d)["hadamard_signs"]
    Pi = O.hadamard_rotation(sig)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) < 1e-12
    # the sign diagonal is applied first: column j of Pi is sigma_j H[:, j]/sqrt(d)
    j = d - 1
    np.testing.assert_allclose(Pi[:, j] * math.sqrt(d), sig[j] * H[:, j], rtol=0, atol=1e-14)


def test_hadamard_rotation_against_recursive_butterfly():
    """Pi x computed by an in-place butterfly (a different route than the matrix)."""
    d = 128
    rng = np.random.default_rng(3)
    x = rng.standard_normal(d)
    sig = W.method_draws(d, d)["hadamard_signs"].astype(np.float64)
    y = (x * sig).copy()
    h = 1
    while h < d:
        for i in range(0, d, 2 * h):
            a = y[i:i + h].copy()
            b = y[i + h:i + 2 * h].copy()
            y[i:i + h], y[i + h:i + 2 * h] = a + b, a - b
        h *= 2
    y /= math.sqrt(d)
    np.testing.assert_allclose(O.hadamard_rotation(sig) @ x, y, rtol=0, atol=1e-13)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_haar_rotation_orthogonal_and_triangular(d):
    g = W.method_draws(d, d)["haar_gaussian"]
    Pi = O.haar_rotation(g)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(d))) < 1e-12
    R = Pi.T @ g                      # must be the R factor: upper triangular, diag > 0
    assert np.max(np.abs(np.tril(R, -1))) < 1e-10
    assert np.all(np.diag(R) > 0)


def test_haar_rotation_is_uniform_in_distribution():
    """Mean of Pi[0,0]^2 is 1/d and Pi[0,0] is symmetric (Haar invariance), d=8."""
    d, reps = 8, 20000
    rng = np.random.default_rng(11)
    vals = np.array([O.haar_rotation(rng.standard_normal((d, d)))[0, 0] for _ in range(reps)])
    se = np.std(vals ** 2) / math.sqrt(reps)
    assert abs(np.mean(vals ** 2) - 1.0 / d) < 4 * se
    assert abs(np.mean(vals)) < 4 * np.std(vals) / math.sqrt(reps)


# ---------------------------------------------------------------- Lloyd-Max

def test_gaussian_lloyd_max_matches_max_table():
    for r in _read_rows("gaussian_lloyd_max.txt"):
        parts = r.split()
        bits, mse = int(parts[0]), float(parts[1])
        cents = [float(x) for x in parts[2:]]
        c, t = O.lloyd_max_gaussian(bits)
        got = O.quantizer_mse(O.gaussian_pdf, -40, 40, c, t)
        assert abs(got - mse) / mse < 5e-4, (bits, got, mse)   # 4 significant figures
        np.testing.assert_allclose(c[len(c) // 2:], cents, rtol=0, atol=1e-3)


def test_gaussian_one_bit_closed_form():
    c, t = O.lloyd_max_gaussian(1)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-12
    assert abs(t[0]) < 1e-15
    got = O.quantizer_mse(O.gaussian_pdf, -40, 40, c, t)
    assert abs(got - (1 - 2 / math.pi)) < 1e-11


@pytest.mark.parametrize("d", [64, 128, 256])
def test_sphere_one_bit_closed_form(d):
    # E[x | x > 0] for the sphere-coordinate law: Gamma(d/2)/(sqrt(pi) Gamma((d+1)/2))
    c, t = O.lloyd_max_sphere(d, 1)
    want = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    assert abs(c[1] - want) < 1e-13
    assert abs(c[0] + want) < 1e-13


def _sphere_cell_mean(a, b, d):
    """E[x | a <= x < b] for the sphere-coordinate law by another route:
    first moment from the antiderivative of x(1-x^2)^al, mass from the
    regularized incomplete beta function (x^2 ~ Beta(1/2, (d-1)/2))."""
    al = (d - 3) / 2.0
    logc = math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2)
    first = math.exp(logc) * ((1 - a * a) ** (al + 1) - (1 - b * b) ** (al + 1)) / (2 * (al + 1))

    def cdf(x):
        p = 0.5 * special.betainc(0.5, (d - 1) / 2.0, x * x)
        return 0.5 + math.copysign(p, x)
    return first / (cdf(b) - cdf(a))


@pytest.mark.parametrize("d,bits", [(d, b) for d in (64, 128, 256) for b in (1, 2, 3, 4)] + [(128, 5), (64, 7), (128, 7)])
def test_sphere_lloyd_max_optimality_conditions(d, bits):
    c, t = O.lloyd_max_sphere(d, bits)
    edges = np.concatenate([[-1.0], t, [1.0]])
    for k in range(len(c)):
        assert abs(c[k] - _sphere_cell_mean(edges[k], edges[k + 1], d)) < 1e-12
    np.testing.assert_array_equal(t, 0.5 * (c[:-1] + c[1:]))
    np.testing.assert_array_equal(c, -c[::-1])          # the law is even: the optimum is odd
    if bits > 0:
        assert t[len(t) // 2] == 0.0                       # middle boundary exactly at zero
    assert np.all(np.diff(c) > 0)


def test_sphere_codebook_approaches_gaussian_limit():
    """d * MSE_d -> Gaussian MSE as d grows (the rotated coordinate tends to N(0, 1/d))."""
    for bits in (1, 2, 3):
        cg, tg = O.lloyd_max_gaussian(bits)
        mse_g = O.quantizer_mse(O.gaussian_pdf, -40, 40, cg, tg)
        gaps = []
        for d in (64, 256, 2048):
            c, t = O.lloyd_max(lambda x: O.sphere_coordinate_pdf(x, d), -1, 1, 2 ** bits,
                               1 / math.sqrt(d))
            mse = d * O.quantizer_mse(lambda x: O.sphere_coordinate_pdf(x, d), -1, 1, c, t)
            gaps.append(abs(mse - mse_g) / mse_g)
        assert gaps[0] > gaps[1] > gaps[2]
        assert gaps[2] < 2e-3


def test_sphere_density_by_sampling():
    """Cell means of coordinates of random unit vectors (d=16) match the centroids."""
    d, bits = 16, 2
    c, t = O.lloyd_max_sphere(d, bits)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((400000, d))
    x = (x / np.linalg.norm(x, axis=1, keepdims=True)).ravel()
    cell = np.searchsorted(t, x, side="right")
    for k in range(len(c)):
        xs = x[cell == k]
        assert abs(xs.mean() - c[k]) < 5 * xs.std() / math.sqrt(xs.size)


def test_bucketize_is_nearest_centroid():
    """With midpoint boundaries the cell of y is its nearest centroid (brute force)."""
    c, t = O.device_codebook(128, 2)
    rng = np.random.default_rng(9)
    y = rng.standard_normal(20000) / math.sqrt(128)
    idx = O.bucketize(y, t)
    near = np.argmin(np.abs(y[:, None] - c[None, :]), axis=1)
    np.testing.assert_array_equal(idx, near)
    # ties go to the upper cell
    assert list(O.bucketize(t, t)) == list(range(1, len(t) + 1))


# ---------------------------------------------------------------- packing

def test_packing_hand_examples():
    for r in _read_rows("packing_examples.txt"):
        bits, codes, hexes = [p.strip() for p in r.split(";")]
        bits = int(bits)
        codes = np.array([[int(x) for x in codes.split()]])
        want = bytes.fromhex("".join(hexes.split()))
        got = O.pack_codes(codes, bits)
        assert got.tobytes() == want, (bits, got.tobytes().hex(), want.hex())
        np.testing.assert_array_equal(O.unpack_codes(got, bits, codes.shape[1]), codes)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6, 7])
def test_packing_round_trip_and_bit_positions(bits):
    """Every width the library takes: bits * d / 8 bytes per record, unpack(pack(x)) = x, and
    bit k of code j sits at stream bit bits * j + k (R8), checked bit by bit."""
    rng = np.random.default_rng(bits)
    for d in (32, 64, 128):
        codes = rng.integers(0, 1 << bits, size=(5, d))
        packed = O.pack_codes(codes, bits)
        assert packed.shape == (5, bits * d // 8)
        np.testing.assert_array_equal(O.unpack_codes(packed, bits, d), codes)
        stream = packed[0]
        for j in range(d):
            for k in range(bits):
                pos = bits * j + k
                assert (stream[pos // 8] >> (pos % 8)) & 1 == (codes[0, j] >> k) & 1


def test_sign_packing_bit_order():
    b = np.zeros((1, 16), dtype=np.uint8)
    b[0, 0] = 1
    b[0, 9] = 1
    assert O.pack_signs(b).tobytes() == bytes([0x01, 0x02])


def test_record_sizes_and_skill_card_size_figure():
    vals = {}
    for r in _read_rows("qwen2.5-3b_kv_size.txt"):
        k, v = r.split()
        vals[k] = float(v)
    L, H, d, T = int(vals["layers"]), int(vals["kv_heads"]), int(vals["head_dim"]), int(vals["tokens"])
    mib = 1 << 20
    before = L * 2 * H * T * d * 2
    assert before == 301_989_888
    after = L * 2 * H * T * (3 * d // 8 + 4)
    assert abs(before / mib - vals["page_mb_before"]) / vals["page_mb_before"] < vals["rel_tol"]
    assert abs(after / mib - vals["page_mb_after"]) / vals["page_mb_after"] < vals["rel_tol"]
    # our 3-bit key record: 2-bit Lloyd-Max codes + 1-bit QJL signs + fp16 (n, gamma)
    assert O.k_record_bytes(128, 2, 128) == 3 * 128 // 8 + 4 == 52
    assert O.k_record_bytes(128, 3, 128) == 68
    assert O.v_record_bytes(128, 2) == 48 and O.v_record_bytes(128, 4) == 80
    assert L * H * T * (O.k_record_bytes(128, 2, 128) + O.v_record_bytes(128, 2)) == 58_982_400


def test_fp16_midpoint_distance():
    assert O.fp16_midpoint_distance(np.array([1.0 + 2.0 ** -11]))[0] == 0.0
    # 1.0 opens a binade: the gap below it (2^-11) is half the gap above, so the nearest
    # midpoint is 1 - 2^-12; inside a binade both midpoints are half a gap away
    assert O.fp16_midpoint_distance(np.array([1.0]))[0] == pytest.approx(2.0 ** -12, rel=1e-12)
    assert O.fp16_midpoint_distance(np.array([1.5]))[0] == pytest.approx(2.0 ** -11 / 1.5, rel=1e-12)


def _half_grid_from_fields():
    """Every finite non-negative IEEE binary16 value in ascending order, built from the
    format's fields (exponent e, 10-bit fraction f) without any float16 conversion:
    e = 0 gives the subnormals f * 2^-24, e = 1..30 the normals (1024 + f) * 2^(e - 25)."""
    vals = [f * 2.0 ** -24 for f in range(1024)]
    for e in range(1, 31):
        vals += [(1024 + f) * 2.0 ** (e - 25) for f in range(1024)]
    return np.array(vals)


def test_fp16_midpoint_distance_exhaustive_walk():
    """Every pair of consecutive fp16 values, subnormal range and all 30 normal exponents:
    the midpoint of the pair is at distance exactly 0; the pair's lower end, and points a
    quarter gap either side of the midpoint, are at the distances the gap fixes."""
    g = _half_grid_from_fields()
    assert g.size == 31 * 1024 and g[-1] == 65504.0 and np.all(np.diff(g) > 0)
    lo, hi = g[:-1], g[1:]
    gap = hi - lo
    mid = lo + gap / 2                                   # exact in fp64
    assert np.all(O.fp16_midpoint_distance(mid) == 0.0)
    pos = lo > 0
    # a representable value sits half a gap from the midpoints around it; the nearer one
    # is the lower midpoint at an exponent step (the gap below is half the gap above)
    gap_below = np.concatenate([[np.inf], gap[:-1]])
    d_lo = O.fp16_midpoint_distance(lo[pos])
    np.testing.assert_allclose(d_lo, np.minimum(gap[pos], gap_below[pos]) / 2 / lo[pos], rtol=1e-12)
    for side in (-1.0, 1.0):
        x = mid + side * gap / 4
        np.testing.assert_allclose(O.fp16_midpoint_distance(x), (gap / 4) / x, rtol=1e-12)
    # the overflow threshold between 65504 and the next grid point 65536
    assert O.fp16_midpoint_distance(np.array([65520.0]))[0] == 0.0


# ---------------------------------------------------------------- QJL

def test_qjl_unbiased_monte_carlo():
    """E_S[sqrt(pi/2)/m ||r|| <S x, sign(S r)>] = <x, r>, and its variance is at most
    pi/(2m) ||r||^2 ||x||^2, over independent Gaussian S (d = m = 16)."""
    d = m = 16
    reps = 100000
    rng = np.random.default_rng(17)
    x = rng.standard_normal(d)
    r = 0.3 * rng.standard_normal(d)
    S = rng.standard_normal((reps, m, d))
    sr = np.einsum("kmd,d->km", S, r)
    sx = np.einsum("kmd,d->km", S, x)
    est = O.QJL_CONST / m * np.linalg.norm(r) * np.sum(sx * np.where(sr >= 0, 1.0, -1.0), axis=1)
    truth = x @ r
    se = est.std() / math.sqrt(reps)
    assert abs(est.mean() - truth) < 4 * se
    assert est.var() <= math.pi / (2 * m) * (r @ r) * (x @ x) * 1.02
    # the oracle's own helper gives the same single-draw value
    assert O.qjl_inner_product(x, r, S[0]) == pytest.approx(est[0], rel=1e-12)


def test_whole_estimator_unbiased_over_S():
    """Mean over S draws of the packed-key score estimates <q, k> (d = m = 32)."""
    d = m = 32
    reps = 6000
    rng = np.random.default_rng(23)
    k = rng.standard_normal((1, d))
    q = rng.standard_normal((1, d))
    Pi = O.hadamard_rotation(np.where(rng.integers(0, 2, d) == 1, 1, -1))
    c, t = O.device_codebook(d, 2)
    ests = np.empty(reps)
    for i in range(reps):
        S = rng.standard_normal((m, d))
        pk = O.compress_keys(k, Pi, c, t, S)
        ests[i] = O.key_scores(q, pk, Pi, c, S, d, scale=1.0)[0, 0]
    truth = (q @ k.T).item()
    # the stored fp16 norms add a deterministic relative error below 2^-10
    tol = 4 * ests.std() / math.sqrt(reps) + 2.0 ** -10 * abs(truth) + 1e-3
    assert abs(ests.mean() - truth) < tol


# ---------------------------------------------------------------- scores

def test_scores_brute_force_all_codes_tiny_d():
    """d = m = 4: every 2-bit code word x every sign pattern. The LUT-form score
    equals the dot product with the explicitly decompressed key."""
    d = m = 4
    rng = np.random.default_rng(2)
    Pi = O.hadamard_rotation(np.array([1, -1, -1, 1]))
    S = rng.standard_normal((m, d))
    c = np.array([-1.3, -0.4, 0.4, 1.3])
    q = rng.standard_normal((3, d))
    codes = np.array(np.meshgrid(*[range(4)] * d, indexing="ij")).reshape(d, -1).T
    signs = np.array(np.meshgrid(*[range(2)] * m, indexing="ij")).reshape(m, -1).T
    ci = np.repeat(codes, len(signs), axis=0)
    si = np.tile(signs, (len(codes), 1))
    N = ci.shape[0]
    norms = np.stack([np.full(N, 2.5), np.full(N, 0.75)], axis=1).astype(np.float16).view(np.uint16)
    pk = {"codes": O.pack_codes(ci, 2), "signs": O.pack_signs(si), "norms": norms}
    got = O.key_scores(q, pk, Pi, c, S, d, scale=0.5)
    # explicit: x_hat = n Pi^T (c[idx] + sqrt(pi/2)/m gamma S^T s)
    y_hat = c[ci] + (math.sqrt(math.pi / 2) / m) * 0.75 * ((2.0 * si - 1.0) @ S)
    x_hat = 2.5 * y_hat @ Pi
    np.testing.assert_allclose(got, 0.5 * q @ x_hat.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.decompress_keys(pk, Pi, c, S, d), x_hat, rtol=1e-12, atol=1e-12)


def test_compress_keys_against_hand_computation():
    """d = m = 2, one key, every step done by hand."""
    Pi = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2)      # signs (+1, +1)
    c = np.array([-0.5, 0.5])
    t = np.array([0.0])
    S = np.array([[1.0, 2.0], [-1.0, 0.5]])
    k = np.array([[3.0, 4.0]])                                     # n = 5, u = (0.6, 0.8)
    out = O.compress_keys(k, Pi, c, t, S, with_diagnostics=True)
    y = np.array([1.4, -0.2]) / math.sqrt(2)
    np.testing.assert_allclose(out["y"][0], y, rtol=0, atol=1e-15)
    assert list(out["idx"][0]) == [1, 0]
    r = y - np.array([0.5, -0.5])
    assert out["gamma"][0] == pytest.approx(np.linalg.norm(r), rel=1e-15)
    sbits = [int(S[0] @ r >= 0), int(S[1] @ r >= 0)]
    assert out["signs"][0, 0] == sbits[0] | (sbits[1] << 1)
    assert out["codes"][0, 0] == 0b01
    n16 = np.float16(5.0).view(np.uint16)
    assert out["norms"][0, 0] == n16


def test_zero_key_is_all_zero():
    d = m = 8
    c, t = O.device_codebook(d, 2)
    out = O.compress_keys(np.zeros((1, d)), O.hadamard_rotation(np.ones(d)), c, t, np.ones((m, d)))
    assert not out["codes"].any() and not out["signs"].any() and not out["norms"].any()


# ---------------------------------------------------------------- values

def test_value_quant_hand_example():
    v = np.zeros((1, 32))
    v[0, :4] = [0.0, 1.0, 2.0, 3.0]
    v[0, 4:] = 1.49                  # rounds down to code 1
    out = O.quantize_values(v, 2, with_diagnostics=True)
    assert list(out["code_values"][0, :5]) == [0, 1, 2, 3, 1]
    scale, lo = np.asarray(out["params"][0, 0]).view(np.float16).astype(np.float64)
    assert scale == 1.0 and lo == 0.0
    np.testing.assert_allclose(O.dequantize_values(out, 2, 32)[0, :5], [0, 1, 2, 3, 1])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_value_quant_roundtrip_bound(bits):
    rng = np.random.default_rng(4)
    v = rng.standard_normal((500, 128))
    out = O.quantize_values(v, bits, with_diagnostics=True)
    vh = O.dequantize_values(out, bits, 128)
    scale = np.repeat(out["scale"], 32, axis=1)
    # half a step plus the fp16 rounding of (scale, min), scaled by the largest code
    bound = scale / 2 + 2.0 ** -11 * (np.abs(np.repeat(out["min"], 32, axis=1))
                                      + (2 ** bits - 1) * scale) + 1e-12
    assert np.all(np.abs(vh - v) <= bound)


def test_value_quant_three_bit_hand_example():
    """Values 0..7 (then 3.4) in one group: scale 1, min 0, codes equal to the values (3.4
    rounds to 3); the 3-bit codes straddle bytes in the LSB-first stream (R8, R10)."""
    v = np.zeros((1, 32))
    v[0, :8] = np.arange(8)
    v[0, 8:] = 3.4
    out = O.quantize_values(v, 3, with_diagnostics=True)
    assert list(out["code_values"][0, :9]) == [0, 1, 2, 3, 4, 5, 6, 7, 3]
    scale, lo = np.asarray(out["params"][0, 0]).view(np.float16).astype(np.float64)
    assert scale == 1.0 and lo == 0.0
    # codes 0..7 packed LSB-first: 0b 111 110 101 100 011 010 001 000 = 0xFAC688 (little-endian bytes)
    assert out["codes"][0, :3].tobytes() == bytes([0x88, 0xC6, 0xFA])


def test_value_quant_constant_group():
    v = np.full((2, 64), 0.3125)
    out = O.quantize_values(v, 4)
    assert not out["codes"].any()
    np.testing.assert_array_equal(O.dequantize_values(out, 4, 64), v)


# ---------------------------------------------------------------- decode

def _small_cache(n, d=32, seed=0):
    rng = np.random.default_rng(seed)
    Pi = O.hadamard_rotation(np.where(rng.integers(0, 2, d) == 1, 1, -1))
    S = rng.standard_normal((d, d))
    c, t = O.device_codebook(d, 2)
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    return Pi, S, c, t, K, V


def test_decode_single_key_returns_its_value():
    Pi, S, c, t, K, V = _small_cache(1)
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, 4)
    _, out = O.decode_attention(np.ones((2, 32)), pk, pv, Pi, c, S, 32, 4)
    np.testing.assert_allclose(out, np.repeat(O.dequantize_values(pv, 4, 32), 2, 0), rtol=0, atol=1e-15)


def test_decode_identical_keys_average_values():
    Pi, S, c, t, K, V = _small_cache(5)
    K[:] = K[0]
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, 2)
    _, out = O.decode_attention(np.ones((1, 32)), pk, pv, Pi, c, S, 32, 2)
    np.testing.assert_allclose(out[0], O.dequantize_values(pv, 2, 32).mean(0), rtol=1e-13, atol=1e-13)


def test_decode_matches_textbook_softmax_on_decompressed_keys():
    Pi, S, c, t, K, V = _small_cache(300, seed=3)
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, 4)
    q = np.random.default_rng(8).standard_normal((3, 32))
    scores, out = O.decode_attention(q, pk, pv, Pi, c, S, 32, 4, length=250)
    xk = O.decompress_keys(pk, Pi, c, S, 32)
    logits = q @ xk.T / math.sqrt(32)
    np.testing.assert_allclose(scores, logits, rtol=1e-11, atol=1e-11)
    w = np.exp(logits[:, :250] - logits[:, :250].max(1, keepdims=True))
    w /= w.sum(1, keepdims=True)
    np.testing.assert_allclose(out, w @ O.dequantize_values(pv, 4, 32)[:250], rtol=1e-11, atol=1e-12)


def test_decode_empty_sequence():
    Pi, S, c, t, K, V = _small_cache(4)
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, 4)
    _, out = O.decode_attention(np.ones((1, 32)), pk, pv, Pi, c, S, 32, 4, length=0)
    assert not out.any()


# ---------------------------------------------------------------- split sequence (R15)

def _softmax_by_hand(logits_row, values):
    """Softmax-weighted value sum and log denominator, token by token in Python floats
    (no max shift: only for logits of modest size)."""
    ws = [math.exp(x) for x in logits_row]
    tot = sum(ws)
    out = [sum(w * float(v[j]) for w, v in zip(ws, values)) / tot for j in range(len(values[0]))]
    return out, math.log(tot)


def test_log_partition_brute_force_and_large_logits():
    rng = np.random.default_rng(21)
    s = rng.standard_normal((3, 9))
    want = [math.log(sum(math.exp(x) for x in row[:7])) for row in s]
    np.testing.assert_allclose(O.log_partition(s, 7), want, rtol=1e-14, atol=1e-14)
    # evaluated around the maximum: logits of 1000 stay finite; two equal ones give x + log 2
    np.testing.assert_allclose(O.log_partition(np.array([[1000.0, 1000.0, -np.inf]])),
                               [1000.0 + math.log(2.0)], rtol=1e-15)
    assert np.all(O.log_partition(s, 0) == -np.inf)


def test_merge_of_ranges_is_softmax_over_all_tokens():
    """Tokens split into four ranges (one empty): merging each range's normalized output
    and log-partition equals the softmax over all tokens, computed by hand (R15)."""
    rng = np.random.default_rng(22)
    G, N, d = 2, 23, 5
    logits = rng.standard_normal((G, N)) * 3.0
    vals = rng.standard_normal((N, d))
    cuts = [0, 6, 6, 17, 23]
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o = np.zeros((G, d))
        for g in range(G):
            if b > a:
                o[g] = _softmax_by_hand(logits[g, a:b], vals[a:b])[0]
        outs.append(o)
        lses.append(O.log_partition(logits[:, a:b]))
    out, lse = O.merge_attention(np.stack(outs), np.stack(lses))
    for g in range(G):
        want_o, want_l = _softmax_by_hand(logits[g], vals)
        np.testing.assert_allclose(out[g], want_o, rtol=1e-13, atol=1e-14)
        assert abs(lse[g] - want_l) < 1e-13


def test_merge_special_cases():
    rng = np.random.default_rng(23)
    o = rng.standard_normal((2, 3, 4))
    lse = rng.standard_normal((2, 3))
    out, l1 = O.merge_attention(o[:1], lse[:1])             # one range: itself
    np.testing.assert_array_equal(out, o[0])
    np.testing.assert_allclose(l1, lse[0], rtol=0, atol=1e-15)
    empty = lse.copy()
    empty[1] = -np.inf                                      # an empty range weighs nothing
    out, l2 = O.merge_attention(o, empty)
    np.testing.assert_allclose(out, o[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(l2, lse[0], rtol=0, atol=1e-15)
    out, l3 = O.merge_attention(o, np.full((2, 3), -np.inf))  # all empty
    assert not out.any() and np.all(l3 == -np.inf)
    far = np.array([[0.0] * 3, [800.0] * 3])                # exp(-800) is 0 in fp64
    out, l4 = O.merge_attention(o, far)
    np.testing.assert_array_equal(out, o[1])
    np.testing.assert_array_equal(l4, far[1])


def test_merge_is_order_free_and_composes():
    """Merging parts in any order, or merging merged groups with their log-partitions,
    gives the merge of all parts (R15); shifting every logit by c shifts lse by c."""
    rng = np.random.default_rng(24)
    o = rng.standard_normal((5, 3, 8))
    ls = rng.standard_normal((5, 3)) * 3
    ls[2, 1] = -np.inf
    out, lse = O.merge_attention(o, ls)
    perm = [3, 0, 4, 2, 1]
    out_p, lse_p = O.merge_attention(o[perm], ls[perm])
    np.testing.assert_allclose(out_p, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_p, lse, rtol=1e-13)
    a_out, a_lse = O.merge_attention(o[:2], ls[:2])
    b_out, b_lse = O.merge_attention(o[2:], ls[2:])
    out2, lse2 = O.merge_attention(np.stack([a_out, b_out]), np.stack([a_lse, b_lse]))
    np.testing.assert_allclose(out2, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)
    s = rng.standard_normal((4, 50))
    np.testing.assert_allclose(O.log_partition(s + 7.5), O.log_partition(s) + 7.5, rtol=1e-14)


def test_split_decode_of_a_packed_cache_equals_whole_decode():
    """Decoding token ranges of one packed cache separately and merging them
    reproduces the decode over all valid tokens, and its log-partition (R15)."""
    Pi, S, c, t, K, V = _small_cache(300, seed=5)
    pk = O.compress_keys(K, Pi, c, t, S)
    pv = O.quantize_values(V, 2)
    q = np.random.default_rng(9).standard_normal((4, 32))
    scores, whole = O.decode_attention(q, pk, pv, Pi, c, S, 32, 2, length=281)
    outs, lses = [], []
    cuts = [0, 128, 128, 200, 281]
    for a, b in zip(cuts[:-1], cuts[1:]):
        pk_r = {k: v[a:b] for k, v in pk.items()}
        pv_r = {k: v[a:b] for k, v in pv.items()}
        sc, o = O.decode_attention(q, pk_r, pv_r, Pi, c, S, 32, 2, length=b - a)
        np.testing.assert_array_equal(sc, scores[:, a:b])
        outs.append(o)
        lses.append(O.log_partition(sc, b - a))
    out, lse = O.merge_attention(np.stack(outs), np.stack(lses))
    np.testing.assert_allclose(out, whole, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, O.log_partition(scores, 281), rtol=1e-14)


def test_compression_distortion_is_near_lloyd_max():
    """Relative MSE of the LM stage alone is d*MSE_d of the codebook (rotation makes
    every coordinate follow the sphere law), checked on 4096 random keys at d=128."""
    d = 128
    dr = W.method_draws(d, d)
    Pi = O.hadamard_rotation(dr["hadamard_signs"])
    c, t = O.device_codebook(d, 2)
    K = np.random.default_rng(1).standard_normal((4096, d))
    out = O.compress_keys(K, Pi, c, t, dr["qjl_S"], with_diagnostics=True)
    rel = np.mean(out["gamma"] ** 2)
    cl, tl = O.lloyd_max_sphere(d, 2)
    want = d * O.quantizer_mse(lambda x: O.sphere_coordinate_pdf(x, d), -1, 1, cl, tl)
    assert abs(rel - want) / want < 0.02


def test_keys_without_qjl_stage():
    """m = 0 (Lloyd-Max codes only, no QJL signs): the score from the codes equals the score
    against the reconstruction n Pi^T c[idx], and the reconstruction's relative squared error
    averages d times the per-coordinate MSE the sphere codebook was solved for (quadrature),
    d = 64, 2-bit codes, 20000 uniformly random unit directions (well within 4 sigma)."""
    d, bits, n = 64, 2, 20000
    rng = np.random.default_rng(42)
    Pi = O.haar_rotation(rng.standard_normal((d, d)))
    c, t = O.lloyd_max_sphere(d, bits)
    S = np.zeros((0, d))
    K = rng.standard_normal((n, d)) * rng.uniform(0.5, 3.0, size=(n, 1))
    pk = O.compress_keys(K, Pi, c, t, S)
    assert pk["signs"].shape == (n, 0)
    packed = {"codes": pk["codes"], "signs": pk["signs"], "norms": pk["norms"]}
    q = rng.standard_normal((3, d))
    xh = O.decompress_keys(packed, Pi, c, S, d)
    np.testing.assert_allclose(O.key_scores(q, packed, Pi, c, S, d), q @ xh.T / np.sqrt(d), rtol=1e-12, atol=1e-12)
    # with the exact norm (the stored one is fp16) the error is that of the unit direction
    nrm = np.linalg.norm(K, axis=1)
    n16 = pk["norms"][:, 0].view(np.float16).astype(np.float64)
    err = np.sum((K / nrm[:, None] - xh / n16[:, None]) ** 2, axis=1)
    want = d * O.quantizer_mse(lambda x: O.sphere_coordinate_pdf(x, d), -1, 1, c, t)
    assert abs(err.mean() - want) < 4 * err.std() / np.sqrt(n)


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 3), (256, 4)])
def test_newton_and_lloyd_reach_the_same_codebook(d, bits):
    """Newton's method on the boundaries (used from 5 bits on) and plain Lloyd iteration are
    two routes to the same fixed point of the Lloyd-Max conditions."""
    c1, _ = O.lloyd_max_sphere(d, bits)                     # Lloyd iteration
    c2, _ = O.lloyd_max_newton(lambda x: O.sphere_coordinate_pdf(x, d), -1.0, 1.0, 2 ** bits)
    np.testing.assert_allclose(c2, c1, rtol=0, atol=1e-12)
