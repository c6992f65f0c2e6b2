"""Plain, slow fp64 restatement of TurboQuant compression and compressed-cache decode.

TEST INFRASTRUCTURE ONLY: imported by tests, by ``__graft_entry__.smoke()`` and by
the benchmark's CPU-baseline leg; never by the library.

Sources (web pages about TurboQuant; none of them prints an equation):

* "turboquant-pytorch" skill card, section "Что делает": keys and values are
  compressed by random orthogonal rotations, a Lloyd-Max quantizer and a one-bit
  QJL correction of the residual; the point is to preserve inner products for
  attention scoring; ``TurboQuantProd`` scores attention directly from the
  compressed keys; a 3-bit Qwen2.5-3B cache at 8K shrinks from 289 MB to 58 MB;
  codebooks are computed with scipy.
* discosf.com TurboQuant news item, section "一句话看懂：TurboQuant 是什么":
  (1) random orthogonal rotation, (2) Lloyd-Max scalar quantization of keys with
  pre-generated codebooks, (3) QJL projection keeping the residual as 1-bit
  signs, (4) values group-quantized to 2/4 bits, four 2-bit values per byte.
* tproger.ru, "TurboQuant неделю спустя", section "Реализации TurboQuant": the
  O(d^2) rotation is the slow part; a Walsh-Hadamard transform brings it to
  O(d log d).

Every step the pages leave open is resolved by the plainest reading and listed
here; each function says which reading it takes.

R1  Rotation input is the unit vector u = k/||k||; ||k|| is stored (fp16).
R2  Randomized Hadamard rotation is Pi = H_d diag(sigma) / sqrt(d), Sylvester
    H_d[i][j] = (-1)^popcount(i & j), one sign diagonal applied first.
R3  Dense rotation is a Haar orthogonal matrix: Q of the QR factorisation of a
    Gaussian matrix with R's diagonal made positive.
R4  The Lloyd-Max codebook is the optimal scalar quantizer of one coordinate of a
    uniformly random unit vector in R^d (the exact law of (Pi u)_j), with
    boundaries at centroid midpoints; the device holds it in fp32 and both sides
    bucketize against the fp32 values.
R5  Bucketize: idx = #{k : y >= t_k}, so a tie goes to the upper cell.
R6  The QJL residual is taken in the rotated domain: r = y - c[idx], gamma = ||r||,
    sign bit i = [(S r)_i >= 0], S an m x d matrix of N(0,1) draws.
R7  The inner-product estimate is <q,k> ~= n (<Pi q, c[idx]> + sqrt(pi/2)/m *
    gamma * <S Pi q, s>), s in {-1,+1}^m (the standard QJL estimator).
R8  Packing: code j occupies bits [b*j, b*j+b) of a little-endian bit stream
    (least significant bit first); sign i is bit i%8 of byte i/8.
R9  Side info (n, gamma) and the value group (scale, min) are stored as fp16,
    rounded to nearest even.
R10 Values: groups of 32 consecutive coordinates of one vector; asymmetric
    min/max uniform quantizer with 2^b - 1 steps, code = clamp(floor((v-min)/scale
    + 1/2)); a constant group (scale 0) gets code 0; dequant uses stored fp16.
R11 A zero key stores all-zero bytes.
R12 Attention logits are scaled by 1/sqrt(d) unless the caller gives a scale;
    the softmax is exact (max-subtracted, two passes).
R15 A sequence whose tokens are split into disjoint ranges (one per GPU) is
    decoded range by range: each range yields its own normalized output o_r and
    the log of its softmax denominator, lse_r = log sum_t exp(l_t); the output
    over all tokens is sum_r exp(lse_r) o_r / sum_r exp(lse_r). This is an
    identity of the softmax, not an approximation; an empty range has lse = -inf
    and weighs nothing.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import integrate

__all__ = [
    "sphere_coordinate_pdf", "gaussian_pdf", "lloyd_max", "lloyd_max_newton", "lloyd_max_sphere",
    "lloyd_max_gaussian", "quantizer_mse", "device_codebook", "hadamard_matrix",
    "hadamard_rotation", "haar_rotation", "bucketize", "pack_codes", "unpack_codes",
    "pack_signs", "unpack_signs", "compress_keys", "decompress_keys",
    "quantize_values", "dequantize_values", "prepare_query", "key_scores",
    "decode_attention", "log_partition", "merge_attention", "qjl_inner_product", "fp16_midpoint_distance",
    "k_record_bytes", "v_record_bytes", "QJL_CONST",
]

QJL_CONST = math.sqrt(math.pi / 2.0)  # E|g| = sqrt(2/pi) for g ~ N(0,1)


# --------------------------------------------------------------------------
# Densities of the rotated coordinate (R4)
# --------------------------------------------------------------------------

def sphere_coordinate_pdf(x, d: int):
    """Density of one coordinate of a uniform random unit vector in R^d.

    f_d(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2) on [-1, 1].
    After a random orthogonal rotation each coordinate of Pi u has this law,
    which is why one codebook per d serves every key (skill card, "Что делает";
    discosf, "一句话看懂" step 2: codebooks per dimension).
    """
    logc = math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)
    x = np.asarray(x, dtype=np.float64)
    return np.exp(logc) * np.clip(1.0 - x * x, 0.0, None) ** ((d - 3) / 2.0)


def gaussian_pdf(x, sigma: float = 1.0):
    x = np.asarray(x, dtype=np.float64)
    return np.exp(-0.5 * (x / sigma) ** 2) / (sigma * math.sqrt(2.0 * math.pi))


def _quad(fn, a, b):
    return integrate.quad(fn, a, b, epsabs=0.0, epsrel=1e-13, limit=400)[0]


def lloyd_max(pdf, lo: float, hi: float, levels: int, scale: float,
              tol: float = 1e-15, max_iter: int = 20000):
    """Lloyd-Max scalar quantizer for density ``pdf`` on [lo, hi].

    Alternates the two optimality conditions until the centroids move by less
    than ``tol``: boundaries at centroid midpoints, t_k = (c_{k-1} + c_k)/2, and
    centroids at cell means, c_k = int x f / int f over [t_k, t_{k+1}).
    Integrals by adaptive quadrature (the skill card computes its codebooks with
    scipy as well). ``scale`` sets the initial spread (centroids start evenly
    spaced in [-2 scale, 2 scale]). Returns fp64 (centroids, boundaries).
    """
    c = np.linspace(-2.0 * scale, 2.0 * scale, levels) if levels > 1 else np.zeros(1)
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[lo], t, [hi]])
        new = np.empty(levels)
        for k in range(levels):
            a, b = edges[k], edges[k + 1]
            mass = _quad(lambda x: float(pdf(x)), a, b)
            first = _quad(lambda x: x * float(pdf(x)), a, b)
            new[k] = first / mass
        moved = np.max(np.abs(new - c))
        c = new
        if moved < tol:
            break
    else:  # pragma: no cover - the densities used here always converge
        raise RuntimeError("Lloyd-Max iteration did not converge")
    return c, 0.5 * (c[:-1] + c[1:])


def _point_density_edges(pdf, lo: float, hi: float, levels: int, grid: int = 200001):
    """Initial boundaries from the high-resolution optimal point density, proportional to
    pdf^(1/3) (Panter and Dite): the (i/L)-quantiles of that normalized density."""
    x = np.linspace(lo, hi, grid)
    g = np.cbrt(np.array([float(pdf(v)) for v in x]))
    cdf = np.concatenate([[0.0], np.cumsum(0.5 * (g[1:] + g[:-1]) * np.diff(x))])
    return np.interp(np.arange(1, levels) / levels * cdf[-1], cdf, x)


def _solve_tridiagonal(lower, diag, upper, rhs):
    """Thomas algorithm for a tridiagonal system (lower[i] multiplies x[i], row i + 1)."""
    n = diag.size
    cp, dp = np.empty(n), np.empty(n)
    cp[0] = upper[0] / diag[0] if n > 1 else 0.0
    dp[0] = rhs[0] / diag[0]
    for i in range(1, n):
        den = diag[i] - lower[i - 1] * cp[i - 1]
        cp[i] = upper[i] / den if i < n - 1 else 0.0
        dp[i] = (rhs[i] - lower[i - 1] * dp[i - 1]) / den
    out = np.empty(n)
    out[-1] = dp[-1]
    for i in range(n - 2, -1, -1):
        out[i] = dp[i] - cp[i] * out[i + 1]
    return out


def lloyd_max_newton(pdf, lo: float, hi: float, levels: int, tol: float = 1e-14, max_iter: int = 60):
    """The Lloyd-Max conditions (boundaries at centroid midpoints, centroids at cell means)
    solved by Newton's method on the L - 1 boundaries, from the point-density start.

    Residual R_i = t_i - (c_i + c_{i+1}) / 2 with c_k = int x f / int f over cell k; a
    centroid moves with its cell's edges as dc/d(right edge b) = f(b)(b - c)/M0 and
    dc/d(left edge a) = f(a)(c - a)/M0, so the Jacobian is tridiagonal. Steps are halved
    until the boundaries stay ordered inside (lo, hi). Same fixed point as ``lloyd_max``,
    reached in a few iterations where plain Lloyd iteration needs very many (many levels).
    """
    e = _point_density_edges(pdf, lo, hi, levels)

    def cells(e):
        edges = np.concatenate([[lo], e, [hi]])
        m0 = np.array([_quad(lambda x: float(pdf(x)), edges[k], edges[k + 1]) for k in range(levels)])
        m1 = np.array([_quad(lambda x: x * float(pdf(x)), edges[k], edges[k + 1]) for k in range(levels)])
        return m0, m1 / m0

    for _ in range(max_iter):
        m0, c = cells(e)
        res = e - 0.5 * (c[:-1] + c[1:])
        fe = np.array([float(pdf(v)) for v in e])
        right = fe * (e - c[:-1]) / m0[:-1]    # d c_i / d t_i (t_i is cell i's right edge)
        left = fe * (c[1:] - e) / m0[1:]       # d c_{i+1} / d t_i (cell i+1's left edge)
        diag = 1.0 - 0.5 * (right + left)
        step = _solve_tridiagonal(-0.5 * left[:-1], diag, -0.5 * right[1:], res)
        lam = 1.0
        while True:
            cand = e - lam * step
            if np.all(np.diff(cand) > 0) and cand[0] > lo and cand[-1] < hi:
                break
            lam *= 0.5
        e = cand
        if np.max(np.abs(lam * step)) < tol:
            break
    else:  # pragma: no cover
        raise RuntimeError("Lloyd-Max Newton iteration did not converge")
    _, c = cells(e)
    return c, 0.5 * (c[:-1] + c[1:])


_SPHERE_CACHE: dict = {}


def lloyd_max_sphere(d: int, bits: int):
    """Codebook (centroids, boundaries) for the rotated coordinate at dimension d (R4)."""
    key = (d, bits)
    if key not in _SPHERE_CACHE:
        pdf = lambda x: sphere_coordinate_pdf(x, d)  # noqa: E731
        if bits <= 4:
            c, _ = lloyd_max(pdf, -1.0, 1.0, 2 ** bits, 1.0 / math.sqrt(d))
        else:  # many levels: Newton's method on the same two conditions
            c, _ = lloyd_max_newton(pdf, -1.0, 1.0, 2 ** bits)
        # The law is even, so the exact optimum is odd (c_k = -c_{L-1-k}); imposing it
        # removes round-off asymmetry and puts the middle boundary exactly at 0.
        c = 0.5 * (c - c[::-1])
        _SPHERE_CACHE[key] = (c, 0.5 * (c[:-1] + c[1:]))
    c, t = _SPHERE_CACHE[key]
    return c.copy(), t.copy()


def lloyd_max_gaussian(bits: int, sigma: float = 1.0):
    """Codebook of N(0, sigma^2): the d -> infinity limit of ``lloyd_max_sphere``."""
    return lloyd_max(lambda x: gaussian_pdf(x, sigma), -40.0 * sigma, 40.0 * sigma,
                     2 ** bits, sigma)


def quantizer_mse(pdf, lo, hi, centroids, boundaries):
    """E[(x - Q(x))^2] of a scalar quantizer under ``pdf`` (quadrature per cell)."""
    edges = np.concatenate([[lo], boundaries, [hi]])
    total = 0.0
    for k, ck in enumerate(centroids):
        total += _quad(lambda x: (x - ck) ** 2 * float(pdf(x)), edges[k], edges[k + 1])
    return total


def device_codebook(d: int, bits: int):
    """The codebook as the device holds it: fp32-rounded values, widened to fp64 (R4).

    Boundaries are the fp64 midpoints of the fp64 centroids, then rounded.
    """
    c, t = lloyd_max_sphere(d, bits)
    return c.astype(np.float32).astype(np.float64), t.astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Rotations (R2, R3)
# --------------------------------------------------------------------------

def hadamard_matrix(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix written entry by entry: H[i][j] = (-1)^popcount(i & j)."""
    if d <= 0 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.empty((d, d))
    for i in range(d):
        for j in range(d):
            H[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return H


def hadamard_rotation(signs) -> np.ndarray:
    """Pi = H diag(sigma) / sqrt(d) (R2; tproger, "Реализации TurboQuant": the
    Walsh-Hadamard transform is the O(d log d) rotation)."""
    s = np.asarray(signs, dtype=np.float64)
    d = s.shape[0]
    return hadamard_matrix(d) * s[None, :] / math.sqrt(d)


def haar_rotation(gaussian) -> np.ndarray:
    """Haar orthogonal matrix from a Gaussian matrix: QR with diag(R) > 0 (R3)."""
    g = np.asarray(gaussian, dtype=np.float64)
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


# --------------------------------------------------------------------------
# Bit packing (R8)
# --------------------------------------------------------------------------

def pack_codes(codes, bits: int) -> np.ndarray:
    """Pack integer codes [N, d] (each < 2^bits) into a LSB-first stream [N, bits*d/8] (R8).

    Four 2-bit values share a byte (discosf, "一句话看懂" step 4)."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    stream = np.zeros((n, d * bits), dtype=np.uint8)
    for b in range(bits):
        stream[:, b::bits] = (codes >> b) & 1
    return np.packbits(stream, axis=1, bitorder="little")


def unpack_codes(packed, bits: int, d: int) -> np.ndarray:
    stream = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, bitorder="little")
    stream = stream[:, : d * bits].astype(np.int64)
    codes = np.zeros((stream.shape[0], d), dtype=np.int64)
    for b in range(bits):
        codes |= stream[:, b::bits] << b
    return codes


def pack_signs(bits01) -> np.ndarray:
    return np.packbits(np.asarray(bits01, dtype=np.uint8), axis=1, bitorder="little")


def unpack_signs(packed, m: int) -> np.ndarray:
    return np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, bitorder="little")[:, :m]


def k_record_bytes(d: int, lm_bits: int, m: int) -> int:
    """Bytes of one packed key: codes + sign bits + two fp16 (n, gamma)."""
    return lm_bits * d // 8 + m // 8 + 4


def v_record_bytes(d: int, v_bits: int, group: int = 32) -> int:
    """Bytes of one packed value: codes + one fp16 (scale, min) pair per group."""
    return v_bits * d // 8 + (d // group) * 4


def _fp16_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


def fp16_midpoint_distance(x) -> np.ndarray:
    """Relative distance of |x| to the nearest fp16 rounding midpoint (for exemptions).

    The fp16 values lo <= |x| < hi bracket |x|; the midpoints that can be nearest are the
    one of (lo, hi) and, when |x| is itself an fp16 value at the bottom of a binade, the one
    below lo, half of the smaller gap beneath it. Past the largest finite value 65504 the
    next grid point is 65536, so the overflow threshold 65520 is the last midpoint.
    """
    x = np.abs(np.asarray(x, dtype=np.float64))
    with np.errstate(over="ignore"):
        h = x.astype(np.float16)
    hb = h.view(np.uint16).astype(np.int64)
    lo = np.where(h.astype(np.float64) > x, hb - 1, hb)
    lo = np.clip(lo, 0, 0x7BFF)

    def val(bits):
        v = np.clip(bits, 0, 0x7BFF).astype(np.uint16).view(np.float16).astype(np.float64)
        return np.where(bits > 0x7BFF, 65536.0, v)

    lo_v = val(lo)
    mid_up = 0.5 * (lo_v + val(lo + 1))
    mid_dn = np.where(lo > 0, 0.5 * (lo_v + val(lo - 1)), -np.inf)
    dist = np.minimum(np.abs(x - mid_up), np.abs(x - mid_dn))
    with np.errstate(divide="ignore", invalid="ignore"):
        rel = dist / np.where(x > 0, x, 1.0)
    return np.where(x > 0, rel, np.inf)


# --------------------------------------------------------------------------
# Key compression: rotation -> Lloyd-Max -> QJL signs -> packing
# --------------------------------------------------------------------------

def bucketize(y, boundaries) -> np.ndarray:
    """idx_j = #{k : y_j >= t_k} (R5): the Lloyd-Max cell of each rotated coordinate."""
    y = np.asarray(y, dtype=np.float64)
    t = np.asarray(boundaries, dtype=np.float64)
    return np.sum(y[..., None] >= t, axis=-1).astype(np.int64)


def compress_keys(K, Pi, centroids, boundaries, S, with_diagnostics: bool = False):
    """TurboQuantProd compression of keys K [N, d] (fp64 throughout).

    Steps (discosf, "一句话看懂" 1-3; skill card "Что делает"):
      n = ||k||, u = k/n (R1); y = Pi u; idx = bucketize(y) against the Lloyd-Max
      boundaries (R4, R5); r = y - c[idx], gamma = ||r||; sign bits of S r (R6);
      pack codes and signs (R8); store (n, gamma) as fp16 (R9). Zero keys: R11.

    Returns dict(codes [N, b d/8] u8, signs [N, m/8] u8, norms [N, 2] u16 fp16 bits)
    and, if asked, the fp64 intermediates used to decide exemptions.
    """
    K = np.asarray(K, dtype=np.float64)
    Pi = np.asarray(Pi, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    t = np.asarray(boundaries, dtype=np.float64)
    bits = int(round(math.log2(c.shape[0])))
    n_vec, d = K.shape
    m = S.shape[0]

    n = np.sqrt(np.sum(K * K, axis=1))
    nz = n > 0
    u = np.zeros_like(K)
    u[nz] = K[nz] / n[nz, None]
    y = u @ Pi.T
    idx = bucketize(y, t)
    r = y - c[idx]
    gamma = np.sqrt(np.sum(r * r, axis=1))
    proj = r @ S.T
    sbits = (proj >= 0).astype(np.uint8)

    idx[~nz] = 0
    sbits[~nz] = 0
    gamma[~nz] = 0.0
    out = {
        "codes": pack_codes(idx, bits),
        "signs": pack_signs(sbits),
        "norms": np.stack([_fp16_bits(n), _fp16_bits(gamma)], axis=1),
    }
    if with_diagnostics:
        dist = np.min(np.abs(y[..., None] - t), axis=-1) if t.size else np.full_like(y, np.inf)
        out.update({"n": n, "gamma": gamma, "y": y, "idx": idx, "proj": proj,
                    "boundary_distance": dist})
    return out


def decompress_keys(packed: dict, Pi, centroids, S, d: int):
    """x_hat = n Pi^T (c[idx] + sqrt(pi/2)/m * gamma * S^T s): the key the estimator
    of R7 implicitly scores against (fp64; uses the stored fp16 n, gamma)."""
    c = np.asarray(centroids, dtype=np.float64)
    S = np.asarray(S, dtype=np.float64)
    bits = int(round(math.log2(c.shape[0])))
    m = S.shape[0]
    idx = unpack_codes(packed["codes"], bits, d)
    s = 2.0 * unpack_signs(packed["signs"], m).astype(np.float64) - 1.0
    norms = np.asarray(packed["norms"], dtype=np.uint16).view(np.float16).astype(np.float64)
    n, gamma = norms[:, 0], norms[:, 1]
    y_hat = c[idx] + (QJL_CONST / m) * gamma[:, None] * (s @ S) if m else c[idx]  # m = 0: codes alone
    return n[:, None] * (y_hat @ np.asarray(Pi, dtype=np.float64))


# --------------------------------------------------------------------------
# Value group quantization (R10)
# --------------------------------------------------------------------------

def quantize_values(V, bits: int, group: int = 32, with_diagnostics: bool = False):
    """Asymmetric min/max group quantization of values V [N, d] (discosf step 4, R10).

    Returns dict(codes [N, bits d/8] u8, params [N, d/group, 2] u16 = fp16 (scale, min)).
    """
    V = np.asarray(V, dtype=np.float64)
    n_vec, d = V.shape
    g = V.reshape(n_vec, d // group, group)
    lo = g.min(axis=2)
    hi = g.max(axis=2)
    levels = 2 ** bits - 1
    scale = (hi - lo) / levels
    safe = np.where(scale > 0, scale, 1.0)
    x = (g - lo[..., None]) / safe[..., None]
    x = np.where(scale[..., None] > 0, x, 0.0)
    codes = np.clip(np.floor(x + 0.5), 0, levels).astype(np.int64).reshape(n_vec, d)
    out = {
        "codes": pack_codes(codes, bits),
        "params": np.stack([_fp16_bits(scale), _fp16_bits(lo)], axis=2),
    }
    if with_diagnostics:
        frac = x - np.floor(x)
        out.update({"x": x.reshape(n_vec, d), "code_values": codes,
                    "half_distance": np.abs(frac - 0.5).reshape(n_vec, d),
                    "scale": scale, "min": lo})
    return out


def dequantize_values(packed: dict, bits: int, d: int, group: int = 32):
    """v_hat = min16 + scale16 * code (R10)."""
    codes = unpack_codes(packed["codes"], bits, d).astype(np.float64)
    p = np.asarray(packed["params"], dtype=np.uint16).view(np.float16).astype(np.float64)
    scale = np.repeat(p[:, :, 0], group, axis=1)
    lo = np.repeat(p[:, :, 1], group, axis=1)
    return lo + scale * codes


# --------------------------------------------------------------------------
# Decode: scores straight from the packed keys, exact softmax, dequantized V
# --------------------------------------------------------------------------

def prepare_query(q, Pi, S):
    """qr = Pi q and sq = S qr for each query row (fp64)."""
    qr = np.asarray(q, dtype=np.float64) @ np.asarray(Pi, dtype=np.float64).T
    return qr, qr @ np.asarray(S, dtype=np.float64).T


def key_scores(q, packed_k: dict, Pi, centroids, S, d: int, scale: float | None = None):
    """Attention logits of queries q [G, d] against packed keys, without dequantizing.

    l_t = scale * n_t * (<Pi q, c[idx_t]> + sqrt(pi/2)/m * gamma_t * <S Pi q, s_t>)
    (R7, R12; skill card "Что делает": TurboQuantProd scores attention directly
    from the compressed keys). Returns [G, N] fp64.
    """
    c = np.asarray(centroids, dtype=np.float64)
    bits = int(round(math.log2(c.shape[0])))
    m = np.asarray(S).shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    qr, sq = prepare_query(np.atleast_2d(q), Pi, S)
    idx = unpack_codes(packed_k["codes"], bits, d)
    s = 2.0 * unpack_signs(packed_k["signs"], m).astype(np.float64) - 1.0
    norms = np.asarray(packed_k["norms"], dtype=np.uint16).view(np.float16).astype(np.float64)
    n, gamma = norms[:, 0], norms[:, 1]
    lut = c[idx] @ qr.T                       # [N, G]
    qjl = (QJL_CONST / m) * gamma[:, None] * (s @ sq.T) if m else 0.0  # m = 0: no QJL stage
    return (scale * n[:, None] * (lut + qjl)).T


def decode_attention(q, packed_k: dict, packed_v: dict, Pi, centroids, S, d: int,
                     v_bits: int, group: int = 32, length: int | None = None,
                     scale: float | None = None):
    """One decode step of attention over a compressed cache (one KV head).

    Scores from the packed keys (``key_scores``), exact max-subtracted softmax
    over the first ``length`` keys (R12), then the softmax-weighted sum of the
    group-dequantized values. Returns (scores [G, N], out [G, d]) in fp64.
    """
    scores = key_scores(q, packed_k, Pi, centroids, S, d, scale)
    N = scores.shape[1] if length is None else length
    vals = dequantize_values(packed_v, v_bits, d, group)
    if N == 0:
        return scores, np.zeros((scores.shape[0], d))
    s = scores[:, :N]
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return scores, (p @ vals[:N]) / p.sum(axis=1, keepdims=True)


def log_partition(scores, length: int | None = None):
    """lse_g = log sum_{t < N} exp(l_{g,t}) of logits [G, N'] over the first N tokens,
    evaluated around the row maximum (R12, R15); -inf for every row when N = 0."""
    s = np.atleast_2d(np.asarray(scores, dtype=np.float64))
    N = s.shape[1] if length is None else length
    if N == 0:
        return np.full(s.shape[0], -np.inf)
    mx = s[:, :N].max(axis=1)
    return mx + np.log(np.exp(s[:, :N] - mx[:, None]).sum(axis=1))


def merge_attention(outs, lses):
    """Attention over the union of R disjoint token ranges from each range's output
    o_r [R, G, d] and log-partition lse_r [R, G] (R15): weights exp(lse_r - max_r lse_r),
    o = sum_r w_r o_r / sum_r w_r, lse = max + log sum_r w_r. Ranges with lse = -inf get
    weight 0; a row whose ranges are all empty gets a zero output and lse = -inf.
    Returns (out [G, d], lse [G]) in fp64."""
    o = np.asarray(outs, dtype=np.float64)
    ls = np.asarray(lses, dtype=np.float64)
    G, d = o.shape[1], o.shape[2]
    out, lse = np.zeros((G, d)), np.full(G, -np.inf)
    for g in range(G):
        mx = ls[:, g].max()
        if mx == -np.inf:
            continue
        w = np.where(ls[:, g] == -np.inf, 0.0, np.exp(ls[:, g] - mx))
        out[g] = (w[:, None] * o[:, g, :]).sum(axis=0) / w.sum()
        lse[g] = mx + math.log(w.sum())
    return out, lse


def qjl_inner_product(x, r, S):
    """QJL estimate of <x, r> from the signs of S r: sqrt(pi/2)/m * ||r|| * <S x, sign(S r)>."""
    S = np.asarray(S, dtype=np.float64)
    m = S.shape[0]
    sr = np.asarray(r, dtype=np.float64) @ S.T
    s = np.where(sr >= 0, 1.0, -1.0)
    return QJL_CONST / m * np.linalg.norm(r, axis=-1) * np.sum((np.asarray(x) @ S.T) * s, axis=-1)
