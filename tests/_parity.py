"""Helpers shared by the parity tests: building both sides from the same seeded
draws, and comparing packed records under the exemption rule.

Exemption rule (decision points): a packed field may differ from the oracle only
where the oracle's exact value lies within 1e-6 of a decision point -
a Lloyd-Max boundary (rotated unit-norm domain), zero for a QJL sign (residual
of the unit-norm key), a half-step of (v - min)/scale for a value code, or an
fp16 rounding midpoint (relative) for n, gamma and a value scale. A key with an
exempt code also has its signs and gamma exempt. Non-exempt mismatches must not
exceed 1e-6 of all coordinates.
"""
from __future__ import annotations

import math

import numpy as np

import oracle as O
import workloads as W

EPS = 1e-6


def oracle_setup(d, lm_bits, m=None, rotation="hadamard", seed=1234):
    m = m or d
    dr = W.method_draws(d, m, seed)
    if rotation == "hadamard":
        Pi = O.hadamard_rotation(dr["hadamard_signs"])
    else:
        Pi = O.haar_rotation(dr["haar_gaussian"])
    c, t = O.device_codebook(d, lm_bits)
    return Pi, c, t, dr["qjl_S"]


def make_ctx(T, d, lm_bits, v_bits, m=None, rotation="hadamard", seed=1234):
    """Library context built only from the seeded draws and the library's own
    host routines (codebook solver, Haar construction)."""
    m = m or d
    dr = W.method_draws(d, m, seed)
    c, t = T.tq_lloyd_max_codebook(d, lm_bits)
    haar = T.tq_haar_from_gaussian(dr["haar_gaussian"]) if rotation == "haar" else None
    return T.tq_codebook_load(d, lm_bits, v_bits, c, t, dr["qjl_S"], rotation=rotation,
                              hadamard_signs=dr["hadamard_signs"], haar=haar)


def to_np(packed: dict) -> dict:
    out = {}
    for k, v in packed.items():
        a = v.cpu().numpy()
        if a.dtype == np.int16:
            a = a.view(np.uint16)
        out[k] = a
    return out


def compare_keys(gpu: dict, ora: dict, d: int, lm_bits: int, m: int) -> dict:
    """Count exempt and non-exempt mismatches between packed key records."""
    gi = O.unpack_codes(gpu["k_codes"], lm_bits, d)
    oi = ora["idx"]
    code_ex = ora["boundary_distance"] < EPS
    vec_ex = code_ex.any(axis=1)
    code_bad = (gi != oi) & ~code_ex
    gs = O.unpack_signs(gpu["k_signs"], m)
    os_ = O.unpack_signs(ora["signs"], m)
    sign_ex = (np.abs(ora["proj"]) < EPS) | vec_ex[:, None]
    zero = ora["n"] == 0
    sign_ex[zero] = False
    sign_bad = (gs != os_) & ~sign_ex
    gn = gpu["k_norms"].view(np.uint16)
    on = ora["norms"].view(np.uint16)
    n_ex = O.fp16_midpoint_distance(ora["n"]) < EPS
    g_ex = (O.fp16_midpoint_distance(ora["gamma"]) < EPS) | vec_ex
    n_ex[zero] = False
    g_ex[zero] = False
    n_bad = (gn[:, 0] != on[:, 0]) & ~n_ex
    g_bad = (gn[:, 1] != on[:, 1]) & ~g_ex
    return {
        "coords": gi.size,
        "code_exempt": int(code_ex.sum()), "code_mismatch_exempt": int(((gi != oi) & code_ex).sum()),
        "code_bad": int(code_bad.sum()),
        "sign_bad": int(sign_bad.sum()), "sign_mismatch_exempt": int(((gs != os_) & sign_ex).sum()),
        "norm_bad": int(n_bad.sum()), "gamma_bad": int(g_bad.sum()),
        "zero_bytes_ok": bool(not gpu["k_codes"][zero].any() and not gpu["k_signs"][zero].any()
                              and not gn[zero].any()),
    }


def compare_values(gpu: dict, ora: dict, d: int, v_bits: int) -> dict:
    gc = O.unpack_codes(gpu["v_codes"], v_bits, d)
    oc = ora["code_values"]
    ex = ora["half_distance"] < EPS
    bad = (gc != oc) & ~ex
    gp = gpu["v_params"].view(np.uint16)
    op = ora["params"].view(np.uint16)
    sc_ex = O.fp16_midpoint_distance(ora["scale"]) < EPS
    sc_bad = (gp[..., 0] != op[..., 0]) & ~sc_ex
    mn_bad = gp[..., 1] != op[..., 1]
    return {"coords": gc.size, "code_bad": int(bad.sum()), "code_exempt": int(ex.sum()),
            "scale_bad": int(sc_bad.sum()), "min_bad": int(mn_bad.sum())}


def assert_key_parity(stats: dict):
    budget = math.floor(EPS * stats["coords"])
    bad = stats["code_bad"] + stats["sign_bad"] + stats["norm_bad"] + stats["gamma_bad"]
    assert stats["zero_bytes_ok"], stats
    assert bad <= budget, stats


def assert_value_parity(stats: dict):
    budget = math.floor(EPS * stats["coords"])
    assert stats["code_bad"] + stats["scale_bad"] <= budget, stats
    assert stats["min_bad"] == 0, stats


def assert_close(got, want, rtol=1e-3, atol=1e-4, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    lim = atol + rtol * np.abs(want)
    bad = ~(err <= lim)
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside |g-o| <= {atol} + {rtol}|o|; "
                           f"worst excess {float(np.max(err - lim)):.3g}")
