"""The synthetic input recipe (no GPU): shapes and packed sizes of the benchmark
workloads, the properties the Qwen2.5-3B-shaped cache is built to have, and the
reproducibility and exactness of the method's random draws."""
import numpy as np
import pytest

import workloads as W


@pytest.mark.parametrize("name,packed", [
    ("qwen2.5-3b_8k_k3v2", 72 * 8192 * 100),           # 58,982,400 B: K3 (52 B) + V2 (48 B) per token
    ("llama8b_b32_32k_k3v2", 256 * 32768 * 100),       # 838,860,800 B
    ("long_1m_k4v4", 4 * 1048576 * 148),               # 620,756,992 B: K4 (68 B) + V4 (80 B)
    ("llama8b_b32_32k_mse3v2", 256 * 32768 * 100),     # 3-bit codes, no sign bytes: the same 100 B record
    ("single_head_d128_n4096", 4096 * (52 + 80)),
])
def test_packed_bytes_of_the_workloads(name, packed):
    assert W.WORKLOADS[name].packed_bytes() == packed


def test_workload_shapes():
    w = W.WORKLOADS["long_1m_k4v4"]
    assert (w.units, w.group, w.lm_bits, w.m, w.v_bits) == (4, 6, 3, 128, 4)
    w = W.WORKLOADS["llama8b_b32_32k_mse3v2"]
    assert (w.units, w.group, w.lm_bits, w.m) == (256, 4, 3, 0)
    w = W.WORKLOADS["qwen2.5-3b_8k_k3v2"]
    assert (w.units, w.group, w.lm_bits, w.m, w.dtype) == (72, 8, 2, 128, "bf16")


def test_qwen_shaped_keys_carry_outlier_channels_and_large_norms():
    """Keys: lognormal channel scales with 4 channels x20; values 0.1 N(0,1): key norms come
    out about two orders of magnitude above value norms (the K/V norm ratio the pages report
    for real models is 100-180x)."""
    K, V = W.qwen_layer_head_kv(3, 1, tokens=2048)
    assert K.shape == V.shape == (2048, 128)
    ratio = np.linalg.norm(K, axis=1).mean() / np.linalg.norm(V, axis=1).mean()
    assert 30 < ratio < 1000, ratio
    ch = np.sqrt((K.astype(np.float64) ** 2).mean(0))       # per-channel RMS
    top = np.sort(ch)[::-1]
    assert top[3] > 5 * np.median(ch)                        # four channels stand far out
    assert abs(np.sqrt((V.astype(np.float64) ** 2).mean()) - 0.1) < 0.005


def test_method_draws_are_reproducible_and_plain_fp32_gaussians():
    a, b = W.method_draws(128, 128), W.method_draws(128, 128)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    assert set(np.unique(a["hadamard_signs"])) <= {-1, 1}
    S = a["qjl_S"]
    np.testing.assert_array_equal(S.astype(np.float32).astype(np.float64), S)  # exact in fp32
    # not narrowed to any coarser grid: almost no entry is representable in fp16
    assert np.mean(S.astype(np.float16).astype(np.float64) == S) < 0.01
    assert abs(S.std() - 1.0) < 0.02
    c = W.method_draws(128, 128, seed=99)
    assert not np.array_equal(a["qjl_S"], c["qjl_S"])


def test_random_packed_cache_side_info_is_on_the_fp16_grid():
    pk = W.random_packed_cache(1000, 128, 2, 128, 4, seed=3)
    assert pk["k_codes"].shape == (1000, 32) and pk["k_signs"].shape == (1000, 16)
    assert pk["v_codes"].shape == (1000, 64) and pk["v_params"].shape == (1000, 4, 2)
    n = pk["k_norms"].view(np.float16).astype(np.float64)
    assert np.all(n[:, 0] > 0) and np.all((n[:, 1] > 0.09) & (n[:, 1] < 0.61))
    assert np.isfinite(pk["v_params"].view(np.float16)).all()
