"""Seeded synthetic workloads shared by the tests, the oracle checks and the benchmark.

This module only draws random numbers and names shapes. It holds none of the
TurboQuant arithmetic (no rotation, quantization, packing or attention), so both
the CUDA library and the fp64 oracle can take their inputs from it without
sharing any of the method's code.

The shapes follow the workloads the TurboQuant pages talk about:

* a single 128-dim head of fp32 N(0,1) keys/values (the PyTorch skill card,
  "turboquant-pytorch", section "Что делает", describes compressing one layer's
  K/V at 3 bits);
* a Qwen2.5-3B-shaped cache at 8K context (same card: 289 MB shrinking to 58 MB)
  whose keys carry per-channel scales and outlier channels so that key norms sit
  about 100x above value norms (tproger, "TurboQuant неделю спустя", section
  "Проблема K-тензоров": K/V norm ratios of 100-180x);
* batched and long-context decode with asymmetric K3/V2 and K4/V4 bit widths
  (discosf news item, "一句话看懂" steps 1-4; GarraRUST "TurboQuant+ Setup",
  section "Descoberta-chave");
* a prefill-style compression sweep over d and bit width.

All draws use numpy's PCG64 ``default_rng`` so CPU and GPU sides see identical
numbers; large benchmark inputs can instead be drawn on the device with a seeded
torch generator (``device_normal``), which is only used where no oracle compares
element by element.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "method_draws", "single_head_kvq", "normal_f32", "bf16_round",
    "fp16_round", "unit_keys_values", "qwen_layer_head_kv", "queries",
    "random_packed_cache", "device_normal",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and bit-width of one benchmark/parity workload."""
    name: str
    d: int
    batch: int          # sequences (or layers for the Qwen-shaped cache)
    hkv: int            # KV heads per sequence
    hq: int             # query heads per sequence
    tokens: int         # cached tokens per (sequence, KV head)
    k_bits: int         # total key bits = Lloyd-Max bits + 1 QJL bit (Lloyd-Max bits alone if not qjl)
    v_bits: int
    dtype: str          # "f32" or "bf16"
    qjl_m: int = 0      # 0 => m = d
    v_group: int = 32
    rotation: str = "hadamard"
    qjl: bool = True    # False: keys without the QJL stage (m = 0)

    @property
    def m(self) -> int:
        return (self.qjl_m or self.d) if self.qjl else 0

    @property
    def lm_bits(self) -> int:
        return self.k_bits - 1 if self.qjl else self.k_bits

    @property
    def units(self) -> int:
        return self.batch * self.hkv

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    def k_record_bytes(self) -> int:
        return self.lm_bits * self.d // 8 + self.m // 8 + 4

    def v_record_bytes(self) -> int:
        return self.v_bits * self.d // 8 + (self.d // self.v_group) * 4

    def packed_bytes(self) -> int:
        return self.units * self.tokens * (self.k_record_bytes() + self.v_record_bytes())


WORKLOADS = {
    # single head, 4096 fp32 keys/values, 8 queries: the parity-sized case
    "single_head_d128_n4096": Workload("single_head_d128_n4096", 128, 1, 1, 8, 4096, 3, 4, "f32"),
    # Qwen2.5-3B-shaped: 36 layers x 2 KV heads x 8192 tokens, 16 query heads per layer
    "qwen2.5-3b_8k_k3v2": Workload("qwen2.5-3b_8k_k3v2", 128, 36, 2, 16, 8192, 3, 2, "bf16"),
    # Llama-8B-like layer, 32 sequences x 8 KV heads x 32768 tokens, 32 query heads
    "llama8b_b32_32k_k3v2": Workload("llama8b_b32_32k_k3v2", 128, 32, 8, 32, 32768, 3, 2, "bf16"),
    # long context: one sequence of 1,048,576 tokens, 4 KV heads, 24 query heads
    "long_1m_k4v4": Workload("long_1m_k4v4", 128, 1, 4, 24, 1 << 20, 4, 4, "bf16"),
    # the Llama-shaped batch with 3-bit Lloyd-Max keys and no QJL stage (same 100 B record)
    "llama8b_b32_32k_mse3v2": Workload("llama8b_b32_32k_mse3v2", 128, 32, 8, 32, 32768, 3, 2, "bf16", qjl=False),
}

# compression sweep: 16384 tokens x 64 heads of bf16 N(0,1) vectors
SWEEP_VECTORS = 16384 * 64
SWEEP_D = (64, 128, 256)
SWEEP_BITS = (2, 3, 4)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bfloat16 (ties to even); returns fp32."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def fp16_round(x: np.ndarray) -> np.ndarray:
    """Round to the fp16 grid (numpy's correctly rounded conversion); returns fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32)


def method_draws(d: int, m: int, seed: int = 1234) -> dict:
    """The random draws the method makes once per (d, m): returned, never derived.

    * ``hadamard_signs``: the diagonal sign vector of the randomized
      Walsh-Hadamard rotation (int8, +-1);
    * ``haar_gaussian``: a d x d matrix of i.i.d. N(0,1) (fp64) from which each
      side builds its own Haar-distributed orthogonal matrix;
    * ``qjl_S``: the m x d QJL projection, i.i.d. N(0,1) draws in fp32 (an fp64
      array holding the fp32 values: the library takes S as fp32, so both sides
      see exactly the same matrix).
    """
    rng = np.random.default_rng([seed, d, m])
    signs = np.where(rng.integers(0, 2, size=d) == 1, 1, -1).astype(np.int8)
    haar_gaussian = rng.standard_normal((d, d))
    S = rng.standard_normal((m, d), dtype=np.float32).astype(np.float64)
    return {"hadamard_signs": signs, "haar_gaussian": haar_gaussian, "qjl_S": S}


def single_head_kvq(tokens: int = 4096, d: int = 128, n_queries: int = 8, seed: int = 0):
    """K [tokens, d], V [tokens, d], Q [n_queries, d] fp32 N(0,1), drawn in that
    order from one PCG64 generator seeded with ``seed``."""
    rng = np.random.default_rng(seed)
    K = normal_f32(rng, (tokens, d))
    V = normal_f32(rng, (tokens, d))
    Q = normal_f32(rng, (n_queries, d))
    return K, V, Q


def unit_keys_values(w: Workload, unit: int, seed: int = 0):
    """fp32 N(0,1) keys and values for one (sequence, KV head) unit.

    Each unit has its own generator (seeded by ``[seed, unit]``) so any unit can
    be regenerated alone. Returns (K, V) as fp32 arrays [tokens, d]
    (bf16-rounded when the workload is bf16).
    """
    rng = np.random.default_rng([seed, unit])
    K = normal_f32(rng, (w.tokens, w.d))
    V = normal_f32(rng, (w.tokens, w.d))
    if w.dtype == "bf16":
        K, V = bf16_round(K), bf16_round(V)
    return K, V


def qwen_layer_head_kv(layer: int, head: int, tokens: int = 8192, d: int = 128):
    """Keys/values of one (layer, KV head) of the Qwen2.5-3B-shaped cache.

    Keys: N(0,1) scaled per channel by lognormal(0,1) factors, with 4 channels
    (chosen without replacement) multiplied by 20. Values: 0.1 * N(0,1).
    Both rounded to bf16. Seed 1000 + 2*layer + head.
    """
    rng = np.random.default_rng(1000 + 2 * layer + head)
    lam = rng.lognormal(0.0, 1.0, size=d).astype(np.float32)
    outliers = rng.choice(d, size=4, replace=False)
    lam[outliers] *= 20.0
    K = normal_f32(rng, (tokens, d)) * lam[None, :]
    V = np.float32(0.1) * normal_f32(rng, (tokens, d))
    return bf16_round(K), bf16_round(V)


def queries(shape, seed: int = 7, dtype: str = "f32") -> np.ndarray:
    rng = np.random.default_rng([seed, 99])
    q = normal_f32(rng, shape)
    return bf16_round(q) if dtype == "bf16" else q


def random_packed_cache(n_vec: int, d: int, lm_bits: int, m: int, v_bits: int,
                        v_group: int = 32, seed: int = 5,
                        k_norm_scale: float = 1.0) -> dict:
    """Random packed K/V records (bytes, not derived from any compression).

    Codes and sign bits are uniform random bytes; norms are drawn in the range
    a unit-variance d-dim key produces (n ~ sqrt(d), gamma ~ 0.1-0.6); V scales
    and minima are drawn like those of N(0,1) groups. All side info is on the
    fp16 grid and returned as uint16 bit patterns.
    """
    rng = np.random.default_rng([seed, n_vec, d])
    k_codes = rng.integers(0, 256, size=(n_vec, lm_bits * d // 8), dtype=np.uint8)
    k_signs = rng.integers(0, 256, size=(n_vec, m // 8), dtype=np.uint8)
    n = k_norm_scale * math.sqrt(d) * (1.0 + 0.1 * rng.standard_normal(n_vec))
    g = rng.uniform(0.1, 0.6, size=n_vec)
    k_norms = np.stack([np.abs(n), g], axis=1).astype(np.float16).view(np.uint16)
    v_codes = rng.integers(0, 256, size=(n_vec, v_bits * d // 8), dtype=np.uint8)
    ng = d // v_group
    lo = -2.0 + 0.3 * rng.standard_normal((n_vec, ng))
    span = 4.0 + 0.5 * rng.standard_normal((n_vec, ng))
    sc = np.abs(span) / (2 ** v_bits - 1)
    v_params = np.stack([sc, lo], axis=2).astype(np.float16).view(np.uint16)
    return {"k_codes": k_codes, "k_signs": k_signs, "k_norms": np.ascontiguousarray(k_norms),
            "v_codes": v_codes, "v_params": np.ascontiguousarray(v_params)}


def device_normal(shape, seed: int, device: str = "cuda", dtype=None):
    """Seeded N(0,1) draws made on the device (torch Philox); for benchmark-sized inputs."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32 if dtype is None else dtype)
