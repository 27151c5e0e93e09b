"""Seeded synthetic inputs for the grouped-int4 expert FFN workloads.

Input generation only: random numbers with the shapes and distributions of the
workloads, nothing of the method's arithmetic (no packing, no dequantisation, no
routing).  Both the CUDA path and the oracle take their inputs from here.

Weights: q ~ U{-8..7} i.i.d. per weight.  A packed byte holds two independent weights,
so i.i.d. uniform q is the same distribution as i.i.d. uniform bytes; the large
configurations therefore draw packed bytes directly (``rng.bytes``) instead of q.  The
small ones draw q (int8) so that the packer itself can be tested.

Every tensor has its own sub-stream: ``default_rng([seed, tensor_id, index])`` so an
expert's weights can be regenerated alone (the oracle only needs the experts its
sampled tokens visit).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# tensor ids for sub-streams
_T_Q, _T_S, _T_X, _T_LOGIT, _T_HOT = 1, 2, 3, 4, 5
_GATE, _UP, _DOWN, _DENSE = 10, 11, 12, 13


def rng(seed: int, *path: int) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [int(p) for p in path])


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """f32 -> bf16 bit patterns (uint16), round to nearest even (input generation only)."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def q_uniform(seed, O, I, *path) -> np.ndarray:
    """int8 [O][I], uniform in -8..7."""
    return rng(seed, _T_Q, *path).integers(-8, 8, size=(O, I), dtype=np.int8)


def packed_uniform(seed, O, I, *path) -> np.ndarray:
    """uint8 [O][I/2] of i.i.d. uniform bytes (= packed i.i.d. uniform q); I even."""
    assert I % 2 == 0
    return np.frombuffer(rng(seed, _T_Q, *path).bytes(O * I // 2), np.uint8).reshape(O, I // 2)


def scales_uniform(seed, O, ng, lo, hi, *path) -> np.ndarray:
    return rng(seed, _T_S, *path).uniform(lo, hi, size=(O, ng)).astype(np.float32)


def x_normal(seed, T, I, dtype: str, *path) -> np.ndarray:
    """activations ~ N(0,1): float32 or bf16 bit patterns (uint16)."""
    x = rng(seed, _T_X, *path).standard_normal((T, I), dtype=np.float32)
    return to_bf16_bits(x) if dtype == "bf16" else x


def logits_normal(seed, T, E, sigma=1.0, n_hot=0, hot_bias=0.0):
    """router logits ~ N(0, sigma^2), plus hot_bias on n_hot seeded distinct experts."""
    lg = (rng(seed, _T_LOGIT).standard_normal((T, E)) * sigma).astype(np.float32)
    hot = np.zeros(0, np.int64)
    if n_hot:
        hot = np.sort(rng(seed, _T_HOT).choice(E, size=n_hot, replace=False))
        lg[:, hot] += np.float32(hot_bias)
    return lg, hot


# ---------------------------------------------------------------------------------
# Workloads (shapes and distributions of the five configurations)
# ---------------------------------------------------------------------------------
GS = 64


@dataclass
class MoEConfig:
    name: str
    T: int
    H: int
    E: int
    F: int
    K: int
    seed: int
    sigma: float = 1.0
    n_hot: int = 0
    hot_bias: float = 0.0
    scale_lo: float = 0.002
    scale_hi: float = 0.02
    x_dtype: str = "bf16"
    oracle_sample: int = 0  # 0: every token

    def logits(self):
        return logits_normal(self.seed, self.T, self.E, self.sigma, self.n_hot, self.hot_bias)

    def x(self):
        return x_normal(self.seed, self.T, self.H, self.x_dtype)

    # per-expert tensors (packed bytes + scales), regenerable one expert at a time
    def gate(self, e):
        return (packed_uniform(self.seed, self.F, self.H, _GATE, e),
                scales_uniform(self.seed, self.F, self.H // GS, self.scale_lo, self.scale_hi, _GATE, e))

    def up(self, e):
        return (packed_uniform(self.seed, self.F, self.H, _UP, e),
                scales_uniform(self.seed, self.F, self.H // GS, self.scale_lo, self.scale_hi, _UP, e))

    def down(self, e):
        return (packed_uniform(self.seed, self.H, self.F, _DOWN, e),
                scales_uniform(self.seed, self.H, self.F // GS, self.scale_lo, self.scale_hi, _DOWN, e))

    def sample_tokens(self):
        if not self.oracle_sample or self.oracle_sample >= self.T:
            return np.arange(self.T, dtype=np.int64)
        return np.sort(rng(self.seed, 99).choice(self.T, size=self.oracle_sample, replace=False)).astype(np.int64)


MOE_DECODE = MoEConfig("moe_decode_t1_h4096_e128_f1536_k8", T=1, H=4096, E=128, F=1536, K=8, seed=1002)
# "N(0,2)" read as variance 2 (sigma = sqrt 2); 16 seeded hot experts get +3
MOE_BATCHED = MoEConfig("moe_batched_decode_t32_h6144_e256_f2048_k8", T=32, H=6144, E=256, F=2048,
                        K=8, seed=1003, sigma=float(np.sqrt(2.0)), n_hot=16, hot_bias=3.0)
MOE_PREFILL = MoEConfig("moe_prefill_t4096_h6144_e256_f2048_k8", T=4096, H=6144, E=256, F=2048,
                        K=8, seed=1004, oracle_sample=256)

# profiling case: the batched-decode shapes and routing with 32 experts (0.68 GB of
# weights: larger than L2, small enough for multi-pass counter captures)
MOE_BATCHED_E32 = MoEConfig("moe_batched_decode_t32_h6144_e32_f2048_k8", T=32, H=6144, E=32, F=2048,
                            K=8, seed=1003, sigma=float(np.sqrt(2.0)), n_hot=4, hot_bias=3.0)

# profiling case of the prefill kernels: 128 rows per expert as at full size, 32 experts
MOE_PREFILL_E32 = MoEConfig("moe_prefill_t512_h6144_e32_f2048_k8", T=512, H=6144, E=32, F=2048, K=8,
                            seed=1004, oracle_sample=64)

MOE_CONFIGS = {c.name: c for c in (MOE_DECODE, MOE_BATCHED, MOE_PREFILL, MOE_BATCHED_E32, MOE_PREFILL_E32)}

DENSE_SHAPES = [(4096, 4096), (14336, 4096), (4096, 14336), (151936, 4096)]


def dense_matvec(O, I, seed=1001, dtype="bf16"):
    """one gq4_matvec case of the dense sweep: packed bytes, scales U(0.002,0.02), x N(0,1)."""
    return (packed_uniform(seed, O, I, _DENSE, O, I),
            scales_uniform(seed, O, I // GS, 0.002, 0.02, _DENSE, O, I),
            x_normal(seed, 1, I, dtype, O, I))


@dataclass
class SingleExpert:
    """x f32 [1,1024]; gate/up [2048,1024] (q drawn as int8), down [1024,2048];
    scales U(0.005, 0.02)."""
    seed: int = 1000
    H: int = 1024
    F: int = 2048
    qg: np.ndarray = field(init=False)
    qu: np.ndarray = field(init=False)
    qd: np.ndarray = field(init=False)

    def __post_init__(self):
        self.qg = q_uniform(self.seed, self.F, self.H, _GATE)
        self.qu = q_uniform(self.seed, self.F, self.H, _UP)
        self.qd = q_uniform(self.seed, self.H, self.F, _DOWN)
        self.sg = scales_uniform(self.seed, self.F, self.H // GS, 0.005, 0.02, _GATE)
        self.su = scales_uniform(self.seed, self.F, self.H // GS, 0.005, 0.02, _UP)
        self.sd = scales_uniform(self.seed, self.H, self.F // GS, 0.005, 0.02, _DOWN)
        self.x = x_normal(self.seed, 1, self.H, "f32")
