"""Seeded synthetic inputs for the streamed NF4 LoRA path.

This module holds none of the method's arithmetic: it only draws seeded
normal samples, rounds them to bf16 bit patterns (the inputs' storage type)
and lists the projection shapes of the model families the path is sized
for.  Both the CUDA-path tests and the oracle tests take their inputs from
here, so that the two sides see identical bytes.

Input recipe (synthetic throughout -- the Poros API reference, under
PorosTrainer.train, notes that token content does not change memory,
throughput or parity, so no dataset is used):
  * base weight W [N_out, K_in] ~ N(0, 0.02^2), rounded to bf16;
  * adapter A [r, K_in] ~ N(0, (1/16)^2), B [N_out, r] ~ N(0, 0.01^2), bf16;
  * activations X [T, K_in] and upstream gradients dY [T, N_out] ~ N(0, 1), bf16;
  * rank 16, alpha 32 (the Poros defaults).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

RANK = 16
ALPHA = 32.0
W_STD = 0.02
A_STD = 1.0 / 16.0
B_STD = 0.01

PROJ_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class Family:
    """Decoder shape of one model family (only what the 7 projections need)."""
    name: str
    hidden: int
    inter: int
    heads: int
    kv_heads: int
    head_dim: int
    layers: int

    def projections(self):
        """[(name, N_out, K_in)] of the 7 LoRA-targeted linears of one layer."""
        h, i, d = self.hidden, self.inter, self.head_dim
        q, kv = self.heads * d, self.kv_heads * d
        return [("q", q, h), ("k", kv, h), ("v", kv, h), ("o", h, q),
                ("gate", i, h), ("up", i, h), ("down", h, i)]


FAMILIES = {
    "qwen2.5-7b": Family("qwen2.5-7b", 3584, 18944, 28, 4, 128, 28),
    "llama-3.1-8b": Family("llama-3.1-8b", 4096, 14336, 32, 8, 128, 32),
    "qwen2.5-32b": Family("qwen2.5-32b", 5120, 27648, 40, 8, 128, 64),
    "qwen2.5-72b": Family("qwen2.5-72b", 8192, 29568, 64, 8, 128, 80),
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), round to nearest even.

    Only used to give a sampled input its bf16 storage form."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bits_to_f32(h: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact widening)."""
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def sub_seed(seed: int, *keys: int) -> int:
    """Deterministic per-(layer, projection, ...) sub-seed."""
    ss = np.random.SeedSequence([seed, *keys])
    return int(ss.generate_state(1, dtype=np.uint64)[0])


@dataclass
class LinearCase:
    """One LoRA linear's inputs, all bf16 bit patterns (uint16)."""
    W: np.ndarray   # [N, K]
    X: np.ndarray   # [T, K]
    A: np.ndarray   # [r, K]
    B: np.ndarray   # [N, r]
    dY: np.ndarray  # [T, N]
    alpha: float = ALPHA

    @property
    def shape(self):
        return self.X.shape[0], self.W.shape[0], self.W.shape[1], self.A.shape[0]


def linear_case(seed: int, T: int, N: int, K: int, r: int = RANK, alpha: float = ALPHA,
                w_std: float = W_STD, a_std: float = A_STD, b_std: float = B_STD) -> LinearCase:
    rng = np.random.default_rng(seed)
    W = normal_bf16(rng, (N, K), w_std)
    A = normal_bf16(rng, (r, K), a_std)
    B = normal_bf16(rng, (N, r), b_std)
    X = normal_bf16(rng, (T, K), 1.0)
    dY = normal_bf16(rng, (T, N), 1.0)
    return LinearCase(W, X, A, B, dY, alpha)
