"""Seeded synthetic inputs shared by the CPU oracle tests, the GPU tests and the benchmark.

This module holds no arithmetic of the decoding method: it only draws numbers.
Everything it returns is a plain NumPy array, so neither the oracle nor the CUDA
library depends on the other through it.

- Model shapes: a tiny 2-layer decoder and the Qwen3-8B shape (36 layers, hidden
  4096, 32 query / 8 key-value heads, head_dim 128, FFN 12288, vocab 151936),
  each with a same-shaped draft attention module per layer (Orthrus,
  "Approach": a trainable diffusion attention path per layer that shares the
  frozen backbone's KV cache).
- Weights: N(0, 0.02) float32 from NumPy PCG64, one SeedSequence per tensor
  chunk, rounded to bfloat16 (round-to-nearest-even) and returned as uint16 bit
  patterns. Norm gains are 1.0 unless ``gain_std`` asks for random gains.
- Prompts: uniform token ids.
- Planted drafts: a per-step accept length ``a`` from a geometric law and the
  drafts that realise it against a given greedy token stream.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np

__all__ = [
    "ModelShape", "TINY", "TINY_QK", "QWEN3_8B", "tensor_specs", "make_weights",
    "make_prompt", "round_to_bf16_bits", "bf16_bits_to_f32", "planted_accepts",
    "planted_accepts_stratified", "capped_geometric_mean", "planted_drafts", "uniform_tokens", "normal_bf16",
]


@dataclass(frozen=True)
class ModelShape:
    """Decoder shape. ``mask_id`` is the token placed at draft-block positions 2..K."""

    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    d_ff: int
    vocab: int
    qk_norm: bool
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6

    @property
    def mask_id(self) -> int:
        return self.vocab - 1

    @property
    def group(self) -> int:
        return self.n_heads // self.n_kv_heads

    @property
    def qkv_rows(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim


TINY = ModelShape("tiny", 2, 256, 4, 2, 64, 768, 1024, qk_norm=False)
TINY_QK = replace(TINY, name="tiny_qk", qk_norm=True)
QWEN3_8B = ModelShape("qwen3_8b", 36, 4096, 32, 8, 128, 12288, 151936, qk_norm=True)


def tensor_specs(shape: ModelShape):
    """Ordered list of (name, dims, kind) with kind in {"base", "draft", "gain"}.

    Layout conventions (row-major, rows = output features):
      w_qkv   [(H + 2 Hkv) d, D]  rows: q heads, then k heads, then v heads
      w_o     [D, H d]
      w_gate_up [2F, D]           rows 0..F-1 gate, F..2F-1 up
      w_down  [D, F]
      lm_head [V, D], embed [V, D]
    """
    D, H, Hkv, d, F, V = (shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                          shape.d_ff, shape.vocab)
    specs = [("embed", (V, D), "base")]
    for l in range(shape.n_layers):
        p = f"l{l}."
        specs += [
            (p + "attn_norm", (D,), "gain"),
            (p + "w_qkv", (shape.qkv_rows, D), "base"),
            (p + "w_o", (D, H * d), "base"),
            (p + "q_norm", (d,), "gain"),
            (p + "k_norm", (d,), "gain"),
            (p + "mlp_norm", (D,), "gain"),
            (p + "w_gate_up", (2 * F, D), "base"),
            (p + "w_down", (D, F), "base"),
            (p + "wd_qkv", (shape.qkv_rows, D), "draft"),
            (p + "wd_o", (D, H * d), "draft"),
            (p + "wd_q_norm", (d,), "gain"),
            (p + "wd_k_norm", (d,), "gain"),
        ]
    specs += [("final_norm", (D,), "gain"), ("lm_head", (V, D), "base")]
    return specs


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


_CHUNK = 1 << 24  # elements per independently seeded chunk


def _normal_bf16(seed: int, tensor_index: int, n: int, std: float, out: np.ndarray, pool) -> None:
    def job(c):
        lo = c * _CHUNK
        hi = min(n, lo + _CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(tensor_index, c))))
        a = g.standard_normal(hi - lo, dtype=np.float32)
        a *= np.float32(std)
        out[lo:hi] = round_to_bf16_bits(a)
    list(pool.map(job, range((n + _CHUNK - 1) // _CHUNK)))


def make_weights(shape: ModelShape, seed_base: int, seed_draft: int, std: float = 0.02,
                 gain_std: float = 0.0, gain_seed: int = 7, threads: int | None = None):
    """Return {name: array}: uint16 bf16 bits for matrices, float32 for norm gains.

    Base tensors draw from ``seed_base``, draft-module tensors from ``seed_draft``;
    each tensor is seeded by its index in ``tensor_specs`` so values do not depend
    on thread count. Gains are exactly 1.0 when ``gain_std == 0``.
    """
    threads = threads or max(1, len(os.sched_getaffinity(0)))
    out = {}
    with ThreadPoolExecutor(threads) as pool:
        for idx, (name, dims, kind) in enumerate(tensor_specs(shape)):
            n = int(np.prod(dims))
            if kind == "gain":
                if gain_std == 0.0:
                    out[name] = np.ones(dims, dtype=np.float32)
                else:
                    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(gain_seed, spawn_key=(idx,))))
                    out[name] = (1.0 + gain_std * g.standard_normal(n)).astype(np.float32).reshape(dims)
                continue
            buf = np.empty(n, dtype=np.uint16)
            _normal_bf16(seed_base if kind == "base" else seed_draft, idx, n, std, buf, pool)
            out[name] = buf.reshape(dims)
    return out


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    """N(0, std) float32 rounded to bfloat16; uint16 bit patterns of the given shape."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(0xB16,))))
    a = g.standard_normal(int(np.prod(shape)), dtype=np.float32) * np.float32(std)
    return round_to_bf16_bits(a).reshape(shape)


def uniform_tokens(vocab: int, n: int, seed: int) -> np.ndarray:
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(0xC0DE,))))
    return g.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_prompt(shape: ModelShape, length: int, seed: int) -> np.ndarray:
    """Uniform token ids in [0, vocab)."""
    return uniform_tokens(shape.vocab, length, seed)


def planted_accepts(n_steps: int, mean: float, K: int, seed: int) -> np.ndarray:
    """Accept lengths a_t ~ Geometric on {0,1,...} with E[a] = mean, then capped at K.

    P(a = k) = p (1 - p)^k with p = 1 / (mean + 1).
    """
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(0xACC,))))
    p = 1.0 / (mean + 1.0)
    a = g.geometric(p, size=n_steps) - 1  # numpy's geometric counts trials, support {1,2,...}
    return np.minimum(a, K).astype(np.int32)


def capped_geometric_mean(mean: float, K: int) -> float:
    """E[min(a, K)] for a ~ Geometric on {0,1,...} with E[a] = mean:
    sum_{k=1..K} P(a >= k) = (1 - p) (1 - (1 - p)^K) / p with p = 1 / (mean + 1)."""
    p = 1.0 / (mean + 1.0)
    return (1.0 - p) * (1.0 - (1.0 - p) ** K) / p


def planted_accepts_stratified(n_steps: int, mean: float, K: int, seed: int) -> np.ndarray:
    """n_steps accept lengths of the same capped geometric law, drawn by stratified
    sampling: the law's quantiles at u = (i + 1/2) / n_steps, i = 0..n_steps-1, in a
    seeded random order. Their mean follows the law's mean to O(1/n_steps) rather than
    O(1/sqrt(n_steps)), so a short timed window commits a reproducible number of tokens.

    Quantile: the smallest k with P(a <= k) = 1 - (1 - p)^(k+1) >= u, i.e.
    k = ceil(log(1 - u) / log(1 - p)) - 1, then capped at K.
    """
    p = 1.0 / (mean + 1.0)
    u = (np.arange(n_steps, dtype=np.float64) + 0.5) / n_steps
    k = np.ceil(np.log1p(-u) / np.log1p(-p)) - 1.0
    a = np.clip(k, 0, K).astype(np.int32)
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(0x57A,))))
    g.shuffle(a)
    return a


def planted_drafts(stream: np.ndarray, n: int, a: int, K: int, vocab: int, rng: np.random.Generator) -> np.ndarray:
    """Drafts d_1..d_K for a step whose cache holds positions [0, n) and whose pending
    token is ``stream[n]``: d_i = stream[n + i] for i <= a; if a < K, d_{a+1} differs
    from ``stream[n + a + 1]`` by construction; the rest are uniform ids.
    """
    d = rng.integers(0, vocab, size=K, dtype=np.int64)
    d[:a] = stream[n + 1:n + 1 + a]
    if a < K:
        u = int(rng.integers(0, vocab - 1))
        d[a] = (int(stream[n + a + 1]) + 1 + u) % vocab
    return d.astype(np.int32)
