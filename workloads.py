"""Seeded synthetic inputs for the int3 + low-rank-compensator MoE forward.

This module only draws random numbers and shapes them: it holds none of the
method's arithmetic (no quantisation, no routing, no GEMM).  The same host
arrays feed the CUDA library and the CPU oracle, so both sides see identical
bits.

Workloads (the MoE shapes follow the "Background" and "Experimental Setup &
Results" sections of "MiLo: Efficient Quantized MoE Inference with Mixture of
Low-Rank Compensators", which evaluate Mixtral-8x7B and DeepSeekMoE-style
models in W3A16):

* ``single``   one expert, decode: x fp16 [1, 1024] ~ N(0,1); W fp16
  [1024, 1024] ~ N(0, 0.02) with 0.1 % of the entries multiplied by 20; rank
  16 compensator U [1024, 16], V [16, 1024] ~ N(0, 0.01).
* ``mixtral``  Mixtral-8x7B-shaped SwiGLU MoE layer, decode: H 4096, I 14336,
  8 experts, top-2 renormalised softmax over fp16 logits ~ N(0,1), ranks drawn
  per expert from {0, 16, 32, 64}, 16 tokens of bf16 ~ N(0,1).
* ``deepseek`` DeepSeekMoE-16B-shaped layer: H 2048, I 1408, 64 routed experts
  top-6 (full softmax, no renormalisation) plus 2 always-on shared experts,
  ranks from {0, 8, 16, 32}, 64 bf16 tokens, logits ~ N(0,1) plus a fixed
  per-expert bias ~ N(0, 0.5) that skews the load.
* ``sweep``    the Mixtral w1 projection (4096 -> 14336, 8 experts, rank 32)
  with T in {1, 4, 16, 64, 256, 1024} rows, each row given one expert drawn
  from a truncated Zipf law P(e) ~ (e+1)^-1.1.
* ``prefill``  the Mixtral-shaped layer with 8192 tokens, iid N(0,1) logits
  (uniform-random top-2 by symmetry) and rank 64 on every expert.

Every weight matrix uses the single-expert recipe (N(0, 0.02) plus 0.1 %
outliers x20); every compensator uses N(0, 0.01).
"""
from __future__ import annotations

import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

SEED = 0


# ----------------------------------------------------------------------------
# bit-level helpers (storage formats only)
# ----------------------------------------------------------------------------

def f32_to_f16_bits(a: np.ndarray) -> np.ndarray:
    """IEEE round-to-nearest-even fp32 -> fp16, returned as uint16 bits."""
    return np.asarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 (finite inputs), as uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float32)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# random streams
# ----------------------------------------------------------------------------

def rng_for(workload: str, tensor: str, index: int = 0, seed: int = SEED) -> np.random.Generator:
    """One independent PCG64 stream per (seed, workload, tensor, index)."""
    key = [seed, zlib.crc32(workload.encode()), zlib.crc32(tensor.encode()), index]
    return np.random.default_rng(np.random.SeedSequence(key))


def gen_weight(rng: np.random.Generator, n: int, k: int, std: float = 0.02,
               outlier_frac: float = 0.001, outlier_mul: float = 20.0) -> np.ndarray:
    """fp16 bits [n, k]: N(0, std) with round(frac*n*k) distinct entries x mul."""
    w = rng.standard_normal(n * k, dtype=np.float32)
    w *= np.float32(std)
    n_out = int(round(outlier_frac * n * k))
    if n_out:
        idx = rng.choice(n * k, size=n_out, replace=False)
        w[idx] *= np.float32(outlier_mul)
    return f32_to_f16_bits(w).reshape(n, k)


def gen_normal_f16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    a = rng.standard_normal(int(np.prod(shape)), dtype=np.float32) * np.float32(std)
    return f32_to_f16_bits(a).reshape(shape)


def gen_activations(rng: np.random.Generator, t: int, h: int, dtype: str) -> np.ndarray:
    a = rng.standard_normal(t * h, dtype=np.float32).reshape(t, h)
    return f32_to_bf16_bits(a) if dtype == "bf16" else f32_to_f16_bits(a)


def gen_zipf_ids(rng: np.random.Generator, t: int, e: int, s: float = 1.1) -> np.ndarray:
    p = (np.arange(e, dtype=np.float64) + 1.0) ** (-s)
    p /= p.sum()
    return rng.choice(e, size=t, p=p).astype(np.int32)


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

@dataclass
class Projection:
    """One fp16 weight W [n, k] and its rank-r compensator U [n, r], V [r, k]."""
    W: np.ndarray
    U: np.ndarray
    V: np.ndarray

    @property
    def n(self) -> int:
        return self.W.shape[0]

    @property
    def k(self) -> int:
        return self.W.shape[1]

    @property
    def rank(self) -> int:
        return self.U.shape[1]


@dataclass
class MoEWorkload:
    name: str
    hidden: int
    inter: int
    n_routed: int
    n_shared: int
    top_k: int
    renorm: bool
    T: int
    x_dtype: str
    x: np.ndarray                     # uint16 bits [T, H]
    logits: np.ndarray | None         # fp16 bits [T, E] (None when ids are given)
    ids: np.ndarray | None            # int32 [T, k] when routing is given
    ranks: list = field(default_factory=list)
    experts: list = field(default_factory=list)   # list of dict(w1=, w3=, w2=) Projections

    @property
    def n_experts(self) -> int:
        return self.n_routed + self.n_shared


def make_projection(workload: str, tensor: str, index: int, n: int, k: int, rank: int) -> Projection:
    W = gen_weight(rng_for(workload, tensor + ".W", index), n, k)
    r_u = rng_for(workload, tensor + ".U", index)
    r_v = rng_for(workload, tensor + ".V", index)
    U = gen_normal_f16(r_u, (n, rank), 0.01)
    V = gen_normal_f16(r_v, (rank, k), 0.01)
    return Projection(W, U, V)


def _experts(name: str, hidden: int, inter: int, ranks: list, threads: int = 8,
             which=("w1", "w3", "w2")) -> list:
    jobs = []
    for e, r in enumerate(ranks):
        for wname in which:
            n, k = (inter, hidden) if wname in ("w1", "w3") else (hidden, inter)
            jobs.append((e, wname, n, k, r))
    with ThreadPoolExecutor(threads) as ex:
        projs = list(ex.map(lambda j: make_projection(name, j[1], j[0], j[2], j[3], j[4]), jobs))
    out = [dict() for _ in ranks]
    for (e, wname, *_), p in zip(jobs, projs):
        out[e][wname] = p
    return out


def single(seed_workload: str = "single", n: int = 1024, k: int = 1024, rank: int = 16,
           T: int = 1) -> tuple:
    """The single-expert decode case: returns (x fp16 bits [T, k], Projection)."""
    x = gen_activations(rng_for(seed_workload, "x"), T, k, "f16")
    return x, make_projection(seed_workload, "w", 0, n, k, rank)


def mixtral(T: int = 16, name: str = "mixtral", hidden: int = 4096, inter: int = 14336,
            ranks=None, rank_choices=(0, 16, 32, 64), n_experts: int = 8) -> MoEWorkload:
    E = n_experts
    if ranks is None:
        ranks = list(rng_for(name, "ranks").choice(rank_choices, size=E).astype(int))
    x = gen_activations(rng_for(name, "x"), T, hidden, "bf16")
    logits = gen_normal_f16(rng_for(name, "logits"), (T, E), 1.0)
    return MoEWorkload(name, hidden, inter, E, 0, 2, True, T, "bf16", x, logits, None,
                       ranks, _experts(name, hidden, inter, ranks))


def deepseek(T: int = 64, name: str = "deepseek", hidden: int = 2048, inter: int = 1408,
             rank_choices=(0, 8, 16, 32)) -> MoEWorkload:
    E, S = 64, 2
    ranks = list(rng_for(name, "ranks").choice(rank_choices, size=E + S).astype(int))
    x = gen_activations(rng_for(name, "x"), T, hidden, "bf16")
    bias = rng_for(name, "bias").standard_normal(E, dtype=np.float32) * np.float32(0.5)
    raw = rng_for(name, "logits").standard_normal(T * E, dtype=np.float32).reshape(T, E)
    logits = f32_to_f16_bits(raw + bias[None, :])
    return MoEWorkload(name, hidden, inter, E, S, 6, False, T, "bf16", x, logits, None,
                       ranks, _experts(name, hidden, inter, ranks))


def prefill(T: int = 8192, name: str = "prefill", n_experts: int = 8) -> MoEWorkload:
    return mixtral(T=T, name=name, ranks=[64] * n_experts, n_experts=n_experts)


def sweep(T: int, name: str = "sweep", hidden: int = 4096, inter: int = 14336,
          rank: int = 32) -> MoEWorkload:
    """Single w1 projection, each row routed to one Zipf-drawn expert (k = 1)."""
    E = 8
    ranks = [rank] * E
    x = gen_activations(rng_for(name, "x", T), T, hidden, "bf16")
    ids = gen_zipf_ids(rng_for(name, "ids", T), T, E).reshape(T, 1)
    exps = _experts(name, hidden, inter, ranks, which=("w1",))
    return MoEWorkload(name, hidden, inter, E, 0, 1, False, T, "bf16", x, None, ids, ranks, exps)


def small_moe(name: str = "small", T: int = 5, hidden: int = 256, inter: int = 384,
              n_routed: int = 4, n_shared: int = 1, top_k: int = 2, renorm: bool = True,
              rank_choices=(0, 8, 16), x_dtype: str = "bf16") -> MoEWorkload:
    """A reduced layer (same recipe, small shapes) that the oracle finishes in seconds."""
    ranks = list(rng_for(name, "ranks").choice(rank_choices, size=n_routed + n_shared).astype(int))
    x = gen_activations(rng_for(name, "x"), T, hidden, x_dtype)
    logits = gen_normal_f16(rng_for(name, "logits"), (T, n_routed), 1.0)
    return MoEWorkload(name, hidden, inter, n_routed, n_shared, top_k, renorm, T, x_dtype, x,
                       logits, None, ranks, _experts(name, hidden, inter, ranks))
