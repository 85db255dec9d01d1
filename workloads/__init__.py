"""Seeded synthetic inputs for the MoE token-routing pipeline.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It holds random draws and their shaping only (Gaussian
activations rounded to bf16, routing maps, router weights, fp32 expert
weights); none of the routing, quantisation, GEMV or combine arithmetic lives
here.

Recipe (one generator per (seed, stream)):
  stream 0      activations  x ~ N(0,1) fp32, rounded to bf16 (RNE), all N rows
  stream 1      routing      distinct experts per real row; garbage ids in
                             padding rows (uniform, repeats allowed), so a
                             missed mask routes them to real experts
  stream 2      router logits N(0,1); softmax over top_k, or sigmoid
                             normalised to sum 1
  stream 3      outlier mask (Bernoulli(p) per element, x *= mult)
  stream 4 + e  fp32 weights of expert e ~ N(0, 0.02), shape [N_out, K]
  stream 5000   synthetic expert outputs y (combine stage tests only)

Distinct sampling without replacement uses the Gumbel-top-k construction:
the k largest of log(p_e) + Gumbel noise are a draw of k experts in
successive-sampling order (uniform routing is the special case p = 1/E).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import ml_dtypes
import numpy as np

__all__ = [
    "Config", "CONFIGS", "config", "small_config",
    "activations_bf16", "routing", "router_weights", "expert_weights_f32",
    "expert_outputs_bf16", "bf16_bits_to_f32", "f32_to_bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    N: int                 # token rows (capacity, possibly a padded graph bucket)
    real: int              # real_token_count (rows >= real are padding)
    K: int                 # hidden size
    E: int                 # experts
    top_k: int
    N_out: int             # expert output width
    modes: tuple           # GEMV variants run on this workload: "w4a16", "w4a4"
    routing: str = "uniform"   # "uniform" | "zipf"
    zipf_s: float = 0.0
    router: str = "softmax"    # "softmax" | "sigmoid_norm"
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    epilogue: str = "none"     # combine epilogue: "none" | "identity" | "scale"
    seed: int = 0

    @property
    def slots(self) -> int:
        return self.N * self.top_k

    @property
    def routed_pairs(self) -> int:
        return min(max(self.real, 0), self.N) * self.top_k


# The five workloads: shapes, value distributions and routing skew as stated
# for the method's benchmark configurations.
CONFIGS = {
    "tiny": Config("tiny", N=16, real=13, K=256, E=8, top_k=2, N_out=256,
                   modes=("w4a16", "w4a4"), seed=101),
    "decode_30b_a3b": Config("decode_30b_a3b", N=128, real=128, K=2048, E=128, top_k=8,
                             N_out=768, modes=("w4a16",), seed=102),
    "decode_large_expert": Config("decode_large_expert", N=640, real=512, K=7168, E=256,
                                  top_k=8, N_out=2048, modes=("w4a4",), routing="zipf",
                                  zipf_s=1.1, router="sigmoid_norm", seed=103),
    "prefill_index_stress": Config("prefill_index_stress", N=16384, real=16384, K=4096, E=64,
                                   top_k=6, N_out=1408, modes=("w4a16",),
                                   epilogue="identity", seed=104),
    "gpt_oss_120b_w4a4": Config("gpt_oss_120b_w4a4", N=4096, real=3000, K=2880, E=128,
                                top_k=4, N_out=2880, modes=("w4a4",), routing="zipf",
                                zipf_s=0.8, outlier_frac=0.01, outlier_mult=20.0, seed=105),
}


def config(name: str) -> Config:
    return CONFIGS[name]


def small_config(name: str = "small", **kw) -> Config:
    """A reduced workload for tests: defaults span several tiles and a ragged tail."""
    base = dict(N=40, real=37, K=320, E=12, top_k=3, N_out=200, modes=("w4a16", "w4a4"),
                seed=7)
    base.update(kw)
    return Config(name, **base)


def _rng(cfg: Config, stream: int) -> np.random.Generator:
    return np.random.default_rng([cfg.seed, stream])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the raw uint16 bits."""
    return np.ascontiguousarray(np.asarray(x, np.float32).astype(ml_dtypes.bfloat16)).view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations_bf16(cfg: Config) -> np.ndarray:
    """x [N, K] as bf16 bits (uint16)."""
    x = _rng(cfg, 0).standard_normal((cfg.N, cfg.K), dtype=np.float32)
    if cfg.outlier_frac > 0:
        mask = _rng(cfg, 3).random((cfg.N, cfg.K)) < cfg.outlier_frac
        x = np.where(mask, x * np.float32(cfg.outlier_mult), x)
    return f32_to_bf16_bits(x)


def _expert_probs(cfg: Config, rng: np.random.Generator) -> np.ndarray:
    if cfg.routing == "uniform":
        return np.full(cfg.E, 1.0 / cfg.E)
    if cfg.routing == "zipf":
        perm = rng.permutation(cfg.E)
        p = np.empty(cfg.E)
        p[perm] = (np.arange(cfg.E) + 1.0) ** (-cfg.zipf_s)
        return p / p.sum()
    raise ValueError(cfg.routing)


def routing(cfg: Config) -> np.ndarray:
    """topk_ids [N, top_k] int64.

    Rows < real hold top_k distinct experts drawn from the routing
    distribution (slot order = draw order); rows >= real hold uniform garbage
    ids in [0, E) with repeats allowed.
    """
    rng = _rng(cfg, 1)
    p = _expert_probs(cfg, rng)
    real = min(max(cfg.real, 0), cfg.N)
    ids = np.empty((cfg.N, cfg.top_k), np.int64)
    if real:
        g = rng.gumbel(size=(real, cfg.E))
        keys = np.log(p)[None, :] + g
        order = np.argsort(-keys, axis=1, kind="stable")
        ids[:real] = order[:, : cfg.top_k]
    if cfg.N > real:
        ids[real:] = rng.integers(0, cfg.E, size=(cfg.N - real, cfg.top_k))
    return ids


def router_weights(cfg: Config) -> np.ndarray:
    """router_weights [N, top_k] fp32."""
    logits = _rng(cfg, 2).standard_normal((cfg.N, cfg.top_k))
    if cfg.router == "softmax":
        z = np.exp(logits - logits.max(axis=1, keepdims=True))
        w = z / z.sum(axis=1, keepdims=True)
    elif cfg.router == "sigmoid_norm":
        s = 1.0 / (1.0 + np.exp(-logits))
        w = s / s.sum(axis=1, keepdims=True)
    else:
        raise ValueError(cfg.router)
    return w.astype(np.float32)


def expert_weights_f32(cfg: Config, e: int, std: float = 0.02) -> np.ndarray:
    """fp32 weights of expert e, [N_out, K] ~ N(0, std)."""
    w = _rng(cfg, 4 + e).standard_normal((cfg.N_out, cfg.K), dtype=np.float32)
    return w * np.float32(std)


def expert_outputs_bf16(cfg: Config, scale: float = 1.0) -> np.ndarray:
    """Synthetic expert outputs y [N, top_k, N_out] as bf16 bits, for combine-only tests."""
    y = _rng(cfg, 5000).standard_normal((cfg.N, cfg.top_k, cfg.N_out), dtype=np.float32)
    return f32_to_bf16_bits(y * np.float32(scale))


def all_expert_weights_f32(cfg: Config, experts: Optional[list] = None) -> np.ndarray:
    """Stacked fp32 weights [E, N_out, K] (only for small configs)."""
    es = range(cfg.E) if experts is None else experts
    return np.stack([expert_weights_f32(cfg, e) for e in es])


def expert_weights_f32_many(cfg: Config, experts, threads: int = 8) -> np.ndarray:
    """Stacked fp32 weights of several experts, generated on a thread pool
    (numpy's generators release the GIL; every expert keeps its own stream)."""
    from concurrent.futures import ThreadPoolExecutor
    experts = list(experts)
    out = np.empty((len(experts), cfg.N_out, cfg.K), np.float32)

    def fill(i):
        out[i] = expert_weights_f32(cfg, experts[i])

    with ThreadPoolExecutor(max(1, min(threads, len(experts)))) as ex:
        list(ex.map(fill, range(len(experts))))
    return out
