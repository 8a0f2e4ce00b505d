"""Seeded synthetic inputs for the grouped NF4 expert block.

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the method's arithmetic (no routing, no NF4
table, no quantisation, no GEMM).  Both the CUDA path and the CPU oracle take
their inputs from here.

Recipe (all streams seeded from ``(seed, tensor id)``):

* ``x`` bf16 [T, H] ~ N(0, 1); ``dY`` bf16 [T, H] ~ N(0, 1).
* router logits float32 [T, E]: ``"normal"`` is i.i.d. N(0, 1) (exchangeable,
  so every expert has the same expected load); ``"zipf"`` is
  ``log p[pi(e)] + Gumbel(0, 1)`` with ``p_i ~ i^-s`` (s = 1.1) and ``pi`` a
  seeded permutation of the experts -- top-k of Gumbel-perturbed log
  probabilities samples k distinct experts with probabilities ~ p, so group
  sizes range from a handful of tokens to nearly every token.
* NF4 stacks: codes i.i.d. uniform over the 16 levels (two per byte), and
  absmax per block of 64 distributed as the largest |w| of 64 draws of
  N(0, sigma^2), sampled exactly through its CDF ``(2 Phi(m/sigma) - 1)^64``.
  NF4's levels are equal-probability quantiles of the normal, so uniform codes
  are the code statistics of quantised normal weights up to the slight
  concentration toward the central levels that normalising by the block's own
  maximum causes.
* LoRA ``A[e]`` bf16 ~ N(0, 1/sqrt(in)) (the second argument is the standard
  deviation); ``B[e]`` bf16 ~ N(0, 0.01), or exactly zero for the B = 0
  variant (the method's initial state).
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict

import numpy as np
import torch
from scipy.special import ndtri

BLOCK = 64


@dataclass(frozen=True)
class Config:
    name: str
    E: int
    H: int
    I: int  # noqa: E741
    top_k: int
    T: int
    r: int
    alpha: float
    routing: str          # "normal" or "zipf"
    seed: int
    b_zero: bool = False
    sigma_w: float = 0.02
    zipf_s: float = 1.1
    passes: tuple = ("fwd",)
    note: str = ""

    @property
    def N(self) -> int:
        return self.T * self.top_k

    @property
    def scaling(self) -> float:
        return self.alpha / self.r


# The five workloads (and the B = 0 variant of the tiny one).
CONFIGS: Dict[str, Config] = {
    "tiny": Config("tiny", E=4, H=64, I=128, top_k=2, T=32, r=8, alpha=16.0,
                   routing="normal", seed=1, passes=("fwd", "dgrad", "wgrad"),
                   note="tiny MoE block, E4 H64 I128 top-2 T32 r8"),
    "tiny_b0": Config("tiny_b0", E=4, H=64, I=128, top_k=2, T=32, r=8, alpha=16.0,
                      routing="normal", seed=11, b_zero=True,
                      passes=("fwd", "dgrad", "wgrad"),
                      note="tiny MoE block with B = 0"),
    "mixtral": Config("mixtral", E=8, H=4096, I=14336, top_k=2, T=4096, r=16,
                      alpha=32.0, routing="normal", seed=2, passes=("fwd",),
                      note="Mixtral-like layer, E8 H4096 I14336 top-2 T4096 r16"),
    "finegrained": Config("finegrained", E=128, H=2048, I=768, top_k=8, T=8192,
                          r=16, alpha=32.0, routing="zipf", seed=3,
                          passes=("fwd", "dgrad"),
                          note="fine-grained layer, E128 H2048 I768 top-8 T8192 r16, Zipf(1.1)"),
    "decode": Config("decode", E=128, H=2048, I=768, top_k=8, T=16, r=16,
                     alpha=32.0, routing="normal", seed=4, passes=("fwd",),
                     note="decode batch, E128 H2048 I768 top-8 T16 r16"),
    "train": Config("train", E=128, H=2048, I=768, top_k=8, T=8192, r=64,
                    alpha=128.0, routing="zipf", seed=5,
                    passes=("fwd", "dgrad", "wgrad"),
                    note="full QLoRA step, E128 H2048 I768 top-8 T8192 r64 a128, Zipf(1.1)"),
}


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 values -> bfloat16 bit patterns (torch's conversion)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, stream]))


def _normal_bf16(rng, shape, std) -> np.ndarray:
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


def _nf4_stack(rng, E, rows, K, sigma):
    codes = rng.integers(0, 256, size=(E, rows, K // 2), dtype=np.uint8)
    u = rng.random((E, rows, K // BLOCK))
    m = ndtri((1.0 + u ** (1.0 / BLOCK)) / 2.0)
    absmax = (sigma * m).astype(np.float32)
    return codes, absmax


def router_logits(cfg: Config, T: int = None, data_rank: int = 0) -> np.ndarray:
    T = cfg.T if T is None else T
    rng = _rng(cfg.seed, 2 + 1000 * data_rank)
    if cfg.routing == "normal":
        return rng.standard_normal((T, cfg.E), dtype=np.float32)
    if cfg.routing == "zipf":
        p = np.arange(1, cfg.E + 1, dtype=np.float64) ** (-cfg.zipf_s)
        p /= p.sum()
        perm = _rng(cfg.seed, 10).permutation(cfg.E)  # the expert popularity order is a model property
        logp = np.log(p[perm])
        u = rng.random((T, cfg.E))
        gumbel = -np.log(-np.log(u))
        return (logp[None, :] + gumbel).astype(np.float32)
    raise ValueError(cfg.routing)


@dataclass
class Problem:
    cfg: Config
    x: np.ndarray                 # uint16 bf16 bits [T, H]
    logits: np.ndarray            # float32 [T, E]
    gate_up_nf4: np.ndarray       # uint8 [E, 2I, H/2]
    gate_up_absmax: np.ndarray    # float32 [E, 2I, H/64]
    down_nf4: np.ndarray          # uint8 [E, H, I/2]
    down_absmax: np.ndarray       # float32 [E, H, I/64]
    A_gu: np.ndarray              # uint16 [E, r, H]
    B_gu: np.ndarray              # uint16 [E, 2I, r]
    A_d: np.ndarray               # uint16 [E, r, I]
    B_d: np.ndarray               # uint16 [E, H, r]
    dY: np.ndarray                # uint16 [T, H]
    extra: dict = field(default_factory=dict)


def make_problem(cfg: Config, T: int = None, data_rank: int = 0) -> Problem:
    """All inputs of one workload (``T`` overrides the token count).

    ``data_rank`` selects an independent batch (tokens, logits, upstream
    gradient) over the same weights, as data-parallel ranks see it.
    """
    T = cfg.T if T is None else T
    E, H, I, r = cfg.E, cfg.H, cfg.I, cfg.r
    x = _normal_bf16(_rng(cfg.seed, 1 + 1000 * data_rank), (T, H), 1.0)
    logits = router_logits(cfg, T, data_rank)
    gu_codes, gu_absmax = _nf4_stack(_rng(cfg.seed, 3), E, 2 * I, H, cfg.sigma_w)
    d_codes, d_absmax = _nf4_stack(_rng(cfg.seed, 4), E, H, I, cfg.sigma_w)
    A_gu = _normal_bf16(_rng(cfg.seed, 5), (E, r, H), 1.0 / np.sqrt(H))
    A_d = _normal_bf16(_rng(cfg.seed, 6), (E, r, I), 1.0 / np.sqrt(I))
    if cfg.b_zero:
        B_gu = np.zeros((E, 2 * I, r), dtype=np.uint16)
        B_d = np.zeros((E, H, r), dtype=np.uint16)
    else:
        B_gu = _normal_bf16(_rng(cfg.seed, 7), (E, 2 * I, r), 0.01)
        B_d = _normal_bf16(_rng(cfg.seed, 8), (E, H, r), 0.01)
    dY = _normal_bf16(_rng(cfg.seed, 9 + 1000 * data_rank), (T, H), 1.0)
    return Problem(cfg, x, logits, gu_codes, gu_absmax, d_codes, d_absmax,
                   A_gu, B_gu, A_d, B_d, dY)


def dense_expert_weights(cfg: Config):
    """Dense bf16 expert stacks drawn ~ N(0, sigma_w): ``gate_up`` [E, 2I, H] and ``down`` [E, H, I]
    (bf16 bit patterns), the weights the workloads describe before NF4 quantisation.  Random draws only:
    quantising them is the caller's step."""
    E, H, I = cfg.E, cfg.H, cfg.I
    gu = _normal_bf16(_rng(cfg.seed, 13), (E, 2 * I, H), cfg.sigma_w)
    dn = _normal_bf16(_rng(cfg.seed, 14), (E, H, I), cfg.sigma_w)
    return gu, dn


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
