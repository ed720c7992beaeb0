"""Seeded synthetic inputs for the Gemma-4-26B-A4B MoE feed-forward block.

This module only draws random numbers and stores them as bf16 bit patterns
(uint16 numpy arrays). It holds none of the block's arithmetic, so both the
CUDA path and the CPU oracle can take their inputs from it.

Recipe (no trained checkpoint is available, so weights are random-init of the
published architecture):

* weights: one seeded ``torch.Generator`` (CPU) stream, drawn in the order
  router, expert gate, expert up, expert down, shared gate, shared up, shared
  down, each float32 ``N(0, 0.02^2)`` (the checkpoint's ``initializer_range``
  0.02), rounded to bf16 with round-to-nearest-even;
* activations ``x``: seed 1, float32 ``N(0, 1)`` rounded to bf16;
* the skewed-routing benchmark adds a per-expert router bias
  ``2.0 * ln(p_r)`` with ``p_r`` the Zipf(s=1.1) probability of rank
  ``r = e + 1`` over the experts.

Shapes follow the layer's statement: embed_dim 2816, 128 experts of width 704,
top-8, a dense shared MLP of width 2112 (gemma-llm ``Gemma4_26B_A4B``
TransformerConfig; HF ``config.json`` text_config).
"""

from __future__ import annotations

import dataclasses

import numpy as np

EMBED_DIM = 2816
NUM_EXPERTS = 128
EXPERT_DIM = 704
HIDDEN_DIM = 2112
TOP_K = 8
INIT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Dims:
    embed_dim: int = EMBED_DIM
    num_experts: int = NUM_EXPERTS
    expert_dim: int = EXPERT_DIM
    hidden_dim: int = HIDDEN_DIM


GEMMA4_26B_A4B = Dims()


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(gen, shape, std: float) -> np.ndarray:
    import torch

    a = torch.empty(tuple(shape), dtype=torch.float32).normal_(0.0, std, generator=gen)
    return a.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _generator(seed: int):
    import torch

    return torch.Generator().manual_seed(seed)


@dataclasses.dataclass
class BlockWeights:
    """bf16 bit patterns, row-major, in the layouts the C ABI takes."""

    w_router: np.ndarray  # [D, E]
    wg: np.ndarray  # [E, D, F]
    wu: np.ndarray  # [E, D, F]
    wd: np.ndarray  # [E, F, D]
    sg: np.ndarray  # [D, S]
    su: np.ndarray  # [D, S]
    sd: np.ndarray  # [S, D]

    @property
    def dims(self) -> Dims:
        return Dims(self.w_router.shape[0], self.w_router.shape[1], self.wg.shape[2], self.sg.shape[1])


def make_weights(dims: Dims = GEMMA4_26B_A4B, seed: int = 0, std: float = INIT_STD) -> BlockWeights:
    d, e, f, s = dims.embed_dim, dims.num_experts, dims.expert_dim, dims.hidden_dim
    rng = _generator(seed)
    return BlockWeights(
        w_router=_normal_bf16(rng, (d, e), std),
        wg=_normal_bf16(rng, (e, d, f), std),
        wu=_normal_bf16(rng, (e, d, f), std),
        wd=_normal_bf16(rng, (e, f, d), std),
        sg=_normal_bf16(rng, (d, s), std),
        su=_normal_bf16(rng, (d, s), std),
        sd=_normal_bf16(rng, (s, d), std),
    )


# The dense E4B sibling (gm.nn.Gemma4_E4B TransformerConfig: embed_dim 2560,
# hidden_dim 10240, enable_moe=False).
E4B_EMBED_DIM = 2560
E4B_HIDDEN_DIM = 10240


@dataclasses.dataclass
class DenseWeights:
    wg: np.ndarray  # [D, S]
    wu: np.ndarray  # [D, S]
    wd: np.ndarray  # [S, D]


def make_dense_weights(embed_dim: int = E4B_EMBED_DIM, hidden_dim: int = E4B_HIDDEN_DIM, seed: int = 0,
                       std: float = INIT_STD) -> DenseWeights:
    """Gate, up, down of a dense GeGLU FFN from one seeded stream, N(0, std^2) -> bf16 bits."""
    rng = _generator(seed)
    return DenseWeights(
        wg=_normal_bf16(rng, (embed_dim, hidden_dim), std),
        wu=_normal_bf16(rng, (embed_dim, hidden_dim), std),
        wd=_normal_bf16(rng, (hidden_dim, embed_dim), std),
    )


def make_x(tokens: int, embed_dim: int = EMBED_DIM, seed: int = 1) -> np.ndarray:
    return _normal_bf16(_generator(seed), (tokens, embed_dim), 1.0)


def zipf_router_bias(num_experts: int = NUM_EXPERTS, s: float = 1.1, amplitude: float = 2.0) -> np.ndarray:
    """Per-expert router bias of the skewed-routing workload (float32)."""
    ranks = np.arange(1, num_experts + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    return (amplitude * np.log(p)).astype(np.float32)


def sample_tokens(tokens: int, count: int, seed: int = 3) -> np.ndarray:
    """A seeded sorted subset of token indices (all of them when count >= tokens)."""
    if count >= tokens:
        return np.arange(tokens)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(tokens, size=count, replace=False))
