"""Parameter counts implied by the layer shapes the oracle uses.

Test infrastructure only (see the package docstring). These pin the shapes
(embed_dim, num_experts, expert_dim, top_k, shared width) to the checkpoint
counts that the Gemma-4-26B-A4B model card prints ("Calculated ... safetensors
headers" rows) and to the TransformerConfig of gm.nn.Gemma4_26B_A4B.

Norm scale vectors are left out: they are a few thousand parameters per layer
and vanish in the printed rounding (0.1M / 0.001B).
"""

from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Gemma4Config:
    """Fields of gm.nn.Gemma4_26B_A4B's TransformerConfig that set parameter counts."""

    num_embed: int = 262144
    embed_dim: int = 2816
    hidden_dim: int = 2112  # = moe_dense_hidden_dim, the shared MLP width
    num_heads: int = 16
    head_dim: int = 256
    num_kv_heads: int = 8
    num_global_kv_heads: int = 2
    global_key_size: int = 512
    k_eq_v_global: bool = True
    num_experts: int = 128
    expert_dim: int = 704
    top_k_experts: int = 8
    num_layers: int = 30
    global_every: int = 6  # attention_types: five LOCAL_SLIDING then one GLOBAL, repeated


def expert_params_per_layer(c: Gemma4Config) -> int:
    """gate + up [D, F] and down [F, D] for each of the E experts."""
    return c.num_experts * 3 * c.embed_dim * c.expert_dim


def active_expert_params_per_layer(c: Gemma4Config) -> int:
    """The top_k of E experts a token runs through."""
    return expert_params_per_layer(c) * c.top_k_experts // c.num_experts


def shared_mlp_params(c: Gemma4Config) -> int:
    return 3 * c.embed_dim * c.hidden_dim


def router_params(c: Gemma4Config) -> int:
    return c.embed_dim * c.num_experts


def local_attention_params(c: Gemma4Config) -> int:
    q = c.embed_dim * c.num_heads * c.head_dim
    kv = 2 * c.embed_dim * c.num_kv_heads * c.head_dim
    o = c.num_heads * c.head_dim * c.embed_dim
    return q + kv + o


def global_attention_params(c: Gemma4Config) -> int:
    q = c.embed_dim * c.num_heads * c.global_key_size
    k = c.embed_dim * c.num_global_kv_heads * c.global_key_size
    v = 0 if c.k_eq_v_global else k
    o = c.num_heads * c.global_key_size * c.embed_dim
    return q + k + v + o


def layer_counts(c: Gemma4Config = Gemma4Config()) -> dict:
    n_global = c.num_layers // c.global_every
    n_local = c.num_layers - n_global
    ffn_dense = shared_mlp_params(c) + router_params(c)
    non_expert = c.num_layers * ffn_dense + n_local * local_attention_params(c) + n_global * global_attention_params(c)
    return {
        "expert_per_layer": expert_params_per_layer(c),
        "active_expert_per_layer": active_expert_params_per_layer(c),
        "largest_layer": global_attention_params(c) + ffn_dense + expert_params_per_layer(c),
        "backbone_total": non_expert + c.num_layers * expert_params_per_layer(c),
        "backbone_active": non_expert + c.num_layers * active_expert_params_per_layer(c),
        "embedding": c.num_embed * c.embed_dim,
    }


def block_flops_per_token(c: Gemma4Config = Gemma4Config()) -> dict:
    """Multiply-add FLOPs (2 per MAC) of one block per token."""
    d, f, s, e, k = c.embed_dim, c.expert_dim, c.hidden_dim, c.num_experts, c.top_k_experts
    return {
        "router": 2 * d * e,
        "expert_gate_up": k * 2 * 2 * d * f,
        "expert_down": k * 2 * f * d,
        "shared": 3 * 2 * d * s,
    }
