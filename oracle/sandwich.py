"""Float64 CPU oracle of the normalisation sandwich around the MoE block.

Test infrastructure only (see the package docstring).

What it computes, with the passage each step follows:

* The block normalisation layers are RMSNorm [Gemma-4-26B-A4B model card,
  "Normalization layer type in the blocks": RMSNorm] with epsilon 1e-6
  [model card, "Epsilon of the block normalization layers": 1e-06].
* They sit on both sides of the feed-forward block, "sandwich" = pre and post
  [model card, "Pre-norm, post-norm, or sandwich"; gm.nn.Gemma4_26B_A4B
  TransformerConfig use_post_ffw_norm=True].
* The block's output adds to the residual stream of width embed_dim
  [model card, "Residual stream width": 2816].

Readings where the pages are silent:

* RMSNorm(v) = gamma * v / sqrt(mean(v^2) + eps), a learned per-channel scale
  gamma [embed_dim] that multiplies (no offset);
* one pre-norm feeds the whole block: router, experts and shared MLP all read
  the normalised input, which is stored in bf16 (round to nearest even), the
  dtype the block computes in;
* the post-norm acts on the block output before any rounding, and the residual
  adds the raw block input x.
"""

from __future__ import annotations

import numpy as np

from oracle import moe_oracle as mo


def rms_norm(v, gamma=None, eps: float = mo.RMS_EPS) -> np.ndarray:
    """gamma * v / sqrt(mean(v^2) + eps) per row (gamma None: no scale)."""
    v = mo.f64(v)
    out = v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)
    return out if gamma is None else out * mo.f64(gamma)


def bf16_rne(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits),
    ties to even, straight from float64 (no intermediate float32). Returns
    float64 values that bf16 represents exactly; zeros stay zero."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)  # v = m * 2^e, 0.5 <= |m| < 1
    q = np.ldexp(np.round(np.ldexp(v, 8 - e)), e - 8)  # np.round: half to even
    return np.where(v == 0, 0.0, q)


def bf16_bits(v) -> np.ndarray:
    """bf16 bit patterns (uint16) of values that bf16 represents exactly."""
    f = np.asarray(v, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def sandwich_block(x, w_router, wg, wu, wd, sg, su, sd, gamma_pre, gamma_post, top_k: int = 8, bias=None,
                   routing=None, residual: bool = True):
    """out = x + RMSNorm_post(block(bf16(RMSNorm_pre(x)))).

    Returns a dict: out [T, D]; x_norm (the block input, bf16 bit patterns);
    ffn (the block's output); post (its normalised value); and the block's
    idx, w, logits."""
    x64 = mo.f64(x)
    xn = bf16_bits(bf16_rne(rms_norm(x64, gamma_pre)))
    blk = mo.moe_block(xn, w_router, wg, wu, wd, sg, su, sd, top_k=top_k, bias=bias, routing=routing)
    post = rms_norm(blk["out"], gamma_post)
    out = x64 + post if residual else post
    return {"out": out, "x_norm": xn, "ffn": blk["out"], "post": post, "idx": blk["idx"], "w": blk["w"],
            "logits": blk["logits"]}
