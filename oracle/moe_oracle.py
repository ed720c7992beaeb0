"""Float64 CPU oracle of one Gemma-4-26B-A4B MoE feed-forward block.

Test infrastructure only (see the package docstring).

What the block computes, with the passage each step follows:

* Every layer's FFN is two branches, a mixture-of-experts branch and a dense
  shared MLP branch, whose outputs add [gm.nn.Gemma4_26B_A4B, class
  docstring: "Each layer has: A MoE branch ... A dense shared MLP branch";
  Gemma-4-26B-A4B model card, "Always-on experts per MoE layer": 1].
* Router: one linear map embed_dim -> num_experts of the block input, no bias
  [G4-MeroMero-26B-A4B-NVFP4 config.json, quantization_config.ignore lists
  ``layers.N.router.proj``; model card, "FFN projections have bias terms": No].
* Gating is a softmax over the expert logits [model card, "Gating function over
  expert logits": softmax]; the top_k_experts = 8 largest are kept
  [TransformerConfig top_k_experts=8; model card "Routed experts selected per
  token": 8] and their weights renormalised to sum to one [model card,
  "Selected expert weights are renormalized to sum to 1": Yes].
* Each routed expert and the shared MLP is a bias-free GeGLU with the tanh
  approximation of GELU [model card, "FFN activation": GeGLU (tanh-approximate
  GELU); config.json text_config.hidden_activation gelu_pytorch_tanh], widths
  expert_dim = 704 and moe_dense_hidden_dim = 2112 [TransformerConfig].

Readings where the pages are silent:

* equal logits: the lower expert index ranks first;
* the order of the k selected experts ("slots") is by descending logit;
* GeGLU applies GELU to the gate projection and multiplies the up projection;
* the shared MLP is ungated (weight 1) and always present;
* the optional ``bias`` (skewed-routing workload only) adds to the logits
  before the softmax, so it moves both the selection and the weights.

Inputs may be float arrays or bf16 bit patterns (uint16); bf16 widens exactly.
"""

from __future__ import annotations

import numpy as np

GELU_C = np.sqrt(2.0 / np.pi)
GELU_A = 0.044715
RMS_EPS = 1e-6  # model card, "Epsilon of the block normalization layers": 1e-06


def f64(a) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) or any float array to float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ----------------------------------------------------------------- routing


def router_logits(x, w_router, bias=None) -> np.ndarray:
    """l[t, e] = sum_d x[t, d] * W_r[d, e]  (+ bias[e] when given)."""
    logits = f64(x) @ f64(w_router)
    if bias is not None:
        logits = logits + f64(bias)[None, :]
    return logits


def softmax(logits: np.ndarray) -> np.ndarray:
    """Softmax along the last axis (max-shifted; exact up to rounding)."""
    z = logits - logits.max(axis=-1, keepdims=True)
    p = np.exp(z)
    return p / p.sum(axis=-1, keepdims=True)


def select_top_k(logits: np.ndarray, k: int) -> np.ndarray:
    """Per row, the k expert indices with the largest logits, largest first.

    Equal logits rank the lower expert index first.
    """
    t_count, e_count = logits.shape
    out = np.empty((t_count, k), dtype=np.int64)
    experts = np.arange(e_count)
    for t in range(t_count):
        # lexsort: last key is primary -> descending logit, then ascending index
        order = np.lexsort((experts, -logits[t]))
        out[t] = order[:k]
    return out


def route(x, w_router, top_k: int, bias=None):
    """Softmax over all experts, keep the top_k, renormalise the kept weights.

    Returns (idx [T, k] int64, w [T, k] float64, logits [T, E] float64).
    """
    logits = router_logits(x, w_router, bias)
    p = softmax(logits)
    idx = select_top_k(logits, top_k)
    kept = np.take_along_axis(p, idx, axis=1)
    w = kept / kept.sum(axis=1, keepdims=True)
    return idx, w, logits


def top_k_gap(logits: np.ndarray, k: int) -> np.ndarray:
    """Per token, the logit gap between the k-th and (k+1)-th ranked expert.

    A token whose gap is tiny may legitimately be routed differently by an
    implementation that accumulates the logits in another order or precision.
    """
    s = -np.sort(-logits, axis=1)
    if k >= logits.shape[1]:
        return np.full(logits.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


def permutation(idx: np.ndarray, num_experts: int):
    """Expert-major ordering of the T*k (token, slot) assignments.

    Rows of expert e occupy [off[e], off[e] + cnt[e]) in ascending token order.
    Returns cnt [E], off [E+1] (exclusive scan), row_of [T, k], token_of [T*k].
    """
    t_count, k = idx.shape
    cnt = np.zeros(num_experts, dtype=np.int64)
    for t in range(t_count):
        for j in range(k):
            cnt[idx[t, j]] += 1
    off = np.zeros(num_experts + 1, dtype=np.int64)
    for e in range(num_experts):
        off[e + 1] = off[e] + cnt[e]
    fill = off[:-1].copy()
    row_of = np.empty((t_count, k), dtype=np.int64)
    token_of = np.empty(t_count * k, dtype=np.int64)
    for t in range(t_count):
        for j in range(k):
            e = idx[t, j]
            row_of[t, j] = fill[e]
            token_of[fill[e]] = t
            fill[e] += 1
    return cnt, off, row_of, token_of


# ------------------------------------------------------------------- GeGLU


def gelu_tanh(z):
    """GELU, tanh approximation: z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3)))."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(GELU_C * (z + GELU_A * z * z * z)))


def geglu_hidden(x, w_gate, w_up) -> np.ndarray:
    """h = gelu_tanh(x W_gate) * (x W_up)."""
    x = f64(x)
    return gelu_tanh(x @ f64(w_gate)) * (x @ f64(w_up))


def geglu_ffn(x, w_gate, w_up, w_down) -> np.ndarray:
    """GeGLU feed-forward: (gelu_tanh(x W_gate) * (x W_up)) W_down, no biases."""
    return geglu_hidden(x, w_gate, w_up) @ f64(w_down)


# ------------------------------------------------------------------- block


def dense_ffn(x, w_gate, w_up, w_down) -> np.ndarray:
    """The feed-forward of the dense E4B sibling [gm.nn.Gemma4_E4B TransformerConfig:
    enable_moe=False, hidden_dim=10240, embed_dim=2560]: the same bias-free
    GeGLU as the 26B-A4B block's shared MLP (reading: the pages give the E4B
    config only; its FFN is the family's gated FFN with gelu_pytorch_tanh)."""
    return geglu_ffn(x, w_gate, w_up, w_down)


def moe_block(x, w_router, wg, wu, wd, sg, su, sd, top_k: int = 8, bias=None, routing=None):
    """out = shared_mlp(x) + sum_k w[t, k] * expert_{idx[t, k]}(x[t]).

    ``routing`` = (idx, w) replaces the router's own choice (used to check the
    rest of the block given another implementation's routing).
    Returns a dict with out [T, D], idx, w, logits (None when routing is given),
    the shared branch ``shared`` and the routed sum ``routed``.
    """
    x = f64(x)
    t_count = x.shape[0]
    if routing is None:
        idx, w, logits = route(x, w_router, top_k, bias)
    else:
        idx, w = (np.asarray(routing[0], dtype=np.int64), np.asarray(routing[1], dtype=np.float64))
        logits = None
    shared = geglu_ffn(x, sg, su, sd) if t_count else np.zeros((0, x.shape[1]))
    routed = np.zeros_like(shared)
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        y = geglu_ffn(x[tok], wg[e], wu[e], wd[e])
        routed[tok] += w[tok, slot][:, None] * y
    return {"out": shared + routed, "idx": idx, "w": w, "logits": logits, "shared": shared, "routed": routed}


def moe_block_dense(x, w_router, wg, wu, wd, sg, su, sd, bias=None) -> np.ndarray:
    """The block with every expert kept (top_k = num_experts): the dense softmax mixture.

    out[t] = shared(x[t]) + sum_e softmax(l[t])_e * expert_e(x[t]). Evaluated
    token by token and expert by expert, without routing or permutation.
    """
    x = f64(x)
    p = softmax(router_logits(x, w_router, bias))
    out = np.zeros((x.shape[0], x.shape[1]))
    for t in range(x.shape[0]):
        xt = x[t : t + 1]
        out[t] = geglu_ffn(xt, sg, su, sd)[0]
        for e in range(p.shape[1]):
            out[t] += p[t, e] * geglu_ffn(xt, wg[e], wu[e], wd[e])[0]
    return out


def rms_normalize(x, eps: float = RMS_EPS) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) per row, no learned scale (inter-block norm of the stack workload)."""
    x = f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
