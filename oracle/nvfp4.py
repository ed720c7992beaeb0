"""NVFP4 (e2m1 values, e4m3 group scales, fp32 tensor scale) in plain numpy.

Test infrastructure only (see the package docstring).

The checkpoint's quantisation recipe [G4-MeroMero-26B-A4B-NVFP4 config.json,
quantization_config.config_groups.group_0]: every Linear except the routers
holds 4-bit floats ("type": float, "num_bits": 4) in groups of 16 along the
input dimension ("group_size": 16), one ``float8_e4m3fn`` scale per group
("scale_dtype"), symmetric, strategy ``tensor_group`` (a per-tensor fp32 scale
above the group scales); weights are static ("dynamic": false), input
activations are quantised per call ("dynamic": "local") under a scale fixed
by calibration ("observer": static_minmax). The routers stay bf16 (the
``ignore`` list names every ``layers.N.router.proj``).

Reading of the arithmetic the page leaves open:

* tensor scale  G = 448 * 6 / amax(tensor), fp32 (G = 1 for an all-zero tensor);
* group scale   s = e4m3(fp32(fp32(amax_group / 6) * G)), round to nearest even,
                saturating at 448; s = 0 makes the whole group zero;
* value code    q = e2m1(fp32(x * fp32(G / s))), round to nearest even,
                saturating at 6 (IEEE sign kept, so tiny negatives give -0);
* dequantised   x^ = e2m1(q) * e4m3(s) / G.

The rounding decisions are taken in float32, the precision the format is
defined in, so an implementation that follows the same steps with IEEE fp32
operations reaches the same codes bit for bit.

Formats (OCP Microscaling spec): e2m1 = 1 sign, 2 exponent (bias 1), 1
mantissa bit, magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; e4m3 ("fn") = 1 sign, 4
exponent (bias 7), 3 mantissa bits, no infinities, 0x7F / 0xFF are NaN,
largest finite 448, smallest subnormal 2^-9.
"""

from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0
E4M3_MAX = 448.0
GROUP = 16


# ------------------------------------------------------------------- e2m1


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -mag, mag)


def e2m1_encode(v) -> np.ndarray:
    """Nearest e2m1 code (ties to the even code), saturating at +-6, sign kept."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    # distance to each of the 8 magnitudes; ties go to the even code
    d = np.abs(a[..., None] - E2M1_MAGNITUDES)
    best = np.argmin(d, axis=-1)
    dmin = np.take_along_axis(d, best[..., None], -1)[..., 0]
    # an exact tie can only be with the next code up: prefer whichever is even
    nxt = np.minimum(best + 1, 7)
    tie = (np.take_along_axis(d, nxt[..., None], -1)[..., 0] == dmin) & (nxt != best)
    best = np.where(tie & (best % 2 == 1), nxt, best)
    sign = np.signbit(v).astype(np.uint8) << 3
    return (best.astype(np.uint8) | sign).astype(np.uint8)


# ------------------------------------------------------------------- e4m3


def e4m3_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where(code & 0x80, -1.0, 1.0)
    e = (code >> 3) & 0xF
    m = code & 7
    mag = np.where(e == 0, m * 2.0**-9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((code & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def e4m3_encode(v) -> np.ndarray:
    """Nearest e4m3 code (ties to even), saturating at +-448 (finite inputs)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    sub = a < 2.0**-6
    # subnormal range: multiples of 2^-9; code 8 is the smallest normal 2^-6
    code_sub = np.rint(a / 2.0**-9)
    # normal range: a = f * 2^ex with f in [0.5, 1), so the binade exponent is ex - 1
    _, ex = np.frexp(np.where(sub, 1.0, a))
    e = ex - 1
    m = np.rint(a / np.exp2(e) * 8.0) - 8.0  # 0..8; 8 carries into the next binade
    code_norm = (e + 7) * 8 + m
    code = np.where(sub, code_sub, code_norm)
    code = np.where(a >= E4M3_MAX, 0x7E, np.minimum(code, 0x7E)).astype(np.int64)
    sign = np.signbit(v).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


# --------------------------------------------------------------- quantiser


def tensor_scale(amax) -> np.float32:
    """G = 448 * 6 / amax in fp32; 1 when the tensor is all zero."""
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(np.float32(E4M3_MAX * E2M1_MAX) / amax)


def quantize(x, g) -> tuple[np.ndarray, np.ndarray]:
    """Quantise the last axis of ``x`` in groups of 16 under tensor scale ``g``.

    Returns (codes uint8 [..., K], group scale codes uint8 [..., K/16]).
    """
    x = np.asarray(x, dtype=np.float32)
    g = np.float32(g)
    k = x.shape[-1]
    assert k % GROUP == 0
    grp = x.reshape(*x.shape[:-1], k // GROUP, GROUP)
    amax = np.abs(grp).max(axis=-1)
    s_req = (amax / np.float32(E2M1_MAX)).astype(np.float32) * g  # two fp32 roundings
    s_code = e4m3_encode(s_req.astype(np.float32))
    s_val = e4m3_decode(s_code).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(s_val > 0, (g / s_val).astype(np.float32), np.float32(0)).astype(np.float32)
    v = (grp * r[..., None]).astype(np.float32)
    q = e2m1_encode(v)
    q = np.where((s_val > 0)[..., None], q, np.uint8(0)).astype(np.uint8)
    return q.reshape(x.shape), s_code


def dequantize(q, s_code, g) -> np.ndarray:
    """x^ = e2m1(q) * e4m3(s) / G, float64."""
    q = np.asarray(q)
    k = q.shape[-1]
    vals = e2m1_decode(q).reshape(*q.shape[:-1], k // GROUP, GROUP)
    scale = e4m3_decode(s_code)[..., None]
    return (vals * scale / np.float64(np.float32(g))).reshape(q.shape)


def fake_quantize(x, g) -> np.ndarray:
    """dequantize(quantize(x, g)) along the last axis, float64."""
    q, s = quantize(x, g)
    return dequantize(q, s, g)


def weight_fake_quantize(w_kn, g=None):
    """Quantise a [K, N] Linear weight in groups of 16 along K (the input axis).

    Returns (dequantised float64 [K, N], G). ``g`` defaults to the tensor's own
    amax-derived scale (weights are static, observer memoryless_minmax).
    """
    wt = np.ascontiguousarray(np.asarray(w_kn, dtype=np.float32).T)  # [N, K]
    if g is None:
        g = tensor_scale(np.abs(wt).max() if wt.size else 0.0)
    return dequantize(*quantize(wt, g), g).T, np.float32(g)


# ------------------------------------------------------------ NVFP4 block


def act_scales_from_calibration(x_calib, w_router, wg, wu, wd, sg, su, sd, top_k: int = 8, bias=None):
    """Static activation tensor scales from one calibration batch (observer: min/max).

    Runs the bf16 block in float64 on ``x_calib`` and returns fp32 tensor scales
    (g_x, g_h, g_hs) for the block input, the routed experts' GeGLU hidden rows
    (all experts share one scale) and the shared MLP's hidden rows.
    """
    from oracle import moe_oracle as mo

    x = mo.f64(x_calib)
    idx, _, _ = mo.route(x, w_router, top_k, bias)
    amax_h = 0.0
    for e in np.unique(idx):
        tok, _ = np.nonzero(idx == e)
        h = mo.geglu_hidden(x[tok], wg[e], wu[e]).astype(np.float32)
        amax_h = max(amax_h, float(np.abs(h).max()))
    hs = mo.geglu_hidden(x, sg, su).astype(np.float32)
    amax_x = float(np.abs(x.astype(np.float32)).max())
    return tensor_scale(amax_x), tensor_scale(amax_h), tensor_scale(float(np.abs(hs).max()))


def geglu_ffn_nvfp4(xq, w_gate, w_up, w_down, g_hidden) -> np.ndarray:
    """GeGLU on quantised activations and weights; the hidden rows are
    quantised (fp32 decisions) under ``g_hidden`` before the down projection."""
    from oracle import moe_oracle as mo

    gq, _ = weight_fake_quantize(mo.f64(w_gate).astype(np.float32))
    uq, _ = weight_fake_quantize(mo.f64(w_up).astype(np.float32))
    dq, _ = weight_fake_quantize(mo.f64(w_down).astype(np.float32))
    h = mo.gelu_tanh(xq @ gq) * (xq @ uq)
    hq = fake_quantize(h.astype(np.float32), g_hidden)
    return hq @ dq


def moe_block_nvfp4(x, w_router, wg, wu, wd, sg, su, sd, g_x, g_h, g_hs, top_k: int = 8, bias=None, routing=None):
    """The block with NVFP4 Linears: the bf16 router picks and weighs the
    experts; expert and shared projections see quantised activations (tensor
    scales g_x for the block input, g_h / g_hs for the hidden rows) and
    quantised weights (each matrix under its own amax-derived tensor scale)."""
    from oracle import moe_oracle as mo

    x = mo.f64(x)
    if routing is None:
        idx, w, logits = mo.route(x, w_router, top_k, bias)
    else:
        idx, w, logits = np.asarray(routing[0], np.int64), np.asarray(routing[1], np.float64), None
    xq = fake_quantize(x.astype(np.float32), g_x)
    shared = geglu_ffn_nvfp4(xq, sg, su, sd, g_hs)
    routed = np.zeros_like(shared)
    for e in np.unique(idx):
        tok, slot = np.nonzero(idx == e)
        routed[tok] += w[tok, slot][:, None] * geglu_ffn_nvfp4(xq[tok], wg[e], wu[e], wd[e], g_h)
    return {"out": shared + routed, "idx": idx, "w": w, "logits": logits}
