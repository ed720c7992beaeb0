"""Weight-only formats the pages name by footprint: SFP8 and Q4_0.

Test infrastructure only (see the package docstring).

The pages give these formats only as resident footprints of the whole model
["MEMORY IS SET BY TOTAL, NOT ACTIVE": 57.7 GB bf16, 28.8 GB at SFP8, 14.4 GB
at Q4_0], that is ~8 and ~4.5 bits per weight; they print neither format.
Readings (stated, not taken from the pages):

Q4_0 - the published 4-bit block format of that name (ggml):

* blocks of 32 consecutive weights along a Linear's input dimension K, each
  with one fp16 scale d and 32 codes q in [0, 15];
* m = the block's element of largest magnitude, sign kept (the first one on
  ties); d = m / -8 in fp32, stored as fp16 (round to nearest even);
* q_i = min(15, trunc(fp32(fp32(x_i * id) + 8.5))) with id = fp32(1 / d)
  computed from the fp32 d (id = 0 when d = 0);
* dequantised x^_i = (q_i - 8) * fp16(d).

SFP8 - an 8-bit "switching" floating point, sign and magnitude:

* bit 7 is the sign; the magnitude code m (7 bits) switches between two
  exponent / mantissa splits so that larger values keep 3 mantissa bits and
  smaller ones trade a mantissa bit for range:
    m = 0                 zero
    m in [1, 63]          (1 + (m & 3) / 4) * 2^((m >> 2) - 23)      2^-23 ... 2^-8 binades
    m in [64, 127]        (1 + (m & 7) / 8) * 2^(((m >> 3) & 7) - 7)  2^-7 ... 2^0 binades
  (monotone in m, largest magnitude 1.875);
* one fp32 scale per matrix S = amax / 1.875 (1 for an all-zero matrix); a
  weight is encoded as the nearest magnitude to fp32(|x| / S) (ties to the
  even code, saturating at 1.875) with its sign;
* dequantised x^ = value(code) * S.

Both formats quantise along K with the weights stored as the block takes them
([K, N], N contiguous); the router stays bf16 and the activations stay bf16
(weight-only formats).
"""

from __future__ import annotations

import numpy as np

Q4_BLOCK = 32
SFP_MAX = 1.875


# -------------------------------------------------------------------- Q4_0


def q4_0_quantize(x):
    """Quantise the last axis of x (float32, length a multiple of 32).

    Returns (codes uint8 [..., K] in [0, 15], scales float16 [..., K/32])."""
    x = np.asarray(x, dtype=np.float32)
    k = x.shape[-1]
    assert k % Q4_BLOCK == 0
    blk = x.reshape(*x.shape[:-1], k // Q4_BLOCK, Q4_BLOCK)
    first = np.argmax(np.abs(blk), axis=-1)  # first element of largest magnitude
    m = np.take_along_axis(blk, first[..., None], -1)[..., 0]
    d = (m / np.float32(-8.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d != 0, (np.float32(1.0) / d).astype(np.float32), np.float32(0.0)).astype(np.float32)
    v = ((blk * inv[..., None]).astype(np.float32) + np.float32(8.5)).astype(np.float32)
    q = np.minimum(15, np.trunc(v)).astype(np.uint8)
    return q.reshape(x.shape), d.astype(np.float16)


def q4_0_dequantize(q, d16) -> np.ndarray:
    """(q - 8) * d per block of 32, float64."""
    q = np.asarray(q).astype(np.float64)
    k = q.shape[-1]
    vals = (q - 8.0).reshape(*q.shape[:-1], k // Q4_BLOCK, Q4_BLOCK)
    return (vals * np.asarray(d16, np.float64)[..., None]).reshape(q.shape)


# -------------------------------------------------------------------- SFP8


def sfp8_magnitudes() -> np.ndarray:
    """Value of each magnitude code m = 0..127."""
    m = np.arange(128)
    small = (1 + (m & 3) / 4.0) * np.exp2((m >> 2) - 23.0)
    large = (1 + (m & 7) / 8.0) * np.exp2(((m >> 3) & 7) - 7.0)
    out = np.where(m >= 64, large, small)
    out[0] = 0.0
    return out


SFP8_TABLE = sfp8_magnitudes()


def sfp8_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = SFP8_TABLE[code & 0x7F]
    return np.where(code & 0x80, -mag, mag)


def sfp8_encode(v) -> np.ndarray:
    """Nearest SFP8 code of each value (ties to the even code), saturating at 1.875, sign kept."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), SFP_MAX)
    # the table is increasing: the nearest is one of the two codes around a
    hi = np.clip(np.searchsorted(SFP8_TABLE, a, side="left"), 0, 127)
    lo = np.clip(hi - 1, 0, 127)
    d_lo, d_hi = a - SFP8_TABLE[lo], SFP8_TABLE[hi] - a
    pick = np.where(d_hi < d_lo, hi, np.where(d_lo < d_hi, lo, np.where(hi % 2 == 0, hi, lo)))
    sign = np.signbit(v).astype(np.uint8) << 7
    return (pick.astype(np.uint8) | sign).astype(np.uint8)


def sfp8_scale(amax) -> np.float32:
    """S = amax / 1.875 in fp32; 1 for an all-zero tensor."""
    amax = np.float32(amax)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(SFP_MAX))


def sfp8_quantize(x, scale) -> np.ndarray:
    """Codes of fp32(x / scale)."""
    x = np.asarray(x, dtype=np.float32)
    return sfp8_encode((x / np.float32(scale)).astype(np.float32))


# ------------------------------------------------------------ weight matrices


def weight_fake_quantize(w_kn, fmt: str):
    """Dequantised copy (float64 [K, N]) of a [K, N] Linear weight in `fmt`
    ("q4_0" or "sfp8"), quantised along K (the input axis)."""
    wt = np.ascontiguousarray(np.asarray(w_kn, dtype=np.float32).T)  # [N, K]
    if fmt == "q4_0":
        q, d = q4_0_quantize(wt)
        return q4_0_dequantize(q, d).T
    if fmt == "sfp8":
        s = sfp8_scale(np.abs(wt).max() if wt.size else 0.0)
        return (sfp8_decode(sfp8_quantize(wt, s)) * np.float64(s)).T
    raise ValueError(fmt)


def moe_block_wq(x, w_router, wg, wu, wd, sg, su, sd, fmt: str, top_k: int = 8, bias=None, routing=None):
    """The block with every expert and shared Linear weight in `fmt` (each
    matrix quantised on its own; router and activations bf16): the oracle's
    block on the dequantised weights."""
    from oracle import moe_oracle as mo

    def deq(m):
        return weight_fake_quantize(mo.f64(m).astype(np.float32), fmt)

    if routing is None:
        idx, w, _ = mo.route(x, w_router, top_k, bias)
        routing = (idx, w)
    # only the experts the routing uses are quantised; the others stay zero
    wgq, wuq, wdq = (np.zeros(a.shape) for a in (wg, wu, wd))
    for e in np.unique(np.asarray(routing[0])):
        wgq[e], wuq[e], wdq[e] = deq(wg[e]), deq(wu[e]), deq(wd[e])
    return mo.moe_block(x, w_router, wgq, wuq, wdq, deq(sg), deq(su), deq(sd), top_k=top_k, bias=bias,
                        routing=routing)
