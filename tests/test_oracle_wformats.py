"""Pins of the oracle's weight-only formats, SFP8 and Q4_0 (no GPU needed).

The pages name these formats only by footprint; their readings are stated in
oracle/wformats.py and fixed in tests/golden/ (q4_0_format.json,
sfp8_format.json). Pinned here against those constants, scalar brute force,
exact round trips and closed forms.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from conftest import GOLDEN
from mixture_experts_transformer_b200 import inputs
from oracle import moe_oracle as mo
from oracle import wformats as wf

F32 = np.float32


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# -------------------------------------------------------------------- Q4_0


def _q4_scalar(block):
    """One block of 32 by scalar steps from the format definition."""
    fmt = _load("q4_0_format.json")
    m = F32(0.0)
    for v in block:  # first element of largest magnitude, sign kept
        if abs(F32(v)) > abs(m):
            m = F32(v)
    d = F32(m / F32(fmt["scale_divisor"]))
    inv = F32(F32(1.0) / d) if d != 0 else F32(0.0)
    codes = []
    for v in block:
        t = F32(F32(F32(v) * inv) + F32(fmt["code_offset"] + 0.5))
        codes.append(min(2 ** fmt["code_bits"] - 1, int(math.trunc(float(t)))))
    return codes, np.float16(d)


def test_q4_0_against_scalar_definition():
    rng = np.random.default_rng(40)
    x = (rng.standard_normal((50, 128)) * np.exp(rng.uniform(-6, 2, (50, 1)))).astype(np.float32)
    x[3, 64:96] = 0.0  # an all-zero block (the third of the row)
    x[7, 0:32] = -x[7, 0:32]
    x[9, 5] = -np.abs(x[9]).max() * 1.5  # a negative block maximum
    q, d = wf.q4_0_quantize(x)
    assert q.shape == x.shape and d.shape == (50, 4) and d.dtype == np.float16
    for r in range(50):
        for b in range(4):
            codes, dref = _q4_scalar(x[r, 32 * b : 32 * b + 32])
            assert list(q[r, 32 * b : 32 * b + 32]) == codes, (r, b)
            assert d[r, b] == dref or (np.isnan(d[r, b]) and np.isnan(dref))
    # a zero block: scale 0, every code 8, dequantised to 0
    assert d[3, 2] == 0 and np.all(q[3, 64:96] == 8) and not wf.q4_0_dequantize(q, d)[3, 64:96].any()
    # halfway cases round up (trunc of x / d + 8.5): with maximum -8 (d = 1),
    # 2.5 -> code 11 and -2.5 -> code 6, where round-half-even would give 10, 6
    blk = np.zeros(32, np.float32)
    blk[0], blk[1], blk[2], blk[3] = -8.0, 2.5, -2.5, 3.5
    qb, db = wf.q4_0_quantize(blk)
    assert db[0] == 1.0 and list(qb[:4]) == [0, 11, 6, 12]
    # equal magnitudes of opposite sign: the first one sets the sign of d
    blk = np.zeros(32, np.float32)
    blk[4], blk[9] = 4.0, -4.0
    qb, db = wf.q4_0_quantize(blk)
    assert db[0] == -0.5 and qb[4] == 0 and qb[9] == 15


def test_q4_0_round_trip_and_extremes():
    """Blocks built as (q - 8) * d, with an fp16 d and a code 0 in every block,
    come back exactly; the block maximum always takes code 0 (value -8 d = m)."""
    rng = np.random.default_rng(41)
    d = (rng.uniform(0.5, 2.0, (20, 2)) * np.exp2(rng.integers(-12, 2, (20, 2)))).astype(np.float16)
    q = rng.integers(1, 16, (20, 64)).astype(np.uint8)
    q[:, 0] = 0
    q[:, 32] = 0
    x = wf.q4_0_dequantize(q, d).astype(np.float32)
    q2, d2 = wf.q4_0_quantize(x)
    np.testing.assert_array_equal(d2, d)
    np.testing.assert_array_equal(q2, q)
    # codes stay in [0, 15]; the dequantised error is at most half a step |d| / 2,
    # except above 7.5 |d| on the side opposite the block maximum, where the
    # top code 15 (7 d) clamps and the error reaches at most |d|
    y = (rng.standard_normal((30, 96)) * 3).astype(np.float32)
    qy, dy = wf.q4_0_quantize(y)
    assert qy.max() <= 15
    err = np.abs(wf.q4_0_dequantize(qy, dy) - y).reshape(30, 3, 32)
    step = np.abs(dy.astype(np.float64))[..., None] * (1 + 2e-3)  # fp16 rounding of d
    clamped = (qy.reshape(30, 3, 32) == 15) & (err > 0.5 * step)
    assert np.all(err[~clamped] <= 0.5 * np.broadcast_to(step, err.shape)[~clamped] + 1e-12)
    assert np.all(err <= np.broadcast_to(step, err.shape) + 1e-12)


# -------------------------------------------------------------------- SFP8


def test_sfp8_table_against_format_constants():
    f = _load("sfp8_format.json")
    t = wf.SFP8_TABLE
    assert t[0] == 0 and np.all(np.diff(t) > 0)  # strictly increasing magnitudes
    assert t[127] == f["largest"] and t[1] == f["smallest_nonzero"] and t[64] == f["switch_at"]
    # 2^-23 .. 2^1: 24 binades; 3 mantissa bits at and above the switch, 2 below
    nz = t[1:]
    e = np.floor(np.log2(nz))
    assert e.min() == -23 and e.max() == 0 and len(np.unique(e)) == f["binades"]
    mant = nz / np.exp2(e) - 1
    large = nz >= f["switch_at"]
    assert np.all(mant[large] * 2 ** f["mantissa_bits_large"] % 1 == 0)
    assert np.all(mant[~large] * 2 ** f["mantissa_bits_small"] % 1 == 0)
    assert len(np.unique(e[large])) == 8 and len(np.unique(e[~large])) == 16


def test_sfp8_values_are_exact_in_bf16():
    """Every decoded value is a bf16 number: the tensor cores can take the
    decoded weights as they are and apply the matrix scale to the fp32 sums."""
    v = torch.from_numpy(wf.sfp8_decode(np.arange(256, dtype=np.uint8)).astype(np.float32))
    np.testing.assert_array_equal(v.to(torch.bfloat16).float().numpy(), v.numpy())


def test_sfp8_round_trip_and_nearest_even():
    codes = np.arange(256, dtype=np.uint8)
    np.testing.assert_array_equal(wf.sfp8_encode(wf.sfp8_decode(codes)), codes)
    t = wf.SFP8_TABLE
    mids = (t[1:] + t[:-1]) / 2
    vals = np.concatenate([mids, np.linspace(0, 2.5, 5001), np.geomspace(1e-9, 1.0, 4000)])
    got = wf.sfp8_encode(vals)
    for v, c in zip(vals, got):
        a = min(v, 1.875)
        dist = np.abs(t - a)
        cands = np.flatnonzero(dist == dist.min())
        want = cands[0] if len(cands) == 1 else [k for k in cands if k % 2 == 0][0]
        assert c == want, (v, c, want)
    assert wf.sfp8_encode(np.array([-0.3]))[0] == wf.sfp8_encode(np.array([0.3]))[0] | 0x80


def test_sfp8_matrix_scale():
    """S = amax / 1.875 maps the matrix's largest magnitude to the top code;
    an all-zero matrix has scale 1."""
    rng = np.random.default_rng(42)
    w = (rng.standard_normal((64, 16)) * 0.03).astype(np.float32)
    s = wf.sfp8_scale(np.abs(w).max())
    assert s == F32(F32(np.abs(w).max()) / F32(1.875))
    q = wf.sfp8_quantize(w, s)
    assert (q[np.unravel_index(np.argmax(np.abs(w)), w.shape)] & 0x7F) == 127
    assert wf.sfp8_scale(0.0) == 1.0


# ---------------------------------------------------------- block and matrices


@pytest.mark.parametrize("fmt", ["q4_0", "sfp8"])
def test_weight_fake_quantize_runs_along_k_per_matrix(fmt):
    rng = np.random.default_rng(43)
    w = (rng.standard_normal((64, 24)) * 0.05).astype(np.float32)
    w[3, 7] = 0.5  # holds the matrix's amax
    base = wf.weight_fake_quantize(w, fmt)
    w2 = w.copy()
    w2[32:64, 5] *= 0.37  # one block of 32 along K of one column
    moved = wf.weight_fake_quantize(w2, fmt)
    changed = np.argwhere(moved != base)
    assert changed.size and set(changed[:, 1]) == {5} and changed[:, 0].min() >= 32
    # a power-of-two rescaling of the matrix rescales its dequantised copy exactly
    np.testing.assert_array_equal(wf.weight_fake_quantize(4 * w, fmt), 4 * base)


@pytest.mark.parametrize("fmt", ["q4_0", "sfp8"])
def test_block_on_representable_weights_is_the_bf16_block(fmt):
    """Weights already on the format's grid quantise to themselves, so the
    format's block equals the plain block; off the grid they differ."""
    dims = inputs.Dims(embed_dim=64, num_experts=4, expert_dim=32, hidden_dim=32)
    w = inputs.make_weights(dims, seed=44, std=0.1)
    f = lambda a: np.stack([wf.weight_fake_quantize(mo.f64(m).astype(np.float32), fmt) for m in a])  # noqa: E731
    g = lambda m: wf.weight_fake_quantize(mo.f64(m).astype(np.float32), fmt)  # noqa: E731
    # a dequantised matrix is on the grid: Q4_0 keeps each block's maximum at
    # code 0 (value -8 d), so re-quantising returns the same d and codes
    on = (f(w.wg), f(w.wu), f(w.wd), g(w.sg), g(w.su), g(w.sd))
    x = inputs.make_x(6, dims.embed_dim, seed=45)
    ref = mo.moe_block(x, w.w_router, *on[:3], *on[3:], top_k=2)["out"]
    got = wf.moe_block_wq(x, w.w_router, *(a.astype(np.float32) for a in on), fmt=fmt, top_k=2)["out"]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)
    plain = mo.moe_block(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=2)["out"]
    assert np.abs(plain - ref).max() > 1e-4 * np.abs(ref).max()
