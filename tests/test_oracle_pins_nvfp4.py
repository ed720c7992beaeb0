"""Pins of the oracle's NVFP4 block composition (no GPU needed).

The codec pins (e2m1 grid, e4m3 against torch, the group quantiser's
properties) live in test_oracle_pins.py. Here the parts built on top of them
are pinned against an independent evaluation:

* a scalar-loop NVFP4 block that quantises by brute-force search over the
  format's codes, whose values it derives from the format constants in
  tests/golden/ (not from the oracle's codecs), with groups of 16 along each
  Linear's input dimension K, one tensor scale per matrix, x quantised under
  g_x, the routed hidden rows under g_h and the shared ones under g_hs
  [G4-MeroMero-26B-A4B-NVFP4 config.json, quantization_config.config_groups.
  group_0: group_size 16, float8_e4m3fn scales, strategy tensor_group,
  input_activations dynamic "local"];
* direct tests of the weight grouping axis and of the per-matrix tensor scale;
* the calibration observer against a per-token dense evaluation's amax.
"""

import json
import math
import os

import numpy as np

from conftest import GOLDEN
from mixture_experts_transformer_b200 import inputs
from oracle import moe_oracle as mo
from oracle import nvfp4

F32 = np.float32


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ----------------------------------------------- brute-force format tables


def _e4m3_table():
    """Value of every non-negative finite e4m3 code, from the format's field widths."""
    f = _load("e4m3_format.json")
    mbits, bias = f["mantissa_bits"], f["exponent_bias"]
    vals = []
    for code in range(f["max_finite_code"] + 1):
        e, m = code >> mbits, code & ((1 << mbits) - 1)
        if e == 0:  # subnormal: m * 2^(1 - bias - mbits)
            v = m * 2.0 ** (1 - bias - mbits)
        else:
            v = (1 + m / 2.0**mbits) * 2.0 ** (e - bias)
        vals.append(v)
    assert vals[-1] == f["max_finite"] and vals[1] == f["min_subnormal"] and vals[8] == f["min_normal"]
    return vals


E4M3 = _e4m3_table()
E2M1 = _load("e2m1_grid.json")["magnitudes"]


def _nearest_even(table, v):
    """Index of the table value nearest to v >= 0; an exact tie takes the even
    index (the code whose mantissa bit is 0); v past the last value saturates."""
    if v >= table[-1]:
        return len(table) - 1
    best = None
    for i, t in enumerate(table):
        d = abs(t - v)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def _quantize_group(xs, g):
    """Dequantised values of one group of 16 fp32 values under tensor scale g (fp32)."""
    amax = F32(max(abs(F32(v)) for v in xs))
    s_req = F32(F32(amax / F32(6.0)) * g)
    s = F32(E4M3[_nearest_even(E4M3, float(s_req))])
    if s == 0:
        return [0.0] * len(xs)
    r = F32(g / s)
    out = []
    for v in xs:
        q = F32(F32(v) * r)
        mag = E2M1[_nearest_even(E2M1, abs(float(q)))]
        out.append(math.copysign(mag, float(q)) * float(s) / float(g))
    return out


def _tensor_scale(values):
    amax = F32(max(abs(F32(v)) for v in values))
    return F32(1.0) if amax == 0 else F32(F32(448.0 * 6.0) / amax)


def _quantize_matrix(w_kn):
    """[K, N] weight -> its dequantised copy: one tensor scale for the matrix,
    groups of 16 running down each column (along K)."""
    k_dim, n_dim = w_kn.shape
    g = _tensor_scale(w_kn.ravel())
    out = np.zeros((k_dim, n_dim))
    for n in range(n_dim):
        for k0 in range(0, k_dim, 16):
            out[k0 : k0 + 16, n] = _quantize_group([F32(w_kn[k, n]) for k in range(k0, k0 + 16)], g)
    return out, g


def _quantize_row(row, g):
    out = []
    for k0 in range(0, len(row), 16):
        out += _quantize_group([F32(v) for v in row[k0 : k0 + 16]], g)
    return out


def _gelu(z):
    return 0.5 * z * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (z + 0.044715 * z**3)))


def _ffn_scalar(xq, g_kn, u_kn, d_kn, g_hidden):
    """Scalar-loop GeGLU with quantised operands; the hidden row is quantised
    (from its fp32 value) under g_hidden before the down projection."""
    d_dim, f_dim = g_kn.shape
    h = []
    for j in range(f_dim):
        a = sum(xq[i] * g_kn[i, j] for i in range(d_dim))
        b = sum(xq[i] * u_kn[i, j] for i in range(d_dim))
        h.append(F32(_gelu(a) * b))
    hq = _quantize_row(h, g_hidden)
    return [sum(hq[j] * d_kn[j, i] for j in range(f_dim)) for i in range(d_kn.shape[1])]


def _nvfp4_block_scalar(x, w, k, g_x, g_h, g_hs):
    """The NVFP4 block by scalar loops: bf16 router, top-k by repeated arg-max
    (lower index wins ties), softmax renormalised over the kept experts."""
    xf = mo.f64(x)
    wr = mo.f64(w.w_router)
    mats = lambda a: [mo.f64(a[e]) for e in range(a.shape[0])]  # noqa: E731
    wg, wu, wd = mats(w.wg), mats(w.wu), mats(w.wd)
    qg = [_quantize_matrix(m)[0] for m in wg]
    qu = [_quantize_matrix(m)[0] for m in wu]
    qd = [_quantize_matrix(m)[0] for m in wd]
    qsg, qsu, qsd = (_quantize_matrix(mo.f64(m))[0] for m in (w.sg, w.su, w.sd))
    out = np.zeros_like(xf)
    for t in range(xf.shape[0]):
        logit = [sum(xf[t, i] * wr[i, e] for i in range(xf.shape[1])) for e in range(wr.shape[1])]
        chosen = []
        for _ in range(k):
            best = None
            for e in range(len(logit)):
                if e not in chosen and (best is None or logit[e] > logit[best]):
                    best = e
            chosen.append(best)
        m = max(logit[e] for e in chosen)
        p = [math.exp(logit[e] - m) for e in chosen]
        xq = _quantize_row([F32(v) for v in xf[t]], g_x)
        acc = np.array(_ffn_scalar(xq, qsg, qsu, qsd, g_hs))
        for j, e in enumerate(chosen):
            acc += p[j] / sum(p) * np.array(_ffn_scalar(xq, qg[e], qu[e], qd[e], g_h))
        out[t] = acc
    return out


def _tiny_nvfp4_weights():
    dims = inputs.Dims(embed_dim=32, num_experts=4, expert_dim=16, hidden_dim=16)
    w = inputs.make_weights(dims, seed=11, std=0.2)
    # give every expert matrix its own amax, so a tensor scale shared across
    # the expert stack would move the other experts' codes
    spread = np.array([1.0, 2.7, 0.35, 1.6], np.float32)

    def rescale(a):
        f = inputs.bf16_bits_to_f32(a) * spread[:, None, None]
        return inputs.f32_to_bf16_bits(f)

    return inputs.BlockWeights(w.w_router, rescale(w.wg), rescale(w.wu), rescale(w.wd), w.sg, w.su, w.sd)


def test_e4m3_table_matches_the_oracle_codec():
    """The brute-force table and the oracle's decoder agree code by code."""
    np.testing.assert_array_equal(nvfp4.e4m3_decode(np.arange(len(E4M3))), E4M3)


def test_nvfp4_block_against_scalar_brute_force():
    """moe_block_nvfp4 == the scalar-loop NVFP4 block, to rounding."""
    w = _tiny_nvfp4_weights()
    x = inputs.make_x(8, 32, seed=12)
    # activation tensor scales: deliberately far apart, so quantising x under
    # g_h, or h under g_x, changes the result
    g_x, g_h, g_hs = F32(40.0), F32(230.0), F32(9.0)
    args = (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    got = nvfp4.moe_block_nvfp4(x, *args, g_x, g_h, g_hs, top_k=2)["out"]
    ref = _nvfp4_block_scalar(x, w, 2, g_x, g_h, g_hs)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
    # and it is not the bf16 block: the quantisation is really applied
    bf = mo.moe_block(x, *args, top_k=2)["out"]
    assert np.abs(bf - ref).max() > 1e-3 * np.abs(ref).max()


def test_nvfp4_block_each_hidden_scale_matters():
    """Changing g_h moves only the routed branch; g_hs only the shared one."""
    w = _tiny_nvfp4_weights()
    x = inputs.make_x(8, 32, seed=12)
    args = (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    base = nvfp4.moe_block_nvfp4(x, *args, F32(40.0), F32(230.0), F32(9.0), top_k=2)["out"]
    moved_h = nvfp4.moe_block_nvfp4(x, *args, F32(40.0), F32(23.0), F32(9.0), top_k=2)["out"]
    moved_hs = nvfp4.moe_block_nvfp4(x, *args, F32(40.0), F32(230.0), F32(90.0), top_k=2)["out"]
    ref_h = _nvfp4_block_scalar(x, w, 2, F32(40.0), F32(23.0), F32(9.0))
    ref_hs = _nvfp4_block_scalar(x, w, 2, F32(40.0), F32(230.0), F32(90.0))
    assert np.abs(moved_h - base).max() > 0 and np.abs(moved_hs - base).max() > 0
    np.testing.assert_allclose(moved_h, ref_h, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(moved_hs, ref_hs, rtol=1e-10, atol=1e-12)


def test_weight_fake_quantize_groups_run_along_k():
    """Scaling one 16-long K-group of one column moves that group alone."""
    rng = np.random.default_rng(21)
    w = (rng.standard_normal((64, 24)) * 0.05).astype(np.float32)
    w[3, 7] = 1.0  # the tensor's amax stays put, so its tensor scale does too
    base, g = nvfp4.weight_fake_quantize(w)
    w2 = w.copy()
    w2[32:48, 5] *= 0.3
    moved, g2 = nvfp4.weight_fake_quantize(w2)
    assert g2 == g
    changed = np.argwhere(moved != base)
    assert changed.size
    assert set(changed[:, 1]) == {5} and changed[:, 0].min() >= 32 and changed[:, 0].max() < 48
    # against the brute force, element for element
    ref, g_ref = _quantize_matrix(w2)
    assert g_ref == g2
    np.testing.assert_array_equal(moved, ref)


def test_weight_fake_quantize_one_tensor_scale_per_matrix():
    """G = 448 * 6 / amax of the matrix itself; a power-of-two rescaling of the
    matrix rescales its dequantised values exactly (G absorbs it)."""
    rng = np.random.default_rng(22)
    w = (rng.standard_normal((32, 16)) * 0.03).astype(np.float32)
    deq, g = nvfp4.weight_fake_quantize(w)
    assert g == F32(F32(2688.0) / F32(np.abs(w).max()))
    deq4, g4 = nvfp4.weight_fake_quantize(4 * w)
    assert g4 == g / 4
    np.testing.assert_array_equal(deq4, 4 * deq)


def test_act_scales_from_calibration_against_per_token_amax():
    """The calibration observer's three tensor scales equal 448 * 6 / amax of a
    token-by-token dense evaluation: x itself, the GeGLU rows of each token's
    top-k experts, and the shared MLP's GeGLU rows."""
    dims = inputs.Dims(embed_dim=64, num_experts=8, expert_dim=32, hidden_dim=48)
    w = inputs.make_weights(dims, seed=13, std=0.1)
    x = inputs.make_x(24, 64, seed=14)
    got = nvfp4.act_scales_from_calibration(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=3)
    xf = mo.f64(x)
    wr = mo.f64(w.w_router)
    amax_x = amax_h = amax_hs = 0.0
    for t in range(xf.shape[0]):
        xt = xf[t]
        amax_x = max(amax_x, float(np.abs(xt).max()))
        logits = [float(xt @ wr[:, e]) for e in range(dims.num_experts)]
        top = [e for _, e in sorted((-l, e) for e, l in enumerate(logits))][:3]
        for e in top:
            for j in range(dims.expert_dim):
                a = float(xt @ mo.f64(w.wg[e][:, j]))
                b = float(xt @ mo.f64(w.wu[e][:, j]))
                amax_h = max(amax_h, abs(_gelu(a) * b))
        for j in range(dims.hidden_dim):
            a = float(xt @ mo.f64(w.sg[:, j]))
            b = float(xt @ mo.f64(w.su[:, j]))
            amax_hs = max(amax_hs, abs(_gelu(a) * b))
    want = [F32(2688.0) / F32(a) for a in (amax_x, amax_h, amax_hs)]
    np.testing.assert_allclose(np.array(got, np.float64), np.array(want, np.float64), rtol=2e-7)
    assert got[0] == want[0]  # x is exact: bf16 values, no arithmetic
    # an all-zero tensor has scale 1
    z = np.zeros_like(x)
    assert nvfp4.act_scales_from_calibration(z, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=3) == (1, 1, 1)
