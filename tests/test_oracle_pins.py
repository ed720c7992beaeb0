"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test names what it pins against: values printed on the pages, a library
routine the pages name, a closed form, an invariant, or a brute-force
re-derivation on tiny inputs by a different algorithm.
"""

import json
import os

import numpy as np
import pytest
import torch
from scipy.special import erf

from conftest import GOLDEN
from mixture_experts_transformer_b200 import inputs
from oracle import counts, moe_oracle as mo, nvfp4

TINY = inputs.Dims(embed_dim=32, num_experts=8, expert_dim=16, hidden_dim=24)
SMALL = inputs.Dims(embed_dim=128, num_experts=16, expert_dim=64, hidden_dim=64)


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------ shapes / counts


def test_param_counts_reproduce_model_card():
    """Layer shapes -> the checkpoint counts printed on the model card."""
    gold = _load("param_counts.json")
    got = counts.layer_counts()
    for key, ref in gold.items():
        if key.startswith("_"):
            continue
        assert abs(got[key] - ref["printed"]) <= ref["resolution"], (key, got[key], ref)


def test_default_dims_match_config():
    c = counts.Gemma4Config()
    d = inputs.GEMMA4_26B_A4B
    assert (d.embed_dim, d.num_experts, d.expert_dim, d.hidden_dim) == (
        c.embed_dim,
        c.num_experts,
        c.expert_dim,
        c.hidden_dim,
    )
    assert inputs.TOP_K == c.top_k_experts == 8


# --------------------------------------------------------------------- GELU


def test_gelu_tanh_matches_pytorch_tanh_gelu():
    """config.json names hidden_activation gelu_pytorch_tanh: PyTorch's own tanh GELU."""
    z = np.linspace(-12, 12, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(z), approximate="tanh").numpy()
    np.testing.assert_allclose(mo.gelu_tanh(z), ref, rtol=0, atol=1e-14)


def test_gelu_tanh_close_to_exact_gelu():
    """The tanh form approximates x*Phi(x) (Hendrycks & Gimpel) to within 4.8e-4."""
    z = np.linspace(-10, 10, 200001)
    exact = 0.5 * z * (1 + erf(z / np.sqrt(2)))
    assert np.abs(mo.gelu_tanh(z) - exact).max() < 4.8e-4


def test_gelu_closed_forms():
    z = np.linspace(-6, 6, 1201)
    assert mo.gelu_tanh(0.0) == 0.0
    # odd part: 0.5 z (1 + tanh(u)) - 0.5 (-z)(1 - tanh(u)) = z
    np.testing.assert_allclose(mo.gelu_tanh(z) - mo.gelu_tanh(-z), z, atol=1e-13)
    assert abs(mo.gelu_tanh(40.0) - 40.0) < 1e-12 and abs(mo.gelu_tanh(-40.0)) < 1e-12


# ------------------------------------------------------------------ routing


def _rand_block(dims, tokens, seed=0, std=0.2):
    w = inputs.make_weights(dims, seed=seed, std=std)
    x = inputs.make_x(tokens, dims.embed_dim, seed=seed + 1)
    return x, w


def test_routing_invariants():
    x, w = _rand_block(SMALL, 97)
    idx, wt, logits = mo.route(x, w.w_router, 8)
    assert idx.shape == (97, 8)
    for t in range(97):
        assert len(set(idx[t])) == 8
    np.testing.assert_allclose(wt.sum(1), 1.0, atol=1e-12)
    assert np.all(np.diff(wt, axis=1) <= 1e-15)
    # the kept experts are the 8 largest logits
    for t in range(97):
        kept = logits[t, idx[t]]
        rest = np.delete(logits[t], idx[t])
        assert kept.min() >= rest.max()


def test_renormalised_softmax_equals_softmax_of_kept_logits():
    """softmax over all experts then renormalise == softmax over the kept logits alone."""
    x, w = _rand_block(SMALL, 40)
    idx, wt, logits = mo.route(x, w.w_router, 8)
    kept = np.take_along_axis(logits, idx, 1)
    e = np.exp(kept - kept.max(1, keepdims=True))
    np.testing.assert_allclose(wt, e / e.sum(1, keepdims=True), rtol=1e-13)


def test_top_k_brute_force_and_ties():
    """Selection against Python's sorted() on (-logit, index); duplicated router
    columns give exactly equal logits, and the lower index must win."""
    rng = np.random.default_rng(5)
    d, e = 64, 16
    wr = rng.standard_normal((d, e))
    wr[:, 9] = wr[:, 3]  # expert 9 ties with expert 3
    wr[:, 12] = wr[:, 0]
    wr[:, 7] = wr[:, 0]
    x = rng.standard_normal((50, d))
    logits = mo.router_logits(x, wr)
    assert np.all(logits[:, 9] == logits[:, 3])
    for k in (1, 3, 8, 16):
        got = mo.select_top_k(logits, k)
        for t in range(50):
            ref = [i for _, i in sorted((-logits[t, i], i) for i in range(e))][:k]
            assert list(got[t]) == ref


def test_top_1_weight_is_one():
    x, w = _rand_block(SMALL, 33)
    idx, wt, _ = mo.route(x, w.w_router, 1)
    assert np.all(wt == 1.0)


def test_skewed_bias_sends_half_the_assignments_to_a_tenth_of_the_experts():
    """The skewed-routing workload is specified by its effect: a router bias of
    2 ln(Zipf(1.1) rank probability) per expert, so that 10% of the experts
    receive more than half of the assignments. Pinned two ways: exp(bias / 2)
    is the Zipf pmf (sums to one, strictly decreasing with the rank), and on
    512 seeded tokens routed by the oracle with the benchmark's router weights
    (the first draw of the weight stream, seed 0) the 13 most-chosen of the
    128 experts take more than half of the 8 x 512 assignments."""
    bias = inputs.zipf_router_bias()
    pmf = np.exp(bias.astype(np.float64) / 2)
    assert abs(pmf.sum() - 1.0) < 1e-5
    assert np.all(np.diff(pmf) < 0)
    w_r = inputs._normal_bf16(inputs._generator(0), (inputs.EMBED_DIM, inputs.NUM_EXPERTS), inputs.INIT_STD)
    x = inputs.make_x(512)
    idx, w, _ = mo.route(x, w_r, 8, bias=bias)
    cnt = np.bincount(idx.ravel(), minlength=inputs.NUM_EXPERTS)
    assert cnt.sum() == 8 * 512
    assert np.sort(cnt)[::-1][:13].sum() > 0.5 * cnt.sum()
    # without the bias the same tokens spread out: no tenth of the experts takes half
    idx0, _, _ = mo.route(x, w_r, 8)
    cnt0 = np.bincount(idx0.ravel(), minlength=inputs.NUM_EXPERTS)
    assert np.sort(cnt0)[::-1][:13].sum() < 0.25 * cnt0.sum()


def test_permutation_against_stable_sort():
    """Counting-based permutation == a library stable sort of (expert, token) keys."""
    rng = np.random.default_rng(2)
    t_count, e, k = 301, 16, 8
    idx = np.stack([rng.permutation(e)[:k] for _ in range(t_count)])
    cnt, off, row_of, token_of = mo.permutation(idx, e)
    assert cnt.sum() == t_count * k
    np.testing.assert_array_equal(cnt, np.bincount(idx.ravel(), minlength=e))
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(cnt)]))
    key = idx.ravel() * t_count + np.repeat(np.arange(t_count), k)
    order = np.argsort(key, kind="stable")
    np.testing.assert_array_equal(token_of, order // k)
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    np.testing.assert_array_equal(row_of.ravel(), inv)
    # bijection
    assert sorted(row_of.ravel()) == list(range(t_count * k))


# -------------------------------------------------------------------- block


def _naive_block(x, w, k, bias=None):
    """Scalar loops straight from the definition, no matrices, no permutation."""
    x = mo.f64(x)
    d_count = x.shape[1]
    wr, wg, wu, wd = (mo.f64(a) for a in (w.w_router, w.wg, w.wu, w.wd))
    sg, su, sd = (mo.f64(a) for a in (w.sg, w.su, w.sd))
    e_count, f_count, s_count = wr.shape[1], wg.shape[2], sg.shape[1]

    def gelu(v):
        return 0.5 * v * (1 + np.tanh(np.sqrt(2 / np.pi) * (v + 0.044715 * v**3)))

    def ffn(xt, g, u, dn, width):
        out = [0.0] * d_count
        for j in range(width):
            a = sum(xt[i] * g[i, j] for i in range(d_count))
            b = sum(xt[i] * u[i, j] for i in range(d_count))
            hj = gelu(a) * b
            for i in range(d_count):
                out[i] += hj * dn[j, i]
        return np.array(out)

    res = np.zeros_like(x)
    for t in range(x.shape[0]):
        xt = x[t]
        logit = [sum(xt[i] * wr[i, e] for i in range(d_count)) + (0 if bias is None else bias[e]) for e in range(e_count)]
        m = max(logit)
        p = [np.exp(l - m) for l in logit]
        z = sum(p)
        p = [v / z for v in p]
        chosen = []
        for _ in range(k):  # repeated arg-max scan, first index wins ties
            best = None
            for e in range(e_count):
                if e in chosen:
                    continue
                if best is None or logit[e] > logit[best]:
                    best = e
            chosen.append(best)
        norm = sum(p[e] for e in chosen)
        res[t] = ffn(xt, sg, su, sd, s_count)
        for e in chosen:
            res[t] += p[e] / norm * ffn(xt, wg[e], wu[e], wd[e], f_count)
    return res


@pytest.mark.parametrize("k", [2, 3])
def test_block_against_naive_loops(k):
    x, w = _rand_block(TINY, 6, seed=4)
    bias = np.linspace(-1, 1, TINY.num_experts)
    got = mo.moe_block(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=k, bias=bias)["out"]
    ref = _naive_block(x, w, k, bias)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_all_experts_kept_equals_dense_mixture():
    x, w = _rand_block(SMALL, 5, seed=6)
    e = SMALL.num_experts
    got = mo.moe_block(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=e)["out"]
    ref = mo.moe_block_dense(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-12)


def test_zero_experts_leave_shared_branch():
    x, w = _rand_block(SMALL, 9, seed=7)
    z = np.zeros_like(w.wg)
    res = mo.moe_block(x, w.w_router, z, z, np.zeros_like(w.wd), w.sg, w.su, w.sd)
    np.testing.assert_array_equal(res["out"], mo.geglu_ffn(x, w.sg, w.su, w.sd))


def test_given_routing_reproduces_own_routing():
    x, w = _rand_block(SMALL, 12, seed=8)
    a = mo.moe_block(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    b = mo.moe_block(x, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, routing=(a["idx"], a["w"]))
    np.testing.assert_array_equal(a["out"], b["out"])


def test_rms_normalize():
    """Closed forms of x / sqrt(mean(x^2) + 1e-6) (model card: epsilon 1e-06)."""
    rng = np.random.default_rng(0)
    # a constant row c gives c / sqrt(c^2 + eps) everywhere; at c = 1e-3 the
    # epsilon equals the mean square, so dropping it would give 1, not 1/sqrt(2)
    for c in (1e-3, -2.0, 3e-4):
        got = mo.rms_normalize(np.full((1, 96), c))
        np.testing.assert_allclose(got, c / np.sqrt(c * c + 1e-6), rtol=1e-14)
    np.testing.assert_allclose(mo.rms_normalize(np.full((1, 8), 1e-3)), 2.0**-0.5, rtol=1e-12)
    # the output's mean square is ms / (ms + eps) for any row of mean square ms
    x = rng.standard_normal((7, 256)) * rng.uniform(1e-4, 3, (7, 1))
    ms = np.mean(x * x, axis=1)
    y = mo.rms_normalize(x)
    np.testing.assert_allclose(np.mean(y * y, axis=1), ms / (ms + 1e-6), rtol=1e-12)
    # every row is scaled by one positive factor (direction kept), zero stays zero
    np.testing.assert_allclose(y / x, (y / x)[:, :1] * np.ones((1, 256)), rtol=1e-12)
    assert not mo.rms_normalize(np.zeros((2, 16))).any()


def test_top_k_gap_brute_force():
    """k-th minus (k+1)-th largest logit per row, against Python's sorted()."""
    rng = np.random.default_rng(8)
    logits = rng.standard_normal((40, 16))
    logits[3, 5] = logits[3, 9]  # a tie across the k / k+1 boundary
    logits[3] = np.where(logits[3] > logits[3, 5], -5.0, logits[3])
    for k in (1, 2, 8, 15):
        got = mo.top_k_gap(logits, k)
        for t in range(40):
            s = sorted(logits[t].tolist(), reverse=True)
            assert got[t] == s[k - 1] - s[k], (k, t)
    assert mo.top_k_gap(logits, 1)[3] == 0.0  # the tied pair leads row 3
    assert np.all(np.isinf(mo.top_k_gap(logits, 16)))


# -------------------------------------------------------------------- NVFP4


def test_e2m1_grid():
    g = _load("e2m1_grid.json")
    np.testing.assert_array_equal(nvfp4.e2m1_decode(np.arange(8)), g["magnitudes"])
    np.testing.assert_array_equal(nvfp4.e2m1_decode(np.arange(8) | 8), -np.array(g["magnitudes"]))
    # every grid value encodes to its own code
    np.testing.assert_array_equal(nvfp4.e2m1_encode(np.array(g["magnitudes"])), np.arange(8))
    assert nvfp4.e2m1_encode(np.array([7.5, 1e9, -100.0])).tolist() == [7, 7, 15]


def test_e2m1_round_to_nearest_even_brute_force():
    """Nearest grid value; at an exact midpoint, the code with mantissa bit 0."""
    mags = np.array(_load("e2m1_grid.json")["magnitudes"])
    vals = np.concatenate([np.linspace(0, 7, 2801), (mags[1:] + mags[:-1]) / 2])
    got = nvfp4.e2m1_encode(vals)
    for v, c in zip(vals, got):
        d = np.abs(np.minimum(v, 6.0) - mags)
        cands = np.flatnonzero(d == d.min())
        want = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert c == want, (v, c, want)


def test_e4m3_against_torch_float8_e4m3fn():
    """Encoding == torch's float32 -> float8_e4m3fn cast (RNE) inside the finite range."""
    rng = np.random.default_rng(1)
    v = np.concatenate(
        [
            rng.uniform(-448, 448, 200000),
            rng.uniform(-0.02, 0.02, 50000),
            np.exp(rng.uniform(np.log(2.0**-10), np.log(448), 100000)),
        ]
    ).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(nvfp4.e4m3_encode(v), ref)


def test_e4m3_round_trip_and_format_constants():
    f = _load("e4m3_format.json")
    codes = np.arange(256, dtype=np.uint8)
    vals = nvfp4.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    assert np.sum(~finite) == 2 and np.isnan(vals[f["nan_code"]])
    back = nvfp4.e4m3_encode(vals[finite])
    np.testing.assert_array_equal(back, codes[finite])
    assert vals[f["max_finite_code"]] == f["max_finite"] == np.nanmax(vals)
    assert vals[1] == f["min_subnormal"] and vals[8] == f["min_normal"]
    assert nvfp4.e4m3_encode(np.array([500.0, 1e6])).tolist() == [126, 126]
    # torch agrees on every finite code
    ref = torch.from_numpy(vals[finite].astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ref, codes[finite])


def test_nvfp4_quantize_properties():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float32)
    g = nvfp4.tensor_scale(np.abs(x).max())
    q, s = nvfp4.quantize(x, g)
    assert q.shape == x.shape and s.shape == (64, 16)
    xh = nvfp4.dequantize(q, s, g)
    # the tensor's largest element sits at the top of the grid and comes back exactly
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert abs(abs(nvfp4.e2m1_decode(q[i])) - 6.0) == 0
    assert abs(xh[i] - x[i]) <= 2.0**-22 * abs(x[i])
    # every value lands on the nearest grid point of its scaled value (or saturates)
    sv = nvfp4.e4m3_decode(s).astype(np.float32)
    r = (g / sv).astype(np.float32)
    v = (x.reshape(64, 16, 16) * r[..., None]).astype(np.float32).reshape(64, 256)
    gap = np.where(np.abs(v) < 2, 0.25, np.where(np.abs(v) < 4, 0.5, 1.0))
    err = np.abs(nvfp4.e2m1_decode(q) - np.clip(v, -6, 6))
    assert np.all(err <= gap + 1e-12)
    # groups run along the last axis: scaling one group of 16 moves only its scale
    x2 = x.copy()
    x2[5, 32:48] *= 0.25
    _, s2 = nvfp4.quantize(x2, g)
    changed = np.argwhere(s2 != s)
    assert changed.size and np.all(changed == [5, 2])


def test_nvfp4_exact_values_round_trip():
    """Values built as grid * scale / G come back unchanged."""
    rng = np.random.default_rng(4)
    g = np.float32(1.0)
    scale_codes = rng.integers(40, 100, size=(8, 4)).astype(np.uint8)
    mags = nvfp4.E2M1_MAGNITUDES
    q = rng.integers(0, 16, size=(8, 4, 16)).astype(np.uint8)
    q[..., 0] = 7  # each group holds its maximum magnitude 6, so amax/6 == scale
    x = (nvfp4.e2m1_decode(q) * nvfp4.e4m3_decode(scale_codes)[..., None]).astype(np.float32).reshape(8, 64)
    q2, s2 = nvfp4.quantize(x, g)
    np.testing.assert_array_equal(s2, scale_codes)
    np.testing.assert_array_equal(nvfp4.dequantize(q2, s2, g), x.astype(np.float64))
    assert mags[7] == 6.0


def test_nvfp4_block_near_bf16_block():
    """FP4 weights and activations perturb the block by a bounded relative amount."""
    x, w = _rand_block(SMALL, 16, seed=9, std=0.05)
    args = (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    ref = mo.moe_block(x, *args)
    gx, gh, ghs = nvfp4.act_scales_from_calibration(inputs.make_x(64, SMALL.embed_dim, seed=2), *args)
    got = nvfp4.moe_block_nvfp4(x, *args, gx, gh, ghs)
    np.testing.assert_array_equal(got["idx"], ref["idx"])  # the router stays bf16
    rms = np.sqrt(np.mean(ref["out"] ** 2))
    rel = np.sqrt(np.mean((got["out"] - ref["out"]) ** 2)) / rms
    # one fp4 rounding costs ~9.5% RMS per element, a dot product ~13%; the
    # GeGLU chain compounds x, W, h and W_down roundings to ~25%
    assert 0.1 < rel < 0.4, rel
