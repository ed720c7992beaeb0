"""Pins of the sandwich oracle (RMSNorm with a learned scale, bf16 rounding,
pre/post norm and residual) against closed forms and library routines."""

import numpy as np
import torch

from mixture_experts_transformer_b200 import inputs
from oracle import moe_oracle as mo
from oracle import sandwich as sw

EPS = mo.RMS_EPS


def test_rms_norm_worked_example():
    # [3, 4]: mean square 12.5, so the row divides by sqrt(12.5 + 1e-6)
    got = sw.rms_norm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]))
    r = np.sqrt(12.5 + 1e-6)
    np.testing.assert_allclose(got, [[3.0 / r, 8.0 / r]], rtol=1e-15)
    np.testing.assert_allclose(got, [[0.848528, 2.262742]], rtol=1e-6)


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(5)
    # a constant row c: every output is gamma * c / sqrt(c^2 + eps)
    for c in (-3.0, 1e-3, 7.5):
        got = sw.rms_norm(np.full((1, 64), c), np.full(64, 0.5))
        np.testing.assert_allclose(got, 0.5 * c / np.sqrt(c * c + EPS), rtol=1e-14)
    # unscaled output mean square is ms / (ms + eps)
    v = rng.standard_normal((6, 2816)) * rng.uniform(0.01, 10, (6, 1))
    ms = np.mean(v * v, axis=1)
    np.testing.assert_allclose(np.mean(sw.rms_norm(v) ** 2, axis=1), ms / (ms + EPS), rtol=1e-12)
    # scale invariance once eps is negligible; zero row -> zero
    np.testing.assert_allclose(sw.rms_norm(1e3 * v), sw.rms_norm(v), rtol=1e-5)
    assert not sw.rms_norm(np.zeros((1, 8)), np.ones(8)).any()


def test_bf16_rne_matches_torch_on_float32_values():
    rng = np.random.default_rng(6)
    f = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(sw.bf16_rne(f.astype(np.float64)), ref)


def test_bf16_rne_ties_to_even():
    # 1 + 2^-8 sits halfway between 1 and 1 + 2^-7: even mantissa (1) wins;
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: 1 + 2^-6 wins
    got = sw.bf16_rne(np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, -(1 + 2.0**-8), 1 + 2.0**-8 + 2.0**-30]))
    np.testing.assert_array_equal(got, [1.0, 1 + 2.0**-6, -1.0, 1 + 2.0**-7])


def test_sandwich_reduces_to_residual():
    d = inputs.Dims(embed_dim=64, num_experts=8, expert_dim=64, hidden_dim=64)
    w = inputs.make_weights(d, seed=3, std=0.1)
    x = inputs.make_x(5, d.embed_dim, seed=4)
    args = (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)
    g_pre = np.linspace(0.5, 1.5, d.embed_dim)
    # gamma_post = 0: the block's output is scaled away, out is x exactly
    r = sw.sandwich_block(x, *args, g_pre, np.zeros(d.embed_dim), top_k=2)
    np.testing.assert_array_equal(r["out"], mo.f64(x))
    # zero weights: the block outputs 0 and RMSNorm(0) = 0
    z = [np.zeros_like(a) for a in args]
    r = sw.sandwich_block(x, *z, g_pre, np.ones(d.embed_dim), top_k=2)
    np.testing.assert_array_equal(r["out"], mo.f64(x))
    # no residual: the normalised block output has unit mean square scaled by gamma_post^2
    r = sw.sandwich_block(x, *args, g_pre, np.full(d.embed_dim, 2.0), top_k=2, residual=False)
    ms = np.mean(r["ffn"] ** 2, axis=1)
    np.testing.assert_allclose(np.mean(r["out"] ** 2, axis=1), 4.0 * ms / (ms + EPS), rtol=1e-12)
    # the block's input is the bf16 pre-norm of x
    xn = sw.rms_norm(x, g_pre)
    assert np.abs(mo.f64(r["x_norm"]) - xn).max() <= 2.0**-8 * np.abs(xn).max()
