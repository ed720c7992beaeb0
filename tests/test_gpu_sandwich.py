"""The normalisation sandwich on a B200 against the oracle: pre-FFN RMSNorm
with a learned scale (bf16 block input), post-FFN RMSNorm with a learned
scale, residual add; each part alone and all three together."""

import numpy as np
import pytest
import torch

from gpu_common import (ACC_SLACK, BF16_SLACK, OUT_TOL, SMALL, bf16_storage_cost, check_routing, device_weights,
                        require_gpu, rne_bf16, to_np, w_args, weights)
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs
from oracle import moe_oracle as mo
from oracle import sandwich as sw

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _gammas(D, seed=9):
    rng = np.random.default_rng(seed)
    return tuple(inputs.f32_to_bf16_bits(rng.uniform(0.5, 1.5, D).astype(np.float32)) for _ in range(2))


def _run(dims, w, dw, T, k, pre, post, res, seed):
    D = dims.embed_dim
    x_bits = inputs.make_x(T, D, seed=seed)
    g_pre, g_post = _gammas(D)
    ws, lay = block.workspace_for(dims, T, k)
    r = block.forward(dw, block.bf16_tensor(x_bits), top_k=k, debug=True, workspace=ws,
                      norm_pre=block.bf16_tensor(g_pre) if pre else None,
                      norm_post=block.bf16_tensor(g_post) if post else None, residual=res)
    assert B.moe_get_device_status() == B.MOE_OK
    x64 = mo.f64(x_bits)
    idx, wts = to_np(r.idx), to_np(r.w)
    if pre:
        # (a) the block input, element by element: the GPU rounds its fp32 value,
        # the oracle its float64 value, so they may sit one bf16 step apart
        xn_gpu = to_np(ws[lay.x_norm:lay.x_norm + T * D * 2].view(torch.int16)).view(np.uint16).reshape(T, D)
        xn_ref = sw.bf16_bits(sw.bf16_rne(sw.rms_norm(x_bits, g_pre)))
        diff = xn_gpu != xn_ref
        assert diff.mean() <= 1e-3, diff.mean()
        a, b = mo.f64(xn_gpu[diff]), mo.f64(xn_ref[diff])
        assert np.all(np.abs(a - b) <= 2.0**-7 * np.abs(b)), np.abs(a - b).max()
        xin = xn_gpu
    else:
        xin = x_bits
    # (b) routing on the block's actual input
    ri, rw, logits = mo.route(xin, w.w_router, k)
    check_routing(logits, ri, rw, idx, wts, k)
    # (c) the output given that input and the GPU's routing
    blk = mo.moe_block(xin, *w_args(w), routing=(idx, wts))["out"]
    rms_f = np.sqrt(np.mean(blk**2))
    tol_f = max(OUT_TOL, BF16_SLACK * bf16_storage_cost(xin, w, idx, wts) / rms_f + ACC_SLACK)
    got = to_np(r.out_f32).astype(np.float64) - (x64 if res else 0.0)
    if post:
        ref = sw.rms_norm(blk, g_post)
        n_ref = sw.rms_norm(blk)
        # a block error |df| <= tol_f * rms(f) moves f / rms(f) by at most
        # tol_f * (1 + |n|) per element (the rms itself moves by <= rms(df)),
        # then times the learned scale
        bound = mo.f64(g_post).max() * tol_f * (1.0 + np.abs(n_ref).max())
    else:
        ref = blk
        bound = tol_f * rms_f
    err = np.abs(got - ref).max()
    assert err <= bound, (err, bound)
    np.testing.assert_array_equal(r.out.float().cpu().numpy(), rne_bf16(to_np(r.out_f32)))
    return err


@pytest.mark.parametrize("pre,post,res", [(1, 0, 0), (0, 1, 0), (0, 0, 1), (1, 1, 1)])
def test_sandwich_parts_small_dims(pre, post, res):
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    _run(SMALL, w, dw, 65, 4, pre, post, res, seed=31)


@pytest.mark.parametrize("T,k", [(7, 4), (300, 4), (1100, 8)])
def test_sandwich_small_dims(T, k):
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    _run(SMALL, w, dw, T, k, 1, 1, 1, seed=40 + T)


def test_sandwich_gemma_T64():
    _run(inputs.GEMMA4_26B_A4B, weights(), device_weights(), 64, 8, 1, 1, 1, seed=5)


def test_sandwich_gemma_prefill_sampled():
    """T=4096 (the prefill launch configuration): routing and output checked on
    a sample of tokens, the pre-norm on every element."""
    T, k = 4096, 8
    dims = inputs.GEMMA4_26B_A4B
    w, dw = weights(), device_weights()
    x_bits = inputs.make_x(T, seed=7)
    g_pre, g_post = _gammas(dims.embed_dim)
    ws, lay = block.workspace_for(dims, T, k)
    r = block.forward(dw, block.bf16_tensor(x_bits), top_k=k, debug=True, workspace=ws,
                      norm_pre=block.bf16_tensor(g_pre), norm_post=block.bf16_tensor(g_post), residual=True)
    assert B.moe_get_device_status() == B.MOE_OK
    D = dims.embed_dim
    xn_gpu = to_np(ws[lay.x_norm:lay.x_norm + T * D * 2].view(torch.int16)).view(np.uint16).reshape(T, D)
    xn_ref = mo.f64(sw.bf16_bits(sw.bf16_rne(sw.rms_norm(x_bits, g_pre))))
    assert (mo.f64(xn_gpu) != xn_ref).mean() <= 1e-3
    tok = np.random.default_rng(3).choice(T, 48, replace=False)
    idx, wts = to_np(r.idx)[tok], to_np(r.w)[tok]
    xin = xn_gpu[tok]
    ri, rw, logits = mo.route(xin, w.w_router, k)
    check_routing(logits, ri, rw, idx, wts, k)
    blk = mo.moe_block(xin, *w_args(w), routing=(idx, wts))["out"]
    ref = sw.rms_norm(blk, g_post)
    got = to_np(r.out_f32)[tok].astype(np.float64) - mo.f64(x_bits[tok])
    bound = mo.f64(g_post).max() * OUT_TOL * (1.0 + np.abs(sw.rms_norm(blk)).max())
    assert np.abs(got - ref).max() <= bound
    np.testing.assert_array_equal(r.out.float().cpu().numpy(), rne_bf16(to_np(r.out_f32)))
