"""Parity of the CUDA path (through the C ABI) with the CPU oracle on a B200."""

import numpy as np
import pytest
import torch

from gpu_common import (
    SMALL,
    bf16_to_f32,
    check_block_output,
    check_routing,
    device_weights,
    require_gpu,
    LOGIT_TOL,
    run_block,
    tile_covering_tokens,
    to_np,
    w_args,
    weights,
)
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs
from oracle import moe_oracle as mo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


# ------------------------------------------------------------------ router


@pytest.mark.parametrize("T,skew", [(64, False), (4096, False), (4096, True)])
def test_router_logits_against_oracle(T, skew):
    """The router's fp32 logits (tensor-core products of bf16 values, exact in
    fp32, accumulated in the hardware's order, split partials summed in split
    order) against the oracle's fp64 logits, element by element. The measured
    error sets the routing tolerance LOGIT_TOL of the other tests."""
    w = weights()
    dw = device_weights()
    bias = inputs.zipf_router_bias() if skew else None
    x_bits = inputs.make_x(T, seed=90 + T)
    res = run_block(dw, x_bits, bias=bias)
    ref = mo.router_logits(x_bits, w.w_router, bias)
    got = to_np(res.logits).astype(np.float64)
    err = np.abs(got - ref)
    print(f"router logits T={T} skew={skew}: max |err| {err.max():.3e}, "
          f"99.9th pct {np.quantile(err, 0.999):.3e}, |logit| max {np.abs(ref).max():.2f}")
    assert err.max() <= LOGIT_TOL, err.max()


@pytest.mark.parametrize("T", [1, 7, 64, 257, 1025, 2048])
def test_route_gemma(T):
    """Routing against the oracle; from T = 1024 the top-k takes two tokens per
    warp (1025: the last warp's second half has no token)."""
    w = weights()
    dw = device_weights()
    x_bits = inputs.make_x(T, seed=11 + T)
    x = block.bf16_tensor(x_bits)
    idx = torch.empty((T, 8), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    p = B.make_params(T, x, dw.w_router, top_k=8)
    B.check(B.moe_route(p, idx, wt), "moe_route")
    assert B.moe_get_device_status() == B.MOE_OK
    ref_idx, ref_w, logits = mo.route(x_bits, w.w_router, 8)
    check_routing(logits, ref_idx, ref_w, to_np(idx), to_np(wt), 8)


@pytest.mark.parametrize("T", [96, 1030])
def test_route_ties_pick_lower_index(T):
    """Duplicated router columns give bitwise-equal fp32 logits on the GPU too;
    the lower expert index must be selected first (one token per warp at
    T = 96, two at T = 1030)."""
    rng = np.random.default_rng(3)
    d, e = 256, 16
    wr = inputs.f32_to_bf16_bits(rng.standard_normal((d, e)).astype(np.float32) * 0.1)
    wr[:, 9] = wr[:, 3]
    wr[:, 14] = wr[:, 3]
    wr[:, 5] = wr[:, 0]
    x_bits = inputs.make_x(T, d, seed=5)
    idx = torch.empty((T, 4), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, 4), dtype=torch.float32, device="cuda")
    p = B.make_params(
        T, block.bf16_tensor(x_bits), block.bf16_tensor(wr), top_k=4, dims=inputs.Dims(d, e, 64, 64)
    )
    B.check(B.moe_route(p, idx, wt), "moe_route")
    gi = to_np(idx)
    for t in range(T):
        row = list(gi[t])
        for lo, hi in ((3, 9), (3, 14), (9, 14), (0, 5)):
            if hi in row:
                assert lo in row and row.index(lo) < row.index(hi), (t, row)


# ------------------------------------------------------------- permutation


@pytest.mark.parametrize("T,skew", [(1, False), (5, False), (128, False), (129, True), (1000, False), (4099, True)])
def test_permute_bit_exact(T, skew):
    E, k = 128, 8
    rng = np.random.default_rng(T)
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
        idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    else:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    d_idx = torch.from_numpy(idx.astype(np.int32)).cuda()
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty((T, k), dtype=torch.int32, device="cuda")
    token_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    p = B.make_params(T, top_k=k)
    B.check(B.moe_permute(p, d_idx, cnt, off, row_of, token_of), "moe_permute")
    assert B.moe_get_device_status() == B.MOE_OK
    r_cnt, r_off, r_row, r_tok = mo.permutation(idx, E)
    np.testing.assert_array_equal(to_np(cnt), r_cnt)
    np.testing.assert_array_equal(to_np(off), r_off)
    np.testing.assert_array_equal(to_np(row_of), r_row)
    np.testing.assert_array_equal(to_np(token_of), r_tok)


# -------------------------------------------------------------- the block


@pytest.mark.parametrize("T,k", [(1, 4), (7, 4), (65, 4), (300, 4), (300, 1), (513, 8), (1100, 8)])
def test_block_small_dims(T, k):
    """Dims 256/16/192/320 put a 64-column tail tile on every GEMM; T spans
    partial and multiple 128-row tiles. T*k = 4104 takes the paired gate|up
    GEMM (>= 160 rows per expert on average), 8800 the paired down GEMM too
    (>= 512)."""
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    x_bits = inputs.make_x(T, SMALL.embed_dim, seed=T)
    res = run_block(dw, x_bits, top_k=k)
    check_block_output(w, x_bits, res, k, derived_tol=True)
    if k == 1:
        assert np.all(to_np(res.w) == 1.0)
    assert to_np(res.cnt).sum() == T * k


def test_block_all_experts_is_dense_mixture():
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    x_bits = inputs.make_x(20, SMALL.embed_dim, seed=2)
    res = run_block(dw, x_bits, top_k=SMALL.num_experts)
    ref = mo.moe_block_dense(x_bits, *w_args(w))
    rms = np.sqrt(np.mean(ref**2))
    assert np.abs(to_np(res.out_f32) - ref).max() <= 1e-2 * rms


def test_block_zero_experts_leave_shared():
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    z = block.DeviceWeights(
        SMALL, dw.w_router, torch.zeros_like(dw.wg), torch.zeros_like(dw.wu), torch.zeros_like(dw.wd), dw.sg, dw.su, dw.sd
    )
    x_bits = inputs.make_x(40, SMALL.embed_dim, seed=3)
    res = run_block(z, x_bits, top_k=4)
    ref = mo.geglu_ffn(x_bits, w.sg, w.su, w.sd)
    rms = np.sqrt(np.mean(ref**2))
    assert np.abs(to_np(res.out_f32) - ref).max() <= 1e-2 * rms


def test_block_intermediates_via_workspace():
    """x_perm, h and y in a caller workspace against the oracle given the GPU routing."""
    T, k = 200, 4
    w = weights(SMALL, seed=1, std=0.05)
    dw = device_weights(SMALL, seed=1, std=0.05)
    ws, lay = block.workspace_for(SMALL, T, k)
    x_bits = inputs.make_x(T, SMALL.embed_dim, seed=9)
    res = run_block(dw, x_bits, top_k=k, workspace=ws)
    D, F, R = SMALL.embed_dim, SMALL.expert_dim, T * k

    def view(off, n, dtype):
        return ws[off : off + n * torch.tensor([], dtype=dtype).element_size()].view(dtype)

    idx = to_np(res.idx)
    cnt, off, row_of, token_of = mo.permutation(idx, SMALL.num_experts)
    np.testing.assert_array_equal(to_np(view(lay.token_of, R, torch.int32)), token_of)
    np.testing.assert_array_equal(to_np(view(lay.row_of, R, torch.int32)).reshape(T, k), row_of)
    xp = to_np(view(lay.x_perm, R * D, torch.int16)).view(np.uint16).reshape(R, D)
    np.testing.assert_array_equal(xp, x_bits[token_of])
    h = bf16_to_f32(view(lay.h, R * F, torch.bfloat16).reshape(R, F))
    y = bf16_to_f32(view(lay.y, R * D, torch.bfloat16).reshape(R, D))
    for e in range(SMALL.num_experts):
        rows = slice(off[e], off[e + 1])
        if off[e + 1] == off[e]:
            continue
        # h and y are stored in bf16: each element within half an ulp (2^-8
        # relative) of the exact value, plus 2e-3 * RMS for fp32 accumulation
        # order and the tanh approximation
        xe = mo.f64(x_bits[token_of[rows]])
        h_ref = mo.geglu_hidden(xe, w.wg[e], w.wu[e])
        slack = 2e-3 * np.sqrt(np.mean(h_ref**2))
        assert np.all(np.abs(h[rows] - h_ref) <= 2.0**-8 * np.abs(h_ref) + slack), e
        y_ref = mo.f64(h[rows]) @ mo.f64(w.wd[e])  # down projection of the GPU's own h
        slack = 2e-3 * np.sqrt(np.mean(y_ref**2))
        assert np.all(np.abs(y[rows] - y_ref) <= 2.0**-8 * np.abs(y_ref) + slack), e


@pytest.mark.parametrize("T", [8, 64])
def test_block_gemma(T):
    w = weights()
    dw = device_weights()
    x_bits = inputs.make_x(T)
    res = run_block(dw, x_bits)
    check_block_output(w, x_bits, res, 8)


def test_block_gemma_prefill_sampled():
    """T = 4096 in the benchmark's launch configuration (paired gate|up, down
    on SM pairs): 512 seeded random tokens plus the first and last token of
    every 128-row block of every expert against the oracle (tokens are
    independent in the block), so every row tile of both GEMMs is compared."""
    T = 4096
    w = weights()
    dw = device_weights()
    x_bits = inputs.make_x(T)
    ws, lay = block.workspace_for(inputs.GEMMA4_26B_A4B, T)
    res = run_block(dw, x_bits, workspace=ws)
    cnt = to_np(res.cnt)
    assert cnt.sum() == 8 * T and cnt.min() > 0
    tiles = tile_covering_tokens(ws, lay, T, 8, inputs.NUM_EXPERTS)
    tokens = np.union1d(inputs.sample_tokens(T, 512), tiles)
    assert len(tokens) >= 512
    check_block_output(w, x_bits, res, 8, tokens=tokens, derived_tol=True)


def test_block_gemma_skewed_every_tile():
    """T = 16384 with the Zipf(1.1) router bias: a few experts take most rows
    (the hottest holds almost every token, ~128 row blocks). The sample is the
    first and last token of every 128-row block of every expert, read from the
    GPU's own permutation, so every tile of the long tail and of the hot
    expert is compared with the oracle."""
    T = 16384
    w = weights()
    dw = device_weights()
    bias = inputs.zipf_router_bias()
    x_bits = inputs.make_x(T)
    ws, lay = block.workspace_for(inputs.GEMMA4_26B_A4B, T)
    res = run_block(dw, x_bits, bias=bias, workspace=ws)
    cnt = np.sort(to_np(res.cnt))[::-1]
    assert cnt[:13].sum() > 0.5 * 8 * T
    tokens = tile_covering_tokens(ws, lay, T, 8, inputs.NUM_EXPERTS)
    assert len(tokens) >= 512
    check_block_output(w, x_bits, res, 8, bias=bias, tokens=tokens, derived_tol=True)


def test_deterministic():
    dw = device_weights(SMALL, seed=1, std=0.05)
    x_bits = inputs.make_x(300, SMALL.embed_dim, seed=4)
    a = run_block(dw, x_bits, top_k=4)
    b = run_block(dw, x_bits, top_k=4)
    assert torch.equal(a.out_f32, b.out_f32) and torch.equal(a.out, b.out) and torch.equal(a.idx, b.idx)


def test_empty_batch_and_bad_args():
    dw = device_weights(SMALL, seed=1, std=0.05)
    x = torch.zeros((0, SMALL.embed_dim), dtype=torch.bfloat16, device="cuda")
    res = block.forward(dw, x, top_k=4)
    assert res.out.shape == (0, SMALL.embed_dim)
    x = torch.zeros((9, SMALL.embed_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((9 * SMALL.embed_dim + 8,), dtype=torch.bfloat16, device="cuda")
    p = B.make_params(9, x, *dw.args(), out.data_ptr() + 2, top_k=4, dims=SMALL)
    assert B.moe_block_forward_ex(p) == B.MOE_ERR_ALIGNMENT
    small_ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    p = B.make_params(9, x, *dw.args(), out, top_k=4, dims=SMALL, workspace=small_ws)
    assert B.moe_block_forward_ex(p) == B.MOE_ERR_WORKSPACE


def test_bounded_wait_reports_timeout():
    """A kernel whose barrier nobody completes gives up after 1 ms, records the
    timeout and returns; the context stays usable afterwards."""
    assert B.moe_get_device_status() == B.MOE_OK
    B.check(B.moe_debug_timeout_probe(1000), "probe")
    assert B.moe_get_device_status() == B.MOE_ERR_DEVICE_TIMEOUT
    assert B.moe_get_device_status() == B.MOE_OK  # the word was cleared
    dw = device_weights(SMALL, seed=1, std=0.05)
    x_bits = inputs.make_x(16, SMALL.embed_dim, seed=6)
    res = run_block(dw, x_bits, top_k=4)
    assert torch.isfinite(res.out_f32).all()
