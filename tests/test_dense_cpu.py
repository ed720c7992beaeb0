"""The dense GeGLU FFN of the E4B sibling: the oracle against the page's
config and a scalar-loop evaluation, and the C ABI's host-side validation."""

import ctypes
import json
import math
import os

import numpy as np
import pytest

from conftest import GOLDEN, ROOT
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import build as mbuild
from mixture_experts_transformer_b200 import inputs
from oracle import moe_oracle as mo


def test_e4b_dims_match_config():
    cfg = json.load(open(os.path.join(GOLDEN, "e4b_config.json")))
    assert not cfg["enable_moe"]
    assert (inputs.E4B_EMBED_DIM, inputs.E4B_HIDDEN_DIM) == (cfg["embed_dim"], cfg["hidden_dim"])
    assert (B.E4B_EMBED_DIM, B.E4B_HIDDEN_DIM) == (cfg["embed_dim"], cfg["hidden_dim"])
    hdr = open(os.path.join(ROOT, "include", "moe_block.h")).read()
    assert f"#define MOE_E4B_EMBED_DIM {cfg['embed_dim']}" in hdr
    assert f"#define MOE_E4B_HIDDEN_DIM {cfg['hidden_dim']}" in hdr


def test_dense_ffn_scalar_loops():
    rng = np.random.default_rng(11)
    T, D, S = 3, 5, 4
    x, wg, wu, wd = (rng.standard_normal(sh) for sh in ((T, D), (D, S), (D, S), (S, D)))
    ref = np.zeros((T, D))
    for t in range(T):
        h = []
        for j in range(S):
            g = sum(x[t, d] * wg[d, j] for d in range(D))
            u = sum(x[t, d] * wu[d, j] for d in range(D))
            gel = 0.5 * g * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (g + 0.044715 * g**3)))
            h.append(gel * u)
        for i in range(D):
            ref[t, i] = sum(h[j] * wd[j, i] for j in range(S))
    np.testing.assert_allclose(mo.dense_ffn(x, wg, wu, wd), ref, rtol=1e-12, atol=1e-12)


def test_dense_ffn_is_the_shared_branch():
    d = inputs.Dims(embed_dim=64, num_experts=8, expert_dim=64, hidden_dim=128)
    w = inputs.make_weights(d, seed=2, std=0.1)
    x = inputs.make_x(6, d.embed_dim, seed=3)
    zero = np.zeros_like(w.wd)  # routed experts output nothing
    blk = mo.moe_block(x, w.w_router, w.wg, w.wu, zero, w.sg, w.su, w.sd, top_k=2)
    np.testing.assert_array_equal(blk["out"], mo.dense_ffn(x, w.sg, w.su, w.sd))


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return B.lib()


def test_dense_host_validation(lib):
    f = lambda p: lib.moe_dense_ffn_forward(ctypes.byref(p), None)  # noqa: E731
    good = dict(x=16, wg=16, wu=16, wd=16, out=1 << 40)
    assert f(B.make_dense_params(0, **good)) == B.MOE_OK  # empty batch: no-op
    assert f(B.make_dense_params(-1, **good)) == B.MOE_ERR_INVALID_ARG
    assert f(B.make_dense_params(4, **{**good, "x": 0})) == B.MOE_ERR_INVALID_ARG
    assert f(B.make_dense_params(4, **{**good, "wd": 24})) == B.MOE_ERR_ALIGNMENT
    assert f(B.make_dense_params(4, **good, embed_dim=100)) == B.MOE_ERR_INVALID_ARG  # not a multiple of 64
    assert f(B.make_dense_params(4, **{**good, "out": 16})) == B.MOE_ERR_INVALID_ARG  # out overlaps x
    assert lib.moe_dense_ffn_forward(None, None) == B.MOE_ERR_INVALID_ARG
    p = B.make_dense_params(64)
    assert B.moe_dense_workspace_bytes(p) >= 64 * inputs.E4B_HIDDEN_DIM * 2


def test_dense_workspace_holds_split_k_partials(lib):
    """Small batches cut the down GEMM's reduction into K ranges whose fp32
    partial sums live in the workspace (about one wave of (column tile, K
    range) items at 148 SMs, at least 4 K blocks each): at the E4B decode
    shape, 10 column tiles of 256 give 14 ranges of 160 K blocks, i.e. 14
    partial [64, 2560] fp32 planes beyond the bf16 hidden rows. Large batches
    (T >= 256, paired GEMMs) never split."""
    D, S = inputs.E4B_EMBED_DIM, inputs.E4B_HIDDEN_DIM
    dec = B.moe_dense_workspace_bytes(B.make_dense_params(64))
    assert dec >= 64 * S * 2 + 14 * 64 * D * 4
    # a hidden dim too short to split (K blocks / 4 < 2) keeps one range
    small = B.moe_dense_workspace_bytes(B.make_dense_params(64, embed_dim=256, hidden_dim=320))
    assert small < 64 * 320 * 2 + 2 * 64 * 256 * 4
    # T = 256 takes the paired kernels: no partial planes at all
    big = B.moe_dense_workspace_bytes(B.make_dense_params(256))
    assert big < 256 * S * 2 + 256 * D * 4

