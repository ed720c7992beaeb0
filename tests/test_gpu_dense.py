"""The dense GeGLU FFN (the E4B sibling's feed-forward) on a B200 against the
oracle, at reduced shapes (several tiles and a ragged tail) and at the E4B
shapes (embed_dim 2560, hidden_dim 10240) in the launch configurations of
small and large batches."""

import functools

import numpy as np
import pytest
import torch

from gpu_common import ACC_SLACK, BF16_SLACK, OUT_TOL, require_gpu, rne_bf16, to_np
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs
from oracle import moe_oracle as mo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@functools.lru_cache(maxsize=2)
def _weights(D, S, std):
    w = inputs.make_dense_weights(D, S, seed=4, std=std)
    return w, tuple(block.bf16_tensor(a) for a in (w.wg, w.wu, w.wd))


def _hidden_rounding_cost(xs, w):
    """max |out(hidden rows rounded to bf16) - out(exact)|: the designed storage
    precision of the hidden rows (float64 otherwise)."""
    h = mo.geglu_hidden(mo.f64(xs), w.wg, w.wu)
    hr = torch.from_numpy(h.astype(np.float32)).to(torch.bfloat16).double().numpy()
    wd = mo.f64(w.wd)
    return np.abs(hr @ wd - h @ wd).max()


def _check(D, S, T, std, tokens=None, seed=21):
    w, dev = _weights(D, S, std)
    x_bits = inputs.make_x(T, D, seed=seed + T)
    r = block.dense_forward(block.bf16_tensor(x_bits), *dev, debug=True)
    assert B.moe_get_device_status() == B.MOE_OK
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = mo.dense_ffn(x_bits[tok], w.wg, w.wu, w.wd)
    got = to_np(r.out_f32)[tok].astype(np.float64)
    rms = np.sqrt(np.mean(ref**2))
    bound = max(OUT_TOL * rms, BF16_SLACK * _hidden_rounding_cost(x_bits[tok], w) + ACC_SLACK * rms)
    err = np.abs(got - ref).max()
    assert err <= bound, (err / rms, bound / rms)
    np.testing.assert_array_equal(r.out.float().cpu().numpy(), rne_bf16(to_np(r.out_f32)))


@pytest.mark.parametrize("T", [1, 37, 300, 1100])
def test_dense_small_dims(T):
    """embed 256 / hidden 320: a 64-column tail on every gate|up tile row;
    T=300 and 1100 take the paired gate|up and the SM-pair down GEMM."""
    _check(256, 320, T, std=0.05)


@pytest.mark.parametrize("T", [1, 20, 200])
def test_dense_split_k(T):
    """hidden 2048 at small batches: the down GEMM is cut along its reduction
    (8 K ranges of 4 blocks) and the fp32 partial sums are added in order."""
    _check(256, 2048, T, std=0.05)


def test_dense_e4b_decode():
    _check(inputs.E4B_EMBED_DIM, inputs.E4B_HIDDEN_DIM, 64, std=inputs.INIT_STD)


def test_dense_e4b_prefill_sampled():
    T = 4096
    tok = np.random.default_rng(8).choice(T, 40, replace=False)
    _check(inputs.E4B_EMBED_DIM, inputs.E4B_HIDDEN_DIM, T, std=inputs.INIT_STD, tokens=tok)


def test_dense_bf16_out_without_debug():
    """Without out_f32 the down GEMM writes the bf16 output itself; it equals
    the rounding of the debug run's fp32 output."""
    D, S, T = 256, 320, 300
    w, dev = _weights(D, S, 0.05)
    x = block.bf16_tensor(inputs.make_x(T, D, seed=99))
    a = block.dense_forward(x, *dev, debug=True)
    b = block.dense_forward(x, *dev)
    torch.cuda.synchronize()
    assert torch.equal(a.out, b.out)
