"""The allocation-free router entry point against the regular one.

moe_route_noalloc serves callers that may not allocate device memory; its
scratch is a fixed array inside the library. Two calls in a row (different
batch sizes, so the second reuses the first call's leftovers) must reproduce
moe_route exactly. This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

from gpu_common import W_REL, device_weights, require_gpu, to_np
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs

pytestmark = pytest.mark.gpu


def _route(fn, dw, x, T, bias=None):
    idx = torch.full((T, 8), -1, dtype=torch.int32, device="cuda")
    wt = torch.full((T, 8), -1.0, dtype=torch.float32, device="cuda")
    p = B.make_params(T, x, dw.w_router, top_k=8, router_bias=bias)
    B.check(fn(p, idx, wt), fn.__name__)
    assert B.moe_get_device_status() == B.MOE_OK
    return to_np(idx), to_np(wt)


def test_route_noalloc_matches_route_twice():
    require_gpu()
    dw = device_weights()
    bias = torch.from_numpy(inputs.zipf_router_bias()).cuda()
    for T, b in ((200, None), (64, bias)):
        x = block.bf16_tensor(inputs.make_x(T, seed=40 + T))
        ref_idx, ref_w = _route(B.moe_route, dw, x, T, b)
        got_idx, got_w = _route(B.moe_route_noalloc, dw, x, T, b)
        np.testing.assert_array_equal(got_idx, ref_idx)
        np.testing.assert_allclose(got_w, ref_w, rtol=W_REL, atol=1e-9)


def test_route_noalloc_rejects_oversized_batch():
    require_gpu()
    dw = device_weights()
    T = 4097
    x = torch.zeros((T, inputs.EMBED_DIM), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, 8), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    p = B.make_params(T, x, dw.w_router, top_k=8)
    assert B.moe_route_noalloc(p, idx, wt) == B.MOE_ERR_WORKSPACE
