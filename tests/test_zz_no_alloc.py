"""The allocation-free router entry point against the regular one.

moe_route_noalloc serves callers that may not allocate device memory: its
scratch is a fixed array inside the library. It runs moe_route's kernels with
moe_route's own split of the reduction, so idx, w and the logits must come
out bit for bit equal, on two calls in a row (different batch sizes, so each
call reuses the previous call's leftovers), up to its 4096-token limit; the
routing is also checked against the oracle. This file is collected last on
purpose.
"""

import numpy as np
import pytest
import torch

from gpu_common import check_routing, device_weights, require_gpu, to_np, weights
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs
from oracle import moe_oracle as mo

pytestmark = pytest.mark.gpu


def _route(fn, dw, x, T, bias=None):
    idx = torch.full((T, 8), -1, dtype=torch.int32, device="cuda")
    wt = torch.full((T, 8), -1.0, dtype=torch.float32, device="cuda")
    logits = torch.full((T, inputs.NUM_EXPERTS), -1.0, dtype=torch.float32, device="cuda")
    p = B.make_params(T, x, dw.w_router, top_k=8, router_bias=bias, logits_out=logits)
    B.check(fn(p, idx, wt), fn.__name__)
    assert B.moe_get_device_status() == B.MOE_OK
    return to_np(idx), to_np(wt), to_np(logits)


def test_route_noalloc_matches_route_twice():
    require_gpu()
    dw = device_weights()
    bias_np = inputs.zipf_router_bias()
    bias = torch.from_numpy(bias_np).cuda()
    for T, b in ((200, None), (64, bias), (4096, None), (1024, bias)):
        x_bits = inputs.make_x(T, seed=40 + T)
        x = block.bf16_tensor(x_bits)
        ref = _route(B.moe_route, dw, x, T, b)
        got = _route(B.moe_route_noalloc, dw, x, T, b)
        for a, r in zip(got, ref):
            np.testing.assert_array_equal(a, r)
        if T >= 1024:
            ref_idx, ref_w, ref_logits = mo.route(x_bits, weights().w_router, 8, None if b is None else bias_np)
            check_routing(ref_logits, ref_idx, ref_w, got[0], got[1], 8)


def test_route_noalloc_rejects_oversized_batch():
    require_gpu()
    dw = device_weights()
    T = 4097
    x = torch.zeros((T, inputs.EMBED_DIM), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((T, 8), dtype=torch.int32, device="cuda")
    wt = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    p = B.make_params(T, x, dw.w_router, top_k=8)
    assert B.moe_route_noalloc(p, idx, wt) == B.MOE_ERR_WORKSPACE
