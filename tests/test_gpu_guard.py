"""Workspace guard words (a debug aid standing in for a memory checker, which
this pool does not offer): a guarded call writes a pattern after its workspace
data and checks it after its last kernel. Nothing here faults a GPU: the
violation is made by the host, which overwrites a guard byte itself."""

import numpy as np
import pytest
import torch

from gpu_common import SMALL, device_weights, require_gpu
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs

pytestmark = pytest.mark.gpu


def test_guarded_call_is_clean_and_unchanged():
    require_gpu()
    dw = device_weights(SMALL, seed=1, std=0.05)
    T = 150
    x = block.bf16_tensor(inputs.make_x(T, SMALL.embed_dim, seed=9))
    ws, lay = block.workspace_for(SMALL, T, top_k=4)
    ref = block.forward(dw, x, top_k=4, debug=True, workspace=ws)
    out = torch.empty_like(ref.out)
    p = B.make_params(T, x, *dw.args(), out, top_k=4, dims=SMALL, workspace=ws, check_guards=True)
    B.check(B.moe_block_forward_ex(p), "guarded forward")
    assert B.moe_last_launch_count() == 7 + 2  # the fill and the check
    assert B.moe_get_device_status() == B.MOE_OK
    assert torch.equal(out, ref.out)
    # the pattern is in place after the call; the guard check alone agrees
    assert ws[lay.guard : lay.guard + 256].any()
    B.check(B.moe_workspace_guard_check(p), "guard check")
    assert B.moe_get_device_status() == B.MOE_OK


def test_overwritten_guard_is_reported():
    require_gpu()
    dw = device_weights(SMALL, seed=1, std=0.05)
    T = 40
    x = block.bf16_tensor(inputs.make_x(T, SMALL.embed_dim, seed=10))
    ws, lay = block.workspace_for(SMALL, T, top_k=4)
    out = torch.empty((T, SMALL.embed_dim), dtype=torch.bfloat16, device="cuda")
    p = B.make_params(T, x, *dw.args(), out, top_k=4, dims=SMALL, workspace=ws, check_guards=True)
    B.check(B.moe_block_forward_ex(p), "guarded forward")
    assert B.moe_get_device_status() == B.MOE_OK
    ws[lay.guard + 77] ^= 0x10  # one flipped bit past the data
    B.check(B.moe_workspace_guard_check(p), "guard check")
    assert B.moe_get_device_status() == B.MOE_ERR_GUARD
    assert B.moe_get_device_status() == B.MOE_OK  # the word was cleared
    # the next guarded call rewrites the pattern and passes
    B.check(B.moe_block_forward_ex(p), "guarded forward")
    assert B.moe_get_device_status() == B.MOE_OK
