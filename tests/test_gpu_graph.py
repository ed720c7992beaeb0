"""The block forward is capture-safe with a caller workspace: captured into a
CUDA graph (on a side stream ordered after the inputs) it replays to the same
bits as direct launches, at the decode and prefill launch configurations."""

import pytest
import torch

from gpu_common import device_weights, require_gpu
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [64, 4096])
def test_graph_replay_matches_direct(T):
    require_gpu()
    dw = device_weights()
    x = block.bf16_tensor(inputs.make_x(T, seed=60))
    ws, _ = block.workspace_for(inputs.GEMMA4_26B_A4B, T)
    out = torch.empty_like(x)
    p = B.make_params(T, x, *dw.args(), out, workspace=ws)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())  # inputs and workspace are ready on s
    with torch.cuda.stream(s):
        for _ in range(3):  # warm up on the capture stream
            B.check(B.moe_block_forward_ex(p, s), "forward")
    torch.cuda.synchronize()
    ref = out.clone()
    out.zero_()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        B.check(B.moe_block_forward_ex(p, torch.cuda.current_stream()), "capture")
    graph.replay()
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == B.MOE_OK
    assert torch.equal(out, ref)
    del graph
