"""A stack of NVFP4 MoE blocks with the unlearned RMSNorm between them (no
attention, no residual): x_{l+1} = RMSNorm(block_l(x_l)), eps 1e-6.

Setup (quantisation and calibration) and the forward loop call the library's
C ABI only; torch provides the device buffers.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import binding as B
from . import block
from .inputs import Dims


@dataclasses.dataclass
class Nvfp4Stack:
    layers: list  # [block.Nvfp4Weights]
    scales: list  # [(g_x, g_h, g_hs)]
    dims: Dims
    top_k: int = B.TOP_K


def build_stack(make_device_weights, n_layers: int, x_calib: torch.Tensor, top_k: int = B.TOP_K, keep_bf16=None):
    """make_device_weights(l) -> block.DeviceWeights for layer l (bf16 on the device).

    Layer l is quantised with the library's quantiser and calibrated on the
    calibration batch as it arrives at layer l: the bf16 block's observer gives
    the activation scales, and the NVFP4 block's normalised output becomes the
    next layer's calibration input. The bf16 weights are dropped after that
    (kept for the layers listed in keep_bf16, e.g. for a CPU baseline)."""
    layers, scales, kept = [], [], {}
    xc = x_calib
    dims = None
    for l in range(n_layers):
        dw = make_device_weights(l)
        dims = dw.dims
        sc, _ = block.calibrate(dw, xc, top_k=top_k)
        nw = block.quantize_block(dw)
        layers.append(nw)
        scales.append(sc)
        xc = block.forward_nvfp4(nw, xc, sc, top_k=top_k, rms_norm_out=True).out
        if keep_bf16 and l in keep_bf16:
            kept[l] = dw
        del dw
    torch.cuda.synchronize()
    return Nvfp4Stack(layers, scales, dims, top_k), kept


def stack_forward(stack: Nvfp4Stack, x: torch.Tensor, bufs=None, workspace=None, stream=None, debug_last=False):
    """Run every layer; returns the last layer's BlockResult (normalised output)."""
    T = x.shape[0]
    if bufs is None:
        bufs = [torch.empty((T, stack.dims.embed_dim), dtype=torch.bfloat16, device=x.device) for _ in range(2)]
    cur = x
    res = None
    n = len(stack.layers)
    for l, (nw, sc) in enumerate(zip(stack.layers, stack.scales)):
        out = bufs[l % 2]
        res = block.forward_nvfp4(
            nw, cur, sc, top_k=stack.top_k, rms_norm_out=True, out=out, workspace=workspace,
            debug=debug_last and l == n - 1, stream=stream,
        )
        cur = out
    return res


def stack_workspace(stack: Nvfp4Stack, T: int, device="cuda") -> torch.Tensor:
    p = block.nvfp4_params(stack.layers[0], T, None, None, stack.scales[0], top_k=stack.top_k)
    return torch.empty(B.moe_nvfp4_workspace_bytes(p), dtype=torch.uint8, device=device)


def fp4_weight_bytes(dims: Dims, touched_experts: int) -> int:
    """NVFP4 bytes (codes + scale atoms) a block reads: touched experts and the shared MLP."""
    d, f, s = dims.embed_dim, dims.expert_dim, dims.hidden_dim

    def lin(K, N):
        return N * K // 2 + ((N + 127) // 128) * (K // 64) * 512

    return touched_experts * (2 * lin(d, f) + lin(f, d)) + 2 * lin(d, s) + lin(s, d)


def act_scale_array(stack: Nvfp4Stack) -> np.ndarray:
    return np.array(stack.scales, dtype=np.float32)
