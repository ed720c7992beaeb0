"""Device-side convenience around the C ABI: upload bf16 weights once, run the block.

Marshalling only. Every computation happens inside libmoeblock.so.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import binding as B
from .inputs import BlockWeights, Dims


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> torch.bfloat16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device != "cpu" else t


@dataclasses.dataclass
class DeviceWeights:
    dims: Dims
    w_router: torch.Tensor
    wg: torch.Tensor
    wu: torch.Tensor
    wd: torch.Tensor
    sg: torch.Tensor
    su: torch.Tensor
    sd: torch.Tensor

    def args(self):
        return (self.w_router, self.wg, self.wu, self.wd, self.sg, self.su, self.sd)


def upload(w: BlockWeights, device="cuda") -> DeviceWeights:
    return DeviceWeights(
        w.dims, *(bf16_tensor(a, device) for a in (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd))
    )


@dataclasses.dataclass
class BlockResult:
    out: torch.Tensor
    out_f32: torch.Tensor | None = None
    idx: torch.Tensor | None = None
    w: torch.Tensor | None = None
    cnt: torch.Tensor | None = None
    logits: torch.Tensor | None = None


def forward(
    dw: DeviceWeights,
    x: torch.Tensor,
    *,
    top_k: int = B.TOP_K,
    router_bias: torch.Tensor | None = None,
    debug: bool = False,
    workspace: torch.Tensor | None = None,
    out: torch.Tensor | None = None,
    stream=None,
    norm_pre: torch.Tensor | None = None,
    norm_post: torch.Tensor | None = None,
    residual: bool = False,
) -> BlockResult:
    """Run one block; with debug=True also return out_f32, the routing, the router logits and the counts.
    norm_pre / norm_post (bf16 [embed_dim]) and residual add the normalisation
    sandwich: out = x + norm_post-RMSNorm(block(norm_pre-RMSNorm(x)))."""
    T = x.shape[0]
    dev = x.device
    if out is None:
        out = torch.empty((T, dw.dims.embed_dim), dtype=torch.bfloat16, device=dev)
    res = BlockResult(out=out)
    if debug:
        res.out_f32 = torch.empty((T, dw.dims.embed_dim), dtype=torch.float32, device=dev)
        res.idx = torch.empty((T, top_k), dtype=torch.int32, device=dev)
        res.w = torch.empty((T, top_k), dtype=torch.float32, device=dev)
        res.cnt = torch.empty((dw.dims.num_experts,), dtype=torch.int32, device=dev)
        res.logits = torch.empty((T, dw.dims.num_experts), dtype=torch.float32, device=dev)
    p = B.make_params(
        T,
        x,
        *dw.args(),
        out,
        top_k=top_k,
        dims=dw.dims,
        router_bias=router_bias,
        out_f32=res.out_f32,
        idx_out=res.idx,
        w_out=res.w,
        cnt_out=res.cnt,
        workspace=workspace,
        norm_pre=norm_pre,
        norm_post=norm_post,
        residual=residual,
        logits_out=res.logits,
    )
    B.check(B.moe_block_forward_ex(p, stream), "moe_block_forward_ex")
    return res


def workspace_for(dims: Dims, T: int, top_k: int = B.TOP_K, device="cuda") -> tuple[torch.Tensor, B.MoeWsLayout]:
    """A caller-owned workspace (uint8) and its layout."""
    p = B.make_params(T, top_k=top_k, dims=dims)
    lay = B.moe_workspace_layout(p)
    return torch.empty(lay.total_bytes, dtype=torch.uint8, device=device), lay


# ----------------------------------------------------------------- NVFP4


@dataclasses.dataclass
class Nvfp4Linear:
    """One quantised Linear stack on the device: codes, scale atoms, tensor scales."""

    q: torch.Tensor
    sf: torch.Tensor
    g: torch.Tensor
    groups: int
    K: int
    N: int

    def struct(self) -> B.MoeNvfp4Linear:
        return B.MoeNvfp4Linear(self.q.data_ptr(), self.sf.data_ptr(), self.g.data_ptr())


def quantize_linear(w: torch.Tensor, stream=None) -> Nvfp4Linear:
    """w [G][K][N] (or [K][N]) bf16 on the device -> NVFP4 (the library's quantiser)."""
    w3 = w if w.dim() == 3 else w.unsqueeze(0)
    G, K, N = w3.shape
    qb, sfb = B.moe_nvfp4_weight_bytes(G, K, N)
    q = torch.empty(qb, dtype=torch.uint8, device=w.device)
    sf = torch.empty(sfb, dtype=torch.uint8, device=w.device)
    g = torch.empty(G, dtype=torch.float32, device=w.device)
    B.check(B.moe_nvfp4_quantize_weight(w3, G, K, N, q, sf, g, stream), "moe_nvfp4_quantize_weight")
    return Nvfp4Linear(q, sf, g, G, K, N)


@dataclasses.dataclass
class Nvfp4Weights:
    dims: Dims
    w_router: torch.Tensor
    wg: Nvfp4Linear
    wu: Nvfp4Linear
    wd: Nvfp4Linear
    sg: Nvfp4Linear
    su: Nvfp4Linear
    sd: Nvfp4Linear


def quantize_block(dw: DeviceWeights, stream=None) -> Nvfp4Weights:
    return Nvfp4Weights(
        dw.dims,
        dw.w_router,
        *(quantize_linear(t, stream) for t in (dw.wg, dw.wu, dw.wd, dw.sg, dw.su, dw.sd)),
    )


def forward_nvfp4(
    nw: Nvfp4Weights,
    x: torch.Tensor,
    act_scales,
    *,
    top_k: int = B.TOP_K,
    router_bias: torch.Tensor | None = None,
    rms_norm_out: bool = False,
    debug: bool = False,
    workspace: torch.Tensor | None = None,
    out: torch.Tensor | None = None,
    stream=None,
) -> BlockResult:
    """One NVFP4 block; act_scales = (g_x, g_h, g_hs)."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, nw.dims.embed_dim), dtype=torch.bfloat16, device=x.device)
    res = BlockResult(out=out)
    if debug:
        res.out_f32 = torch.empty((T, nw.dims.embed_dim), dtype=torch.float32, device=x.device)
        res.idx = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
        res.w = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
        res.cnt = torch.empty((nw.dims.num_experts,), dtype=torch.int32, device=x.device)
    p = nvfp4_params(nw, T, x, out, act_scales, top_k=top_k, router_bias=router_bias, rms_norm_out=rms_norm_out,
                     res=res, workspace=workspace)
    B.check(B.moe_block_forward_nvfp4(p, stream), "moe_block_forward_nvfp4")
    return res


def nvfp4_params(nw, T, x, out, act_scales, *, top_k=B.TOP_K, router_bias=None, rms_norm_out=False, res=None,
                 workspace=None) -> B.MoeNvfp4Params:
    p = B.MoeNvfp4Params()
    p.T, p.top_k_experts = T, top_k
    d = nw.dims
    p.embed_dim, p.num_experts, p.expert_dim, p.hidden_dim = d.embed_dim, d.num_experts, d.expert_dim, d.hidden_dim
    p.x, p.w_router, p.router_bias = B.ptr(x), B.ptr(nw.w_router), B.ptr(router_bias)
    for name in ("wg", "wu", "wd", "sg", "su", "sd"):
        setattr(p, name, getattr(nw, name).struct())
    p.g_x, p.g_h, p.g_hs = (float(v) for v in act_scales)
    p.rms_norm_out = 1 if rms_norm_out else 0
    p.out = B.ptr(out)
    if res is not None:
        p.out_f32, p.idx_out, p.w_out, p.cnt_out = (B.ptr(res.out_f32), B.ptr(res.idx), B.ptr(res.w), B.ptr(res.cnt))
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel()
    return p


def calibrate(dw: DeviceWeights, x: torch.Tensor, top_k: int = B.TOP_K, router_bias=None, stream=None):
    """Static NVFP4 activation tensor scales (g_x, g_h, g_hs) from one calibration
    batch run through the bf16 block: the library's observer writes the amax
    values and the scales on the device; they are copied back here.
    Returns ((g_x, g_h, g_hs) as float32, amax [3] float32)."""
    ws, _ = workspace_for(dw.dims, x.shape[0], top_k, device=x.device)
    out = torch.empty((x.shape[0], dw.dims.embed_dim), dtype=torch.bfloat16, device=x.device)
    amax = torch.zeros(3, dtype=torch.float32, device=x.device)
    scales = torch.zeros(3, dtype=torch.float32, device=x.device)
    p = B.make_params(x.shape[0], x, *dw.args(), out, top_k=top_k, dims=dw.dims, router_bias=router_bias, workspace=ws)
    B.check(B.moe_nvfp4_calibrate(p, amax, scales, stream), "moe_nvfp4_calibrate")
    g = scales.cpu().numpy().astype(np.float32)
    return tuple(np.float32(v) for v in g), amax.cpu().numpy().astype(np.float32)


# ------------------------------------------------ weight-only SFP8 / Q4_0


@dataclasses.dataclass
class WqLinear:
    """G stacked [K, N] Linears in a weight-only format: the library's blocks
    (uint8) and, for SFP8, the fp32 matrix scales [G]."""

    q: torch.Tensor
    scale: torch.Tensor | None

    def struct(self) -> B.MoeWqLinear:
        return B.MoeWqLinear(B.ptr(self.q), B.ptr(self.scale))


@dataclasses.dataclass
class WqWeights:
    dims: Dims
    fmt: str
    w_router: torch.Tensor
    wg: WqLinear
    wu: WqLinear
    wd: WqLinear
    sg: WqLinear
    su: WqLinear
    sd: WqLinear


def quantize_wq_linear(w: torch.Tensor, fmt: str, stream=None) -> WqLinear:
    """w [G, K, N] or [K, N] bf16 (device) -> the library's format `fmt`."""
    w3 = w if w.dim() == 3 else w.unsqueeze(0)
    G, K, N = w3.shape
    code = B.WFORMATS[fmt]
    q = torch.empty(B.moe_wq_weight_bytes(code, G, K, N), dtype=torch.uint8, device=w.device)
    scale = torch.empty(G, dtype=torch.float32, device=w.device) if fmt == "sfp8" else None
    B.check(B.moe_wq_quantize_weight(code, w3, G, K, N, q, scale, stream), "moe_wq_quantize_weight")
    return WqLinear(q, scale)


def quantize_wq(dw: DeviceWeights, fmt: str, stream=None) -> WqWeights:
    return WqWeights(dw.dims, fmt, dw.w_router,
                     *(quantize_wq_linear(t, fmt, stream) for t in (dw.wg, dw.wu, dw.wd, dw.sg, dw.su, dw.sd)))


def wq_params(ww: WqWeights, T: int, x, out, *, top_k=B.TOP_K, router_bias=None, res=None,
              workspace=None) -> B.MoeWqParams:
    p = B.MoeWqParams()
    p.T, p.top_k_experts, p.format = T, top_k, B.WFORMATS[ww.fmt]
    d = ww.dims
    p.embed_dim, p.num_experts, p.expert_dim, p.hidden_dim = d.embed_dim, d.num_experts, d.expert_dim, d.hidden_dim
    p.x, p.w_router, p.router_bias = B.ptr(x), B.ptr(ww.w_router), B.ptr(router_bias)
    for name in ("wg", "wu", "wd", "sg", "su", "sd"):
        setattr(p, name, getattr(ww, name).struct())
    p.out = B.ptr(out)
    if res is not None:
        p.out_f32, p.idx_out, p.w_out, p.cnt_out = (B.ptr(res.out_f32), B.ptr(res.idx), B.ptr(res.w), B.ptr(res.cnt))
    if workspace is not None:
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = workspace.numel()
    return p


def forward_wq(ww: WqWeights, x: torch.Tensor, *, top_k: int = B.TOP_K, router_bias=None, debug: bool = False,
               workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> BlockResult:
    """One block with weight-only SFP8 / Q4_0 expert and shared Linears."""
    T = x.shape[0]
    if out is None:
        out = torch.empty((T, ww.dims.embed_dim), dtype=torch.bfloat16, device=x.device)
    res = BlockResult(out=out)
    if debug:
        res.out_f32 = torch.empty((T, ww.dims.embed_dim), dtype=torch.float32, device=x.device)
        res.idx = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
        res.w = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
        res.cnt = torch.empty((ww.dims.num_experts,), dtype=torch.int32, device=x.device)
    p = wq_params(ww, T, x, out, top_k=top_k, router_bias=router_bias, res=res, workspace=workspace)
    B.check(B.moe_block_forward_wq(p, stream), "moe_block_forward_wq")
    return res


# ---------------------------------------------------------------- dense FFN


def dense_forward(x: torch.Tensor, wg: torch.Tensor, wu: torch.Tensor, wd: torch.Tensor, *, debug: bool = False,
                  workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> BlockResult:
    """The dense GeGLU FFN: out = (gelu_tanh(x wg) * (x wu)) wd; wg, wu [D, S], wd [S, D] bf16."""
    T, D = x.shape
    S = wg.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=torch.bfloat16, device=x.device)
    res = BlockResult(out=out)
    if debug:
        res.out_f32 = torch.empty((T, D), dtype=torch.float32, device=x.device)
    p = B.make_dense_params(T, x, wg, wu, wd, out, embed_dim=D, hidden_dim=S, out_f32=res.out_f32,
                            workspace=workspace)
    B.check(B.moe_dense_ffn_forward(p, stream), "moe_dense_ffn_forward")
    return res
