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
) -> BlockResult:
    """Run one block; with debug=True also return out_f32, the routing and the counts."""
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
    )
    B.check(B.moe_block_forward_ex(p, stream), "moe_block_forward_ex")
    return res


def workspace_for(dims: Dims, T: int, top_k: int = B.TOP_K, device="cuda") -> tuple[torch.Tensor, B.MoeWsLayout]:
    """A caller-owned workspace (uint8) and its layout."""
    p = B.make_params(T, top_k=top_k, dims=dims)
    lay = B.moe_workspace_layout(p)
    return torch.empty(lay.total_bytes, dtype=torch.uint8, device=device), lay
