"""Expert parallelism: one MoE block split over G devices.

The layer is two branches that add (gm.nn.Gemma4_26B_A4B class docstring: a
MoE branch of 128 experts and a dense shared MLP branch), so it splits without
approximation:

* rank r of G holds experts [r E / G, (r + 1) E / G) and a slice of the shared
  MLP's hidden units (whole 64-unit chunks, as even as the width allows); the
  router (embed_dim x num_experts) is replicated, so every rank routes every
  token exactly as the whole layer would;
* GeGLU acts per hidden unit, so each rank's shared-MLP slice gives a partial
  sum of the shared output, and its experts give the part of the weighted
  expert sum whose slots chose them;
* the partial sums (fp32) of all ranks add up to the block's output.

One forward pass of the data-parallel-in, expert-parallel-out decode layout:
all-gather every rank's tokens, run the library's expert-shard block on all of
them (its fp32 partial sums), reduce-scatter the partial sums so that each
rank receives the full sums of its own tokens, and round them to bf16 with the
library. Only the collectives move data between devices; every step of the
block runs in the library's kernels. The sum across ranks is taken in the
collective's order, so results are deterministic for a given G (and equal, up
to fp32 summation order, to the single-device block).
"""

from __future__ import annotations

import dataclasses

import torch

from . import binding as B
from .block import DeviceWeights
from .inputs import Dims

HIDDEN_CHUNK = 64  # the library's GEMMs take hidden widths in multiples of 64


def expert_range(num_experts: int, world: int, rank: int) -> tuple[int, int]:
    """(first expert, count) of rank `rank` of `world`; the experts must split evenly."""
    if world < 1 or not 0 <= rank < world or num_experts % world:
        raise ValueError(f"{num_experts} experts do not split over {world} ranks")
    per = num_experts // world
    return rank * per, per


def hidden_slice(hidden_dim: int, world: int, rank: int, chunk: int = HIDDEN_CHUNK) -> tuple[int, int]:
    """[begin, end) of the shared MLP's hidden units held by `rank`: whole
    `chunk`-unit pieces, the first (hidden_dim / chunk) % world ranks one more."""
    if hidden_dim % chunk:
        raise ValueError(f"hidden_dim {hidden_dim} is not a multiple of {chunk}")
    n = hidden_dim // chunk
    if n < world:
        raise ValueError(f"{n} chunks of the shared MLP cannot feed {world} ranks")
    base, extra = divmod(n, world)
    begin = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return begin * chunk, (begin + count) * chunk


@dataclasses.dataclass
class Shard:
    """One rank's part of a block: its experts' weights, its slice of the
    shared MLP, the replicated router, and where they sit in the whole layer."""

    dims: Dims  # the whole layer's dims (num_experts: all experts the router scores)
    world: int
    rank: int
    expert_begin: int
    expert_count: int
    hidden_begin: int
    hidden_end: int
    w_router: torch.Tensor
    wg: torch.Tensor
    wu: torch.Tensor
    wd: torch.Tensor
    sg: torch.Tensor
    su: torch.Tensor
    sd: torch.Tensor

    @property
    def hidden_dim(self) -> int:
        return self.hidden_end - self.hidden_begin

    def args(self):
        return (self.w_router, self.wg, self.wu, self.wd, self.sg, self.su, self.sd)


def shard_of(dw: DeviceWeights, world: int, rank: int) -> Shard:
    """Rank `rank`'s shard of a whole block's weights (copies, contiguous)."""
    d = dw.dims
    e0, ec = expert_range(d.num_experts, world, rank)
    h0, h1 = hidden_slice(d.hidden_dim, world, rank)
    return Shard(
        d, world, rank, e0, ec, h0, h1,
        dw.w_router,
        dw.wg[e0 : e0 + ec].contiguous(),
        dw.wu[e0 : e0 + ec].contiguous(),
        dw.wd[e0 : e0 + ec].contiguous(),
        dw.sg[:, h0:h1].contiguous(),
        dw.su[:, h0:h1].contiguous(),
        dw.sd[h0:h1].contiguous(),
    )


def shard_params(shard: Shard, T: int, x: torch.Tensor, partial: torch.Tensor, *, top_k: int = B.TOP_K,
                 router_bias=None, workspace=None, idx_out=None, w_out=None, cnt_out=None) -> B.MoeParams:
    """C-ABI parameters of the shard's block: its fp32 partial sums into `partial`."""
    d = shard.dims
    dims = Dims(d.embed_dim, d.num_experts, d.expert_dim, shard.hidden_dim)
    return B.make_params(T, x, *shard.args(), None, top_k=top_k, dims=dims, router_bias=router_bias,
                         out_f32=partial, idx_out=idx_out, w_out=w_out, cnt_out=cnt_out, workspace=workspace,
                         expert_begin=shard.expert_begin, expert_count=shard.expert_count)


def shard_partial(shard: Shard, x: torch.Tensor, *, top_k: int = B.TOP_K, router_bias=None, workspace=None,
                  stream=None) -> torch.Tensor:
    """The shard's partial sums [T, embed_dim] fp32 of the block over x [T, embed_dim]."""
    T = x.shape[0]
    partial = torch.empty((T, shard.dims.embed_dim), dtype=torch.float32, device=x.device)
    p = shard_params(shard, T, x, partial, top_k=top_k, router_bias=router_bias, workspace=workspace)
    B.check(B.moe_block_forward_ex(p, stream), "moe_block_forward_ex (expert shard)")
    return partial


def round_bf16(src: torch.Tensor, stream=None) -> torch.Tensor:
    """The library's round-to-nearest-even of fp32 sums into bf16."""
    out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    B.check(B.moe_round_bf16(src, out, src.numel(), stream), "moe_round_bf16")
    return out


def _reduce_scatter_sum(partial: torch.Tensor, world: int, rank: int, group) -> torch.Tensor:
    """Each rank's own rows of the sum over ranks of `partial` [world * T, D]."""
    import torch.distributed as dist

    T = partial.shape[0] // world
    if dist.get_backend(group) == "nccl":
        mine = torch.empty((T, partial.shape[1]), dtype=partial.dtype, device=partial.device)
        dist.reduce_scatter_tensor(mine, partial, op=dist.ReduceOp.SUM, group=group)
        return mine
    # backends without a reduce-scatter (gloo): the full sum, then this rank's rows
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial[rank * T : (rank + 1) * T].clone()


def ep_forward(shard: Shard, x_local: torch.Tensor, *, group=None, top_k: int = B.TOP_K, router_bias=None,
               workspace=None, stream=None, partial_fn=None, round_fn=None) -> torch.Tensor:
    """One expert-parallel block over this rank's tokens x_local [T, embed_dim]
    (every rank the same T): all-gather the tokens, the shard's partial sums
    over all of them, reduce-scatter, round. Returns this rank's output rows
    (bf16). partial_fn(shard, x_all) and round_fn(sums) default to the
    library's kernels."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if (world, rank) != (shard.world, shard.rank):
        raise ValueError(f"shard {shard.rank}/{shard.world} used on rank {rank}/{world}")
    x_all = torch.empty((world * x_local.shape[0], x_local.shape[1]), dtype=x_local.dtype, device=x_local.device)
    dist.all_gather_into_tensor(x_all, x_local.contiguous(), group=group)
    if partial_fn is None:
        partial = shard_partial(shard, x_all, top_k=top_k, router_bias=router_bias, workspace=workspace,
                                stream=stream)
    else:
        partial = partial_fn(shard, x_all)
    sums = _reduce_scatter_sum(partial, world, rank, group)
    return round_bf16(sums, stream) if round_fn is None else round_fn(sums)
