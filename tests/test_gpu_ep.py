"""Expert shards of the block on one B200, through the C ABI.

Each of G shards (its experts, its slice of the shared MLP's hidden units, the
replicated router) runs on the same tokens; their fp32 partial sums must add
up to the whole block: against the oracle within the block's tolerance, and
against the library's own single-call block to fp32 summation order. Each
partial is also checked against the oracle's partial of that shard (given the
GPU's routing). The multi-device collectives of ep_forward are exercised on
one rank here (NCCL, world size 1) and on CPU ranks in test_ep_cpu.py.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

from gpu_common import (ACC_SLACK, BF16_SLACK, OUT_TOL, SMALL, bf16_storage_cost, device_weights, require_gpu,
                        run_block, to_np, w_args, weights)
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, ep, inputs
from oracle import moe_oracle as mo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _oracle_shard_partial(w_host, x_bits, shard, idx, wts):
    """Shared-MLP slice plus the slots whose experts the shard holds (float64)."""
    h0, h1 = shard.hidden_begin, shard.hidden_end
    part = mo.geglu_ffn(x_bits, w_host.sg[:, h0:h1], w_host.su[:, h0:h1], w_host.sd[h0:h1])
    x = mo.f64(x_bits)
    for e in range(shard.expert_begin, shard.expert_begin + shard.expert_count):
        tok, slot = np.nonzero(idx == e)
        if tok.size:
            part[tok] += wts[tok, slot][:, None] * mo.geglu_ffn(x[tok], w_host.wg[e], w_host.wu[e], w_host.wd[e])
    return part


@pytest.mark.parametrize("dims_name,T,k,G", [("gemma", 64, 8, 2), ("gemma", 64, 8, 4), ("small", 300, 4, 2),
                                             ("gemma", 1024, 8, 8)])
def test_shards_add_up_to_the_block(dims_name, T, k, G):
    dims = inputs.GEMMA4_26B_A4B if dims_name == "gemma" else SMALL
    seed, std = (0, inputs.INIT_STD) if dims_name == "gemma" else (1, 0.05)
    w = weights(dims, seed, std)
    dw = device_weights(dims, seed, std)
    x_bits = inputs.make_x(T, dims.embed_dim, seed=60 + T)
    x = block.bf16_tensor(x_bits)
    full = run_block(dw, x_bits, top_k=k)
    idx, wts = to_np(full.idx), to_np(full.w)
    ref = mo.moe_block(x_bits, *w_args(w), routing=(idx, wts))["out"]
    rms = np.sqrt(np.mean(ref**2))
    total = np.zeros((T, dims.embed_dim))
    for r in range(G):
        shard = ep.shard_of(dw, G, r)
        part = torch.empty((T, dims.embed_dim), dtype=torch.float32, device="cuda")
        s_idx = torch.empty_like(full.idx)
        s_w = torch.empty_like(full.w)
        s_cnt = torch.empty_like(full.cnt)
        p = ep.shard_params(shard, T, x, part, top_k=k, idx_out=s_idx, w_out=s_w, cnt_out=s_cnt)
        B.check(B.moe_block_forward_ex(p), "shard")
        assert B.moe_get_device_status() == B.MOE_OK
        # every shard routes exactly as the whole block
        assert torch.equal(s_idx, full.idx) and torch.equal(s_w, full.w)
        cnt = to_np(s_cnt)
        e0, e1 = shard.expert_begin, shard.expert_begin + shard.expert_count
        np.testing.assert_array_equal(cnt[e0:e1], to_np(full.cnt)[e0:e1])
        assert not cnt[:e0].any() and not cnt[e1:].any()
        got = to_np(part).astype(np.float64)
        ref_part = _oracle_shard_partial(w, x_bits, shard, idx, wts)
        err = np.abs(got - ref_part).max()
        # the block's bound, or the one derived from the bf16 storage of the
        # shard's own hidden rows and expert outputs (reduced shapes)
        cost = bf16_storage_cost(x_bits, w, idx, wts, hidden=(shard.hidden_begin, shard.hidden_end), experts=(e0, e1))
        assert err <= max(OUT_TOL * rms, BF16_SLACK * cost + ACC_SLACK * rms), (r, err / rms, cost / rms)
        total += got
    # the shards' sum is the block: against the oracle, and against the one-call block
    cost = bf16_storage_cost(x_bits, w, idx, wts)
    assert np.abs(total - ref).max() <= max(OUT_TOL * rms, BF16_SLACK * cost + ACC_SLACK * rms)
    diff = np.abs(total - to_np(full.out_f32)).max()
    assert diff <= 1e-4 * rms, diff / rms


def test_ep_forward_one_rank_is_the_block():
    """ep_forward through NCCL on one rank: the all-gather and reduce-scatter
    are identities, the shard holds the whole layer, so the result equals the
    block's bf16 output bit for bit."""
    import torch.distributed as dist

    dw = device_weights()
    T = 64
    x_bits = inputs.make_x(T, seed=71)
    x = block.bf16_tensor(x_bits)
    full = run_block(dw, x_bits)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        shard = ep.shard_of(dw, 1, 0)
        out = ep.ep_forward(shard, x)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert B.moe_get_device_status() == B.MOE_OK
    assert torch.equal(out, full.out)


def test_round_bf16_matches_torch():
    src = torch.randn((37, 64), device="cuda") * torch.logspace(-20, 20, 64, device="cuda")
    dst = torch.empty(src.shape, dtype=torch.bfloat16, device="cuda")
    B.check(B.moe_round_bf16(src, dst, src.numel()), "round")
    assert torch.equal(dst, src.to(torch.bfloat16))
