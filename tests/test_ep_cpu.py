"""Expert parallelism on CPU: the partitioning and the collectives of
mixture_experts_transformer_b200.ep, run as two and four gloo ranks.

Each rank holds its shard (its experts, its slice of the shared MLP's hidden
units, the replicated router) as cut by ep.shard_of; the block's partial sum of
a shard is evaluated here by the oracle (the library needs a GPU), in float64;
ep_forward all-gathers the tokens, sums the partials across ranks and hands
each rank its own rows. The result must equal the oracle's whole block on all
tokens (the layer splits exactly: gm.nn.Gemma4_26B_A4B, MoE branch plus
shared MLP branch, and GeGLU acts per hidden unit).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mixture_experts_transformer_b200 import ep, inputs

DIMS = inputs.Dims(embed_dim=64, num_experts=8, expert_dim=32, hidden_dim=320)
T_LOCAL, TOP_K = 5, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_weights():
    from mixture_experts_transformer_b200 import block

    w = inputs.make_weights(DIMS, seed=31, std=0.2)
    return w, block.DeviceWeights(DIMS, *(block.bf16_tensor(a, "cpu") for a in
                                          (w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd)))


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_partial(shard, x_all):
    """The shard's partial sum by the oracle: its shared-MLP slice, plus the
    slots of the whole layer's routing whose experts it holds."""
    from oracle import moe_oracle as mo

    x = _bits(x_all)
    idx, w, _ = mo.route(x, _bits(shard.w_router), TOP_K)
    part = mo.geglu_ffn(x, _bits(shard.sg), _bits(shard.su), _bits(shard.sd))
    xf = mo.f64(x)
    for t in range(x.shape[0]):
        for j in range(TOP_K):
            e = int(idx[t, j]) - shard.expert_begin
            if 0 <= e < shard.expert_count:
                part[t] += w[t, j] * mo.geglu_ffn(xf[t : t + 1], _bits(shard.wg[e]), _bits(shard.wu[e]),
                                                  _bits(shard.wd[e]))[0]
    return torch.from_numpy(part)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        _, dw = _cpu_weights()
        shard = ep.shard_of(dw, world, rank)
        x_all = inputs.make_x(world * T_LOCAL, DIMS.embed_dim, seed=32)
        from mixture_experts_transformer_b200 import block

        x_local = block.bf16_tensor(x_all[rank * T_LOCAL : (rank + 1) * T_LOCAL], "cpu")
        y = ep.ep_forward(shard, x_local, partial_fn=_oracle_partial, round_fn=lambda s: s)
        out.put((rank, (shard.expert_begin, shard.expert_count, shard.hidden_begin, shard.hidden_end), y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_block_equals_whole_block(world):
    from oracle import moe_oracle as mo

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the shards tile the experts and the shared MLP's hidden units exactly once
    experts = sorted(e for _, (e0, ec, _, _), _ in res for e in range(e0, e0 + ec))
    assert experts == list(range(DIMS.num_experts))
    units = sorted(u for _, (_, _, h0, h1), _ in res for u in range(h0, h1))
    assert units == list(range(DIMS.hidden_dim))
    assert all((h1 - h0) % 64 == 0 for _, (_, _, h0, h1), _ in res)
    # every rank gets the whole block's output for its own tokens
    w, _ = _cpu_weights()
    x_all = inputs.make_x(world * T_LOCAL, DIMS.embed_dim, seed=32)
    ref = mo.moe_block(x_all, w.w_router, w.wg, w.wu, w.wd, w.sg, w.su, w.sd, top_k=TOP_K)["out"]
    got = np.concatenate([y for _, _, y in res])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_shard_ranges():
    assert [ep.expert_range(128, 8, r) for r in (0, 7)] == [(0, 16), (112, 16)]
    # 2112 = 33 chunks of 64: over 8 ranks the first gets 5 chunks, the rest 4
    sl = [ep.hidden_slice(2112, 8, r) for r in range(8)]
    assert sl[0] == (0, 320) and sl[1] == (320, 576) and sl[-1] == (1856, 2112)
    assert sum(b - a for a, b in sl) == 2112
    with pytest.raises(ValueError):
        ep.expert_range(128, 3, 0)
    with pytest.raises(ValueError):
        ep.hidden_slice(100, 2, 0)
