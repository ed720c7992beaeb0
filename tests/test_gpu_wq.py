"""Weight-only SFP8 and Q4_0 on a B200 against the oracle (oracle/wformats.py):
the quantisers bit-exact, the block within tolerance of the oracle's block on
the exactly dequantised weights (given the GPU's routing).

Tolerance: the block's 1e-2 * RMS, or the bound derived from the designed
roundings - the bf16 storage of h, hs and y (as for the bf16 block) and, for
Q4_0, the rounding of each dequantised weight (q - 8) d to bf16 before the
tensor cores; both are measured by evaluating the oracle's formula with and
without them (SFP8 values are exact in bf16, so only the first applies)."""

import functools

import numpy as np
import pytest
import torch

from gpu_common import (ACC_SLACK, BF16_SLACK, OUT_TOL, SMALL, bf16_storage_cost, check_routing, device_weights,
                        require_gpu, to_np, weights)
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import block, inputs
from oracle import moe_oracle as mo
from oracle import wformats as wf

pytestmark = pytest.mark.gpu
FORMATS = ["sfp8", "q4_0"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _unswizzle(rows: np.ndarray, shift: int, mask: int) -> np.ndarray:
    """[..., 128 rows, pieces, 16 B] stored with piece j of row r at position j ^ ((r >> shift) & mask)
    -> pieces in K order."""
    r = np.arange(128)[:, None]
    j = np.arange(rows.shape[-2])[None, :]
    return rows[..., r, j ^ ((r >> shift) & mask), :]


def decode_layout(q: np.ndarray, fmt: str, G: int, K: int, N: int):
    """The library's blocks -> (codes [G][N][K], Q4_0 scales [G][N][K/32] or None, padding rows)."""
    nb, kb = (N + 127) // 128, K // 64
    if fmt == "sfp8":
        blk = _unswizzle(q.reshape(G, nb, kb, 128, 4, 16), 1, 3).reshape(G, nb, kb, 128, 64)
        codes = blk.transpose(0, 1, 3, 2, 4).reshape(G, nb * 128, K)
        return codes[:, :N], None, codes[:, N:]
    blk = q.reshape(G, nb, kb, 4608)
    cb = _unswizzle(blk[..., :4096].reshape(G, nb, kb, 128, 2, 16), 2, 1).reshape(G, nb, kb, 128, 32)
    nib = np.empty((G, nb, kb, 128, 64), np.uint8)
    nib[..., 0::2] = cb & 0xF
    nib[..., 1::2] = cb >> 4
    codes = nib.transpose(0, 1, 3, 2, 4).reshape(G, nb * 128, K)
    sc = np.ascontiguousarray(blk[..., 4096:]).view(np.float16).reshape(G, nb, kb, 128, 2)
    sc = sc.transpose(0, 1, 3, 2, 4).reshape(G, nb * 128, K // 32)
    pad = np.concatenate([codes[:, N:].reshape(G, -1), sc[:, N:].view(np.uint16).reshape(G, -1)], axis=1)
    return codes[:, :N], sc[:, :N], pad


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("G,K,N", [(3, 256, 192), (1, 2816, 2112), (2, 704, 2816)])
def test_wq_quantizer_bit_exact(fmt, G, K, N):
    """Codes (and scales) equal the oracle's quantiser on the transposed weights;
    padding rows are zero."""
    gen = torch.Generator().manual_seed(50 + K)
    w = (torch.randn((G, K, N), generator=gen) * 0.03).to(torch.bfloat16)
    w[0, :32, 5] = 0.0  # an all-zero Q4_0 block
    lin = block.quantize_wq_linear(w.cuda(), fmt)
    assert B.moe_get_device_status() == B.MOE_OK
    codes, sc, pad = decode_layout(to_np(lin.q), fmt, G, K, N)
    assert not pad.any()
    wt = w.float().numpy().transpose(0, 2, 1)  # [G][N][K]
    for g in range(G):
        if fmt == "sfp8":
            s = wf.sfp8_scale(np.abs(wt[g]).max())
            assert to_np(lin.scale)[g] == s
            np.testing.assert_array_equal(codes[g], wf.sfp8_quantize(wt[g], s))
        else:
            q_ref, d_ref = wf.q4_0_quantize(wt[g])
            np.testing.assert_array_equal(codes[g], q_ref)
            np.testing.assert_array_equal(sc[g].view(np.uint16), d_ref.view(np.uint16))


def _rne_bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).double().numpy()


class _Deq:
    """Dequantised weights (float64) of the experts a routing uses and of the shared MLP."""

    def __init__(self, w, fmt, experts, round_bf16=False):
        f = lambda m: wf.weight_fake_quantize(mo.f64(m).astype(np.float32), fmt)  # noqa: E731
        r = _rne_bf16 if round_bf16 else (lambda a: a)
        self.w_router = w.w_router
        self.wg, self.wu, self.wd = (np.zeros(a.shape) for a in (w.wg, w.wu, w.wd))
        for e in experts:
            self.wg[e], self.wu[e], self.wd[e] = r(f(w.wg[e])), r(f(w.wu[e])), r(f(w.wd[e]))
        self.sg, self.su, self.sd = r(f(w.sg)), r(f(w.su)), r(f(w.sd))

    def args(self):
        return (self.w_router, self.wg, self.wu, self.wd, self.sg, self.su, self.sd)


@functools.lru_cache(maxsize=8)
def _wq_device(dims, seed, std, fmt):
    return block.quantize_wq(device_weights(dims, seed, std), fmt)


def _check_wq_block(fmt, dims, seed, std, T, k, x_seed, tokens=None):
    w = weights(dims, seed, std)
    ww = _wq_device(dims, seed, std, fmt)
    x_bits = inputs.make_x(T, dims.embed_dim, seed=x_seed)
    res = block.forward_wq(ww, block.bf16_tensor(x_bits), top_k=k, debug=True)
    assert B.moe_get_device_status() == B.MOE_OK
    tok = np.arange(T) if tokens is None else tokens
    xs, idx, wts = x_bits[tok], to_np(res.idx)[tok], to_np(res.w)[tok]
    ref_idx, ref_w, logits = mo.route(xs, w.w_router, k)
    check_routing(logits, ref_idx, ref_w, idx, wts, k)  # the router stays bf16
    deq = _Deq(w, fmt, np.unique(idx))
    ref = mo.moe_block(xs, *deq.args(), routing=(idx, wts))["out"]
    rms = np.sqrt(np.mean(ref**2))
    err = np.abs(to_np(res.out_f32)[tok].astype(np.float64) - ref).max()
    cost = bf16_storage_cost(xs, deq, idx, wts)
    if fmt == "q4_0":  # the GPU's weights are the dequantised ones rounded to bf16
        deq_r = _Deq(w, fmt, np.unique(idx), round_bf16=True)
        cost += np.abs(mo.moe_block(xs, *deq_r.args(), routing=(idx, wts))["out"] - ref).max()
    bound = max(OUT_TOL * rms, BF16_SLACK * cost + ACC_SLACK * rms)
    print(f"{fmt} T={T} k={k}: max |err| {err / rms:.4%} of RMS, bound {bound / rms:.4%}")
    assert err <= bound, (err / rms, bound / rms)
    out_bits = res.out.float().cpu().numpy()
    rne = torch.from_numpy(to_np(res.out_f32)).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(out_bits, rne)


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("T,k", [(1, 4), (37, 4), (300, 8)])
def test_wq_block_small_dims(fmt, T, k):
    _check_wq_block(fmt, SMALL, 1, 0.05, T, k, x_seed=30 + T)


@pytest.mark.parametrize("fmt", FORMATS)
def test_wq_block_gemma_T64(fmt):
    _check_wq_block(fmt, inputs.GEMMA4_26B_A4B, 0, inputs.INIT_STD, 64, 8, x_seed=1)


@pytest.mark.parametrize("fmt", FORMATS)
def test_wq_block_gemma_T1024_sampled(fmt):
    """T = 1024: experts hold ~64 rows (one 128-row block each), 256 tokens compared."""
    _check_wq_block(fmt, inputs.GEMMA4_26B_A4B, 0, inputs.INIT_STD, 1024, 8, x_seed=3,
                    tokens=inputs.sample_tokens(1024, 256))
