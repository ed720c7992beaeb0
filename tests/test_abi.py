"""The C-ABI library loads, exports every declared entry point and validates
arguments on the host (no GPU needed: every case here returns before any
CUDA call)."""

import ctypes
import os
import re

import pytest

from conftest import ROOT
from mixture_experts_transformer_b200 import binding as B
from mixture_experts_transformer_b200 import build as mbuild


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return B.lib()


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if not f.endswith(".h"):
            continue
        src = open(os.path.join(inc, f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(B.EXPORTS), set(names) - set(B.EXPORTS)


def test_status_strings(lib):
    for code in range(8):
        assert B.moe_status_string(code).startswith("MOE_")
    assert B.moe_status_string(B.MOE_ERR_GUARD) == "MOE_ERR_GUARD"


def test_workspace_sizes(lib):
    assert B.moe_workspace_bytes(0) > 0
    small = B.moe_workspace_bytes(8)
    big = B.moe_workspace_bytes(4096)
    assert big > small > 0
    # the routed intermediates dominate: x_perm, y (bf16 [8T, 2816]) and h
    assert big >= 4096 * 8 * (2816 * 2 * 2 + 704 * 2)
    p = B.make_params(64)
    lay = B.moe_workspace_layout(p)
    offs = [lay.x_perm, lay.h, lay.y, lay.hs, lay.s, lay.idx, lay.w, lay.cnt, lay.off, lay.row_of, lay.token_of,
            lay.x_norm]
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == len(offs)
    assert lay.total_bytes == B.moe_workspace_bytes(64)
    assert B.moe_workspace_bytes(64, 0) == 0  # top_k 0 is invalid


def _params(**kw):
    base = dict(x=16, w_router=16, wg=16, wu=16, wd=16, sg=16, su=16, sd=16, out=1 << 40)
    base.update(kw)
    return B.make_params(kw.pop("T", 4), **{k: v for k, v in base.items() if k != "T"})


def test_host_validation(lib):
    f = lambda p: lib.moe_block_forward_ex(ctypes.byref(p), None)  # noqa: E731
    assert f(_params(T=0)) == B.MOE_OK  # empty batch: no-op
    assert f(_params(T=-1)) == B.MOE_ERR_INVALID_ARG
    assert f(_params(x=0)) == B.MOE_ERR_INVALID_ARG  # null x
    assert f(_params(x=18)) == B.MOE_ERR_ALIGNMENT
    assert f(_params(out=16)) == B.MOE_ERR_INVALID_ARG  # out aliases x
    p = _params()
    p.top_k_experts = 129
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params()
    p.expert_dim = 700  # not a multiple of 64
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params()
    p.num_experts = 256  # more than one warp's 4 experts per lane
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(norm_pre=18)  # misaligned learned scale
    assert f(p) == B.MOE_ERR_ALIGNMENT
    p = _params(norm_post=16)
    p.embed_dim = 4160  # the post-norm keeps a whole row per CTA: embed_dim <= 4096
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params()
    p.embed_dim, p.residual = 4160, 1
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(norm_pre=16)
    p.embed_dim = 4160
    assert f(p) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_block_forward_ex(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_timeout_probe(0, None) == B.MOE_ERR_INVALID_ARG


def test_expert_shard_validation(lib):
    """Expert-shard fields and the optional bf16 output, checked on the host."""
    f = lambda p: lib.moe_block_forward_ex(ctypes.byref(p), None)  # noqa: E731
    p = _params(expert_begin=120, expert_count=16)  # past the 128 experts
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(expert_begin=-1, expert_count=4)
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(out=None)  # no output at all
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(out=1 << 40 | 8)  # misaligned bf16 output
    assert f(p) == B.MOE_ERR_ALIGNMENT
    # a shard's output is a partial sum: no post-norm, no residual
    p = _params(expert_begin=64, expert_count=64, out=None, out_f32=1 << 41, norm_post=16)
    assert f(p) == B.MOE_ERR_INVALID_ARG
    p = _params(expert_begin=0, expert_count=64, residual=True)
    assert f(p) == B.MOE_ERR_INVALID_ARG
    # fp32 output alone, without the bf16 one, but with the post-norm: refused too
    p = _params(out=None, out_f32=1 << 41, norm_post=16)
    assert f(p) == B.MOE_ERR_INVALID_ARG


def test_round_bf16_validation(lib):
    f = lib.moe_round_bf16
    assert f(None, None, 0, None) == B.MOE_OK  # nothing to do
    assert f(None, 16, 8, None) == B.MOE_ERR_INVALID_ARG
    assert f(16, 1 << 20, 12, None) == B.MOE_ERR_INVALID_ARG  # n not a multiple of 8
    assert f(20, 1 << 20, 8, None) == B.MOE_ERR_ALIGNMENT
    assert f(1 << 20, (1 << 20) + 16, 8, None) == B.MOE_ERR_INVALID_ARG  # overlap


def test_workspace_guard_layout(lib):
    """The layout ends in 256 guard bytes after every data region."""
    for T in (1, 64, 4096):
        lay = B.moe_workspace_layout(B.make_params(T))
        assert lay.guard % 256 == 0 and lay.total_bytes == lay.guard + 256
        assert lay.guard >= max(lay.x_perm, lay.h, lay.y, lay.hs, lay.s, lay.x_norm, lay.token_of)
    p = B.make_params(8)
    assert lib.moe_workspace_guard_check(ctypes.byref(p), None) == B.MOE_ERR_INVALID_ARG  # no workspace
    p = B.make_params(8, workspace=1 << 20, workspace_bytes=64)
    assert lib.moe_workspace_guard_check(ctypes.byref(p), None) == B.MOE_ERR_WORKSPACE
