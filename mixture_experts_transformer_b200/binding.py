"""ctypes binding of libmoeblock.so (include/moe_block.h), same names as the C ABI.

Argument marshalling only: every step of the block runs in the library's CUDA
kernels. torch is used for device memory (``tensor.data_ptr()``) and streams.
There is no fallback: if the library is missing or the GPU is not a B200 the
calls raise.
"""

from __future__ import annotations

import ctypes
import os

from . import build as _build

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_ALIGNMENT = 2
MOE_ERR_ARCH = 3
MOE_ERR_CUDA = 4
MOE_ERR_WORKSPACE = 5
MOE_ERR_DEVICE_TIMEOUT = 6
MOE_ERR_GUARD = 7

EMBED_DIM, NUM_EXPERTS, EXPERT_DIM, HIDDEN_DIM, TOP_K = 2816, 128, 704, 2112, 8

_vp = ctypes.c_void_p


class MoeParams(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int),
        ("top_k_experts", ctypes.c_int),
        ("embed_dim", ctypes.c_int),
        ("num_experts", ctypes.c_int),
        ("expert_dim", ctypes.c_int),
        ("hidden_dim", ctypes.c_int),
        ("x", _vp),
        ("w_router", _vp),
        ("router_bias", _vp),
        ("wg", _vp),
        ("wu", _vp),
        ("wd", _vp),
        ("sg", _vp),
        ("su", _vp),
        ("sd", _vp),
        ("out", _vp),
        ("out_f32", _vp),
        ("idx_out", _vp),
        ("w_out", _vp),
        ("cnt_out", _vp),
        ("workspace", _vp),
        ("workspace_bytes", ctypes.c_size_t),
        ("norm_pre", _vp),
        ("norm_post", _vp),
        ("residual", ctypes.c_int),
        ("logits_out", _vp),
        ("expert_begin", ctypes.c_int),
        ("expert_count", ctypes.c_int),
        ("check_guards", ctypes.c_int),
    ]


class MoeWsLayout(ctypes.Structure):
    _fields_ = [
        (name, ctypes.c_size_t)
        for name in ("total_bytes", "x_perm", "h", "y", "hs", "s", "idx", "w", "cnt", "off", "row_of", "token_of",
                     "x_norm", "guard")
    ]


EXPORTS = {
    "moe_workspace_bytes_ex": (ctypes.c_size_t, [ctypes.POINTER(MoeParams)]),
    "moe_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int]),
    "moe_workspace_layout": (ctypes.c_int, [ctypes.POINTER(MoeParams), ctypes.POINTER(MoeWsLayout)]),
    "moe_block_forward": (ctypes.c_int, [_vp] * 8 + [ctypes.c_int, _vp, _vp]),
    "moe_block_forward_ex": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp]),
    "moe_route": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp, _vp, _vp]),
    "moe_permute": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_get_device_status": (ctypes.c_int, [_vp]),
    "moe_debug_timeout_probe": (ctypes.c_int, [ctypes.c_int, _vp]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_launch_count": (ctypes.c_int, []),
    "moe_round_bf16": (ctypes.c_int, [_vp, _vp, ctypes.c_size_t, _vp]),
    "moe_workspace_guard_check": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp]),
    "moe_block_forward_hostio": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp, _vp, _vp]),
    "moe_profile_begin": (ctypes.c_int, [ctypes.c_uint32]),
    "moe_profile_end": (ctypes.c_int, [_vp, _vp, ctypes.c_int]),
    "moe_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_route_noalloc": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp, _vp, _vp]),
}

_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libmoeblock.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run mixture_experts_transformer_b200.build.build() first")
        handle = ctypes.CDLL(path)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lib().moe_status_string(status).decode()}")


def check(status: int, where: str = "moe") -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def ptr(t) -> int | None:
    """Device address of a tensor (None stays None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_handle(stream=None) -> int | None:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_params(
    T: int,
    x=None,
    w_router=None,
    wg=None,
    wu=None,
    wd=None,
    sg=None,
    su=None,
    sd=None,
    out=None,
    *,
    top_k: int = TOP_K,
    dims=None,
    router_bias=None,
    out_f32=None,
    idx_out=None,
    w_out=None,
    cnt_out=None,
    workspace=None,
    workspace_bytes: int = 0,
    norm_pre=None,
    norm_post=None,
    residual: bool = False,
    logits_out=None,
    expert_begin: int = 0,
    expert_count: int = 0,
    check_guards: bool = False,
) -> MoeParams:
    p = MoeParams()
    p.T = T
    p.top_k_experts = top_k
    if dims is not None:
        p.embed_dim, p.num_experts, p.expert_dim, p.hidden_dim = (
            dims.embed_dim,
            dims.num_experts,
            dims.expert_dim,
            dims.hidden_dim,
        )
    for name, val in (
        ("x", x),
        ("w_router", w_router),
        ("router_bias", router_bias),
        ("wg", wg),
        ("wu", wu),
        ("wd", wd),
        ("sg", sg),
        ("su", su),
        ("sd", sd),
        ("out", out),
        ("out_f32", out_f32),
        ("idx_out", idx_out),
        ("w_out", w_out),
        ("cnt_out", cnt_out),
        ("workspace", workspace),
        ("norm_pre", norm_pre),
        ("norm_post", norm_post),
        ("logits_out", logits_out),
    ):
        setattr(p, name, ptr(val))
    p.residual = 1 if residual else 0
    p.expert_begin, p.expert_count = expert_begin, expert_count
    p.check_guards = 1 if check_guards else 0
    if workspace is not None and not workspace_bytes:
        workspace_bytes = workspace.numel() * workspace.element_size()
    p.workspace_bytes = workspace_bytes
    return p


def moe_workspace_bytes_ex(p: MoeParams) -> int:
    return lib().moe_workspace_bytes_ex(ctypes.byref(p))


def moe_workspace_bytes(T: int, top_k: int = TOP_K) -> int:
    return lib().moe_workspace_bytes(T, top_k)


def moe_workspace_layout(p: MoeParams) -> MoeWsLayout:
    out = MoeWsLayout()
    check(lib().moe_workspace_layout(ctypes.byref(p), ctypes.byref(out)), "moe_workspace_layout")
    return out


def moe_block_forward(x, w_router, wg, wu, wd, sg, su, sd, T, out, stream=None) -> int:
    return lib().moe_block_forward(
        ptr(x), ptr(w_router), ptr(wg), ptr(wu), ptr(wd), ptr(sg), ptr(su), ptr(sd), T, ptr(out), stream_handle(stream)
    )


def moe_block_forward_ex(p: MoeParams, stream=None) -> int:
    return lib().moe_block_forward_ex(ctypes.byref(p), stream_handle(stream))


def moe_route(p: MoeParams, idx, w, stream=None) -> int:
    return lib().moe_route(ctypes.byref(p), ptr(idx), ptr(w), stream_handle(stream))


def moe_permute(p: MoeParams, idx, cnt, off, row_of, token_of, stream=None) -> int:
    return lib().moe_permute(
        ctypes.byref(p), ptr(idx), ptr(cnt), ptr(off), ptr(row_of), ptr(token_of), stream_handle(stream)
    )


def moe_get_device_status(stream=None) -> int:
    return lib().moe_get_device_status(stream_handle(stream))


def moe_debug_timeout_probe(timeout_us: int, stream=None) -> int:
    return lib().moe_debug_timeout_probe(timeout_us, stream_handle(stream))


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def moe_last_launch_count() -> int:
    return lib().moe_last_launch_count()


def moe_workspace_guard_check(p: MoeParams, stream=None) -> int:
    return lib().moe_workspace_guard_check(ctypes.byref(p), stream_handle(stream))


def moe_round_bf16(src, dst, n: int, stream=None) -> int:
    return lib().moe_round_bf16(ptr(src), ptr(dst), n, stream_handle(stream))


def moe_block_forward_hostio(p: MoeParams, x_host, out_host, stream=None) -> int:
    return lib().moe_block_forward_hostio(ctypes.byref(p), ptr(x_host), ptr(out_host), stream_handle(stream))


def kernel_ids() -> dict:
    """{kernel name: id} of the library's kernels."""
    out, i = {}, 0
    while True:
        n = lib().moe_kernel_name(i)
        if n is None:
            return out
        out[n.decode()] = i
        i += 1


def moe_profile_begin(kernels=None) -> int:
    """Record events around the named kernels (all when None)."""
    if kernels is None:
        mask = 0xFFFFFFFF
    else:
        ids = kernel_ids()
        mask = 0
        for k in kernels:
            mask |= 1 << ids[k]
    return lib().moe_profile_begin(mask)


def moe_profile_end(n: int = 32) -> dict:
    """{kernel name: (total ms, launches)} for the kernels recorded since moe_profile_begin()."""
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int * n)()
    k = lib().moe_profile_end(ms, cnt, n)
    out = {}
    for i in range(min(k, n)):
        if cnt[i]:
            out[lib().moe_kernel_name(i).decode()] = (float(ms[i]), int(cnt[i]))
    return out


def moe_route_noalloc(p: MoeParams, idx, w, stream=None) -> int:
    """moe_route with its scratch in the library's fixed device array (no allocation)."""
    return lib().moe_route_noalloc(ctypes.byref(p), ptr(idx), ptr(w), stream_handle(stream))


# ----------------------------------------------------------------- NVFP4


class MoeNvfp4Linear(ctypes.Structure):
    _fields_ = [("q", _vp), ("sf", _vp), ("g", _vp)]


class MoeNvfp4Params(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int),
        ("top_k_experts", ctypes.c_int),
        ("embed_dim", ctypes.c_int),
        ("num_experts", ctypes.c_int),
        ("expert_dim", ctypes.c_int),
        ("hidden_dim", ctypes.c_int),
        ("x", _vp),
        ("w_router", _vp),
        ("router_bias", _vp),
        ("wg", MoeNvfp4Linear),
        ("wu", MoeNvfp4Linear),
        ("wd", MoeNvfp4Linear),
        ("sg", MoeNvfp4Linear),
        ("su", MoeNvfp4Linear),
        ("sd", MoeNvfp4Linear),
        ("g_x", ctypes.c_float),
        ("g_h", ctypes.c_float),
        ("g_hs", ctypes.c_float),
        ("rms_norm_out", ctypes.c_int),
        ("out", _vp),
        ("out_f32", _vp),
        ("idx_out", _vp),
        ("w_out", _vp),
        ("cnt_out", _vp),
        ("workspace", _vp),
        ("workspace_bytes", ctypes.c_size_t),
    ]


class MoeNvfp4WsLayout(ctypes.Structure):
    _fields_ = [
        (name, ctypes.c_size_t)
        for name in ("total_bytes", "xq_perm", "xsf_perm", "xq_tok", "xsf_tok", "hq", "hsf", "hsq", "hssf", "y", "s",
                     "idx", "w", "cnt", "off", "row_of")
    ] + [("routed_rows", ctypes.c_longlong), ("token_rows", ctypes.c_longlong)]


EXPORTS.update(
    {
        "moe_nvfp4_weight_bytes": (
            ctypes.c_int,
            [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t), ctypes.POINTER(ctypes.c_size_t)],
        ),
        "moe_nvfp4_quantize_weight": (
            ctypes.c_int,
            [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp],
        ),
        "moe_nvfp4_quantize_act": (ctypes.c_int, [_vp, ctypes.c_int, ctypes.c_int, ctypes.c_float, _vp, _vp, _vp]),
        "moe_nvfp4_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(MoeNvfp4Params)]),
        "moe_nvfp4_workspace_layout": (ctypes.c_int, [ctypes.POINTER(MoeNvfp4Params),
                                                      ctypes.POINTER(MoeNvfp4WsLayout)]),
        "moe_block_forward_nvfp4": (ctypes.c_int, [ctypes.POINTER(MoeNvfp4Params), _vp]),
        "moe_nvfp4_calibrate": (ctypes.c_int, [ctypes.POINTER(MoeParams), _vp, _vp, _vp]),
    }
)


def moe_nvfp4_weight_bytes(groups: int, K: int, N: int) -> tuple[int, int]:
    q, sf = ctypes.c_size_t(), ctypes.c_size_t()
    check(lib().moe_nvfp4_weight_bytes(groups, K, N, ctypes.byref(q), ctypes.byref(sf)), "moe_nvfp4_weight_bytes")
    return q.value, sf.value


def moe_nvfp4_quantize_weight(w, groups, K, N, q, sf, g, stream=None) -> int:
    return lib().moe_nvfp4_quantize_weight(ptr(w), groups, K, N, ptr(q), ptr(sf), ptr(g), stream_handle(stream))


def moe_nvfp4_quantize_act(x, rows, K, g, q, sf, stream=None) -> int:
    return lib().moe_nvfp4_quantize_act(ptr(x), rows, K, float(g), ptr(q), ptr(sf), stream_handle(stream))


def moe_nvfp4_workspace_bytes(p: MoeNvfp4Params) -> int:
    return lib().moe_nvfp4_workspace_bytes(ctypes.byref(p))


def moe_nvfp4_workspace_layout(p: MoeNvfp4Params) -> "MoeNvfp4WsLayout":
    out = MoeNvfp4WsLayout()
    check(lib().moe_nvfp4_workspace_layout(ctypes.byref(p), ctypes.byref(out)), "moe_nvfp4_workspace_layout")
    return out


def moe_block_forward_nvfp4(p: MoeNvfp4Params, stream=None) -> int:
    return lib().moe_block_forward_nvfp4(ctypes.byref(p), stream_handle(stream))


def moe_nvfp4_calibrate(p: MoeParams, amax, scales, stream=None) -> int:
    return lib().moe_nvfp4_calibrate(ctypes.byref(p), ptr(amax), ptr(scales), stream_handle(stream))


# ------------------------------------------------ weight-only SFP8 / Q4_0

WFMT_SFP8 = 1
WFMT_Q4_0 = 2
WFORMATS = {"sfp8": WFMT_SFP8, "q4_0": WFMT_Q4_0}


class MoeWqLinear(ctypes.Structure):
    _fields_ = [("q", _vp), ("scale", _vp)]


class MoeWqParams(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int),
        ("top_k_experts", ctypes.c_int),
        ("embed_dim", ctypes.c_int),
        ("num_experts", ctypes.c_int),
        ("expert_dim", ctypes.c_int),
        ("hidden_dim", ctypes.c_int),
        ("format", ctypes.c_int),
        ("x", _vp),
        ("w_router", _vp),
        ("router_bias", _vp),
        ("wg", MoeWqLinear),
        ("wu", MoeWqLinear),
        ("wd", MoeWqLinear),
        ("sg", MoeWqLinear),
        ("su", MoeWqLinear),
        ("sd", MoeWqLinear),
        ("out", _vp),
        ("out_f32", _vp),
        ("idx_out", _vp),
        ("w_out", _vp),
        ("cnt_out", _vp),
        ("workspace", _vp),
        ("workspace_bytes", ctypes.c_size_t),
    ]


EXPORTS.update(
    {
        "moe_wq_weight_bytes": (
            ctypes.c_int,
            [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)],
        ),
        "moe_wq_quantize_weight": (
            ctypes.c_int,
            [ctypes.c_int, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp],
        ),
        "moe_wq_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(MoeWqParams)]),
        "moe_block_forward_wq": (ctypes.c_int, [ctypes.POINTER(MoeWqParams), _vp]),
    }
)


def moe_wq_weight_bytes(fmt: int, groups: int, K: int, N: int) -> int:
    n = ctypes.c_size_t()
    check(lib().moe_wq_weight_bytes(fmt, groups, K, N, ctypes.byref(n)), "moe_wq_weight_bytes")
    return n.value


def moe_wq_quantize_weight(fmt, w, groups, K, N, q, scale, stream=None) -> int:
    return lib().moe_wq_quantize_weight(fmt, ptr(w), groups, K, N, ptr(q), ptr(scale), stream_handle(stream))


def moe_wq_workspace_bytes(p: MoeWqParams) -> int:
    return lib().moe_wq_workspace_bytes(ctypes.byref(p))


def moe_block_forward_wq(p: MoeWqParams, stream=None) -> int:
    return lib().moe_block_forward_wq(ctypes.byref(p), stream_handle(stream))


# ------------------------------------------------------------ dense GeGLU FFN

E4B_EMBED_DIM = 2560
E4B_HIDDEN_DIM = 10240


class MoeDenseParams(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int),
        ("embed_dim", ctypes.c_int),
        ("hidden_dim", ctypes.c_int),
        ("x", _vp),
        ("wg", _vp),
        ("wu", _vp),
        ("wd", _vp),
        ("out", _vp),
        ("out_f32", _vp),
        ("workspace", _vp),
        ("workspace_bytes", ctypes.c_size_t),
    ]


EXPORTS.update(
    {
        "moe_dense_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(MoeDenseParams)]),
        "moe_dense_ffn_forward": (ctypes.c_int, [ctypes.POINTER(MoeDenseParams), _vp]),
    }
)


def make_dense_params(T, x=None, wg=None, wu=None, wd=None, out=None, *, embed_dim=0, hidden_dim=0, out_f32=None,
                      workspace=None) -> MoeDenseParams:
    p = MoeDenseParams()
    p.T, p.embed_dim, p.hidden_dim = T, embed_dim, hidden_dim
    for name, val in (("x", x), ("wg", wg), ("wu", wu), ("wd", wd), ("out", out), ("out_f32", out_f32),
                      ("workspace", workspace)):
        setattr(p, name, ptr(val))
    if workspace is not None:
        p.workspace_bytes = workspace.numel() * workspace.element_size()
    return p


def moe_dense_workspace_bytes(p: MoeDenseParams) -> int:
    return lib().moe_dense_workspace_bytes(ctypes.byref(p))


def moe_dense_ffn_forward(p: MoeDenseParams, stream=None) -> int:
    return lib().moe_dense_ffn_forward(ctypes.byref(p), stream_handle(stream))
