"""Python binding of libw8a8 (the C ABI in include/w8a8.h).

Argument marshalling only: each function takes torch CUDA tensors, allocates any output the
caller did not pass, and calls the C entry point of the same name on the current CUDA stream.
Every step of the computation runs in the library's kernels. If the library is missing the
first call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw8a8.so")

W8A8_OK = 0
W8A8_ERR_ARG = -1
W8A8_ERR_UNSUPPORTED = -2
W8A8_ERR_WORKSPACE = -3
W8A8_ERR_LAUNCH = -4
W8A8_ERR_DEVICE = -5
W8A8_W_INT8_PER_CHANNEL = 0
W8A8_W_INT4_PER_GROUP = 1

_c_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_size = ctypes.c_size_t


class W8A8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: status {status} ({status_string(status)})")
        self.status = status


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("topk_ids", "topk_w", "tile_counts", "offsets", "perm", "sx", "sx_sorted", "xq", "h",
                 "s_h", "hq", "o", "logits", "sync", "total")]


class _SharedLayout(ctypes.Structure):
    _fields_ = [("routed", _Layout)] + [(n, ctypes.c_size_t) for n in
                                        ("xq", "sx", "h", "s_h", "hq", "o", "gate", "total")]


# (name, restype, argtypes) of every exported entry point
SIGNATURES = {
    "w8a8_version": (_int, []),
    "w8a8_status_string": (ctypes.c_char_p, [_int]),
    "w8a8_check_status": (_int, [_c_p]),
    "w8a8_quantize_weight_per_channel": (_int, [_c_p, _i64, _i64, _i64, _c_p, _c_p, _c_p]),
    "w8a8_quantize_weight_int4_per_group": (_int, [_c_p, _i64, _i64, _int, _c_p, _c_p, _c_p]),
    "w8a8_quant_act_per_token": (_int, [_c_p, _i64, _i64, _c_p, _c_p, _c_p]),
    "w8a8_moe_route": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _int, _c_p, _c_p, _c_p, _c_p]),
    "w8a8_moe_workspace_layout": (_int, [_i64, _i64, _i64, _int, _i64, ctypes.POINTER(_Layout)]),
    "w8a8_moe_workspace_size": (_size, [_i64, _i64, _i64, _int, _i64]),
    "w8a8_moe_forward": (_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _i64, _int,
                                _c_p, _size, _c_p, _c_p]),
    "w8a8_moe_forward_profiled": (_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _i64,
                                         _int, _c_p, _size, _c_p, _c_p, ctypes.POINTER(_c_p)]),
    "w8a8_moe_forward_noalloc": (_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _i64,
                                        _int, _c_p, _c_p]),
    "w8a8_moe_shared_workspace_layout": (_int, [_i64, _i64, _i64, _int, _i64, _i64, ctypes.POINTER(_SharedLayout)]),
    "w8a8_moe_shared_workspace_size": (_size, [_i64, _i64, _i64, _int, _i64, _i64]),
    "w8a8_moe_forward_shared": (_int, [_c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _i64, _int,
                                       _c_p, _c_p, _c_p, _c_p, _c_p, _i64, _c_p, _size, _c_p, _c_p]),
    "w8a8_linear_workspace_size": (_size, [_i64, _i64, _i64, _int, _int]),
    "w8a8_linear": (_int, [_c_p, _c_p, _c_p, _int, _int, _i64, _i64, _i64, _c_p, _size, _c_p, _c_p]),
    "w8a8_linear_prequant": (_int, [_c_p, _c_p, _c_p, _c_p, _int, _int, _i64, _i64, _i64, _c_p, _c_p]),
    "w8a8_gemm_s8s8s32": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _i64, _c_p]),
    "w8a8_mxfp8_quantize": (_int, [_c_p, _i64, _i64, _c_p, _c_p, _c_p]),
    "w8a8_mxfp8_linear_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "w8a8_mxfp8_linear": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _i64, _c_p, ctypes.c_size_t, _c_p, _c_p]),
    "w8a8_mxfp8_linear_prequant": (_int, [_c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _c_p, _c_p]),
    "w8a8_mxfp4_quantize": (_int, [_c_p, _i64, _i64, _c_p, _c_p, _c_p]),
    "w8a8_moe_route_group": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _i64, _int, _int, _c_p, ctypes.c_size_t, _c_p]),
    "w8a8_moe_experts_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64]),
    "w8a8_moe_experts": (_int, [_c_p, _c_p, ctypes.POINTER(ctypes.c_int), _i64, _i64, _i64, _i64, _i64, _i64, _c_p,
                                _c_p, _c_p, _c_p, _c_p, ctypes.c_size_t, _c_p, _c_p]),
    "w8a8_moe_combine_sorted": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _int, _c_p, _c_p, _c_p]),
    "w8a8_mxfp_a8w4_linear": (_int, [_c_p, _c_p, _c_p, _i64, _i64, _i64, _c_p, ctypes.c_size_t, _c_p, _c_p]),
    "w8a8_mxfp_a8w4_linear_prequant": (_int, [_c_p, _c_p, _c_p, _c_p, _i64, _i64, _i64, _c_p, _c_p]),
    "w8a8_debug_wait_timeout": (_int, [ctypes.c_uint64, _c_p]),
    "w8a8_debug_rcp_approx_ulp": (_int, [ctypes.c_uint32, ctypes.c_uint32, _c_p, _c_p]),
    "w8a8_debug_ex2_approx_ulp": (_int, [ctypes.c_uint32, ctypes.c_uint32, _c_p, _c_p]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Loads libw8a8.so (built in-tree by build.py); raises if it is absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libw8a8.so not found at {LIB_PATH}; run w8a8_int8_quantized_act_b200/build.py")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().w8a8_status_string(status).decode()
    except Exception:  # pragma: no cover - library missing
        return "?"


def _check(rc: int, where: str):
    if rc != W8A8_OK:
        raise W8A8Error(rc, where)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _bf16(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return t


def w8a8_version() -> int:
    return lib().w8a8_version()


def w8a8_check_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status; raises on error."""
    rc = lib().w8a8_check_status(_stream(stream))
    _check(rc, "w8a8_check_status")
    return rc


def w8a8_quantize_weight_per_channel(w: torch.Tensor, q=None, scale=None, stream=None):
    """w bf16 [..., N, K] -> (q int8 [..., N, K], scale fp32 [..., N])."""
    _bf16(w)
    *lead, N, K = w.shape
    G = 1
    for d in lead:
        G *= d
    q = torch.empty(w.shape, dtype=torch.int8, device=w.device) if q is None else q
    scale = torch.empty((*lead, N), dtype=torch.float32, device=w.device) if scale is None else scale
    _check(lib().w8a8_quantize_weight_per_channel(_ptr(w), G, N, K, _ptr(q), _ptr(scale), _stream(stream)),
           "w8a8_quantize_weight_per_channel")
    return q, scale


def w8a8_quantize_weight_int4_per_group(w: torch.Tensor, group: int = 128, packed=None, scale=None, stream=None):
    """w bf16 [N, K] -> (packed uint8 [N, K/2], scale fp32 [N, K/group])."""
    _bf16(w)
    N, K = w.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device) if packed is None else packed
    scale = torch.empty((N, K // group), dtype=torch.float32, device=w.device) if scale is None else scale
    _check(lib().w8a8_quantize_weight_int4_per_group(_ptr(w), N, K, group, _ptr(packed), _ptr(scale),
                                                     _stream(stream)),
           "w8a8_quantize_weight_int4_per_group")
    return packed, scale


def w8a8_quant_act_per_token(x: torch.Tensor, q=None, scale=None, stream=None):
    """x bf16 [T, K] -> (q int8 [T, K], scale fp32 [T])."""
    _bf16(x)
    T, K = x.shape
    q = torch.empty((T, K), dtype=torch.int8, device=x.device) if q is None else q
    scale = torch.empty((T,), dtype=torch.float32, device=x.device) if scale is None else scale
    _check(lib().w8a8_quant_act_per_token(_ptr(x), T, K, _ptr(q), _ptr(scale), _stream(stream)),
           "w8a8_quant_act_per_token")
    return q, scale


def w8a8_moe_route(x: torch.Tensor, wg: torch.Tensor, k: int, renorm: bool = True, bias=None,
                   topk_ids=None, topk_w=None, expert_counts=None, stream=None):
    """Router: (topk_ids int32 [T, k], topk_w fp32 [T, k], expert_counts int32 [E])."""
    _bf16(x), _bf16(wg)
    T, H = x.shape
    E = wg.shape[0]
    dev = x.device
    topk_ids = torch.empty((T, k), dtype=torch.int32, device=dev) if topk_ids is None else topk_ids
    topk_w = torch.empty((T, k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    expert_counts = torch.empty((E,), dtype=torch.int32, device=dev) if expert_counts is None else expert_counts
    _check(lib().w8a8_moe_route(_ptr(x), _ptr(wg), _ptr(bias), T, H, E, k, int(renorm), _ptr(topk_ids),
                                _ptr(topk_w), _ptr(expert_counts), _stream(stream)), "w8a8_moe_route")
    return topk_ids, topk_w, expert_counts


def w8a8_moe_workspace_layout(T: int, H: int, E: int, k: int, I: int) -> dict:
    L = _Layout()
    _check(lib().w8a8_moe_workspace_layout(T, H, E, k, I, ctypes.byref(L)), "w8a8_moe_workspace_layout")
    return {name: getattr(L, name) for name, _ in _Layout._fields_}


def w8a8_moe_workspace_size(T: int, H: int, E: int, k: int, I: int) -> int:
    return lib().w8a8_moe_workspace_size(T, H, E, k, I)


def w8a8_moe_forward(x, wg, wgu, s_gu, wd, s_d, k: int, renorm: bool = True, bias=None, workspace=None,
                     y=None, stream=None):
    """W8A8 MoE expert-FFN forward; returns y bf16 [T, H] (workspace keeps the intermediates)."""
    _bf16(x), _bf16(wg)
    T, H = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    ws_bytes = w8a8_moe_workspace_size(T, H, E, k, I)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_moe_forward(_ptr(x), _ptr(wg), _ptr(bias), _ptr(wgu), _ptr(s_gu), _ptr(wd), _ptr(s_d),
                                  T, H, E, k, I, int(renorm), _ptr(workspace), workspace.numel(), _ptr(y),
                                  _stream(stream)), "w8a8_moe_forward")
    return y


def w8a8_moe_shared_workspace_layout(T: int, H: int, E: int, k: int, I: int, Is: int) -> dict:
    L = _SharedLayout()
    _check(lib().w8a8_moe_shared_workspace_layout(T, H, E, k, I, Is, ctypes.byref(L)),
           "w8a8_moe_shared_workspace_layout")
    out = {name: getattr(L, name) for name, _ in _SharedLayout._fields_ if name != "routed"}
    out["routed"] = {name: getattr(L.routed, name) for name, _ in _Layout._fields_}
    return out


def w8a8_moe_shared_workspace_size(T: int, H: int, E: int, k: int, I: int, Is: int) -> int:
    return lib().w8a8_moe_shared_workspace_size(T, H, E, k, I, Is)


def w8a8_moe_forward_shared(x, wg, wgu, s_gu, wd, s_d, k: int, wsg, wgu_s, s_gu_s, wd_s, s_d_s, renorm: bool = True,
                            bias=None, workspace=None, y=None, stream=None):
    """MoE layer with a shared expert; returns y bf16 [T, H] (workspace keeps the intermediates)."""
    _bf16(x), _bf16(wg), _bf16(wsg)
    T, H = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    Is = wgu_s.shape[0] // 2
    ws_bytes = w8a8_moe_shared_workspace_size(T, H, E, k, I, Is)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_moe_forward_shared(_ptr(x), _ptr(wg), _ptr(bias), _ptr(wgu), _ptr(s_gu), _ptr(wd), _ptr(s_d),
                                         T, H, E, k, I, int(renorm), _ptr(wsg), _ptr(wgu_s), _ptr(s_gu_s), _ptr(wd_s),
                                         _ptr(s_d_s), Is, _ptr(workspace), workspace.numel(), _ptr(y),
                                         _stream(stream)), "w8a8_moe_forward_shared")
    return y


def moe_shared_intermediates(workspace: torch.Tensor, T: int, H: int, E: int, k: int, I: int, Is: int) -> dict:
    """Views of the intermediates w8a8_moe_forward_shared leaves in its workspace: the routed ones
    (as moe_intermediates) and the shared expert's under the key "shared"."""
    L = w8a8_moe_shared_workspace_layout(T, H, E, k, I, Is)

    def view(name, dtype, shape):
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return workspace[L[name]:L[name] + nbytes].view(dtype).view(*shape)

    out = moe_intermediates(workspace, T, H, E, k, I)
    out["shared"] = dict(xq=view("xq", torch.int8, (T, H)), sx=view("sx", torch.float32, (T,)),
                         h=view("h", torch.bfloat16, (T, Is)), s_h=view("s_h", torch.float32, (T,)),
                         hq=view("hq", torch.int8, (T, Is)), o=view("o", torch.bfloat16, (T, H)),
                         gate=view("gate", torch.float32, (T,)))
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20


def w8a8_moe_forward_noalloc(x, wg, wgu, s_gu, wd, s_d, k: int, renorm: bool = True, bias=None, y=None,
                             stream=None):
    """The MoE forward with scratch in the library's own device buffer: for callers that can
    not allocate (see include/w8a8.h). Only y is allocated here, and only when not passed."""
    _bf16(x), _bf16(wg)
    T, H = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_moe_forward_noalloc(_ptr(x), _ptr(wg), _ptr(bias), _ptr(wgu), _ptr(s_gu), _ptr(wd),
                                          _ptr(s_d), T, H, E, k, I, int(renorm), _ptr(y), _stream(stream)),
           "w8a8_moe_forward_noalloc")
    return y


MOE_STAGES = ("router", "group_quant", "gate_up", "requant", "down", "combine")


def w8a8_moe_forward_profiled(x, wg, wgu, s_gu, wd, s_d, k: int, events, renorm: bool = True, bias=None,
                              workspace=None, y=None, stream=None):
    """w8a8_moe_forward recording the 7 torch.cuda.Event objects in `events` at stage boundaries."""
    T, H = x.shape
    E, twoI, _ = wgu.shape
    I = twoI // 2
    if workspace is None:
        workspace = torch.empty(max(w8a8_moe_workspace_size(T, H, E, k, I), 1), dtype=torch.uint8,
                                device=x.device)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device) if y is None else y
    arr = (_c_p * 7)(*[e.cuda_event for e in events])
    _check(lib().w8a8_moe_forward_profiled(_ptr(x), _ptr(wg), _ptr(bias), _ptr(wgu), _ptr(s_gu), _ptr(wd),
                                           _ptr(s_d), T, H, E, k, I, int(renorm), _ptr(workspace),
                                           workspace.numel(), _ptr(y), _stream(stream), arr),
           "w8a8_moe_forward_profiled")
    return y


def w8a8_moe_route_group(x, wg, E: int, k: int, renorm: bool = True, bias=None, workspace=None, stream=None):
    """Steps 1-2 of the forward on local tokens; returns the workspace (the layout of
    w8a8_moe_workspace_layout(T, H, E, k, 128)) whose topk_ids, topk_w, offsets, perm, sx_sorted and
    xq moe_intermediates(workspace, T, H, E, k, 128) views."""
    _bf16(x), _bf16(wg)
    T, H = x.shape
    ws_bytes = w8a8_moe_workspace_size(T, H, E, k, 128)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    _check(lib().w8a8_moe_route_group(_ptr(x), _ptr(wg), _ptr(bias), T, H, E, k, int(renorm), _ptr(workspace),
                                      workspace.numel(), _stream(stream)), "w8a8_moe_route_group")
    return workspace


def w8a8_moe_experts_workspace_size(A: int, H: int, I: int, Ew: int) -> int:
    return int(lib().w8a8_moe_experts_workspace_size(A, H, I, Ew))


def w8a8_moe_experts(xq, sx, group_offsets, wgu, s_gu, wd, s_d, weight_groups: int = 0, A: int = None,
                     workspace=None, o=None, stream=None):
    """Steps 3-5 on received rows: xq int8 [A, H], sx fp32 [A], group_offsets a host sequence of
    G+1 ints; group g uses expert g % weight_groups (0: g). Returns o bf16 [A, H] in input row order."""
    H = xq.shape[1]
    Ew, twoI, _ = wgu.shape
    I = twoI // 2
    offs = [int(v) for v in group_offsets]
    G = len(offs) - 1
    A = offs[-1] if A is None else A
    need = w8a8_moe_experts_workspace_size(A, H, I, Ew)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=xq.device)
    o = torch.empty((A, H), dtype=torch.bfloat16, device=xq.device) if o is None else o
    arr = (ctypes.c_int * (G + 1))(*offs)
    _check(lib().w8a8_moe_experts(_ptr(xq), _ptr(sx), arr, G, weight_groups, A, H, I, Ew, _ptr(wgu), _ptr(s_gu),
                                  _ptr(wd), _ptr(s_d), _ptr(workspace), workspace.numel(), _ptr(o),
                                  _stream(stream)), "w8a8_moe_experts")
    return o


def w8a8_moe_combine_sorted(o_sorted, perm, topk_w, k: int, o_slots=None, y=None, stream=None):
    """Step 6 from expert outputs in sorted-row order: y bf16 [T, H]."""
    A, H = o_sorted.shape
    T = A // k
    o_slots = torch.empty_like(o_sorted) if o_slots is None else o_slots
    y = torch.empty((T, H), dtype=torch.bfloat16, device=o_sorted.device) if y is None else y
    _check(lib().w8a8_moe_combine_sorted(_ptr(o_sorted), _ptr(perm), _ptr(topk_w), T, H, k, _ptr(o_slots), _ptr(y),
                                         _stream(stream)), "w8a8_moe_combine_sorted")
    return y


def moe_intermediates(workspace: torch.Tensor, T: int, H: int, E: int, k: int, I: int) -> dict:
    """Views of the intermediates w8a8_moe_forward leaves in its workspace."""
    L = w8a8_moe_workspace_layout(T, H, E, k, I)
    A = T * k
    Ap = max(1, -(-A // 128)) * 128 if A else 128
    C = -(-T // 128)

    def view(name, dtype, shape):
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        return workspace[L[name]:L[name] + nbytes].view(dtype).view(*shape)

    return dict(
        topk_ids=view("topk_ids", torch.int32, (T, k)), topk_w=view("topk_w", torch.float32, (T, k)),
        tile_counts=view("tile_counts", torch.int32, (C, E)), offsets=view("offsets", torch.int32, (E + 1,)),
        perm=view("perm", torch.int32, (A,)), sx=view("sx", torch.float32, (T,)),
        sx_sorted=view("sx_sorted", torch.float32, (Ap,)), xq=view("xq", torch.int8, (Ap, H)),
        h=view("h", torch.bfloat16, (Ap, I)), s_h=view("s_h", torch.float32, (Ap,)),
        hq=view("hq", torch.int8, (Ap, I)), o=view("o", torch.bfloat16, (A, H)),
        logits=view("logits", torch.float32, (T, E)))


def w8a8_linear_workspace_size(M: int, K: int, N: int, w_format: int, group: int = 128) -> int:
    return lib().w8a8_linear_workspace_size(M, K, N, w_format, group)


def w8a8_linear(x, w, sw, w_format: int = W8A8_W_INT8_PER_CHANNEL, group: int = 128, workspace=None, y=None,
                stream=None):
    """Dense W8A8 / W4A8 linear: y bf16 [M, N] = x [M, K] . W^T."""
    _bf16(x)
    M, K = x.shape
    N = w.shape[0]
    ws_bytes = w8a8_linear_workspace_size(M, K, N, w_format, group)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_linear(_ptr(x), _ptr(w), _ptr(sw), w_format, group, M, K, N, _ptr(workspace),
                             workspace.numel(), _ptr(y), _stream(stream)), "w8a8_linear")
    return y


def w8a8_linear_prequant(xq, sx, w, sw, w_format: int = W8A8_W_INT8_PER_CHANNEL, group: int = 128, y=None,
                         stream=None):
    """The dense linear's GEMM on per-token int8 activations xq [M, K] with scales sx [M]."""
    if xq.dtype != torch.int8 or sx.dtype != torch.float32:
        raise TypeError("expected int8 codes and fp32 scales")
    M, K = xq.shape
    N = w.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device) if y is None else y
    _check(lib().w8a8_linear_prequant(_ptr(xq), _ptr(sx), _ptr(w), _ptr(sw), w_format, group, M, K, N, _ptr(y),
                                      _stream(stream)), "w8a8_linear_prequant")
    return y


def w8a8_mxfp8_quantize(x: torch.Tensor, codes=None, scales=None, stream=None):
    """x bf16 [R, K] -> (codes uint8 [R, K] (E4M3), scales uint8 [R, K/32] (E8M0))."""
    _bf16(x)
    R, K = x.shape
    codes = torch.empty((R, K), dtype=torch.uint8, device=x.device) if codes is None else codes
    scales = torch.empty((R, max(K // 32, 1)), dtype=torch.uint8, device=x.device) if scales is None else scales
    _check(lib().w8a8_mxfp8_quantize(_ptr(x), R, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "w8a8_mxfp8_quantize")
    return codes, scales


def w8a8_mxfp8_linear_workspace_size(M: int, K: int, N: int) -> int:
    return int(lib().w8a8_mxfp8_linear_workspace_size(M, K, N))


def w8a8_mxfp8_linear(x, w_codes, w_scales, workspace=None, y=None, stream=None):
    """Dense MXFP8 A8W8 linear: y bf16 [M, N] = x [M, K] . W^T, W given as MXFP8 codes and scales."""
    _bf16(x)
    M, K = x.shape
    N = w_codes.shape[0]
    ws_bytes = w8a8_mxfp8_linear_workspace_size(M, K, N)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_mxfp8_linear(_ptr(x), _ptr(w_codes), _ptr(w_scales), M, K, N, _ptr(workspace),
                                   workspace.numel(), _ptr(y), _stream(stream)), "w8a8_mxfp8_linear")
    return y


def w8a8_mxfp8_linear_prequant(x_codes, x_scales, w_codes, w_scales, y=None, stream=None):
    """The GEMM of w8a8_mxfp8_linear on activations already in MXFP8 (codes [M, K], scales [M, K/32])."""
    M, K = x_codes.shape
    N = w_codes.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device) if y is None else y
    _check(lib().w8a8_mxfp8_linear_prequant(_ptr(x_codes), _ptr(x_scales), _ptr(w_codes), _ptr(w_scales), M, K, N,
                                            _ptr(y), _stream(stream)), "w8a8_mxfp8_linear_prequant")
    return y


def w8a8_mxfp4_quantize(w: torch.Tensor, packed=None, scales=None, stream=None):
    """w bf16 [R, K] -> (packed uint8 [R, K/2] (two E2M1 codes a byte, even element low),
    scales uint8 [R, K/32] (E8M0))."""
    _bf16(w)
    R, K = w.shape
    packed = torch.empty((R, max(K // 2, 1)), dtype=torch.uint8, device=w.device) if packed is None else packed
    scales = torch.empty((R, max(K // 32, 1)), dtype=torch.uint8, device=w.device) if scales is None else scales
    _check(lib().w8a8_mxfp4_quantize(_ptr(w), R, K, _ptr(packed), _ptr(scales), _stream(stream)),
           "w8a8_mxfp4_quantize")
    return packed, scales


def w8a8_mxfp_a8w4_linear(x, w_packed, w_scales, workspace=None, y=None, stream=None):
    """Dense MXFP A8W4 linear: y bf16 [M, N] = x [M, K] . W^T, x quantised to MXFP8 per token, W
    given as MXFP4 (packed [N, K/2], scales [N, K/32]). The workspace is sized by
    w8a8_mxfp8_linear_workspace_size and receives x's MXFP8 codes and scales."""
    _bf16(x)
    M, K = x.shape
    N = w_packed.shape[0]
    ws_bytes = w8a8_mxfp8_linear_workspace_size(M, K, N)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else y
    _check(lib().w8a8_mxfp_a8w4_linear(_ptr(x), _ptr(w_packed), _ptr(w_scales), M, K, N, _ptr(workspace),
                                       workspace.numel(), _ptr(y), _stream(stream)), "w8a8_mxfp_a8w4_linear")
    return y


def w8a8_mxfp_a8w4_linear_prequant(x_codes, x_scales, w_packed, w_scales, y=None, stream=None):
    """The GEMM of w8a8_mxfp_a8w4_linear on activations already in MXFP8."""
    M, K = x_codes.shape
    N = w_packed.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x_codes.device) if y is None else y
    _check(lib().w8a8_mxfp_a8w4_linear_prequant(_ptr(x_codes), _ptr(x_scales), _ptr(w_packed), _ptr(w_scales), M,
                                                K, N, _ptr(y), _stream(stream)), "w8a8_mxfp_a8w4_linear_prequant")
    return y


def mxfp8_linear_intermediates(workspace, M: int, K: int) -> dict:
    """x's MXFP8 codes [M, K] and scales [M, K/32] that w8a8_mxfp8_linear (or
    w8a8_mxfp_a8w4_linear) left in its workspace."""
    a256 = lambda v: (v + 255) // 256 * 256  # noqa: E731
    codes = workspace[:M * K].view(M, K)
    off = a256(M * K)
    scales = workspace[off:off + M * (K // 32)].view(M, K // 32)
    return dict(codes=codes, scales=scales)


def w8a8_gemm_s8s8s32(a, b, c=None, stream=None):
    """Exact int8 GEMM on the tensor cores: c int32 [M, N] = a [M, K] . b [N, K]^T."""
    M, K = a.shape
    N = b.shape[0]
    c = torch.empty((M, N), dtype=torch.int32, device=a.device) if c is None else c
    _check(lib().w8a8_gemm_s8s8s32(_ptr(a), _ptr(b), _ptr(c), M, N, K, _stream(stream)), "w8a8_gemm_s8s8s32")
    return c


def w8a8_debug_rcp_approx_ulp(first_bits: int, count: int, stream=None) -> int:
    """Largest ulp distance of rcp.approx from the correctly rounded reciprocal over a range of
    fp32 bit patterns."""
    out = torch.empty(1, dtype=torch.int32, device="cuda")
    _check(lib().w8a8_debug_rcp_approx_ulp(first_bits, count, _ptr(out), _stream(stream)),
           "w8a8_debug_rcp_approx_ulp")
    return int(out.cpu().item())


def w8a8_debug_ex2_approx_ulp(first_bits: int, count: int, stream=None) -> int:
    """Largest ulp distance of ex2.approx from 2^x (computed in double, rounded to fp32) over a
    range of fp32 bit patterns."""
    out = torch.empty(1, dtype=torch.int32, device="cuda")
    _check(lib().w8a8_debug_ex2_approx_ulp(first_bits, count, _ptr(out), _stream(stream)),
           "w8a8_debug_ex2_approx_ulp")
    return int(out.cpu().item())


def w8a8_debug_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().w8a8_debug_wait_timeout(timeout_ns, _stream(stream)), "w8a8_debug_wait_timeout")
