"""Thin Python binding of the C ABI in ``include/moe.h`` (argument marshalling only).

Every step of the layer runs in the CUDA library ``libmoe_b200.so``; PyTorch only
provides device memory and the current stream.  If the library is missing the
calls raise -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
                6: "MOE_ERR_BAD_INDEX", 7: "MOE_ERR_TOO_LARGE",
                8: "MOE_ERR_ROUTER_BOUND"}
EXPORTS = ["moe_workspace_size", "moe_max_tiles", "moe_route", "moe_permute", "moe_forward",
           "moe_get_device_status", "moe_set_gemm_ctas", "moe_set_claim_order", "moe_set_gemm_trace",
           "moe_set_pair_mma", "moe_set_fp8_swap_ab",
           "moe_set_stage_events", "moe_forward_noalloc", "moe_set_wait_limit_us",
           "moe_forward_fp8", "moe_quantize_rows_fp8", "moe_workspace_offsets", "moe_set_router_audit",
           "moe_forward_shared", "moe_workspace_size_shared", "moe_forward_mx", "moe_quantize_rows_mx",
           "moe_set_fused_combine", "moe_set_layer_gemm", "moe_forward_plan", "moe_set_direct_a",
           "moe_set_cert_staging", "moe_noalloc_get_device_status"]
DTYPE_BF16, DTYPE_FP8, DTYPE_MX = 0, 1, 2
NOALLOC_SCRATCH_BYTES = 16 << 20
STAGES = ["route", "permute", "gemm_gate_up", "gemm_down", "combine"]
TILE_ROWS = 128


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("top_k", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        D = ctypes.POINTER(Dims)
        L.moe_workspace_size.argtypes = [D, ctypes.c_int]
        L.moe_workspace_size.restype = SZ
        L.moe_max_tiles.argtypes = [D]
        L.moe_max_tiles.restype = I32
        L.moe_route.argtypes = [D, P, P, P, P, P, P, SZ, P]
        L.moe_route.restype = ctypes.c_int
        L.moe_permute.argtypes = [D, P, P, P, P, P, P, P, SZ, P]
        L.moe_permute.restype = ctypes.c_int
        L.moe_forward.argtypes = [D, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_forward.restype = ctypes.c_int
        L.moe_get_device_status.argtypes = [P, P]
        L.moe_get_device_status.restype = ctypes.c_int
        L.moe_set_gemm_ctas.argtypes = [I32]
        L.moe_set_gemm_ctas.restype = None
        L.moe_set_claim_order.argtypes = [I32]
        L.moe_set_claim_order.restype = None
        L.moe_set_gemm_trace.argtypes = [P, I32]
        L.moe_set_gemm_trace.restype = None
        L.moe_set_pair_mma.argtypes = [I32]
        L.moe_set_pair_mma.restype = None
        L.moe_set_fp8_swap_ab.argtypes = [I32]
        L.moe_set_fp8_swap_ab.restype = None
        L.moe_set_stage_events.argtypes = [P, I32]
        L.moe_set_stage_events.restype = None
        L.moe_forward_fp8.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_forward_fp8.restype = ctypes.c_int
        L.moe_quantize_rows_fp8.argtypes = [I32, I32, P, P, P, P]
        L.moe_quantize_rows_fp8.restype = ctypes.c_int
        L.moe_workspace_offsets.argtypes = [D, ctypes.c_int, P, I32]
        L.moe_workspace_offsets.restype = ctypes.c_int
        L.moe_set_wait_limit_us.argtypes = [I32, I32]
        L.moe_set_wait_limit_us.restype = None
        L.moe_forward_shared.argtypes = [D, P, P, P, P, P, P, I32, P, P, P, P, P, SZ, P]
        L.moe_forward_shared.restype = ctypes.c_int
        L.moe_workspace_size_shared.argtypes = [D, I32]
        L.moe_workspace_size_shared.restype = SZ
        L.moe_forward_plan.argtypes = [D, ctypes.c_int]
        L.moe_forward_plan.restype = I32
        L.moe_set_layer_gemm.argtypes = [I32]
        L.moe_set_layer_gemm.restype = None
        L.moe_set_direct_a.argtypes = [I32]
        L.moe_set_direct_a.restype = None
        L.moe_set_cert_staging.argtypes = [I32, I32, I32]
        L.moe_set_cert_staging.restype = None
        L.moe_set_fused_combine.argtypes = [I32]
        L.moe_set_fused_combine.restype = None
        L.moe_forward_mx.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        L.moe_forward_mx.restype = ctypes.c_int
        L.moe_quantize_rows_mx.argtypes = [I32, I32, P, P, P, P]
        L.moe_quantize_rows_mx.restype = ctypes.c_int
        L.moe_set_router_audit.argtypes = [P, P, ctypes.c_int64]
        L.moe_set_router_audit.restype = None
        L.moe_forward_noalloc.argtypes = [D, P, P, P, P, P, P, P, P]
        L.moe_forward_noalloc.restype = ctypes.c_int
        L.moe_noalloc_get_device_status.argtypes = [P]
        L.moe_noalloc_get_device_status.restype = ctypes.c_int
        _lib = L
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != MOE_OK:
        raise MoEError(code, where)


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


def dims(T, H, I, E, top_k) -> Dims:
    return Dims(int(T), int(H), int(I), int(E), int(top_k))


def moe_workspace_size(T, H, I, E, top_k, dtype: int = DTYPE_BF16) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(dims(T, H, I, E, top_k)), int(dtype)))


def moe_max_tiles(T, H, I, E, top_k) -> int:
    return int(lib().moe_max_tiles(ctypes.byref(dims(T, H, I, E, top_k))))


def workspace(T, H, I, E, top_k, device, dtype: int = DTYPE_BF16) -> torch.Tensor:
    n = moe_workspace_size(T, H, I, E, top_k, dtype)
    if n == 0:
        raise MoEError(1, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_route(x, router_w, bias, top_k: int, topk_idx=None, topk_w=None, ws=None, stream=None,
              I: int = 64):
    """Router + softmax top-k; returns (topk_idx int32 [T,k], topk_w fp32 [T,k])."""
    T, H = x.shape
    E = router_w.shape[1]
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    topk_idx = torch.empty((T, top_k), dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty((T, top_k), dtype=torch.float32, device=dev) if topk_w is None else topk_w
    ws = workspace(T, H, I, E, top_k, dev) if ws is None else ws
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_route(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(topk_idx), _p(topk_w),
                           _p(ws), ws.numel(), _stream(stream, dev)), "moe_route")
    return topk_idx, topk_w


def moe_permute(topk_idx, E: int, ws=None, stream=None, H: int = 64, I: int = 64):
    """Stable grouping of the flat assignments by expert; returns a dict of device tensors
    (offsets, sorted_to_flat, flat_to_sorted, tile_list [max_tiles,3], num_tiles [1])."""
    T, k = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    A = T * k
    nt_max = max(moe_max_tiles(T, H, I, E, k), 1)
    res = {"offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
           "sorted_to_flat": torch.empty(max(A, 1), dtype=torch.int32, device=dev),
           "flat_to_sorted": torch.empty(max(A, 1), dtype=torch.int32, device=dev),
           "tile_list": torch.empty((nt_max, 3), dtype=torch.int32, device=dev),
           "num_tiles": torch.zeros(1, dtype=torch.int32, device=dev)}
    ws = workspace(T, H, I, E, k, dev) if ws is None else ws
    d = dims(T, H, I, E, k)
    _check(lib().moe_permute(ctypes.byref(d), _p(topk_idx), _p(res["offsets"]), _p(res["sorted_to_flat"]),
                             _p(res["flat_to_sorted"]), _p(res["tile_list"]), _p(res["num_tiles"]),
                             _p(ws), ws.numel(), _stream(stream, dev)), "moe_permute")
    return res


def moe_forward(x, router_w, bias, w_gate, w_up, w_down, top_k: int, out=None, ws=None, stream=None):
    """The MoE layer forward; returns out bf16 [T,H]."""
    T, H = x.shape
    E, I, _ = w_gate.shape
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    _need(w_gate, torch.bfloat16, (E, I, H), "w_gate")
    _need(w_up, torch.bfloat16, (E, I, H), "w_up")
    _need(w_down, torch.bfloat16, (E, H, I), "w_down")
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, torch.bfloat16, (T, H), "out")
    ws = workspace(T, H, I, E, top_k, dev) if ws is None else ws
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_forward(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(w_gate), _p(w_up),
                             _p(w_down), _p(out), _p(ws), ws.numel(), _stream(stream, dev)),
           "moe_forward")
    return out


def moe_workspace_size_shared(T, H, I, E, top_k, shared_I) -> int:
    return int(lib().moe_workspace_size_shared(ctypes.byref(dims(T, H, I, E, top_k)), int(shared_I)))


def moe_forward_shared(x, router_w, bias, w_gate, w_up, w_down, shared_gate, shared_up, shared_down, top_k: int,
                       out=None, ws=None, stream=None):
    """The MoE layer forward with a shared expert (shared_gate/up [shared_I, H], shared_down
    [H, shared_I] bf16, shared_I a multiple of I); returns out bf16 [T,H]."""
    T, H = x.shape
    E, I, _ = w_gate.shape
    SI = shared_gate.shape[0]
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    _need(w_gate, torch.bfloat16, (E, I, H), "w_gate")
    _need(w_up, torch.bfloat16, (E, I, H), "w_up")
    _need(w_down, torch.bfloat16, (E, H, I), "w_down")
    _need(shared_gate, torch.bfloat16, (SI, H), "shared_gate")
    _need(shared_up, torch.bfloat16, (SI, H), "shared_up")
    _need(shared_down, torch.bfloat16, (H, SI), "shared_down")
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, torch.bfloat16, (T, H), "out")
    if ws is None:
        n = moe_workspace_size_shared(T, H, I, E, top_k, SI)
        if n == 0:
            raise MoEError(1, "moe_workspace_size_shared")
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_forward_shared(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(w_gate), _p(w_up),
                                    _p(w_down), int(SI), _p(shared_gate), _p(shared_up), _p(shared_down), _p(out),
                                    _p(ws), ws.numel(), _stream(stream, dev)),
           "moe_forward_shared")
    return out


def moe_forward_mx(x, router_w, bias, w_gate_p, w_gate_x, w_up_p, w_up_x, w_down_p, w_down_x, top_k: int,
                   out=None, ws=None, stream=None):
    """The MX layer: e2m1 weights packed two per byte ([E,N,K/2] uint8) with e8m0 scale
    codes per 32 along K ([E,N,K/32] uint8); returns out bf16 [T,H]."""
    T, H = x.shape
    E, I, _ = w_gate_p.shape
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    for t, shp, nm in ((w_gate_p, (E, I, H // 2), "w_gate_p"), (w_up_p, (E, I, H // 2), "w_up_p"),
                       (w_down_p, (E, H, I // 2), "w_down_p"), (w_gate_x, (E, I, H // 32), "w_gate_x"),
                       (w_up_x, (E, I, H // 32), "w_up_x"), (w_down_x, (E, H, I // 32), "w_down_x")):
        _need(t, torch.uint8, shp, nm)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, torch.bfloat16, (T, H), "out")
    ws = workspace(T, H, I, E, top_k, dev, DTYPE_MX) if ws is None else ws
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_forward_mx(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(w_gate_p), _p(w_gate_x),
                                _p(w_up_p), _p(w_up_x), _p(w_down_p), _p(w_down_x), _p(out), _p(ws), ws.numel(),
                                _stream(stream, dev)),
           "moe_forward_mx")
    return out


def moe_quantize_rows_mx(a, stream=None):
    """MX e4m3 codes [R,K] and e8m0 scale codes [R,K/32] of a bf16 [R,K] (K % 32 == 0)."""
    R, K = a.shape
    _need(a, torch.bfloat16, (R, K), "a")
    q = torch.empty((R, K), dtype=torch.uint8, device=a.device)
    x = torch.empty((R, K // 32), dtype=torch.uint8, device=a.device)
    _check(lib().moe_quantize_rows_mx(int(R), int(K), _p(a), _p(q), _p(x), _stream(stream, a.device)),
           "moe_quantize_rows_mx")
    return q, x


def moe_forward_fp8(x, router_w, bias, w_gate_q, w_gate_s, w_up_q, w_up_s, w_down_q, w_down_s,
                    top_k: int, out=None, ws=None, stream=None):
    """The FP8 block-scaled layer; weights are uint8 e4m3 codes with fp32 128x128 block
    scales; returns out bf16 [T,H]."""
    T, H = x.shape
    E, I, _ = w_gate_q.shape
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    for t, shp, nm in ((w_gate_q, (E, I, H), "w_gate_q"), (w_up_q, (E, I, H), "w_up_q"),
                       (w_down_q, (E, H, I), "w_down_q")):
        _need(t, torch.uint8, shp, nm)
    for t, shp, nm in ((w_gate_s, (E, I // 128, H // 128), "w_gate_s"), (w_up_s, (E, I // 128, H // 128), "w_up_s"),
                       (w_down_s, (E, H // 128, I // 128), "w_down_s")):
        _need(t, torch.float32, shp, nm)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, torch.bfloat16, (T, H), "out")
    ws = workspace(T, H, I, E, top_k, dev, DTYPE_FP8) if ws is None else ws
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_forward_fp8(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(w_gate_q), _p(w_gate_s),
                                 _p(w_up_q), _p(w_up_s), _p(w_down_q), _p(w_down_s), _p(out), _p(ws),
                                 ws.numel(), _stream(stream, dev)), "moe_forward_fp8")
    return out


def moe_quantize_rows_fp8(a, q=None, s=None, stream=None):
    """Per-row, per-128-column e4m3 quantisation of a bf16 [R,K] matrix on the GPU:
    returns (codes uint8 [R,K], scales fp32 [R,K/128])."""
    R, K = a.shape
    _need(a, torch.bfloat16, (R, K), "a")
    q = torch.empty((R, K), dtype=torch.uint8, device=a.device) if q is None else q
    s = torch.empty((R, K // 128), dtype=torch.float32, device=a.device) if s is None else s
    _check(lib().moe_quantize_rows_fp8(int(R), int(K), _p(a), _p(q), _p(s), _stream(stream, a.device)),
           "moe_quantize_rows_fp8")
    return q, s


def moe_forward_noalloc(x, router_w, bias, w_gate, w_up, w_down, top_k: int, out=None, stream=None):
    """The layer forward without a workspace argument, for callers that cannot allocate
    device memory: the library's fixed internal scratch is used instead (dims that need
    more than NOALLOC_SCRATCH_BYTES raise MOE_ERR_TOO_LARGE).  Calls that overlap on
    the GPU share that scratch and race; ``out`` is the only buffer this binding may
    allocate, and only when the caller passes none."""
    T, H = x.shape
    E, I, _ = w_gate.shape
    dev = x.device
    _need(x, torch.bfloat16, (T, H), "x")
    _need(router_w, torch.bfloat16, (H, E), "router_w")
    if bias is not None:
        _need(bias, torch.float32, (E,), "router_bias")
    _need(w_gate, torch.bfloat16, (E, I, H), "w_gate")
    _need(w_up, torch.bfloat16, (E, I, H), "w_up")
    _need(w_down, torch.bfloat16, (E, H, I), "w_down")
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev) if out is None else out
    _need(out, torch.bfloat16, (T, H), "out")
    d = dims(T, H, I, E, top_k)
    _check(lib().moe_forward_noalloc(ctypes.byref(d), _p(x), _p(router_w), _p(bias), _p(w_gate),
                                     _p(w_up), _p(w_down), _p(out), _stream(stream, dev)),
           "moe_forward_noalloc")
    return out


def forward_routing(ws, T, H, I, E, top_k, dtype: int = DTYPE_BF16) -> dict:
    """Views into the workspace of the routing the last forward on it computed
    (topk_idx, topk_w, offsets, sorted_to_flat, flat_to_sorted, tile_list, num_tiles,
    and the router's fp32 logits [T, E]: every entry for T <= 32, at least the chosen
    experts' entries above)."""
    offs = (ctypes.c_size_t * 8)()
    _check(lib().moe_workspace_offsets(ctypes.byref(dims(T, H, I, E, top_k)), int(dtype), offs, 8),
           "moe_workspace_offsets")
    A = T * top_k
    nt = moe_max_tiles(T, H, I, E, top_k)

    def view(i, n, dt):
        nbytes = n * torch.tensor([], dtype=dt).element_size()
        return ws[offs[i]:offs[i] + nbytes].view(dt)
    return {"topk_idx": view(0, A, torch.int32).view(T, top_k), "topk_w": view(1, A, torch.float32).view(T, top_k),
            "offsets": view(2, E + 1, torch.int32), "sorted_to_flat": view(3, A, torch.int32),
            "flat_to_sorted": view(4, A, torch.int32), "tile_list": view(5, 3 * nt, torch.int32).view(nt, 3),
            "num_tiles": view(6, 1, torch.int32), "logits": view(7, T * E, torch.float32).view(T, E)}


def moe_get_device_status(ws, stream=None) -> int:
    """Synchronise the stream and return (and clear) the workspace's device status word."""
    return int(lib().moe_get_device_status(_p(ws), _stream(stream, ws.device)))


def set_gemm_ctas(n: int):
    lib().moe_set_gemm_ctas(int(n))


def set_wait_limit_us(us: int, stall_test: bool = False):
    """Limit of each GEMM pipeline wait in microseconds (<= 0 restores the 2 s default);
    ``stall_test`` makes every GEMM CTA wait on a barrier nothing signals (tests only)."""
    lib().moe_set_wait_limit_us(int(us), 1 if stall_test else 0)


CLAIM_MODES = {"queue": 0, "queue_desc": 1, "static_items": 2, "static_experts": 3}


def set_claim_order(reverse):
    """False/True: the GEMMs' atomic work queue ascending/descending; or one of the
    CLAIM_MODES names ("static_items", "static_experts" replace the queue)."""
    mode = CLAIM_MODES[reverse] if isinstance(reverse, str) else (1 if reverse else 0)
    lib().moe_set_claim_order(mode)


def set_pair_mma(mode: str):
    """"auto" (default), "always" or "never": the bf16 forward's pair-of-CTA GEMMs."""
    lib().moe_set_pair_mma({"auto": 0, "always": 1, "never": 2}[mode])


PLAN_SMALL_ROUTER, PLAN_PAIR_TILES, PLAN_FUSED_COMBINE, PLAN_LAYER_GEMM, PLAN_DIRECT_A = 1, 2, 4, 8, 16


def forward_plan(T, H, I, E, top_k, dtype: int = DTYPE_BF16) -> int:
    """The kernels a forward would launch now (PLAN_* bits), -1 for invalid dims."""
    return int(lib().moe_forward_plan(ctypes.byref(dims(T, H, I, E, top_k)), int(dtype)))


def set_layer_gemm(mode: str):
    """"auto" (default), "always" or "never": both bf16 expert GEMMs in one persistent launch."""
    lib().moe_set_layer_gemm({"auto": 0, "always": 1, "never": 2}[mode])


def set_direct_a(mode: str):
    """"auto" (default), "always" or "never": bf16 gate/up A rows gathered straight from x
    by the GEMM (never: from a sorted copy of x made by a gather kernel first)."""
    lib().moe_set_direct_a({"auto": 0, "always": 1, "never": 2}[mode])


def noalloc_device_status(stream=None) -> int:
    """moe_noalloc_get_device_status: synchronises the stream, then reads and clears the
    device status word of moe_forward_noalloc's scratch on the current device."""
    return lib().moe_noalloc_get_device_status(_stream(stream, torch.device("cuda", torch.cuda.current_device())))


def set_cert_staging(max_stages: int = 0, min_stages: int = 0, max_boxes: int = 0):
    """The certified router's chain staging: chunks in flight (cap), the count the
    widest chunk must leave, and the chunk width cap in 64-value boxes (1, 2, 4, 8);
    0 keeps each default (3, 2, 8).  Routing is the same either way."""
    lib().moe_set_cert_staging(max_stages, min_stages, max_boxes)


def set_fused_combine(mode: str):
    """"auto" (default), "always" or "never": the bf16 combine inside the down GEMM."""
    lib().moe_set_fused_combine({"auto": 0, "always": 1, "never": 2}[mode])


def set_fp8_swap_ab(mode: str):
    """"auto" (default), "always" or "never": the fp8 gate/up GEMM with swapped MMA operands."""
    lib().moe_set_fp8_swap_ab({"auto": 0, "always": 1, "never": 2}[mode])


def set_gemm_trace(buf):
    """Record per GEMM CTA its start/end %globaltimer into `buf` (a CUDA int64 tensor of
    4 * ctas entries, see moe_set_gemm_trace), or turn the trace off with None."""
    if buf is None:
        lib().moe_set_gemm_trace(None, 0)
    else:
        lib().moe_set_gemm_trace(ctypes.c_void_p(buf.data_ptr()), buf.numel() // 4)


def set_stage_events(events):
    """Record these 6 torch.cuda.Events at the stage boundaries of every later
    moe_forward (None turns it off; a None entry is skipped).  Each event must have
    been recorded once so that its CUDA handle exists."""
    if events is None:
        lib().moe_set_stage_events(None, 0)
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event if e is not None else None)
                                            for e in events])
    set_stage_events._keep = arr
    lib().moe_set_stage_events(arr, len(events))


def set_router_audit(logits, bounds):
    """Every later certified router run (T > 32) writes each (t, e)'s tensor-core logit
    (+bias) into `logits` and its error bound into `bounds` (CUDA fp32 tensors of
    T*E values or more); None turns it off."""
    if logits is None:
        lib().moe_set_router_audit(None, None, 0)
        return
    if logits.dtype != torch.float32 or bounds.dtype != torch.float32 or not (logits.is_cuda and bounds.is_cuda):
        raise ValueError("router audit buffers: CUDA float32 tensors")
    lib().moe_set_router_audit(_p(logits), _p(bounds), min(logits.numel(), bounds.numel()))
