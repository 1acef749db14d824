"""ctypes binding of libdsmoe.so with the C ABI's names.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Torch tensors are passed by data pointer (device tensors for
dsmoe_forward, host tensors for dsmoe_forward_host); streams are torch CUDA
streams or raw cudaStream_t integers. Importing this module raises if the
library has not been built; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
# DSMOE_LIBRARY selects another build of the library, e.g. the profiling build with the
# grouped GEMM's role cycle counters (build.py --role-cycles)
LIB_PATH = os.environ.get("DSMOE_LIBRARY") or os.path.join(_HERE, "libdsmoe.so")

DSMOE_OK, DSMOE_ERR_INVALID_ARG, DSMOE_ERR_UNSUPPORTED, DSMOE_ERR_WORKSPACE, DSMOE_ERR_CUDA, \
    DSMOE_ERR_DEVICE_TIMEOUT = range(6)
DSMOE_SCORE_SOFTMAX, DSMOE_SCORE_SIGMOID, DSMOE_SCORE_SQRT_SOFTPLUS, DSMOE_ROUTE_HASH = range(4)
DSMOE_BIAS_NONE, DSMOE_BIAS_SELECT_ONLY, DSMOE_BIAS_IN_LOGITS = range(3)
DSMOE_GEMM_PAIR, DSMOE_GEMM_SINGLE = range(2)
DSMOE_RANGE_PARTIAL, DSMOE_RANGE_ADD_SHARED = 1, 2

ABI_FUNCTIONS = (
    "dsmoe_abi_version", "dsmoe_status_string", "dsmoe_last_error", "dsmoe_check_config",
    "dsmoe_workspace_bytes", "dsmoe_create", "dsmoe_destroy", "dsmoe_forward", "dsmoe_forward_host",
    "dsmoe_balance_stats", "dsmoe_get_status", "dsmoe_set_wait_limit", "dsmoe_set_timing",
    "dsmoe_stage_times", "dsmoe_stage_name", "dsmoe_launch_count", "dsmoe_workspace_tensor",
    "dsmoe_balance_losses", "dsmoe_sequence_balance", "dsmoe_bias_update",
    "dsmoe_route_noalloc", "dsmoe_set_gemm_kernel", "dsmoe_get_gemm_kernel",
    "dsmoe_set_selection", "dsmoe_get_selection", "dsmoe_set_expert_range", "dsmoe_get_expert_range",
    "dsmoe_round_bf16", "dsmoe_backward_gates", "dsmoe_backward_router", "dsmoe_ep_route", "dsmoe_ep_experts",
    "dsmoe_ep_combine", "dsmoe_forward_host_async", "dsmoe_host_join", "dsmoe_host_sync", "dsmoe_set_training",
    "dsmoe_backward_experts", "dsmoe_backward_weights", "dsmoe_gemm_role_cycles",
)
ROLE_CTAS, ROLE_SLOTS = 160, 9
ROLE_KINDS = ("gemm_down", "gemm_gate_up", "shared_down", "shared_gate_up", "weight_grad")
ROLE_SLOT_NAMES = ("cycles", "nanoseconds", "producer_wait_stage", "mma_wait_stage", "mma_wait_acc", "mma_loop",
                   "epi_wait_acc", "epi_loop", "tiles")


class DsmoeCfg(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_routed", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32),
                ("score", ctypes.c_int32), ("bias_mode", ctypes.c_int32), ("renormalize", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("hash_mult", ctypes.c_uint32), ("hash_mod", ctypes.c_uint32)]


class DsmoeError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {status_string(status)} ({status}): {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python mixture_experts_layer_score_b200/build.py` (there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64, f32p, i32p = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                     ctypes.c_void_p, ctypes.c_void_p)
    cfgp = ctypes.POINTER(DsmoeCfg)
    sig = {
        "dsmoe_abi_version": (i32, []),
        "dsmoe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "dsmoe_last_error": (ctypes.c_char_p, []),
        "dsmoe_check_config": (ctypes.c_int, [cfgp]),
        "dsmoe_workspace_bytes": (ctypes.c_int, [cfgp, ctypes.POINTER(ctypes.c_size_t)]),
        "dsmoe_create": (ctypes.c_int, [cfgp, i32, ctypes.POINTER(vp)]),
        "dsmoe_destroy": (None, [vp]),
        "dsmoe_forward": (ctypes.c_int, [vp, i32] + [vp] * 18 + [vp]),
        "dsmoe_forward_host": (ctypes.c_int, [vp, i32] + [vp] * 16 + [vp]),
        "dsmoe_forward_host_async": (ctypes.c_int, [vp, i32] + [vp] * 16 + [vp]),
        "dsmoe_host_join": (ctypes.c_int, [vp, vp]),
        "dsmoe_host_sync": (ctypes.c_int, [vp]),
        "dsmoe_set_training": (ctypes.c_int, [vp, i32]),
        "dsmoe_backward_experts": (ctypes.c_int, [vp, i32] + [vp] * 10 + [vp]),
        "dsmoe_backward_weights": (ctypes.c_int, [vp, i32] + [vp] * 9 + [vp]),
        "dsmoe_balance_stats": (ctypes.c_int, [vp, i64, vp, vp, vp, vp, vp]),
        "dsmoe_get_status": (ctypes.c_int, [vp]),
        "dsmoe_set_wait_limit": (ctypes.c_int, [vp, u64]),
        "dsmoe_set_timing": (ctypes.c_int, [vp, i32]),
        "dsmoe_set_gemm_kernel": (ctypes.c_int, [vp, i32]),
        "dsmoe_get_gemm_kernel": (i32, [vp]),
        "dsmoe_set_selection": (ctypes.c_int, [vp, i32, i32]),
        "dsmoe_get_selection": (ctypes.c_int, [vp, ctypes.POINTER(i32), ctypes.POINTER(i32)]),
        "dsmoe_stage_times": (ctypes.c_int, [vp, ctypes.POINTER(ctypes.c_float), i32, ctypes.POINTER(i32)]),
        "dsmoe_stage_name": (ctypes.c_char_p, [i32]),
        "dsmoe_launch_count": (ctypes.c_int, [vp, ctypes.POINTER(i64)]),
        "dsmoe_gemm_role_cycles": (ctypes.c_int, [vp, i32]),
        "dsmoe_balance_losses": (ctypes.c_int, [vp, vp, vp, i32, vp, ctypes.c_float, ctypes.c_float, vp, vp, vp,
                                                vp]),
        "dsmoe_sequence_balance": (ctypes.c_int, [vp, i32, i32, vp, vp, ctypes.c_float, vp, vp, vp, vp]),
        "dsmoe_bias_update": (ctypes.c_int, [vp, i64, vp, ctypes.c_float, vp, vp]),
        "dsmoe_workspace_tensor": (ctypes.c_int, [vp, ctypes.c_char_p, ctypes.POINTER(vp),
                                                  ctypes.POINTER(i64), ctypes.POINTER(i64)]),
        "dsmoe_route_noalloc": (ctypes.c_int, [cfgp, i32] + [vp] * 8 + [vp]),
        "dsmoe_set_expert_range": (ctypes.c_int, [vp, i32, i32, i32]),
        "dsmoe_get_expert_range": (ctypes.c_int, [vp, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                                  ctypes.POINTER(i32)]),
        "dsmoe_round_bf16": (ctypes.c_int, [vp, i64, vp, vp, vp]),
        "dsmoe_backward_gates": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp]),
        "dsmoe_ep_route": (ctypes.c_int, [vp, i32] + [vp] * 11 + [i32, vp, vp]),
        "dsmoe_ep_experts": (ctypes.c_int, [vp, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp, vp]),
        "dsmoe_ep_combine": (ctypes.c_int, [vp, i32] + [vp] * 7 + [vp]),
        "dsmoe_backward_router": (ctypes.c_int, [vp, i32, vp, vp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp, vp,
                                                 vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.dsmoe_status_string(int(status)).decode()


def dsmoe_status_string(status: int) -> str:
    return status_string(status)


def dsmoe_last_error() -> str:
    return _lib.dsmoe_last_error().decode()


def _check(status: int, where: str):
    if status != DSMOE_OK:
        raise DsmoeError(status, where, dsmoe_last_error())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_cfg(d_model: int, n_routed: int, top_k: int, d_ff: int, n_shared: int = 0, d_ff_shared: int = 0,
             score: int = DSMOE_SCORE_SOFTMAX, bias_mode: int = DSMOE_BIAS_NONE, renormalize: bool = False,
             max_tokens: int = 1, hash_mult: int = 2654435761, hash_mod: int = 0) -> DsmoeCfg:
    return DsmoeCfg(d_model, n_routed, top_k, d_ff, n_shared, d_ff_shared, score, bias_mode, int(renormalize),
                    max_tokens, hash_mult, hash_mod)


def cfg_from(obj, max_tokens: int) -> DsmoeCfg:
    """dsmoe_cfg from any object with the layer's field names (d_model, n_routed, top_k, ...)."""
    return make_cfg(obj.d_model, obj.n_routed, obj.top_k, obj.d_ff, obj.n_shared, obj.d_ff_shared, obj.score,
                    obj.bias_mode, obj.renormalize, max_tokens, getattr(obj, "hash_mult", 2654435761), 0)


def dsmoe_abi_version() -> int:
    return _lib.dsmoe_abi_version()


def dsmoe_check_config(cfg: DsmoeCfg) -> int:
    return _lib.dsmoe_check_config(ctypes.byref(cfg))


def dsmoe_workspace_bytes(cfg: DsmoeCfg) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.dsmoe_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "dsmoe_workspace_bytes")
    return n.value


def dsmoe_create(cfg: DsmoeCfg, device: int = 0) -> int:
    h = ctypes.c_void_p()
    _check(_lib.dsmoe_create(ctypes.byref(cfg), int(device), ctypes.byref(h)), "dsmoe_create")
    return h.value


def dsmoe_destroy(handle: int) -> None:
    _lib.dsmoe_destroy(handle)


def dsmoe_forward(handle, T, x, token_ids, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down,
                  h, topk_idx, gates, counts, f, P, P_sum=None, scores_dbg=None, stream=None) -> None:
    st = _lib.dsmoe_forward(handle, int(T), *[_ptr(t) for t in (
        x, token_ids, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, h, topk_idx, gates, counts, f,
        P, P_sum, scores_dbg)], _stream(stream))
    _check(st, "dsmoe_forward")


def dsmoe_forward_host(handle, T, x_host, token_ids_host, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up,
                       Ws_down, h_host, topk_idx_host, gates_host, counts_host, f_host, P_host,
                       stream=None) -> None:
    st = _lib.dsmoe_forward_host(handle, int(T), *[_ptr(t) for t in (
        x_host, token_ids_host, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, h_host,
        topk_idx_host, gates_host, counts_host, f_host, P_host)], _stream(stream))
    _check(st, "dsmoe_forward_host")


def dsmoe_forward_host_async(handle, T, x_host, token_ids_host, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up,
                             Ws_down, h_host, topk_idx_host, gates_host, counts_host, f_host, P_host,
                             stream=None) -> None:
    st = _lib.dsmoe_forward_host_async(handle, int(T), *[_ptr(t) for t in (
        x_host, token_ids_host, W_router, b, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, h_host,
        topk_idx_host, gates_host, counts_host, f_host, P_host)], _stream(stream))
    _check(st, "dsmoe_forward_host_async")


def dsmoe_host_join(handle, stream=None) -> None:
    _check(_lib.dsmoe_host_join(handle, _stream(stream)), "dsmoe_host_join")


def dsmoe_host_sync(handle) -> None:
    _check(_lib.dsmoe_host_sync(handle), "dsmoe_host_sync")


def dsmoe_balance_stats(handle, T_total, counts, P_sum, f, P, stream=None) -> None:
    _check(_lib.dsmoe_balance_stats(handle, int(T_total), _ptr(counts), _ptr(P_sum), _ptr(f), _ptr(P),
                                    _stream(stream)), "dsmoe_balance_stats")


def dsmoe_get_status(handle) -> int:
    return _lib.dsmoe_get_status(handle)


def dsmoe_set_wait_limit(handle, ns: int) -> None:
    _check(_lib.dsmoe_set_wait_limit(handle, int(ns)), "dsmoe_set_wait_limit")


def dsmoe_set_gemm_kernel(handle, kind: int) -> None:
    _check(_lib.dsmoe_set_gemm_kernel(handle, int(kind)), "dsmoe_set_gemm_kernel")


def dsmoe_get_gemm_kernel(handle) -> int:
    return int(_lib.dsmoe_get_gemm_kernel(handle))


def dsmoe_set_selection(handle, mask_top: int, k_active: int) -> None:
    _check(_lib.dsmoe_set_selection(handle, int(mask_top), int(k_active)), "dsmoe_set_selection")


def dsmoe_get_selection(handle):
    m, k = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.dsmoe_get_selection(handle, ctypes.byref(m), ctypes.byref(k)), "dsmoe_get_selection")
    return m.value, k.value


def dsmoe_set_expert_range(handle, e_begin: int, e_end: int, flags: int) -> None:
    _check(_lib.dsmoe_set_expert_range(handle, int(e_begin), int(e_end), int(flags)), "dsmoe_set_expert_range")


def dsmoe_get_expert_range(handle):
    b, e, f = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(_lib.dsmoe_get_expert_range(handle, ctypes.byref(b), ctypes.byref(e), ctypes.byref(f)),
           "dsmoe_get_expert_range")
    return b.value, e.value, f.value


def dsmoe_round_bf16(handle, n: int, src, dst, stream=None) -> None:
    _check(_lib.dsmoe_round_bf16(handle, int(n), _ptr(src), _ptr(dst), _stream(stream)), "dsmoe_round_bf16")


def dsmoe_ep_route(handle, T, x, token_ids, W_router, b, topk_idx, gates, counts, f, P, P_sum, scores_dbg, world,
                   send_rows, stream=None) -> None:
    _check(_lib.dsmoe_ep_route(handle, int(T), *[_ptr(t) for t in (
        x, token_ids, W_router, b, topk_idx, gates, counts, f, P, P_sum, scores_dbg)], int(world), _ptr(send_rows),
        _stream(stream)), "dsmoe_ep_route")


def dsmoe_ep_experts(handle, n_src, e_begin, e_end, recv_counts, n_rows, rows, W_gate, W_up, W_down, Y,
                     stream=None) -> None:
    _check(_lib.dsmoe_ep_experts(handle, int(n_src), int(e_begin), int(e_end), _ptr(recv_counts), int(n_rows),
                                 *[_ptr(t) for t in (rows, W_gate, W_up, W_down, Y)], _stream(stream)),
           "dsmoe_ep_experts")


def dsmoe_ep_combine(handle, T, x, Ws_gate, Ws_up, Ws_down, gates, Y, h, stream=None) -> None:
    _check(_lib.dsmoe_ep_combine(handle, int(T), *[_ptr(t) for t in (x, Ws_gate, Ws_up, Ws_down, gates, Y, h)],
                                 _stream(stream)), "dsmoe_ep_combine")


def dsmoe_set_training(handle, enable: bool) -> None:
    _check(_lib.dsmoe_set_training(handle, int(bool(enable))), "dsmoe_set_training")


def dsmoe_backward_experts(handle, T, dh, dY, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, dx_add, dx,
                           stream=None) -> None:
    _check(_lib.dsmoe_backward_experts(handle, int(T), *[_ptr(t) for t in (
        dh, dY, W_gate, W_up, W_down, Ws_gate, Ws_up, Ws_down, dx_add, dx)], _stream(stream)),
        "dsmoe_backward_experts")


def dsmoe_backward_weights(handle, T, dh, dY, x, dW_gate, dW_up, dW_down, dWs_gate, dWs_up, dWs_down,
                           stream=None) -> None:
    _check(_lib.dsmoe_backward_weights(handle, int(T), *[_ptr(t) for t in (
        dh, dY, x, dW_gate, dW_up, dW_down, dWs_gate, dWs_up, dWs_down)], _stream(stream)),
        "dsmoe_backward_weights")


def dsmoe_backward_gates(handle, T, dh, gates, dg, dY, stream=None) -> None:
    _check(_lib.dsmoe_backward_gates(handle, int(T), _ptr(dh), _ptr(gates), _ptr(dg), _ptr(dY), _stream(stream)),
           "dsmoe_backward_gates")


def dsmoe_backward_router(handle, T, x, W_router, topk_idx, gates, scores, dg, f, alpha, dlogits, dx, dW_router,
                          stream=None) -> None:
    _check(_lib.dsmoe_backward_router(handle, int(T), *[_ptr(t) for t in (
        x, W_router, topk_idx, gates, scores, dg, f)], float(alpha), _ptr(dlogits), _ptr(dx), _ptr(dW_router),
        _stream(stream)), "dsmoe_backward_router")


def dsmoe_set_timing(handle, enable: bool) -> None:
    _check(_lib.dsmoe_set_timing(handle, int(bool(enable))), "dsmoe_set_timing")


def dsmoe_stage_name(i: int) -> Optional[str]:
    r = _lib.dsmoe_stage_name(int(i))
    return None if r is None else r.decode()


def stage_names() -> Sequence[str]:
    out, i = [], 0
    while (n := dsmoe_stage_name(i)) is not None:
        out.append(n)
        i += 1
    return out


def dsmoe_stage_times(handle) -> Dict[str, float]:
    names = stage_names()
    buf = (ctypes.c_float * len(names))()
    n = ctypes.c_int32(0)
    _check(_lib.dsmoe_stage_times(handle, buf, len(names), ctypes.byref(n)), "dsmoe_stage_times")
    return {names[i]: float(buf[i]) for i in range(n.value)}


def dsmoe_gemm_role_cycles():
    """The one-CTA grouped GEMM's role counters since the last call, as a uint64 array
    [launch kind, CTA, slot] (kinds ROLE_KINDS, slots ROLE_SLOT_NAMES); a profiling build
    of the library is required (DsmoeError with DSMOE_ERR_UNSUPPORTED otherwise)."""
    import numpy as np
    buf = np.zeros((len(ROLE_KINDS), ROLE_CTAS, ROLE_SLOTS), dtype=np.uint64)
    _check(_lib.dsmoe_gemm_role_cycles(buf.ctypes.data, buf.size), "dsmoe_gemm_role_cycles")
    return buf


def dsmoe_launch_count(handle) -> int:
    n = ctypes.c_int64(0)
    _check(_lib.dsmoe_launch_count(handle, ctypes.byref(n)), "dsmoe_launch_count")
    return n.value


def dsmoe_route_noalloc(cfg: DsmoeCfg, T, x, W_router, b, topk_idx, gates, counts, f, P, stream=None) -> None:
    """The routing stage without a handle or any allocation (scratch is a fixed array in
    the library); for callers that cannot allocate device memory when they route."""
    st = _lib.dsmoe_route_noalloc(ctypes.byref(cfg), int(T), *[_ptr(t) for t in (
        x, W_router, b, topk_idx, gates, counts, f, P)], _stream(stream))
    _check(st, "dsmoe_route_noalloc")


def dsmoe_balance_losses(handle, f, P, n_groups, group_of, alpha1, alpha2, f_dev, P_dev, losses, stream=None):
    _check(_lib.dsmoe_balance_losses(handle, _ptr(f), _ptr(P), int(n_groups), _ptr(group_of), float(alpha1),
                                     float(alpha2), _ptr(f_dev), _ptr(P_dev), _ptr(losses), _stream(stream)),
           "dsmoe_balance_losses")


def dsmoe_sequence_balance(handle, T, seq_len, topk_idx, scores, beta, f_seq, p_seq, loss, stream=None):
    _check(_lib.dsmoe_sequence_balance(handle, int(T), int(seq_len), _ptr(topk_idx), _ptr(scores), float(beta),
                                       _ptr(f_seq), _ptr(p_seq), _ptr(loss), _stream(stream)),
           "dsmoe_sequence_balance")


def dsmoe_bias_update(handle, T, counts, alpha, b, stream=None):
    _check(_lib.dsmoe_bias_update(handle, int(T), _ptr(counts), float(alpha), _ptr(b), _stream(stream)),
           "dsmoe_bias_update")


_WS_DTYPES = {"logits": "float32", "offsets": "int32", "slot_of": "int32", "Xp": "bfloat16",
              "A1": "bfloat16", "A1s": "bfloat16", "Y": "bfloat16", "Hs": "float32", "AB": "bfloat16",
              "ABs": "bfloat16", "dAB": "bfloat16", "dABs": "bfloat16", "dXp": "bfloat16", "dXs": "float32"}


def dsmoe_workspace_tensor(handle, name: str):
    """(device address, rows, cols) of an intermediate workspace buffer."""
    p, r, c = ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_int64()
    _check(_lib.dsmoe_workspace_tensor(handle, name.encode(), ctypes.byref(p), ctypes.byref(r), ctypes.byref(c)),
           "dsmoe_workspace_tensor")
    return p.value, r.value, c.value


def workspace_view(handle, name: str, device: int = 0):
    """A torch tensor aliasing a workspace buffer (copy it before the next forward)."""
    import torch
    ptr, rows, cols = dsmoe_workspace_tensor(handle, name)
    dt = getattr(torch, _WS_DTYPES[name])
    n = rows * cols
    esz = torch.empty((), dtype=dt).element_size()

    class _Buf:  # minimal __cuda_array_interface__ exporter over the raw device pointer
        pass

    b = _Buf()
    typestr = {"float32": "<f4", "int32": "<i4", "bfloat16": "<i2"}[_WS_DTYPES[name]]
    b.__cuda_array_interface__ = dict(shape=(n,), typestr=typestr, data=(ptr, False), version=3)
    with torch.cuda.device(device):
        t = torch.as_tensor(b, device=f"cuda:{device}")
    if _WS_DTYPES[name] == "bfloat16":
        t = t.view(torch.bfloat16)
    assert t.element_size() == esz
    return t.view(rows, cols)


class DSMoE:
    """A handle plus the weight tensors of one layer; forward() allocates the outputs with
    torch (device memory only) and calls dsmoe_forward."""

    def __init__(self, cfg: DsmoeCfg, weights: Dict, device: int = 0):
        self.cfg = cfg
        self.device = device
        self.w = weights
        self.handle = dsmoe_create(cfg, device)
        self.mask_top, self.k_active = 0, cfg.top_k
        self.range_flags = DSMOE_RANGE_ADD_SHARED

    def set_selection(self, mask_top: int = 0, k_active: Optional[int] = None):
        """Selection variant for later forwards (see dsmoe_set_selection)."""
        k = self.cfg.top_k if k_active is None else int(k_active)
        dsmoe_set_selection(self.handle, mask_top, k)
        self.mask_top, self.k_active = int(mask_top), k

    def set_expert_range(self, e_begin: int, e_end: int, partial: bool = True, add_shared: bool = False):
        """Apply only routed experts [e_begin, e_end) in later forwards (see
        dsmoe_set_expert_range); the weights given at construction must then hold those
        experts only. With partial, forward() returns h as fp32 partial sums."""
        flags = (DSMOE_RANGE_PARTIAL if partial else 0) | (DSMOE_RANGE_ADD_SHARED if add_shared else 0)
        dsmoe_set_expert_range(self.handle, e_begin, e_end, flags)
        self.range_flags = flags

    def close(self):
        if self.handle:
            dsmoe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def alloc_outputs(self, T: int, with_scores: bool = False):
        import torch
        dev = torch.device("cuda", self.device)
        c = self.cfg
        h_dtype = torch.float32 if self.range_flags & DSMOE_RANGE_PARTIAL else torch.bfloat16
        out = dict(h=torch.empty((T, c.d_model), dtype=h_dtype, device=dev),
                   topk_idx=torch.empty((T, self.k_active), dtype=torch.int32, device=dev),
                   gates=torch.empty((T, self.k_active), dtype=torch.float32, device=dev),
                   counts=torch.empty((c.n_routed,), dtype=torch.int32, device=dev),
                   f=torch.empty((c.n_routed,), dtype=torch.float32, device=dev),
                   P=torch.empty((c.n_routed,), dtype=torch.float32, device=dev),
                   P_sum=torch.empty((c.n_routed,), dtype=torch.float32, device=dev))
        out["scores"] = (torch.empty((T, c.n_routed), dtype=torch.float32, device=dev)
                         if with_scores and c.score != DSMOE_ROUTE_HASH else None)
        return out

    def forward(self, x, token_ids=None, out=None, with_scores: bool = False, stream=None):
        T = x.shape[0]
        o = self.alloc_outputs(T, with_scores) if out is None else out
        w = self.w
        dsmoe_forward(self.handle, T, x, token_ids, w.get("W_router"), w.get("b"), w["W_gate"], w["W_up"],
                      w["W_down"], w.get("Ws_gate"), w.get("Ws_up"), w.get("Ws_down"), o["h"], o["topk_idx"],
                      o["gates"], o["counts"], o["f"], o["P"], o["P_sum"], o["scores"], stream)
        return o
