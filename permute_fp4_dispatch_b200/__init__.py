"""B200 (sm_100a) MoE token-routing hot path: Python binding of libmoe_route.so.

Thin ctypes marshalling over the C ABI declared in include/moe_route.h; the
functions keep the C names.  Every argument that is a buffer accepts a torch
tensor (its data pointer is passed) or a raw integer address; ``stream``
defaults to torch's current CUDA stream.  Every step runs in the library's
CUDA kernels: there is no Python or CPU fallback, and a missing library
raises at first use.

Pipeline (single GPU):
    moe_mask_padding -> moe_create_indices -> moe_dispatch_mxfp4
    -> [moe_quantize_activations_nvfp4] -> moe_grouped_gemv_nvfp4 -> moe_combine
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "MoeError", "library", "library_path",
    "MOE_W4A16", "MOE_W4A4", "MOE_EPI_NONE", "MOE_EPI_IDENTITY", "MOE_EPI_SCALE",
    "MOE_DEVERR_WAIT_TIMEOUT", "MOE_DEVERR_RECV_OVERFLOW", "MOE_DEVERR_ACT_RANGE",
    "MOE_DEVERR_LIMIT",
    "moe_mask_padding", "moe_create_indices_workspace_bytes", "moe_create_indices",
    "moe_create_indices_static", "MOE_CREATE_INDICES_STATIC_SCRATCH",
    "moe_mask_and_create_indices",
    "moe_mxfp4_row_stride", "moe_dispatch_mxfp4", "moe_quantize_activations_nvfp4",
    "moe_dispatch_mxfp4_quantize_nvfp4",
    "MOE_GEMV_DECODE", "MOE_GEMV_TENSOR_MEMORY", "MOE_GEMV_BLOCK_SCALED",
    "moe_quantize_weights_nvfp4", "moe_grouped_gemv_workspace_bytes", "moe_grouped_gemv_nvfp4",
    "moe_grouped_gemv_plan",
    "moe_combine",
    "moe_status_string", "moe_get_device_error", "moe_version",
]

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_ARCH, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
MOE_W4A16, MOE_W4A4 = 0, 1
MOE_GEMV_DECODE, MOE_GEMV_TENSOR_MEMORY, MOE_GEMV_BLOCK_SCALED = 0, 1, 2
MOE_EPI_NONE, MOE_EPI_IDENTITY, MOE_EPI_SCALE = 0, 1, 2
MOE_DEVERR_WAIT_TIMEOUT, MOE_DEVERR_RECV_OVERFLOW, MOE_DEVERR_ACT_RANGE = 0x1, 0x2, 0x4
MOE_DEVERR_LIMIT = 0x8

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libmoe_route.so")
_lib = None
_lock = threading.Lock()


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")


_P, _I32, _I64, _F32, _SZ = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
_SIGS = {
    "moe_mask_padding": ([_P, _I32, _I32, _P, _I32, _P], _I32),
    "moe_create_indices_workspace_bytes": ([_I64, _I32], _SZ),
    "moe_create_indices": ([_P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "moe_create_indices_static": ([_P, _I64, _I32, _P, _P, _P, _P, _P, _P, _P], _I32),
    "moe_mask_and_create_indices": ([_P, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P,
                                     _P, _SZ, _P], _I32),
    "moe_mxfp4_row_stride": ([_I32], _SZ),
    "moe_dispatch_mxfp4": ([_P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _I64, _P, _P], _I32),
    "moe_quantize_activations_nvfp4": ([_P, _I32, _I32, _F32, _P, _P, _P], _I32),
    "moe_dispatch_mxfp4_quantize_nvfp4": ([_P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _I64,
                                           _P, _F32, _P, _P, _P], _I32),
    "moe_quantize_weights_nvfp4": ([_P, _I32, _I32, _I32, _P, _P, _P, _P], _I32),
    "moe_grouped_gemv_workspace_bytes": ([_I32, _I32, _I32, _I32], _SZ),
    "moe_grouped_gemv_nvfp4": ([_I32, _P, _P, _F32, _P, _I32, _I32, _P, _P, _P, _I32, _I32, _I32,
                                _P, _P, _P, _P, _P, _P, _SZ, _P], _I32),
    "moe_grouped_gemv_plan": ([_I32, _I32, _I32, _I32, _I32, _I32, _I32, _P, _P], _I32),
    "moe_combine": ([_P, _P, _P, _I32, _I32, _I32, _I32, _I32, _F32, _P, _P], _I32),
    "moe_status_string": ([_I32], ctypes.c_char_p),
    "moe_get_device_error": ([_P, _I32], _I32),
    "moe_version": ([], _I32),
}


def library():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(library_path):
                    raise ImportError(
                        f"{library_path} is missing: build it with "
                        "`python -m permute_fp4_dispatch_b200.build` (nvcc, sm_100a)")
                lib = ctypes.CDLL(library_path)
                for name, (args, res) in _SIGS.items():
                    f = getattr(lib, name)
                    f.argtypes = args
                    f.restype = res
                _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    return x.data_ptr() or None


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def moe_status_string(status: int) -> str:
    return library().moe_status_string(status).decode()


def moe_version() -> int:
    return library().moe_version()


def moe_mask_padding(routing_map, N: int, top_k: int, real_token_count, tp_rank: int = 0,
                     stream=None):
    _check(library().moe_mask_padding(_ptr(routing_map), N, top_k, _ptr(real_token_count),
                                      tp_rank, _stream(stream)), "moe_mask_padding")


def moe_create_indices_workspace_bytes(num_slots: int, E: int) -> int:
    return library().moe_create_indices_workspace_bytes(num_slots, E)


def moe_create_indices(topk_ids, num_slots: int, E: int, token_expert_order,
                       expert_start_indices, restore_token_order, expert_ids,
                       expert_usage_stats, scales_offset, workspace, ws_bytes: int,
                       stream=None):
    _check(library().moe_create_indices(
        _ptr(topk_ids), num_slots, E, _ptr(token_expert_order), _ptr(expert_start_indices),
        _ptr(restore_token_order), _ptr(expert_ids), _ptr(expert_usage_stats),
        _ptr(scales_offset), _ptr(workspace), ws_bytes, _stream(stream)), "moe_create_indices")


def moe_mask_and_create_indices(routing_map, N: int, top_k: int, real_token_count,
                                tp_rank: int, E: int, token_expert_order, expert_start_indices,
                                restore_token_order, expert_ids, expert_usage_stats,
                                scales_offset, workspace, ws_bytes: int, stream=None):
    """moe_mask_padding followed by moe_create_indices on the masked map, one
    kernel when N * top_k <= 1024."""
    _check(library().moe_mask_and_create_indices(
        _ptr(routing_map), N, top_k, _ptr(real_token_count), tp_rank, E,
        _ptr(token_expert_order), _ptr(expert_start_indices), _ptr(restore_token_order),
        _ptr(expert_ids), _ptr(expert_usage_stats), _ptr(scales_offset), _ptr(workspace),
        ws_bytes, _stream(stream)), "moe_mask_and_create_indices")


MOE_CREATE_INDICES_STATIC_SCRATCH = 262144


def moe_create_indices_static(topk_ids, num_slots: int, E: int, token_expert_order,
                              expert_start_indices, restore_token_order, expert_ids,
                              expert_usage_stats, scales_offset, stream=None):
    """moe_create_indices without a workspace: the scratch is a fixed array inside the
    library (see include/moe_route.h for the size limit and the sharing rules)."""
    _check(library().moe_create_indices_static(
        _ptr(topk_ids), num_slots, E, _ptr(token_expert_order), _ptr(expert_start_indices),
        _ptr(restore_token_order), _ptr(expert_ids), _ptr(expert_usage_stats),
        _ptr(scales_offset), _stream(stream)), "moe_create_indices_static")


def moe_mxfp4_row_stride(K: int) -> int:
    return library().moe_mxfp4_row_stride(K)


def moe_dispatch_mxfp4(input_tokens, N: int, K: int, top_k: int, E: int, restore_token_order,
                       expert_start_indices, expert_ids, expert_usage_stats, recv_buf,
                       recv_capacity: int, recv_counts, stream=None):
    _check(library().moe_dispatch_mxfp4(
        _ptr(input_tokens), N, K, top_k, E, _ptr(restore_token_order),
        _ptr(expert_start_indices), _ptr(expert_ids), _ptr(expert_usage_stats), _ptr(recv_buf),
        recv_capacity, _ptr(recv_counts), _stream(stream)), "moe_dispatch_mxfp4")


def moe_dispatch_mxfp4_quantize_nvfp4(input_tokens, N: int, K: int, top_k: int, E: int,
                                      restore_token_order, expert_start_indices, expert_ids,
                                      expert_usage_stats, recv_buf, recv_capacity: int,
                                      recv_counts, act_global: float, xq, sfa, stream=None):
    """moe_dispatch_mxfp4 and moe_quantize_activations_nvfp4 from one read of x."""
    _check(library().moe_dispatch_mxfp4_quantize_nvfp4(
        _ptr(input_tokens), N, K, top_k, E, _ptr(restore_token_order),
        _ptr(expert_start_indices), _ptr(expert_ids), _ptr(expert_usage_stats), _ptr(recv_buf),
        recv_capacity, _ptr(recv_counts), act_global, _ptr(xq), _ptr(sfa), _stream(stream)),
        "moe_dispatch_mxfp4_quantize_nvfp4")


def moe_quantize_activations_nvfp4(x, M: int, K: int, act_global: float, xq, sfa, stream=None):
    _check(library().moe_quantize_activations_nvfp4(
        _ptr(x), M, K, act_global, _ptr(xq), _ptr(sfa), _stream(stream)),
        "moe_quantize_activations_nvfp4")


def moe_quantize_weights_nvfp4(w, E: int, N: int, K: int, wq, sfw, w_global, stream=None):
    _check(library().moe_quantize_weights_nvfp4(
        _ptr(w), E, N, K, _ptr(wq), _ptr(sfw), _ptr(w_global), _stream(stream)),
        "moe_quantize_weights_nvfp4")


def moe_grouped_gemv_workspace_bytes(M: int, top_k: int, E: int, K: int) -> int:
    return library().moe_grouped_gemv_workspace_bytes(M, top_k, E, K)


def moe_grouped_gemv_nvfp4(mode: int, act, sfa, act_global: float, indices, M: int, top_k: int,
                           w, sfw, w_global, E: int, N: int, K: int, token_expert_order=None,
                           expert_start_indices=None, expert_ids=None, expert_usage_stats=None,
                           out=None, workspace=None, ws_bytes: int = 0, stream=None):
    """Grouped GEMV over the routing map ``indices`` [M, top_k].  Pass the
    four moe_create_indices outputs for this map, or none of them; a workspace
    of moe_grouped_gemv_workspace_bytes(M, top_k, E, K) bytes serves every
    variant (required without the grouping; with it, W4A16 in the
    tensor-memory variant converts its activations there once)."""
    _check(library().moe_grouped_gemv_nvfp4(
        mode, _ptr(act), _ptr(sfa), act_global, _ptr(indices), M, top_k, _ptr(w), _ptr(sfw),
        _ptr(w_global), E, N, K, _ptr(token_expert_order), _ptr(expert_start_indices),
        _ptr(expert_ids), _ptr(expert_usage_stats), _ptr(out), _ptr(workspace), ws_bytes,
        _stream(stream)), "moe_grouped_gemv_nvfp4")


def moe_grouped_gemv_plan(mode: int, M: int, top_k: int, E: int, N: int, K: int,
                          grouping_given: bool = False) -> tuple[int, bool]:
    """(variant, groups_in_kernel) that moe_grouped_gemv_nvfp4 uses for these shapes."""
    v, g = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(library().moe_grouped_gemv_plan(mode, M, top_k, E, N, K, int(grouping_given),
                                           ctypes.byref(v), ctypes.byref(g)),
           "moe_grouped_gemv_plan")
    return v.value, bool(g.value)


def moe_combine(expert_out, router_weights, topk_ids, M: int, top_k: int, H: int, E: int,
                epi: int, alpha: float, output_tokens, stream=None):
    _check(library().moe_combine(
        _ptr(expert_out), _ptr(router_weights), _ptr(topk_ids), M, top_k, H, E, epi, alpha,
        _ptr(output_tokens), _stream(stream)), "moe_combine")


def moe_get_device_error(clear: bool = True) -> int:
    flags = ctypes.c_uint32(0)
    _check(library().moe_get_device_error(ctypes.byref(flags), int(clear)),
           "moe_get_device_error")
    return flags.value
