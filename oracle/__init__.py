"""CPU oracle for the MoE token-routing pipeline (plain C, single thread, fp64).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The CUDA path never
does, and this package never imports the CUDA path.

Each wrapper restates one step of the method (see the citations in
``moe_oracle.c``):

  mask_padding        Megatron-Core mask_routing_padding
  create_indices      MAX moe_create_indices
  mxfp4_encode_rows / dispatch_mxfp4
                      MAX ep.dispatch_async.mxfp4 (MXFP4 payload, 1 GPU)
  nvfp4_quantize*     FlashRT quantize_activations_nvfp4_bf16 /
                      quantize_weights_nvfp4_bf16
  grouped_gemv        FlashRT grouped_w4a16_gemv_bf16 / grouped_w4a4_gemv_bf16
  combine             MAX ep.combine_wait weighted sum + epilogue

Parity status of every function is pinned by ``tests/test_oracle_*.py``
(library routines, closed forms, invariants, brute force); none is unpinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

EPI = {"none": 0, "identity": 1, "scale": 2}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE single division matters)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-fvisibility=hidden", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _declare(_lib)
    return _lib


P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
F32 = ctypes.c_float


def _declare(L):
    L.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_value.restype = ctypes.c_double
    L.oracle_e2m1_encode.argtypes = [ctypes.c_double]
    L.oracle_e2m1_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_value.restype = ctypes.c_double
    L.oracle_e4m3_encode_satfinite.argtypes = [ctypes.c_double]
    L.oracle_e4m3_encode_satfinite.restype = ctypes.c_uint8
    L.oracle_mask_padding.argtypes = [P, I32, I32, I32, I32]
    L.oracle_mask_padding.restype = None
    L.oracle_create_indices.argtypes = [P, I64, I32, P, P, P, P, P, P]
    L.oracle_create_indices.restype = None
    L.oracle_mxfp4_row_stride.argtypes = [I32]
    L.oracle_mxfp4_row_stride.restype = I32
    L.oracle_mxfp4_encode_row.argtypes = [P, I32, P]
    L.oracle_mxfp4_encode_row.restype = None
    L.oracle_dispatch_mxfp4.argtypes = [P, I32, I32, I32, P, P, P, P, P, P]
    L.oracle_dispatch_mxfp4.restype = None
    L.oracle_nvfp4_quantize.argtypes = [P, I64, I32, F32, P, P]
    L.oracle_nvfp4_quantize.restype = None
    L.oracle_nvfp4_quantize_bf16.argtypes = [P, I64, I32, F32, P, P]
    L.oracle_nvfp4_quantize_bf16.restype = None
    L.oracle_nvfp4_weight_global.argtypes = [P, I64]
    L.oracle_nvfp4_weight_global.restype = F32
    L.oracle_quantize_weights_nvfp4.argtypes = [P, I32, I32, I32, P, P, P]
    L.oracle_quantize_weights_nvfp4.restype = None
    L.oracle_gemv_element.argtypes = [I32, P, P, P, F32, P, I32, P, P, P, I32, I32, I32,
                                      I64, I32, I32, P]
    L.oracle_gemv_element.restype = ctypes.c_int
    L.oracle_grouped_gemv.argtypes = [I32, P, P, P, F32, P, I32, I32, P, P, P, I32, I32, I32, P]
    L.oracle_grouped_gemv.restype = None
    L.oracle_combine.argtypes = [P, P, P, I32, I32, I32, I32, I32, F32, P]
    L.oracle_combine.restype = None


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(P)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(P)


# ---------------------------------------------------------------- scalars
def e2m1_value(code: int) -> float:
    return _load().oracle_e2m1_value(code)


def e2m1_encode(v: float) -> int:
    return _load().oracle_e2m1_encode(v)


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return _load().oracle_e4m3_encode_satfinite(v)


# ---------------------------------------------------------------- step 1
def mask_padding(routing_map: np.ndarray, real_token_count: int, tp_rank: int = 0) -> np.ndarray:
    """Return a masked copy of routing_map [N, top_k] int64."""
    m, pm = _c(routing_map, np.int64)
    m = m.copy()
    N, k = m.shape
    _load().oracle_mask_padding(m.ctypes.data_as(P), N, k, int(real_token_count), int(tp_rank))
    return m


# ---------------------------------------------------------------- step 2
def create_indices(topk_ids: np.ndarray, E: int) -> dict:
    ids, pid = _c(np.asarray(topk_ids).reshape(-1), np.int64)
    S = ids.size
    order = np.empty(S, np.uint32)
    start = np.empty(E + 1, np.uint32)
    restore = np.empty(S, np.uint32)
    eids = np.empty(E, np.int32)
    stats = np.empty(2, np.uint32)
    soff = np.empty(E + 1, np.uint32)
    _load().oracle_create_indices(pid, S, E, _ptr(order), _ptr(start), _ptr(restore),
                                  _ptr(eids), _ptr(stats), _ptr(soff))
    return dict(token_expert_order=order, expert_start_indices=start,
                restore_token_order=restore, expert_ids=eids, expert_usage_stats=stats,
                scales_offset=soff)


# ---------------------------------------------------------------- step 3
def mxfp4_row_stride(K: int) -> int:
    return _load().oracle_mxfp4_row_stride(K)


def mxfp4_encode_rows(x_bf16: np.ndarray) -> np.ndarray:
    """MXFP4 rows [rows, stride] u8 of bf16 rows x [rows, K] (uint16 bits)."""
    x, _ = _c(x_bf16, np.uint16)
    rows, K = x.shape
    st = mxfp4_row_stride(K)
    out = np.zeros((rows, st), np.uint8)
    L = _load()
    for r in range(rows):
        L.oracle_mxfp4_encode_row(x[r].ctypes.data_as(P), K, out[r].ctypes.data_as(P))
    return out


def dispatch_mxfp4(x_bf16: np.ndarray, top_k: int, E: int, idx: dict,
                   recv_rows: int | None = None, fill: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """Expert-grouped MXFP4 buffer [recv_rows, stride] and recv_counts [E]."""
    x, px = _c(x_bf16, np.uint16)
    N, K = x.shape
    st = mxfp4_row_stride(K)
    rows = N * top_k if recv_rows is None else recv_rows
    recv = np.full((rows, st), fill, np.uint8)
    counts = np.empty(E, np.uint32)
    order, _ = _c(idx["token_expert_order"], np.uint32)
    start, _ = _c(idx["expert_start_indices"], np.uint32)
    eids, _ = _c(idx["expert_ids"], np.int32)
    stats, _ = _c(idx["expert_usage_stats"], np.uint32)
    _load().oracle_dispatch_mxfp4(px, K, top_k, E, _ptr(order), _ptr(start), _ptr(eids),
                                  _ptr(stats), _ptr(recv), _ptr(counts))
    return recv, counts


# ---------------------------------------------------------------- step 4 codecs
def nvfp4_quantize(x_f32: np.ndarray, g: float = 1.0) -> tuple[np.ndarray, np.ndarray]:
    x, px = _c(x_f32, np.float32)
    rows, K = x.reshape(-1, x.shape[-1]).shape
    q = np.empty((rows, K // 2), np.uint8)
    sf = np.empty((rows, K // 16), np.uint8)
    _load().oracle_nvfp4_quantize(px, rows, K, float(g), _ptr(q), _ptr(sf))
    return q.reshape(*x.shape[:-1], K // 2), sf.reshape(*x.shape[:-1], K // 16)


def nvfp4_quantize_bf16(x_bf16: np.ndarray, g: float = 1.0) -> tuple[np.ndarray, np.ndarray]:
    x, px = _c(x_bf16, np.uint16)
    rows, K = x.shape
    q = np.empty((rows, K // 2), np.uint8)
    sf = np.empty((rows, K // 16), np.uint8)
    _load().oracle_nvfp4_quantize_bf16(px, rows, K, float(g), _ptr(q), _ptr(sf))
    return q, sf


def nvfp4_weight_global(w: np.ndarray) -> float:
    a, pa = _c(w, np.float32)
    return float(_load().oracle_nvfp4_weight_global(pa, a.size))


def quantize_weights_nvfp4(w_f32: np.ndarray):
    """w [E, N, K] fp32 -> (wq [E,N,K/2] u8, sfw [E,N,K/16] u8, w_global [E] f32)."""
    w, pw = _c(w_f32, np.float32)
    E, N, K = w.shape
    wq = np.empty((E, N, K // 2), np.uint8)
    sfw = np.empty((E, N, K // 16), np.uint8)
    gw = np.empty(E, np.float32)
    _load().oracle_quantize_weights_nvfp4(pw, E, N, K, _ptr(wq), _ptr(sfw), _ptr(gw))
    return wq, sfw, gw


# ---------------------------------------------------------------- step 4 GEMV
def grouped_gemv(mode: str, indices: np.ndarray, wq: np.ndarray, sfw: np.ndarray,
                 w_global: np.ndarray | None, act_bf16: np.ndarray | None = None,
                 xq: np.ndarray | None = None, sfa: np.ndarray | None = None,
                 g_a: float = 1.0, fill: float = np.nan) -> np.ndarray:
    """y [M, top_k, N] float64; unrouted slots hold ``fill``."""
    E, N, K2 = wq.shape
    K = K2 * 2
    idx, pidx = _c(indices, np.int64)
    M, top_k = idx.shape
    wq_, pwq = _c(wq, np.uint8)
    sfw_, psfw = _c(sfw, np.uint8)
    gw = None if w_global is None else np.ascontiguousarray(w_global, np.float32)
    y = np.full((M, top_k, N), fill, np.float64)
    m = 0 if mode == "w4a16" else 1
    a = None if act_bf16 is None else np.ascontiguousarray(act_bf16, np.uint16)
    q = None if xq is None else np.ascontiguousarray(xq, np.uint8)
    s = None if sfa is None else np.ascontiguousarray(sfa, np.uint8)
    _load().oracle_grouped_gemv(m, _ptr(a), _ptr(q), _ptr(s), float(g_a), pidx, M, top_k,
                                pwq, psfw, _ptr(gw), E, N, K, _ptr(y))
    return y


def gemv_elements(mode: str, indices: np.ndarray, wq, sfw, w_global, samples,
                  act_bf16=None, xq=None, sfa=None, g_a: float = 1.0, E: int | None = None,
                  expert_base: int = 0) -> np.ndarray:
    """Selected outputs y[m, j, n] for samples [(m, j, n), ...] (float64, NaN if unrouted).

    ``wq/sfw/w_global`` may hold a subset of experts starting at expert
    ``expert_base``: sampled slots must route to experts inside it.
    """
    Esub, N, K2 = wq.shape
    K = K2 * 2
    idx = np.ascontiguousarray(indices, np.int64)
    if expert_base:
        idx = idx - expert_base
    top_k = idx.shape[1]
    E_ = Esub if E is None else E
    wq_ = np.ascontiguousarray(wq, np.uint8)
    sfw_ = np.ascontiguousarray(sfw, np.uint8)
    gw = None if w_global is None else np.ascontiguousarray(w_global, np.float32)
    a = None if act_bf16 is None else np.ascontiguousarray(act_bf16, np.uint16)
    q = None if xq is None else np.ascontiguousarray(xq, np.uint8)
    s = None if sfa is None else np.ascontiguousarray(sfa, np.uint8)
    L = _load()
    out = np.full(len(samples), np.nan)
    yv = ctypes.c_double()
    m_ = 0 if mode == "w4a16" else 1
    for i, (m, j, n) in enumerate(samples):
        if L.oracle_gemv_element(m_, _ptr(a), _ptr(q), _ptr(s), float(g_a), _ptr(idx), top_k,
                                 _ptr(wq_), _ptr(sfw_), _ptr(gw), min(E_, Esub), N, K,
                                 int(m), int(j), int(n), ctypes.byref(yv)):
            out[i] = yv.value
    return out


# ---------------------------------------------------------------- step 5
def combine(expert_out_bf16: np.ndarray, router_weights: np.ndarray, topk_ids: np.ndarray,
            E: int, epilogue: str = "none", alpha: float = 1.0) -> np.ndarray:
    """out [M, H] float64."""
    y, py = _c(expert_out_bf16, np.uint16)
    M, k, H = y.shape
    w, pw = _c(router_weights, np.float32)
    ids, pids = _c(topk_ids, np.int64)
    out = np.empty((M, H), np.float64)
    _load().oracle_combine(py, pw, pids, M, k, H, E, EPI[epilogue], float(alpha), _ptr(out))
    return out
