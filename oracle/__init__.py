"""CPU oracle for the routed-expert MoE layer (numpy wrapper over moe_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library in ``moe_router_softmax_b200`` and never imports it.

Every function takes and returns numpy arrays in host memory.  bf16 data is
passed as its raw bits (``np.uint16``).  The C source states, function by
function, which page and section of the method each step follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

BF16, INT8, INT4 = 0, 1, 2
FMT_NAMES = {"bf16": BF16, "int8": INT8, "int4": INT4}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc, -ffp-contract=off)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))
    ):
        cmd = [
            "gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
            "-fPIC", "-shared", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm",
        ]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("slot_table", ctypes.c_void_p), ("pool", ctypes.c_void_p), ("home", ctypes.c_void_p),
        ("expert_bytes", ctypes.c_size_t),
    ]


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        c = _lib
        P = ctypes.c_void_p
        i32, i64, sz = ctypes.c_int, ctypes.c_long, ctypes.c_size_t
        c.oracle_expert_bytes.restype = sz
        c.oracle_expert_bytes.argtypes = [i32, i32, i32]
        c.oracle_blob_offsets.argtypes = [i32, i32, i32, P]
        c.oracle_exp_p.restype = ctypes.c_float
        c.oracle_exp_p.argtypes = [ctypes.c_float]
        c.oracle_gelu_tanh.restype = ctypes.c_double
        c.oracle_gelu_tanh.argtypes = [ctypes.c_double]
        c.oracle_bf16_rne.restype = ctypes.c_uint16
        c.oracle_bf16_rne.argtypes = [ctypes.c_float]
        c.oracle_route_topk.argtypes = [P, i32, i32, i32, P, P]
        c.oracle_permute.argtypes = [P, i32, i32, i32, P, P, P, P]
        c.oracle_route_min_weight.argtypes = [P, P, P, i32, i32, i32, ctypes.c_float]
        c.oracle_hits.argtypes = [P, i64, i32, P]
        c.oracle_hits_window.argtypes = [P, i32, i32, P]
        c.oracle_router_logits.argtypes = [P, P, i32, i32, i32, P]
        c.oracle_quantize_int8.argtypes = [P, i32, i32, P, P]
        c.oracle_quantize_int4.argtypes = [P, i32, i32, P, P]
        c.oracle_int4_candidates.argtypes = [P, P, P]
        c.oracle_pack_expert.argtypes = [i32, P, P, P, P, i32, i32, P]
        c.oracle_weight.restype = ctypes.c_double
        c.oracle_weight.argtypes = [i32, P, i32, i32, i32, i32, i32]
        c.oracle_expert_ffn.argtypes = [ctypes.POINTER(_Layer), i32, P, P]
        c.oracle_ffn_routes.argtypes = [ctypes.POINTER(_Layer), P, i32, i32, P, P]
        c.oracle_ffn_some_routes.argtypes = [ctypes.POINTER(_Layer), P, i32, P, P, i32, P]
        c.oracle_combine.argtypes = [P, P, P, i32, i32, i32, i32, P]
        c.oracle_refresh_target.restype = i32
        c.oracle_refresh_target.argtypes = [P, i32, i32, P]
        c.oracle_apply_placement.restype = i32
        c.oracle_apply_placement.argtypes = [P, i32, i32, P, i32, P, P, P, P]
        c.oracle_should_refresh.restype = i32
        c.oracle_should_refresh.argtypes = [i32, i32, i64, i32, i64]
        c.oracle_budget_from_vram.restype = i64
        c.oracle_budget_from_vram.argtypes = [i64, i64, i64, i64, i64, i64]
        c.oracle_set_threads.argtypes = [i32]
        c.oracle_get_threads.restype = i32
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    _L().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_L().oracle_get_threads())


def expert_bytes(fmt: int, H: int, I: int) -> int:
    return int(_L().oracle_expert_bytes(fmt, H, I))


def blob_offsets(fmt: int, H: int, I: int):
    off = np.zeros(4, dtype=np.uint64)
    _L().oracle_blob_offsets(fmt, H, I, _p(off))
    return [int(v) for v in off]


def exp_p(x: float) -> float:
    return float(_L().oracle_exp_p(float(x)))


def exp_p_array(x: np.ndarray) -> np.ndarray:
    f = _L().oracle_exp_p
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()], np.float32).reshape(np.shape(x))


def gelu_tanh(v: float) -> float:
    return float(_L().oracle_gelu_tanh(float(v)))


def bf16_rne(f: float) -> int:
    return int(_L().oracle_bf16_rne(float(f)))


def route_topk(logits: np.ndarray, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    _L().oracle_route_topk(_p(logits), T, E, k, _p(ids), _p(w))
    return ids, w


def route_min_weight(ids: np.ndarray, w: np.ndarray, slot_table, E: int, min_weight: float):
    """Returns new (ids, w) after [miss] min_weight partial routing."""
    ids = _c(ids, np.int32).copy()
    w = _c(w, np.float32).copy()
    T, k = ids.shape
    st = None if slot_table is None else _c(slot_table, np.int32)
    _L().oracle_route_min_weight(_p(ids), _p(w), None if st is None else _p(st), T, k, E, float(min_weight))
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    R = T * k
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    sr = np.zeros(max(R, 1), np.int32)
    rp = np.zeros(max(R, 1), np.int32)
    _L().oracle_permute(_p(ids), T, k, E, _p(counts), _p(offsets), _p(sr), _p(rp))
    sorted_route = sr[:R].copy()
    route_pos = rp[:R].copy()
    return counts, offsets, sorted_route, route_pos


def hits(ids: np.ndarray, E: int, hits_in: np.ndarray | None = None) -> np.ndarray:
    ids = _c(np.ravel(ids), np.int32)
    h = np.zeros(E, np.uint32) if hits_in is None else _c(hits_in, np.uint32).copy()
    _L().oracle_hits(_p(ids), ids.size, E, _p(h))
    return h


def hits_window(ring: np.ndarray) -> np.ndarray:
    """Window sum of per-step hit histograms ring[W, E] -> uint32[E]."""
    ring = _c(ring, np.uint32)
    W, E = ring.shape
    out = np.zeros(E, np.uint32)
    _L().oracle_hits_window(_p(ring), W, E, _p(out))
    return out


def router_logits(x_bits: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """fp64 logits[T, E] of the router projection x[T, H] (bf16 bits) . w_router[E, H]^T (fp32)."""
    x_bits = _c(x_bits, np.uint16)
    w_router = _c(w_router, np.float32)
    T, H = x_bits.shape
    E = w_router.shape[0]
    assert w_router.shape[1] == H
    out = np.zeros((T, E), np.float64)
    _L().oracle_router_logits(_p(x_bits), _p(w_router), T, H, E, _p(out))
    return out


def quantize_int8(w_bits: np.ndarray):
    w_bits = _c(w_bits, np.uint16)
    rows, K = w_bits.shape
    q = np.zeros((rows, K), np.int8)
    s = np.zeros(rows, np.float32)
    _L().oracle_quantize_int8(_p(w_bits), rows, K, _p(q), _p(s))
    return q, s


def quantize_int4(w_bits: np.ndarray):
    w_bits = _c(w_bits, np.uint16)
    rows, K = w_bits.shape
    assert K % 64 == 0
    q = np.zeros((rows, K // 2), np.uint8)
    s = np.zeros((rows, K // 64), np.uint16)
    _L().oracle_quantize_int4(_p(w_bits), rows, K, _p(q), _p(s))
    return q, s


def int4_candidates(w64_bits: np.ndarray):
    w64_bits = _c(w64_bits, np.uint16)
    assert w64_bits.size == 64
    s = np.zeros(16, np.float32)
    e = np.zeros(16, np.float64)
    _L().oracle_int4_candidates(_p(w64_bits), _p(s), _p(e))
    return s, e


def pack_expert(fmt: int, H: int, I: int, w13, s13, w2, s2) -> np.ndarray:
    blob = np.zeros(expert_bytes(fmt, H, I), np.uint8)
    parts = [w13, s13, w2, s2]
    ptrs = []
    keep = []
    for a in parts:
        if a is None:
            ptrs.append(None)
        else:
            a = np.ascontiguousarray(a)
            keep.append(a)
            ptrs.append(a.ctypes.data_as(ctypes.c_void_p))
    _L().oracle_pack_expert(fmt, ptrs[0], ptrs[1], ptrs[2], ptrs[3], H, I, _p(blob))
    return blob


def weight(fmt: int, blob: np.ndarray, H: int, I: int, which: int, row: int, col: int) -> float:
    return float(_L().oracle_weight(fmt, _p(blob), H, I, which, row, col))


class Layer:
    """Host copy of one MoE layer: format, sizes, slot table, pool and home blobs."""

    def __init__(self, fmt: int, E: int, H: int, I: int, home: np.ndarray, pool: np.ndarray | None = None,
                 slot_table: np.ndarray | None = None, expert_bytes_: int | None = None):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.home = _c(home, np.uint8).reshape(-1)
        self.pool = None if pool is None else _c(pool, np.uint8).reshape(-1)
        self.slot_table = None if slot_table is None else _c(slot_table, np.int32)
        self.expert_bytes = expert_bytes_ or expert_bytes(fmt, H, I)
        self._s = _Layer(fmt, E, H, I,
                         None if self.slot_table is None else self.slot_table.ctypes.data,
                         None if self.pool is None else self.pool.ctypes.data,
                         self.home.ctypes.data, self.expert_bytes)

    def ref(self):
        return ctypes.byref(self._s)


def expert_ffn(layer: Layer, e: int, x_row_bits: np.ndarray) -> np.ndarray:
    x = _c(x_row_bits, np.uint16)
    y = np.zeros(layer.H, np.float64)
    _L().oracle_expert_ffn(layer.ref(), e, _p(x), _p(y))
    return y


def ffn_routes(layer: Layer, x_bits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    ids = _c(ids, np.int32)
    T, k = ids.shape
    rows = np.zeros((T * k, layer.H), np.float64)
    _L().oracle_ffn_routes(layer.ref(), _p(x), T, k, _p(ids), _p(rows))
    return rows


def ffn_some_routes(layer: Layer, x_bits: np.ndarray, ids: np.ndarray, which) -> np.ndarray:
    x = _c(x_bits, np.uint16)
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    which = _c(which, np.int32)
    rows = np.zeros((which.size, layer.H), np.float64)
    _L().oracle_ffn_some_routes(layer.ref(), _p(x), k, _p(ids), _p(which), which.size, _p(rows))
    return rows


def combine(rows: np.ndarray, ids: np.ndarray, w: np.ndarray, E: int) -> np.ndarray:
    rows = _c(rows, np.float64)
    ids = _c(ids, np.int32)
    w = _c(w, np.float32)
    T, k = ids.shape
    H = rows.shape[1]
    y = np.zeros((T, H), np.float64)
    _L().oracle_combine(_p(rows), _p(ids), _p(w), T, k, E, H, _p(y))
    return y


def moe_layer(layer: Layer, logits: np.ndarray, x_bits: np.ndarray, k: int):
    ids, w = route_topk(logits, k)
    rows = ffn_routes(layer, x_bits, ids)
    y = combine(rows, ids, w, layer.E)
    return ids, w, rows, y


def refresh_target(hits_: np.ndarray, budget: int) -> np.ndarray:
    h = _c(hits_, np.uint32)
    t = np.zeros(max(budget, 1), np.int32)
    n = _L().oracle_refresh_target(_p(h), h.size, budget, _p(t))
    return t[:n].copy()


def apply_placement(slot_of: np.ndarray, n_slots: int, target: np.ndarray):
    """Returns (new slot_of, promote, demote); raises if no slot is free."""
    so = _c(slot_of, np.int32).copy()
    tg = _c(target, np.int32)
    E = so.size
    pr = np.zeros(max(E, 1), np.int32)
    de = np.zeros(max(E, 1), np.int32)
    npr = ctypes.c_int32(0)
    nde = ctypes.c_int32(0)
    rc = _L().oracle_apply_placement(_p(so), E, n_slots, _p(tg), tg.size, _p(pr), _p(de),
                                     ctypes.byref(npr), ctypes.byref(nde))
    if rc != 0:
        raise RuntimeError("oracle_apply_placement: no free slot")
    return so, pr[: npr.value].copy(), de[: nde.value].copy()


def should_refresh(offload_enabled: bool, mode_refresh: bool, step: int, is_prefill_block: bool,
                   interval: int) -> bool:
    return bool(_L().oracle_should_refresh(int(offload_enabled), int(mode_refresh), step,
                                           int(is_prefill_block), interval))


def budget_from_vram(free_bytes, reserve_bytes, expert_bytes_, layers, max_per_layer, E) -> int:
    return int(_L().oracle_budget_from_vram(free_bytes, reserve_bytes, expert_bytes_, layers,
                                            max_per_layer, E))
