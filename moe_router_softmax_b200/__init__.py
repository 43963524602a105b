"""Python binding of libmoe_b200.so -- the B200 (sm_100a) routed-expert MoE layer.

A thin ctypes layer over the C ABI in ``include/moe.h``: every function here has
the name of the C entry point it calls, checks and marshals its arguments
(torch tensors -> device pointers, the current torch CUDA stream) and raises
``MoeError`` with ``moe_last_error()`` when the call fails.  Every step of the
layer runs in the library's kernels; PyTorch only provides device memory and
streams.  There is no fallback: if the shared library is missing, importing this
package raises ImportError (build it with ``python moe_router_softmax_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run python moe_router_softmax_b200/build.py "
                      "(or __graft_entry__.build())")

_lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(5)
MOE_W_BF16, MOE_W_INT8, MOE_W_INT4 = 0, 1, 2
MOE_FFN_AUTO, MOE_FFN_GEMV, MOE_FFN_TC = 0, 1, 2
FMT = {"bf16": MOE_W_BF16, "int8": MOE_W_INT8, "int4": MOE_W_INT4}

# every symbol include/moe.h declares
EXPORTS = [
    "moe_version", "moe_last_error", "moe_expert_bytes", "moe_blob_offsets", "moe_route_topk", "moe_permute",
    "moe_route_permute", "moe_route_ffn",
    "moe_expert_hits", "moe_grouped_ffn_workspace", "moe_grouped_ffn", "moe_grouped_ffn_path", "moe_combine",
    "moe_layer_forward_workspace", "moe_layer_forward", "moe_quantize_int8", "moe_quantize_int4",
    "moe_pack_expert", "moe_copy_to_slots", "moe_refresh_target", "moe_apply_placement",
    "moe_should_refresh", "moe_budget_from_vram", "moe_grouped_ffn_noalloc", "moe_take_device_errors",
    "moe_route_min_weight", "moe_router_topk", "moe_hits_window", "moe_refresh_device", "moe_promote_copies",
    "moe_gather_rows", "moe_ep_recv_ids", "moe_ep_splits",
]


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"[moe status {status}] {msg}")
        self.status = status


class _CLayer(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("slot_table", ctypes.c_void_p), ("pool", ctypes.c_void_p), ("home", ctypes.c_void_p),
        ("expert_bytes", ctypes.c_uint64), ("pool_slots", ctypes.c_int32),
    ]


P, i32, i64, u64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
LP = ctypes.POINTER(_CLayer)
_SIG = {
    "moe_version": (ctypes.c_char_p, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_expert_bytes": (sz, [i32, i32, i32]),
    "moe_blob_offsets": (i32, [i32, i32, i32, P]),
    "moe_route_topk": (i32, [P, i32, i32, i32, P, P, P]),
    "moe_permute": (i32, [P, i32, i32, i32, P, P, P, P, P, P]),
    "moe_route_permute": (i32, [P, i32, i32, i32, P, P, P, P, P, P, P, P]),
    "moe_route_ffn": (i32, [LP, P, P, i32, i32, P, P, P, P, P, P, P, P, P, sz, P]),
    "moe_expert_hits": (i32, [P, i64, i32, P, P]),
    "moe_grouped_ffn_workspace": (sz, [LP, i32, i32]),
    "moe_grouped_ffn": (i32, [LP, P, i32, i32, P, P, P, P, P, sz, P]),
    "moe_grouped_ffn_path": (i32, [LP, P, i32, i32, P, P, P, P, P, sz, i32, P]),
    "moe_combine": (i32, [P, P, P, i32, i32, i32, P, P]),
    "moe_layer_forward_workspace": (sz, [LP, i32, i32]),
    "moe_layer_forward": (i32, [LP, P, P, i32, i32, P, P, P, P, P, sz, P]),
    "moe_quantize_int8": (i32, [P, i32, i32, P, P, P]),
    "moe_quantize_int4": (i32, [P, i32, i32, P, P, P]),
    "moe_pack_expert": (i32, [i32, P, P, P, P, i32, i32, P, P]),
    "moe_copy_to_slots": (i32, [P, P, u64, P, P, i32, P]),
    "moe_refresh_target": (i32, [P, i32, i32, P, P]),
    "moe_apply_placement": (i32, [P, i32, i32, P, i32, P, P, P, P]),
    "moe_should_refresh": (i32, [i32, i32, i64, i32, i64]),
    "moe_budget_from_vram": (i64, [i64, i64, i64, i64, i64, i64]),
    "moe_grouped_ffn_noalloc": (i32, [LP, P, i32, i32, P, P, P, P, P]),
    "moe_take_device_errors": (i32, [P, P]),
    "moe_route_min_weight": (i32, [P, P, P, i32, i32, i32, ctypes.c_float, P]),
    "moe_router_topk": (i32, [P, P, i32, i32, i32, i32, P, P, P, P]),
    "moe_hits_window": (i32, [P, i32, i32, P]),
    "moe_refresh_device": (i32, [P, i32, i32, P, i32, P, P, P]),
    "moe_promote_copies": (i32, [P, P, u64, P, P, i32, P]),
    "moe_gather_rows": (i32, [P, i32, i32, P, i32, i32, P, P]),
    "moe_ep_recv_ids": (i32, [P, i32, i32, P, i32, P]),
    "moe_ep_splits": (i32, [P, i32, P, i32, P, P]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def _check(st: int) -> None:
    if st != MOE_OK:
        raise MoeError(st, (_lib.moe_last_error() or b"").decode())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor | None, dtype=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _host(a: np.ndarray, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


BF16 = (torch.bfloat16, torch.int16, torch.uint16)


def moe_version() -> str:
    return _lib.moe_version().decode()


def moe_last_error() -> str:
    return (_lib.moe_last_error() or b"").decode()


def moe_expert_bytes(fmt: int, H: int, I: int) -> int:
    return int(_lib.moe_expert_bytes(fmt, H, I))


def moe_blob_offsets(fmt: int, H: int, I: int):
    off = np.zeros(4, np.uint64)
    _check(_lib.moe_blob_offsets(fmt, H, I, off.ctypes.data_as(ctypes.c_void_p)))
    return [int(v) for v in off]


class MoeLayer:
    """One MoE layer's experts: format, sizes and the device memory they live in.

    ``home`` holds E expert blobs (uint8, stride ``expert_bytes``); ``pool`` and
    ``slot_table`` (int32 [E], slot id or -1) are optional.  ``pool_slots`` is the
    number of blobs in ``pool`` (default: as many whole blobs as it holds).  The
    tensors are kept alive by this object.
    """

    def __init__(self, fmt: int, E: int, H: int, I: int, home: torch.Tensor, pool: torch.Tensor | None = None,
                 slot_table: torch.Tensor | None = None, expert_bytes: int | None = None,
                 pool_slots: int | None = None):
        self.fmt, self.E, self.H, self.I = int(fmt), int(E), int(H), int(I)
        self.expert_bytes = int(expert_bytes or (moe_expert_bytes(fmt, H, I) + 255) // 256 * 256)
        self.home, self.pool, self.slot_table = home, pool, slot_table
        if pool_slots is None:
            pool_slots = 0 if pool is None else pool.numel() // self.expert_bytes
        self.pool_slots = int(pool_slots)
        self._c = _CLayer()
        self.refresh()

    def refresh(self):
        """Re-read the tensors' addresses (after replacing pool or slot_table)."""
        self._c.fmt, self._c.E, self._c.H, self._c.I = self.fmt, self.E, self.H, self.I
        self._c.home = _dev(self.home, torch.uint8, "home").value
        self._c.pool = None if self.pool is None else _dev(self.pool, torch.uint8, "pool").value
        self._c.slot_table = None if self.slot_table is None else _dev(self.slot_table, torch.int32, "slot_table").value
        self._c.expert_bytes = self.expert_bytes
        self._c.pool_slots = self.pool_slots
        return self

    def ref(self):
        return ctypes.byref(self._c)


def moe_route_topk(logits: torch.Tensor, k: int, ids: torch.Tensor | None = None, w: torch.Tensor | None = None,
                   stream=None):
    T, E = logits.shape
    ids = torch.empty((T, k), dtype=torch.int32, device=logits.device) if ids is None else ids
    w = torch.empty((T, k), dtype=torch.float32, device=logits.device) if w is None else w
    _check(_lib.moe_route_topk(_dev(logits, torch.float32, "logits"), T, E, k, _dev(ids, torch.int32, "ids"),
                               _dev(w, torch.float32, "w"), _stream(stream)))
    return ids, w


def moe_router_topk(x: torch.Tensor, w_router: torch.Tensor, k: int, logits: torch.Tensor | bool | None = None,
                    ids: torch.Tensor | None = None, w: torch.Tensor | None = None, stream=None):
    """Router projection x[T,H] (bf16) . w_router[E,H]^T (fp32) fused with top-k.
    Returns (ids, w) or, with logits=True or a [T,E] fp32 tensor, (ids, w, logits)."""
    T, H = x.shape
    E = w_router.shape[0]
    if w_router.shape[1] != H:
        raise ValueError("w_router must be [E, H]")
    want_logits = logits is not None and logits is not False
    if logits is True:
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    elif logits is False:
        logits = None
    ids = torch.empty((T, k), dtype=torch.int32, device=x.device) if ids is None else ids
    w = torch.empty((T, k), dtype=torch.float32, device=x.device) if w is None else w
    _check(_lib.moe_router_topk(_dev(x, BF16, "x"), _dev(w_router, torch.float32, "w_router"), T, H, E, k,
                                _dev(logits, torch.float32, "logits"), _dev(ids, torch.int32, "ids"),
                                _dev(w, torch.float32, "w"), _stream(stream)))
    return (ids, w, logits) if want_logits else (ids, w)


def moe_route_min_weight(ids: torch.Tensor, w: torch.Tensor, E: int, min_weight: float,
                         slot_table: torch.Tensor | None = None, stream=None):
    """In place: [miss] min_weight partial routing of moe_route_topk's output."""
    T, k = ids.shape
    _check(_lib.moe_route_min_weight(_dev(ids, torch.int32, "ids"), _dev(w, torch.float32, "w"),
                                     None if slot_table is None else _dev(slot_table, torch.int32, "slot_table"),
                                     T, k, E, float(min_weight), _stream(stream)))
    return ids, w


def moe_permute(ids: torch.Tensor, E: int, hits: torch.Tensor | None = None, out=None, stream=None):
    T, k = ids.shape
    R = T * k
    dev = ids.device
    if out is None:
        out = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R],
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R])
    counts, offsets, sorted_route, route_pos = out
    _check(_lib.moe_permute(_dev(ids, torch.int32, "ids"), T, k, E, _dev(counts, torch.int32, "counts"),
                            _dev(offsets, torch.int32, "offsets"), _dev(sorted_route, torch.int32, "sorted_route"),
                            _dev(route_pos, torch.int32, "route_pos"),
                            None if hits is None else _dev(hits, (torch.int32, torch.uint32), "hits"),
                            _stream(stream)))
    return counts, offsets, sorted_route, route_pos


def moe_route_permute(logits: torch.Tensor, k: int, hits: torch.Tensor | None = None, ids_w=None, out=None,
                      stream=None):
    """moe_route_topk then moe_permute in one call (one launch for T <= 16).
    Returns (ids, w, counts, offsets, sorted_route, route_pos)."""
    T, E = logits.shape
    R = T * k
    dev = logits.device
    ids, w = ids_w if ids_w is not None else (torch.empty((T, k), dtype=torch.int32, device=dev),
                                              torch.empty((T, k), dtype=torch.float32, device=dev))
    if out is None:
        out = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R],
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R])
    counts, offsets, sorted_route, route_pos = out
    _check(_lib.moe_route_permute(_dev(logits, torch.float32, "logits"), T, E, k, _dev(ids, torch.int32, "ids"),
                                  _dev(w, torch.float32, "w"), _dev(counts, torch.int32, "counts"),
                                  _dev(offsets, torch.int32, "offsets"),
                                  _dev(sorted_route, torch.int32, "sorted_route"),
                                  _dev(route_pos, torch.int32, "route_pos"),
                                  None if hits is None else _dev(hits, (torch.int32, torch.uint32), "hits"),
                                  _stream(stream)))
    return ids, w, counts, offsets, sorted_route, route_pos


def moe_expert_hits(ids: torch.Tensor, E: int, hits: torch.Tensor, stream=None) -> torch.Tensor:
    _check(_lib.moe_expert_hits(_dev(ids, torch.int32, "ids"), ids.numel(), E,
                                _dev(hits, (torch.int32, torch.uint32), "hits"), _stream(stream)))
    return hits


def moe_grouped_ffn_workspace(layer: MoeLayer, T: int, k: int) -> int:
    return int(_lib.moe_grouped_ffn_workspace(layer.ref(), T, k))


def moe_grouped_ffn(layer: MoeLayer, x: torch.Tensor, k: int, counts, offsets, sorted_route,
                    rows: torch.Tensor | None = None, ws: torch.Tensor | None = None, path: int = MOE_FFN_AUTO,
                    stream=None) -> torch.Tensor:
    T = x.shape[0]
    if rows is None:
        rows = torch.empty((max(T * k, 1), layer.H), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = torch.empty(max(moe_grouped_ffn_workspace(layer, T, k), 16), dtype=torch.uint8, device=x.device)
    _check(_lib.moe_grouped_ffn_path(layer.ref(), _dev(x, BF16, "x"), T, k, _dev(counts, torch.int32, "counts"),
                                     _dev(offsets, torch.int32, "offsets"),
                                     _dev(sorted_route, torch.int32, "sorted_route"), _dev(rows, torch.float32, "rows"),
                                     _dev(ws, torch.uint8, "ws"), ws.numel(), int(path), _stream(stream)))
    return rows


def moe_route_ffn(layer: MoeLayer, logits: torch.Tensor, x: torch.Tensor, k: int, hits: torch.Tensor | None = None,
                  ids_w=None, out=None, rows: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                  stream=None):
    """moe_route_permute then moe_grouped_ffn in one call (for one token the
    routing runs inside the FFN's launches).  Returns (ids, w, counts, offsets,
    sorted_route, route_pos, rows)."""
    T, E = logits.shape
    R = T * k
    dev = logits.device
    ids, w = ids_w if ids_w is not None else (torch.empty((T, k), dtype=torch.int32, device=dev),
                                              torch.empty((T, k), dtype=torch.float32, device=dev))
    if out is None:
        out = (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R],
               torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R])
    counts, offsets, sorted_route, route_pos = out
    if rows is None:
        rows = torch.empty((max(R, 1), layer.H), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(moe_grouped_ffn_workspace(layer, T, k), 16), dtype=torch.uint8, device=dev)
    _check(_lib.moe_route_ffn(layer.ref(), _dev(logits, torch.float32, "logits"), _dev(x, BF16, "x"), T, k,
                              None if hits is None else _dev(hits, (torch.int32, torch.uint32), "hits"),
                              _dev(ids, torch.int32, "ids"), _dev(w, torch.float32, "w"),
                              _dev(counts, torch.int32, "counts"), _dev(offsets, torch.int32, "offsets"),
                              _dev(sorted_route, torch.int32, "sorted_route"),
                              _dev(route_pos, torch.int32, "route_pos"), _dev(rows, torch.float32, "rows"),
                              _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))
    return ids, w, counts, offsets, sorted_route, route_pos, rows


def moe_combine(rows: torch.Tensor, route_pos: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    T, k = w.shape
    H = rows.shape[1]
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=rows.device)
    _check(_lib.moe_combine(_dev(rows, torch.float32, "rows"), _dev(route_pos, torch.int32, "route_pos"),
                            _dev(w, torch.float32, "w"), T, k, H, _dev(y, BF16, "y"), _stream(stream)))
    return y


def moe_layer_forward_workspace(layer: MoeLayer, T: int, k: int) -> int:
    return int(_lib.moe_layer_forward_workspace(layer.ref(), T, k))


def moe_layer_forward(layer: MoeLayer, logits: torch.Tensor, x: torch.Tensor, k: int, y: torch.Tensor | None = None,
                      hits: torch.Tensor | None = None, ids_out: torch.Tensor | None = None,
                      w_out: torch.Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.H), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = torch.empty(max(moe_layer_forward_workspace(layer, T, k), 16), dtype=torch.uint8, device=x.device)
    _check(_lib.moe_layer_forward(layer.ref(), _dev(logits, torch.float32, "logits"), _dev(x, BF16, "x"), T, k,
                                  None if hits is None else _dev(hits, (torch.int32, torch.uint32), "hits"),
                                  _dev(y, BF16, "y"), None if ids_out is None else _dev(ids_out, torch.int32, "ids_out"),
                                  None if w_out is None else _dev(w_out, torch.float32, "w_out"),
                                  _dev(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))
    return y


def moe_quantize_int8(w: torch.Tensor, q: torch.Tensor | None = None, scale: torch.Tensor | None = None, stream=None):
    rows, K = w.shape
    q = torch.empty((rows, K), dtype=torch.int8, device=w.device) if q is None else q
    scale = torch.empty(rows, dtype=torch.float32, device=w.device) if scale is None else scale
    _check(_lib.moe_quantize_int8(_dev(w, BF16, "w"), rows, K, _dev(q, torch.int8, "q"),
                                  _dev(scale, torch.float32, "scale"), _stream(stream)))
    return q, scale


def moe_quantize_int4(w: torch.Tensor, q: torch.Tensor | None = None, scale: torch.Tensor | None = None, stream=None):
    rows, K = w.shape
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=w.device) if q is None else q
    scale = torch.empty((rows, K // 64), dtype=torch.bfloat16, device=w.device) if scale is None else scale
    _check(_lib.moe_quantize_int4(_dev(w, BF16, "w"), rows, K, _dev(q, torch.uint8, "q"), _dev(scale, BF16, "scale"),
                                  _stream(stream)))
    return q, scale


def moe_pack_expert(fmt: int, w13, s13, w2, s2, H: int, I: int, blob: torch.Tensor, stream=None) -> torch.Tensor:
    _check(_lib.moe_pack_expert(fmt, _dev(w13, None, "w13"), None if s13 is None else _dev(s13, None, "s13"),
                                _dev(w2, None, "w2"), None if s2 is None else _dev(s2, None, "s2"), H, I,
                                _dev(blob, torch.uint8, "blob"), _stream(stream)))
    return blob


def moe_copy_to_slots(home: torch.Tensor, pool: torch.Tensor, expert_bytes: int, experts, slots, stream=None):
    ex, pe = _host(experts, np.int32)
    sl, ps = _host(slots, np.int32)
    assert ex.size == sl.size
    _check(_lib.moe_copy_to_slots(_dev(home, torch.uint8, "home"), _dev(pool, torch.uint8, "pool"), int(expert_bytes),
                                  pe, ps, ex.size, _stream(stream)))


def moe_take_device_errors():
    """Synchronise, then return (code, info) of the first problem a tensor-core
    kernel recorded since the last call ((0, 0) if none)."""
    c, i = ctypes.c_uint32(0), ctypes.c_uint32(0)
    st = _lib.moe_take_device_errors(ctypes.byref(c), ctypes.byref(i))
    if st not in (MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_CUDA):
        _check(st)
    return int(c.value), int(i.value)


def moe_refresh_target(hits: np.ndarray, budget: int) -> np.ndarray:
    h, ph = _host(hits, np.uint32)
    t = np.zeros(max(budget, 1), np.int32)
    n = ctypes.c_int32(0)
    _check(_lib.moe_refresh_target(ph, h.size, budget, t.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)))
    return t[: n.value].copy()


def moe_apply_placement(slot_of: np.ndarray, n_slots: int, target: np.ndarray):
    """Returns (new slot_of, promote, demote) -- host arrays."""
    so = np.ascontiguousarray(slot_of, np.int32).copy()
    tg, pt = _host(target, np.int32)
    E = so.size
    pr = np.zeros(E, np.int32)
    de = np.zeros(E, np.int32)
    npr, nde = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(_lib.moe_apply_placement(so.ctypes.data_as(ctypes.c_void_p), E, n_slots, pt, tg.size,
                                    pr.ctypes.data_as(ctypes.c_void_p), de.ctypes.data_as(ctypes.c_void_p),
                                    ctypes.byref(npr), ctypes.byref(nde)))
    return so, pr[: npr.value].copy(), de[: nde.value].copy()


def moe_hits_window(ring: np.ndarray) -> np.ndarray:
    """Host: window sum of per-step hit histograms ring[W, E] -> uint32[E]."""
    r, pr = _host(ring, np.uint32)
    W, E = r.shape
    out = np.zeros(E, np.uint32)
    _check(_lib.moe_hits_window(pr, W, E, out.ctypes.data_as(ctypes.c_void_p)))
    return out


def moe_refresh_device(hits: torch.Tensor, budget: int, slot_table: torch.Tensor, n_slots: int,
                       promo: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None):
    """Device placement refresh (slot_table updated in place).  Returns (promo, status):
    promo int32 [n_slots, 2] (expert, slot) pairs, status int32 [3] (promotions, demotions, error)."""
    E = slot_table.numel()
    dev = slot_table.device
    promo = torch.empty((max(n_slots, 1), 2), dtype=torch.int32, device=dev) if promo is None else promo
    status = torch.empty(3, dtype=torch.int32, device=dev) if status is None else status
    _check(_lib.moe_refresh_device(_dev(hits, (torch.int32, torch.uint32), "hits"), E, budget,
                                   _dev(slot_table, torch.int32, "slot_table"), n_slots,
                                   _dev(promo, torch.int32, "promo"), _dev(status, torch.int32, "status"),
                                   _stream(stream)))
    return promo, status


def moe_promote_copies(home: torch.Tensor, pool: torch.Tensor, expert_bytes: int, promo: torch.Tensor,
                       status: torch.Tensor, max_promo: int, stream=None) -> None:
    """Copy the promoted blobs listed on the device by moe_refresh_device."""
    _check(_lib.moe_promote_copies(_dev(home, None, "home"), _dev(pool, None, "pool"), expert_bytes,
                                   _dev(promo, torch.int32, "promo"), _dev(status, torch.int32, "status"),
                                   max_promo, _stream(stream)))


def moe_should_refresh(offload_enabled: bool, mode_refresh: bool, step: int, is_prefill_block: bool,
                       interval: int) -> bool:
    return bool(_lib.moe_should_refresh(int(offload_enabled), int(mode_refresh), step, int(is_prefill_block), interval))


def moe_budget_from_vram(free_bytes, reserve_bytes, expert_bytes, layers, max_per_layer, E) -> int:
    return int(_lib.moe_budget_from_vram(free_bytes, reserve_bytes, expert_bytes, layers, max_per_layer, E))


def moe_grouped_ffn_noalloc(layer: MoeLayer, x: torch.Tensor, k: int, counts, offsets, sorted_route,
                            rows: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_grouped_ffn for callers that cannot allocate: the library's fixed
    16 MiB device scratch replaces the workspace (see include/moe.h)."""
    T = x.shape[0]
    if rows is None:
        rows = torch.empty((max(T * k, 1), layer.H), dtype=torch.float32, device=x.device)
    _check(_lib.moe_grouped_ffn_noalloc(layer.ref(), _dev(x, BF16, "x"), T, k, _dev(counts, torch.int32, "counts"),
                                        _dev(offsets, torch.int32, "offsets"),
                                        _dev(sorted_route, torch.int32, "sorted_route"),
                                        _dev(rows, torch.float32, "rows"), _stream(stream)))
    return rows


def moe_gather_rows(src: torch.Tensor, index: torch.Tensor, divisor: int = 1, dst: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """dst[i] = src[index[i] // divisor] for the rows of a 2-D tensor (rows with a
    negative or out-of-range index are left as they are in dst)."""
    n = index.numel()
    if dst is None:
        dst = torch.empty((max(n, 1), src.shape[1]), dtype=src.dtype, device=src.device)
    row_bytes = src.shape[1] * src.element_size()
    if dst.shape[1] * dst.element_size() != row_bytes or dst.shape[0] < n:
        raise ValueError("dst must have at least index.numel() rows of the same size as src's")
    _check(_lib.moe_gather_rows(_dev(src, None, "src"), src.shape[0], row_bytes, _dev(index, torch.int32, "index"),
                                n, int(divisor), _dev(dst, None, "dst"), _stream(stream)))
    return dst[:n] if dst.shape[0] != n else dst


def moe_ep_recv_ids(recv_counts: torch.Tensor, n: int, ids: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Local expert id (int32 [n]) of each received row; recv_counts int32 [N, El]."""
    N, El = recv_counts.shape
    if ids is None:
        ids = torch.empty(max(n, 1), dtype=torch.int32, device=recv_counts.device)[:n]
    _check(_lib.moe_ep_recv_ids(_dev(recv_counts, torch.int32, "recv_counts"), N, El, _dev(ids, torch.int32, "ids"),
                                int(n), _stream(stream)))
    return ids


def moe_ep_splits(counts: np.ndarray, recv_counts: np.ndarray):
    """Host: (send_rows, recv_rows), int32 [N] each, from this rank's counts [E]
    and the received per-expert counts [N, El]."""
    c, pc = _host(np.ravel(counts), np.int32)
    r, pr = _host(recv_counts, np.int32)
    if r.ndim != 2 or r.shape[0] * r.shape[1] != c.size:
        raise ValueError("recv_counts must be [N, E / N]")
    N = r.shape[0]
    send = np.zeros(N, np.int32)
    recv = np.zeros(N, np.int32)
    _check(_lib.moe_ep_splits(pc, c.size, pr, N, send.ctypes.data_as(ctypes.c_void_p),
                              recv.ctypes.data_as(ctypes.c_void_p)))
    return send, recv


# ------------------------------------------------------------------ helpers

def make_layer(fmt: int, w13: torch.Tensor, w2: torch.Tensor, stream=None) -> MoeLayer:
    """Build a layer's home blobs from bf16 weights w13 [E, 2I, H] and w2 [E, H, I]
    (quantised on the GPU by moe_quantize_int8 / moe_quantize_int4 for those
    formats, then packed by moe_pack_expert)."""
    E, I2, H = w13.shape
    I = I2 // 2
    eb = (moe_expert_bytes(fmt, H, I) + 255) // 256 * 256   # blob stride: a multiple of 256 bytes
    home = torch.empty(E * eb, dtype=torch.uint8, device=w13.device)
    for e in range(E):
        blob = home[e * eb:(e + 1) * eb]
        if fmt == MOE_W_BF16:
            moe_pack_expert(fmt, w13[e], None, w2[e], None, H, I, blob, stream)
        elif fmt == MOE_W_INT8:
            q13, s13 = moe_quantize_int8(w13[e], stream=stream)
            q2, s2 = moe_quantize_int8(w2[e], stream=stream)
            moe_pack_expert(fmt, q13, s13, q2, s2, H, I, blob, stream)
        else:
            q13, s13 = moe_quantize_int4(w13[e], stream=stream)
            q2, s2 = moe_quantize_int4(w2[e], stream=stream)
            moe_pack_expert(fmt, q13, s13, q2, s2, H, I, blob, stream)
    return MoeLayer(fmt, E, H, I, home, expert_bytes=eb)
